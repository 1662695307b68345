"""Pins for the CPU oracle: it is checked against facts fixed by the pages and
by mathematics, never against itself.

* the SSA window geometry (QbitAI LoZA article, 1024-token sparse window
  paragraph): closed-form row counts and a hand-derived golden table;
* q = 0 makes every allowed key equally likely, so LSE_i = ln|J(i)| exactly and
  O_i is the plain mean of the allowed values (written from the interval form
  of the window, not the block rule);
* when the window covers the whole prefix, SSA is textbook causal attention
  ("LoZA：ZigZag稀疏注意力机制" §2.1, first formula with j <= i);
* constant values return that value; identical keys give uniform weights;
* a materialised-mask brute force in numpy agrees on tiny inputs;
* decode is invariant to where pages sit, equals prefill row t under the
  shared-latent broadcast, and packed varlen equals per-sequence prefill.
"""
import math
import os

import numpy as np
import pytest

from oracle import ssa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def closed_form_count(i, blk, n_sink, n_local):
    r = i % blk
    return min(i + 1, blk * (n_sink + n_local - 1) + r + 1)


def interval_keys(i, blk, n_sink, n_local):
    """J(i) written as two token intervals: the sink prefix and the local run."""
    b = i // blk
    sink_hi = min(i, n_sink * blk - 1)
    keys = list(range(0, sink_hi + 1))
    lo = max(n_sink * blk, (b - n_local + 1) * blk)
    keys += list(range(lo, i + 1))
    return keys


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 -> bf16 (nearest-even) and return the bit patterns."""
    f = x.astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


# ---------------------------------------------------------------- geometry

def test_golden_row_counts_block128_sink1_local7():
    rows = []
    with open(os.path.join(GOLDEN, "ssa_window_row_counts.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                i, c = line.split()
                rows.append((int(i), int(c)))
    assert len(rows) >= 10
    for i, c in rows:
        assert orc.row_count(i, 128, 1, 7) == c, i


def test_row_count_sink_plus_local_formula():
    # min(i+1, 128*[b>=7] + 768 + (i mod 128) + 1) for 1 sink + 7 local blocks of 128
    for i in list(range(0, 2200, 37)) + [895, 896, 1023, 1024, 5000]:
        b = i // 128
        want = min(i + 1, 128 * (b >= 7) + 768 + (i % 128) + 1)
        assert orc.row_count(i, 128, 1, 7) == want, i


@pytest.mark.parametrize("blk,n_sink,n_local", [(128, 1, 7), (4, 0, 1), (4, 2, 3), (8, 1, 1),
                                                (16, 3, 5), (5, 1, 2), (128, 0, 8)])
def test_row_count_closed_form(blk, n_sink, n_local):
    for i in range(0, blk * (n_sink + n_local + 4), max(1, blk // 8)):
        assert orc.row_count(i, blk, n_sink, n_local) == closed_form_count(i, blk, n_sink, n_local)


@pytest.mark.parametrize("n_sink,n_local", [(1, 7), (0, 1), (2, 3), (3, 1), (1, 12)])
def test_key_blocks_from_mask(n_sink, n_local):
    blk = 8
    for qb in range(0, 30):
        got = orc.key_blocks(qb, seq_len=30 * blk, blk=blk, n_sink=n_sink, n_local=n_local)
        want = sorted(set(range(min(n_sink, qb + 1))) |
                      set(range(max(n_sink, qb - n_local + 1), qb + 1)))
        assert got == want, qb
        assert len(got) == min(qb + 1, n_sink + n_local)


def test_key_blocks_partial_last_block():
    # a ragged final block still touches its own (partial) block
    assert orc.key_blocks(9, seq_len=9 * 128 + 3) == [0, 3, 4, 5, 6, 7, 8, 9]


# ------------------------------------------------------------ attention math

@pytest.mark.parametrize("blk,n_sink,n_local,L", [(128, 1, 7, 1300), (8, 1, 7, 200),
                                                  (4, 0, 2, 50), (6, 2, 3, 97)])
def test_q_zero_gives_log_count_and_mean(blk, n_sink, n_local, L):
    rng = np.random.default_rng(3)
    d = 16
    q = np.zeros((1, 1, L, d))
    k = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, 8))
    o, lse = orc.prefill(q, k, v, blk, n_sink, n_local, scale=0.25)
    for i in range(L):
        keys = interval_keys(i, blk, n_sink, n_local)
        assert len(keys) == closed_form_count(i, blk, n_sink, n_local)
        assert abs(lse[0, 0, i] - math.log(len(keys))) < 1e-12
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, keys].mean(axis=0), rtol=0, atol=1e-12)


@pytest.mark.parametrize("L,blk,n_sink,n_local", [(1024, 128, 1, 7), (700, 128, 1, 7),
                                                  (64, 8, 1, 7), (90, 8, 0, 12), (33, 4, 2, 7)])
def test_full_window_equals_causal(L, blk, n_sink, n_local):
    assert L <= blk * (n_sink + n_local) or n_local >= -(-L // blk)
    rng = np.random.default_rng(L)
    q = rng.standard_normal((1, 2, L, 32))
    k = rng.standard_normal((1, 2, L, 32))
    v = rng.standard_normal((1, 2, L, 24))
    o, lse = orc.prefill(q, k, v, blk, n_sink, n_local, scale=0.3)
    o_ref, lse_ref = orc.causal_attention(q, k, v, scale=0.3)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-11)


def test_beyond_window_differs_from_causal():
    # once the window no longer covers the prefix, SSA must NOT be causal attention
    L = 1400
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, 1, L, 16))
    k = rng.standard_normal((1, 1, L, 16))
    v = rng.standard_normal((1, 1, L, 16))
    o, _ = orc.prefill(q, k, v, scale=0.25)
    o_ref, _ = orc.causal_attention(q, k, v, scale=0.25)
    np.testing.assert_allclose(o[..., :1024, :], o_ref[..., :1024, :], atol=1e-11)
    assert np.abs(o[..., 1024:, :] - o_ref[..., 1024:, :]).max() > 1e-3


def test_constant_values_return_that_value():
    rng = np.random.default_rng(5)
    L = 300
    q = rng.standard_normal((1, 1, L, 16)) * 3
    k = rng.standard_normal((1, 1, L, 16)) * 3
    row = rng.standard_normal(12)
    v = np.broadcast_to(row, (1, 1, L, 12)).copy()
    o, _ = orc.prefill(q, k, v, blk=16, n_sink=1, n_local=3, scale=0.5)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(row, (L, 12)), atol=1e-12)


def test_identical_keys_give_uniform_weights():
    rng = np.random.default_rng(6)
    L, blk, ns, nl = 200, 16, 2, 3
    q = rng.standard_normal((1, 1, L, 8))
    k = np.broadcast_to(rng.standard_normal(8), (1, 1, L, 8)).copy()
    v = rng.standard_normal((1, 1, L, 5))
    o, lse = orc.prefill(q, k, v, blk=blk, n_sink=ns, n_local=nl, scale=0.7)
    s = 0.7 * q[0, 0] @ k[0, 0, 0]
    for i in range(L):
        keys = interval_keys(i, blk, ns, nl)
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, keys].mean(axis=0), atol=1e-12)
        assert abs(lse[0, 0, i] - (s[i] + math.log(len(keys)))) < 1e-11


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_mask_agrees(seed):
    rng = np.random.default_rng(100 + seed)
    blk = int(rng.integers(2, 9))
    n_sink = int(rng.integers(0, 3))
    n_local = int(rng.integers(1, 5))
    L = int(rng.integers(1, 12 * blk))
    q = rng.standard_normal((2, 2, L, 12))
    k = rng.standard_normal((2, 2, L, 12))
    v = rng.standard_normal((2, 2, L, 7))
    o, lse = orc.prefill(q, k, v, blk, n_sink, n_local, scale=0.4)
    o_bf, lse_bf = orc.brute_force_prefill(q, k, v, blk, n_sink, n_local, scale=0.4)
    np.testing.assert_allclose(o, o_bf, atol=1e-11)
    np.testing.assert_allclose(lse, lse_bf, atol=1e-11)


def test_brute_force_block128_two_windows():
    rng = np.random.default_rng(11)
    L = 1300
    q = to_bf16_bits(rng.standard_normal((1, 1, L, 64)))
    k = to_bf16_bits(rng.standard_normal((1, 1, L, 64)))
    v = to_bf16_bits(rng.standard_normal((1, 1, L, 64)))
    o, lse = orc.prefill(q, k, v, scale=0.125)
    o_bf, lse_bf = orc.brute_force_prefill(q, k, v, scale=0.125)
    np.testing.assert_allclose(o, o_bf, atol=1e-11)
    np.testing.assert_allclose(lse, lse_bf, atol=1e-11)


def test_bf16_inputs_are_widened_exactly():
    rng = np.random.default_rng(7)
    bits = [to_bf16_bits(rng.standard_normal((1, 2, 150, 16))) for _ in range(3)]
    wide = [orc.bf16_bits_to_f64(b) for b in bits]
    o1, l1 = orc.prefill(*bits, blk=16, n_sink=1, n_local=2, scale=0.25)
    o2, l2 = orc.prefill(*wide, blk=16, n_sink=1, n_local=2, scale=0.25)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # and the widening itself: bf16 1.5 = 0x3FC0, -2 = 0xC000
    assert orc.bf16_bits_to_f64(np.array([0x3FC0, 0xC000], np.uint16)).tolist() == [1.5, -2.0]


def test_row_subset_matches_full():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((2, 3, 90, 8)) for _ in range(3))
    o, lse = orc.prefill(q, k, v, blk=8, n_sink=1, n_local=2)
    rows = np.array([0, 5, 89, 90, 270, 539])
    os_, ls_ = orc.prefill(q, k, v, blk=8, n_sink=1, n_local=2, rows=rows)
    np.testing.assert_array_equal(os_, o.reshape(-1, 8)[rows])
    np.testing.assert_array_equal(ls_, lse.reshape(-1)[rows])


# ------------------------------------------------------------------- varlen

def test_varlen_equals_per_sequence_prefill():
    rng = np.random.default_rng(9)
    lens = [37, 1, 64, 100, 16]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H, total = 2, int(cu[-1])
    q, k = (rng.standard_normal((H, total, 12)) for _ in range(2))
    v = rng.standard_normal((H, total, 6))
    o, lse = orc.prefill_varlen(q, k, v, cu, blk=8, n_sink=1, n_local=3, scale=0.3)
    for s, n in enumerate(lens):
        a, b = cu[s], cu[s + 1]
        o_s, l_s = orc.prefill(q[None, :, a:b], k[None, :, a:b], v[None, :, a:b], blk=8,
                               n_sink=1, n_local=3, scale=0.3)
        np.testing.assert_array_equal(o[:, a:b], o_s[0])
        np.testing.assert_array_equal(lse[:, a:b], l_s[0])


def test_varlen_short_sequences_equal_causal():
    rng = np.random.default_rng(10)
    lens = [1024, 300, 1]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v = (to_bf16_bits(rng.standard_normal((1, int(cu[-1]), 32))) for _ in range(3))
    o, lse = orc.prefill_varlen(q, k, v, cu, scale=0.2)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        o_c, l_c = orc.causal_attention(q[:, a:b], k[:, a:b], v[:, a:b], scale=0.2)
        np.testing.assert_allclose(o[:, a:b], o_c, atol=1e-11)
        np.testing.assert_allclose(lse[:, a:b], l_c, atol=1e-11)


# ------------------------------------------------------------------- decode

def _decode_case(seed, seq_lens, Hq=4, dqk=24, dv=16, ps=8, permute=True):
    rng = np.random.default_rng(seed)
    pages = [-(-n // ps) for n in seq_lens]
    n_pages = sum(pages) + 3          # a few pages nobody references
    perm = rng.permutation(n_pages) if permute else np.arange(n_pages)
    table = np.full((len(seq_lens), max(pages) + 2), -1, np.int32)
    off = 0
    for b, n in enumerate(pages):
        table[b, :n] = perm[off:off + n]
        off += n
    kv = rng.standard_normal((n_pages, ps, dqk))
    q = rng.standard_normal((len(seq_lens), Hq, dqk))
    return q, kv, table, np.array(seq_lens, np.int32)


def test_decode_matches_brute_force():
    q, kv, pt, sl = _decode_case(1, [1, 8, 9, 61, 100])
    o, lse = orc.decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3, scale=0.3)
    o_bf, lse_bf = orc.brute_force_decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=1,
                                          n_local=3, scale=0.3)
    np.testing.assert_allclose(o, o_bf, atol=1e-11)
    np.testing.assert_allclose(lse, lse_bf, atol=1e-11)


def test_decode_page_permutation_invariant():
    lens = [5, 40, 77]
    q, kv_a, pt_a, sl = _decode_case(2, lens, permute=False)
    # move every page to a new physical slot and rewrite the table to match
    rng = np.random.default_rng(99)
    perm = rng.permutation(kv_a.shape[0])
    kv_b = np.empty_like(kv_a)
    kv_b[perm] = kv_a
    pt_b = np.where(pt_a >= 0, perm[np.maximum(pt_a, 0)], -1).astype(np.int32)
    a = orc.decode(q, kv_a, pt_a, sl, dv=16, page_size=8, n_sink=1, n_local=2)
    b = orc.decode(q, kv_b, pt_b, sl, dv=16, page_size=8, n_sink=1, n_local=2)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_decode_equals_prefill_last_row():
    lens = [70, 33]
    q, kv, pt, sl = _decode_case(3, lens, Hq=3)
    o, lse = orc.decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=2, n_local=3, scale=0.2)
    for b, n in enumerate(lens):
        logical = np.arange(n)
        rows = kv.reshape(-1, kv.shape[-1])[pt[b][logical // 8] * 8 + logical % 8]
        for h in range(3):
            qq = np.zeros((1, 1, n, rows.shape[1]))
            qq[0, 0, n - 1] = q[b, h]
            o_p, l_p = orc.prefill(qq, rows[None, None], rows[None, None, :, :16], blk=8,
                                   n_sink=2, n_local=3, scale=0.2, rows=np.array([n - 1]))
            np.testing.assert_allclose(o[b, h], o_p[0], atol=1e-12)
            assert abs(lse[b, h] - l_p[0]) < 1e-12


def test_decode_rejects_bad_page_id():
    q, kv, pt, sl = _decode_case(4, [20])
    pt[0, 1] = kv.shape[0]          # out of range
    with pytest.raises(ValueError):
        orc.decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)


# --- decode over the window plus selected pages (LongCat sparse-attention
# article, 机制 1 / 机制 3: fixed sink + sliding window plus indexer-chosen pages)

def test_decode_selected_matches_brute_force():
    lens = [1, 9, 61, 100, 100]
    q, kv, pt, sl = _decode_case(11, lens)
    # per sequence: chosen pages with negatives, duplicates, pages already in
    # the window, pages past the query's page
    extra = np.array([[-1, -1, -1, -1, -1],
                      [0, 0, 1, -1, 5],
                      [2, 2, 3, 7, -4],
                      [1, 4, 4, 11, 12],
                      [3, -1, 6, 2, 9]], np.int32)
    o, lse = orc.decode_selected(q, kv, pt, sl, extra, dv=16, page_size=8, n_sink=1, n_local=3,
                                 scale=0.3)
    o_bf, lse_bf = orc.brute_force_decode_selected(q, kv, pt, sl, extra, dv=16, page_size=8,
                                                   n_sink=1, n_local=3, scale=0.3)
    np.testing.assert_allclose(o, o_bf, atol=1e-11)
    np.testing.assert_allclose(lse, lse_bf, atol=1e-11)


def test_decode_selected_with_every_page_is_causal_attention():
    """Listing every page between the sinks and the window turns the key set
    into all keys j <= t: textbook causal attention of the last row."""
    lens = [77, 40]
    q, kv, pt, sl = _decode_case(12, lens, Hq=3)
    extra = np.full((2, 10), -1, np.int32)
    for b, n in enumerate(lens):
        pages = list(range(-(-n // 8)))
        extra[b, :len(pages)] = pages
    o, lse = orc.decode_selected(q, kv, pt, sl, extra, dv=16, page_size=8, n_sink=1, n_local=2,
                                 scale=0.25)
    for b, n in enumerate(lens):
        logical = np.arange(n)
        rows = kv.reshape(-1, kv.shape[-1])[pt[b][logical // 8] * 8 + logical % 8]
        for h in range(3):
            qq = np.zeros((n, rows.shape[1]))
            qq[n - 1] = q[b, h]
            ref_o, ref_lse = orc.causal_attention(qq, rows, rows[:, :16], scale=0.25)
            np.testing.assert_allclose(o[b, h], ref_o[-1], atol=1e-12)
            np.testing.assert_allclose(lse[b, h], ref_lse[-1], atol=1e-12)


def test_decode_selected_key_count():
    """q = 0: LSE = ln |J(t)|, with |J(t)| counted from the definition: the
    window's keys plus 8 keys for every distinct listed page strictly between
    the sinks and the window."""
    lens = [100, 61]
    q, kv, pt, sl = _decode_case(13, lens)
    q[:] = 0.0
    extra = np.array([[2, 2, 5, 11, -1, 12], [1, 3, 3, 0, 6, 7]], np.int32)
    o, lse = orc.decode_selected(q, kv, pt, sl, extra, dv=16, page_size=8, n_sink=1, n_local=3)
    for b, n in enumerate(lens):
        t = n - 1
        qb = t // 8
        lo = max(1, qb - 3 + 1)                       # first local page (n_sink = 1, n_local = 3)
        window = min(t + 1, 8) + sum(min(8, t - 8 * p + 1) for p in range(lo, qb + 1) if p >= 1)
        chosen = {int(e) for e in extra[b] if 1 <= e < lo}
        np.testing.assert_allclose(lse[b], np.log(window + 8 * len(chosen)), atol=1e-12)


def test_decode_selected_without_pages_is_decode():
    q, kv, pt, sl = _decode_case(14, [33, 90])
    extra = np.full((2, 4), -1, np.int32)
    a = orc.decode_selected(q, kv, pt, sl, extra, dv=16, page_size=8, n_sink=1, n_local=3)
    b = orc.decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# --- decode over an FP8 (e4m3 + per-token scale) latent cache


def test_e4m3_known_values():
    v = orc.e4m3_to_f64(np.array([0x00, 0x80, 0x38, 0x7E, 0x01, 0x07, 0x08, 0xC8, 0x3C, 0x77,
                                  0x7F, 0xFF], np.uint8))
    np.testing.assert_array_equal(v[:10], [0.0, -0.0, 1.0, 448.0, 2.0 ** -9, 7 * 2.0 ** -9,
                                           2.0 ** -6, -4.0, 1.5, 240.0])
    assert np.isnan(v[10]) and np.isnan(v[11])


def test_e4m3_matches_torch_float8():
    torch = pytest.importorskip("torch")
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.e4m3_to_f64(codes), ref)


def _fp8_case(seed, seq_lens, Hq=4, dqk=24, ps=8):
    q, kv, pt, sl = _decode_case(seed, seq_lens, Hq=Hq, dqk=dqk, ps=ps)
    rng = np.random.default_rng(seed + 50)
    kv8 = rng.integers(0, 256, size=kv.shape, dtype=np.uint8)
    kv8[(kv8 & 0x7F) == 0x7F] = 0x3C          # no NaN codes
    kv_scale = np.exp(rng.uniform(-4, 4, size=kv.shape[:2]))
    return q, kv8, kv_scale, pt, sl


def test_decode_fp8_matches_brute_force_on_dequantized_cache():
    q, kv8, ksc, pt, sl = _fp8_case(31, [1, 9, 61, 100])
    o, lse = orc.decode_fp8(q, kv8, ksc, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3,
                            scale=0.02)
    kv = orc.e4m3_to_f64(kv8) * ksc[..., None]
    o_bf, lse_bf = orc.brute_force_decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=1,
                                          n_local=3, scale=0.02)
    np.testing.assert_allclose(o, o_bf, rtol=1e-11, atol=1e-9)
    np.testing.assert_allclose(lse, lse_bf, atol=1e-10)


def test_decode_fp8_unit_scales_equal_bf16_decode():
    """Scales of 1: the e4m3 values are exact in bf16, so the decode over the
    bf16 bit patterns of the same values (C oracle, bf16 input path) agrees."""
    torch = pytest.importorskip("torch")
    q, kv8, _, pt, sl = _fp8_case(32, [40, 77])
    ones = np.ones(kv8.shape[:2])
    vals = torch.from_numpy(kv8).view(torch.float8_e4m3fn).to(torch.bfloat16)
    kv_bits = vals.view(torch.int16).numpy().view(np.uint16)
    q_bits = torch.from_numpy(q).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    a = orc.decode_fp8(q_bits, kv8, ones, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)
    b = orc.decode(q_bits, kv_bits, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], atol=1e-13)


def test_decode_fp8_scale_moves_between_cache_and_query():
    """Doubling every token's scale doubles K_j and V_j; halving the attention
    scale as well leaves every score, so the weights and the LSE are unchanged
    and O, a weighted mean of the V_j, doubles."""
    q, kv8, ksc, pt, sl = _fp8_case(33, [70, 33])
    o1, l1 = orc.decode_fp8(q, kv8, ksc, pt, sl, dv=16, page_size=8, scale=0.02)
    o2, l2 = orc.decode_fp8(q, kv8, 2 * ksc, pt, sl, dv=16, page_size=8, scale=0.01)
    np.testing.assert_allclose(o2, 2 * o1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l2, l1, atol=1e-12)


def test_decode_fp8_rejects_nan_codes():
    q, kv8, ksc, pt, sl = _fp8_case(34, [20])
    kv8[0, 0, 0] = 0x7F
    with pytest.raises(ValueError):
        orc.decode_fp8(q, kv8, ksc, pt, sl, dv=16, page_size=8)


# --- full-attention decode (the MLA layers LoZA keeps) and the layer stack


def test_decode_full_is_causal_attention_last_row():
    """Every key 0..t through the page table: the last row of textbook causal
    attention over the sequence's logical key rows."""
    lens = [1, 9, 77, 130]
    q, kv, pt, sl = _decode_case(21, lens, Hq=3)
    o, lse = orc.decode_full(q, kv, pt, sl, dv=16, page_size=8, scale=0.25)
    for b, n in enumerate(lens):
        logical = np.arange(n)
        rows = kv.reshape(-1, kv.shape[-1])[pt[b][logical // 8] * 8 + logical % 8]
        for h in range(3):
            qq = np.zeros((n, rows.shape[1]))
            qq[n - 1] = q[b, h]
            ref_o, ref_lse = orc.causal_attention(qq, rows, rows[:, :16], scale=0.25)
            np.testing.assert_allclose(o[b, h], ref_o[-1], atol=1e-12)
            np.testing.assert_allclose(lse[b, h], ref_lse[-1], atol=1e-12)


def test_decode_full_equals_ssa_decode_when_window_covers_prefix():
    """A sequence no longer than the window (n_sink + n_local pages): the SSA
    decode (C oracle) and the full decode (numpy) see the same keys."""
    lens = [8, 31, 32, 5]
    q, kv, pt, sl = _decode_case(22, lens)
    a = orc.decode_full(q, kv, pt, sl, dv=16, page_size=8, scale=0.3)
    b = orc.decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3, scale=0.3)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)


def test_decode_full_differs_from_ssa_beyond_window():
    q, kv, pt, sl = _decode_case(23, [100])
    a = orc.decode_full(q, kv, pt, sl, dv=16, page_size=8)
    b = orc.decode(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)
    assert np.abs(a[1] - b[1]).max() > 1e-3


def test_decode_full_key_count_and_mean():
    """q = 0: uniform weights over all seq_len keys, so LSE = ln(seq_len) and O
    is the mean of the value rows."""
    lens = [3, 57, 64]
    q, kv, pt, sl = _decode_case(24, lens)
    q[:] = 0.0
    o, lse = orc.decode_full(q, kv, pt, sl, dv=16, page_size=8)
    for b, n in enumerate(lens):
        np.testing.assert_allclose(lse[b], np.log(n), atol=1e-13)
        logical = np.arange(n)
        rows = kv.reshape(-1, kv.shape[-1])[pt[b][logical // 8] * 8 + logical % 8]
        for h in range(o.shape[1]):
            np.testing.assert_allclose(o[b, h], rows[:, :16].mean(axis=0), atol=1e-12)


def test_decode_full_row_subset_and_permutation():
    lens = [40, 77]
    q, kv_a, pt_a, sl = _decode_case(25, lens, permute=False)
    rng = np.random.default_rng(5)
    perm = rng.permutation(kv_a.shape[0])
    kv_b = np.empty_like(kv_a)
    kv_b[perm] = kv_a
    pt_b = np.where(pt_a >= 0, perm[np.maximum(pt_a, 0)], -1).astype(np.int32)
    o_a, l_a = orc.decode_full(q, kv_a, pt_a, sl, dv=16, page_size=8)
    rows = np.array([7, 0, 5, 2])
    o_b, l_b = orc.decode_full(q, kv_b, pt_b, sl, dv=16, page_size=8, rows=rows)
    np.testing.assert_allclose(o_b, o_a.reshape(-1, 16)[rows], atol=1e-13)
    np.testing.assert_allclose(l_b, l_a.reshape(-1)[rows], atol=1e-13)


def test_decode_layers_dispatches_per_layer():
    lens = [100, 20]
    q0, kv0, pt, sl = _decode_case(26, lens)
    q1, kv1, _, _ = _decode_case(27, lens)
    out = orc.decode_layers([(q0, kv0, True), (q1, kv1, False), (q1, kv0, True)], pt, sl, 16,
                            page_size=8, n_sink=1, n_local=3, scale=0.3)
    ref = [orc.brute_force_decode(q0, kv0, pt, sl, 16, 8, n_sink=0, n_local=64, scale=0.3),
           orc.brute_force_decode(q1, kv1, pt, sl, 16, 8, n_sink=1, n_local=3, scale=0.3),
           orc.brute_force_decode(q1, kv0, pt, sl, 16, 8, n_sink=0, n_local=64, scale=0.3)]
    for (o, lse), (o_r, l_r) in zip(out, ref):
        np.testing.assert_allclose(o, o_r, atol=1e-11)
        np.testing.assert_allclose(lse, l_r, atol=1e-11)


# --- decode with several query tokens per sequence (speculative / multi-token
# steps): token k of sequence b is the query at position seq_len - q_len + k

def _mtp_case(seed, seq_lens, q_len, Hq=2, dqk=24):
    q1, kv, pt, sl = _decode_case(seed, seq_lens, Hq=Hq, dqk=dqk)
    rng = np.random.default_rng(seed + 1000)
    q = rng.standard_normal((len(seq_lens), q_len, Hq, dqk))
    return q, kv, pt, sl


def test_decode_mtp_matches_brute_force_per_token():
    q_len = 3
    q, kv, pt, sl = _mtp_case(21, [3, 9, 17, 61, 100], q_len)
    o, lse = orc.decode_mtp(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3, scale=0.3)
    for k in range(q_len):
        # token k alone: a plain decode whose sequence ends at its position
        o_bf, lse_bf = orc.brute_force_decode(q[:, k], kv, pt, sl - q_len + k + 1, dv=16,
                                              page_size=8, n_sink=1, n_local=3, scale=0.3)
        np.testing.assert_allclose(o[:, k], o_bf, atol=1e-11)
        np.testing.assert_allclose(lse[:, k], lse_bf, atol=1e-11)


def test_decode_mtp_equals_masked_prefill_rows():
    """The q_len new tokens are the last q_len rows of a prefill over the
    gathered sequence: checked against the materialised-mask brute force."""
    q_len, n = 4, 45
    q, kv, pt, sl = _mtp_case(22, [n], q_len, Hq=2, dqk=16)
    o, lse = orc.decode_mtp(q, kv, pt, sl, dv=8, page_size=8, n_sink=2, n_local=2, scale=0.25)
    logical = np.arange(n)
    rows = kv.reshape(-1, kv.shape[-1])[pt[0][logical // 8] * 8 + logical % 8]
    for h in range(2):
        qq = np.zeros((n, 16))
        qq[n - q_len:] = q[0, :, h]
        o_p, l_p = orc.brute_force_prefill(qq, rows, rows[:, :8], blk=8, n_sink=2, n_local=2,
                                           scale=0.25)
        np.testing.assert_allclose(o[0, :, h], o_p[n - q_len:], atol=1e-12)
        np.testing.assert_allclose(lse[0, :, h], l_p[n - q_len:], atol=1e-12)


def test_decode_mtp_key_count():
    """q = 0: LSE = ln|J(t)| with |J(t)| = min(t+1, blk*(n_sink+n_local-1) + t%blk + 1)."""
    q_len = 5
    lens = [5, 16, 33, 64, 129]
    q, kv, pt, sl = _mtp_case(23, lens, q_len)
    q[:] = 0.0
    _, lse = orc.decode_mtp(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)
    for b, n in enumerate(lens):
        for k in range(q_len):
            t = n - q_len + k
            count = min(t + 1, 8 * (1 + 3 - 1) + t % 8 + 1)
            np.testing.assert_allclose(lse[b, k], np.log(count), atol=1e-12)


def test_decode_mtp_last_token_is_decode():
    q, kv, pt, sl = _mtp_case(24, [7, 50, 90], 2)
    o, lse = orc.decode_mtp(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)
    o1, lse1 = orc.decode(q[:, -1], kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)
    np.testing.assert_array_equal(o[:, -1], o1)
    np.testing.assert_array_equal(lse[:, -1], lse1)


def test_decode_mtp_rejects_short_sequence():
    q, kv, pt, sl = _mtp_case(25, [2, 40], 3)
    with pytest.raises(ValueError):
        orc.decode_mtp(q, kv, pt, sl, dv=16, page_size=8, n_sink=1, n_local=3)


# --- backward of the dense prefill (gradients of a loss with dL/dO = dout)

def _bwd_case(seed, B=1, H=2, L=13, dqk=5, dv=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, L, dqk)), rng.standard_normal((B, H, L, dqk)),
            rng.standard_normal((B, H, L, dv)), rng.standard_normal((B, H, L, dv)))


def test_prefill_bwd_matches_finite_differences():
    """Central differences of the forward oracle's loss sum(O * dout), every
    element of q, k and v (independent of the backward's formulas)."""
    q, k, v, g = _bwd_case(31)
    kw = dict(blk=4, n_sink=1, n_local=2, scale=0.7)
    dq, dk, dvv = orc.prefill_bwd(q, k, v, g, **kw)

    def loss(qq, kk, vv):
        o, _ = orc.prefill(qq, kk, vv, **kw)
        return float((o * g).sum())

    eps = 1e-5
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dvv)):
        num = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(grad, num, atol=1e-7, err_msg=f"d{name}")


def test_prefill_bwd_matches_masked_brute_force():
    for seed, (n_sink, n_local) in enumerate([(1, 3), (2, 2), (0, 1), (1, 7)]):
        q, k, v, g = _bwd_case(40 + seed, B=2, H=2, L=50, dqk=8, dv=6)
        got = orc.prefill_bwd(q, k, v, g, blk=8, n_sink=n_sink, n_local=n_local, scale=0.4)
        ref = orc.brute_force_prefill_bwd(q, k, v, g, blk=8, n_sink=n_sink, n_local=n_local,
                                          scale=0.4)
        for a, b in zip(got, ref):
            np.testing.assert_allclose(a, b, atol=1e-12)


def test_prefill_bwd_short_sequence_is_causal_autograd():
    """L <= window: SSA is causal attention, whose gradients torch autograd
    computes in float64."""
    import torch
    q, k, v, g = _bwd_case(50, B=1, H=3, L=30, dqk=7, dv=5)
    dq, dk, dvv = orc.prefill_bwd(q, k, v, g, blk=8, n_sink=1, n_local=3, scale=0.5)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    s = 0.5 * tq @ tk.transpose(-1, -2)
    causal = torch.ones(30, 30, dtype=torch.bool).tril()
    o = torch.softmax(s.masked_fill(~causal, float("-inf")), dim=-1) @ tv
    (o * torch.tensor(g)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dvv, tv.grad.numpy(), atol=1e-12)


def test_prefill_bwd_invariants():
    q, k, v, g = _bwd_case(60, B=1, H=2, L=40, dqk=6, dv=4)
    kw = dict(blk=8, n_sink=1, n_local=2, scale=0.6)
    _, dk, _ = orc.prefill_bwd(q, k, v, g, **kw)
    # each row's dS sums to zero, so dK summed over the keys of a plane is 0
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # a value row shared by every key makes O independent of the scores
    v_const = np.broadcast_to(v[:, :, :1], v.shape).copy()
    dq, dk, _ = orc.prefill_bwd(q, k, v_const, g, **kw)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)


def test_prefill_varlen_bwd_matches_per_sequence_finite_differences():
    """Packed sequences: each sequence's gradients are those of its own
    attention problem; checked by central differences of the packed forward
    oracle (keys of one sequence must not leak into another's gradients)."""
    rng = np.random.default_rng(70)
    cu = np.array([0, 9, 12, 25], np.int32)
    H, total, d = 1, 25, 3
    q, k, v, g = (rng.standard_normal((H, total, d)) for _ in range(4))
    kw = dict(blk=4, n_sink=1, n_local=2, scale=0.6)
    dq, dk, dvv = orc.prefill_varlen_bwd(q, k, v, g, cu, **kw)

    def loss(qq, kk, vv):
        o, _ = orc.prefill_varlen(qq, kk, vv, cu, **kw)
        return float((o * g).sum())

    eps = 1e-5
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dvv)):
        num = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(grad, num, atol=1e-7, err_msg=f"d{name}")
