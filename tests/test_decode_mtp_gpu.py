"""Paged decode with several query tokens per sequence (speculative or
multi-token steps) on the GPU against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (LOZA_SSA_DEV_BAD_SEQLEN, loza_ssa_decode,
                                                      loza_ssa_decode_mtp,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu

D_QK, D_V = 576, 512
SCALE = 1 / 24.0


def compact_for_oracle(kv, page_table, seq_lens):
    """Copy the pages the tokens' windows can reach (any sink <= 8 pages, local
    run <= 12 pages, q_len <= 128) to the host and renumber the table."""
    pt = page_table.cpu().numpy()
    sl = seq_lens.cpu().numpy()
    needed = set()
    for b, n in enumerate(sl):
        last = (int(n) - 1) // 128
        for p in range(last + 1):
            if p < 8 or p > last - 14:
                needed.add(int(pt[b, p]))
    order = sorted(needed)
    remap = {p: i for i, p in enumerate(order)}
    small = np.full_like(pt, -1)
    for b in range(pt.shape[0]):
        for p in range(pt.shape[1]):
            if int(pt[b, p]) in remap:
                small[b, p] = remap[int(pt[b, p])]
    idx = torch.as_tensor(order, device=kv.device, dtype=torch.long)
    return synth.bf16_bits(kv[idx]), small, sl


def run(lens, q_len, H_q=128, seed=0, n_sink=1, n_local=7, rows=None):
    q, kv, pt, sl = synth.decode_inputs(lens, H_q, D_QK, seed=seed, device="cuda", q_len=q_len)
    o, lse = loza_ssa_decode_mtp(q, kv, pt, sl, D_V, n_sink=n_sink, n_local=n_local, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    kv_h, pt_h, sl_h = compact_for_oracle(kv, pt, sl)
    o_ref, lse_ref = orc.decode_mtp(synth.bf16_bits(q), kv_h, pt_h, sl_h, D_V, 128, n_sink,
                                    n_local, SCALE, rows=rows)
    if rows is not None:
        r = torch.as_tensor(rows, device="cuda")
        return q, kv, pt, sl, o.reshape(-1, D_V)[r], lse.reshape(-1)[r], o_ref, lse_ref
    return q, kv, pt, sl, o, lse, o_ref, lse_ref


@pytest.mark.parametrize("lens,q_len", [([2, 129, 1000], 2), ([4, 130, 5000, 777], 4),
                                        ([131072, 3000, 256, 257], 3), ([8, 1025, 20000], 8)])
def test_mtp_small_batches(lens, q_len):
    """Token runs that straddle a page boundary (129/130/257 with q_len >= 2),
    start at position 0 (length == q_len) and sit deep in long sequences."""
    *_, o, lse, o_ref, lse_ref = run(lens, q_len, seed=q_len)
    assert_parity(o, lse, o_ref, lse_ref, f"mtp {lens} x {q_len}")


@pytest.mark.parametrize("H_q", [16, 100, 200])
def test_mtp_head_counts(H_q):
    *_, o, lse, o_ref, lse_ref = run([3000, 640], 2, H_q=H_q, seed=H_q)
    assert_parity(o, lse, o_ref, lse_ref, f"mtp H_q={H_q}")


@pytest.mark.parametrize("n_sink,n_local", [(0, 1), (2, 3)])
def test_mtp_window_shapes(n_sink, n_local):
    *_, o, lse, o_ref, lse_ref = run([4000, 300, 2049], 3, H_q=64, seed=7, n_sink=n_sink,
                                     n_local=n_local)
    assert_parity(o, lse, o_ref, lse_ref, f"mtp sink={n_sink} local={n_local}")


def test_mtp_one_token_is_decode_bitwise():
    lens = [5000, 300, 2049]
    q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=8, device="cuda", q_len=1)
    a = loza_ssa_decode_mtp(q, kv, pt, sl, D_V, scale=SCALE)
    b = loza_ssa_decode(q[:, 0].contiguous(), kv, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(a[0][:, 0], b[0]) and torch.equal(a[1][:, 0], b[1])


def test_mtp_short_sequence_is_flagged():
    """A sequence shorter than q_len sets the status bit and its rows come out
    empty (O = 0, LSE = -inf); the other sequences are unaffected."""
    lens = [2, 3000]
    q, kv, pt, sl = synth.decode_inputs([3, 3000], 64, D_QK, seed=9, device="cuda", q_len=3)
    sl_bad = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = loza_ssa_decode_mtp(q, kv, pt, sl_bad, D_V, scale=SCALE)
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_SEQLEN
    assert torch.all(lse[0] == -float("inf")) and torch.all(o[0] == 0)
    good, _ = loza_ssa_decode_mtp(q, kv, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(o[1], good[1])


def test_mtp_full_size_sampled():
    """The 32-sequence decode workload with 2 query tokens per sequence (one
    speculative token), 256 sampled (sequence, token, head) rows."""
    s = synth.DECODE
    lens = synth.decode_seq_lens(0, s.B, s.len_lo, s.len_hi)
    rows = np.sort(np.random.default_rng(0).choice(s.B * 2 * s.H_q, size=256, replace=False))
    *_, o, lse, o_ref, lse_ref = run(lens, 2, H_q=s.H_q, seed=0, rows=rows)
    assert_parity(o, lse, o_ref, lse_ref, "mtp full size")
