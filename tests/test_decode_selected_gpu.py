"""Paged decode over the SSA window plus per-sequence chosen pages (the
page-level selection of the LongCat sparse-attention article, 机制 1 / 机制 3)
on the GPU against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_decode, loza_ssa_decode_selected,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu

D_QK, D_V = 576, 512
SCALE = 1 / 24.0


def compact_for_oracle(kv, page_table, seq_lens, extra):
    """Copy the pages the windows (any sink <= 8, local run <= 12 pages) and the
    chosen lists can reach to the host and renumber the table (host bookkeeping;
    the oracle walks the table itself)."""
    pt = page_table.cpu().numpy()
    sl = seq_lens.cpu().numpy()
    ex = extra.cpu().numpy()
    needed = set()
    for b, n in enumerate(sl):
        last = (int(n) - 1) // 128
        reach = [p for p in range(last + 1) if p < 8 or p > last - 12]
        reach += [int(e) for e in ex[b] if 0 <= e <= last]
        for p in reach:
            needed.add(int(pt[b, p]))
    order = sorted(needed)
    remap = {p: i for i, p in enumerate(order)}
    small = np.full_like(pt, -1)
    for b in range(pt.shape[0]):
        for p in range(pt.shape[1]):
            if int(pt[b, p]) in remap:
                small[b, p] = remap[int(pt[b, p])]
    idx = torch.as_tensor(order, device=kv.device, dtype=torch.long)
    return synth.bf16_bits(kv[idx]), small, sl, ex


def random_extra(lens, max_extra, seed, junk=True):
    """Chosen pages per sequence: mostly valid ones between the sink and the
    local run, plus (junk=True) negatives, duplicates, window and future pages."""
    rng = np.random.default_rng(seed)
    ex = np.full((len(lens), max_extra), -1, np.int32)
    for b, n in enumerate(lens):
        qb = (n - 1) // 128
        for j in range(max_extra):
            if junk and rng.random() < 0.3:
                ex[b, j] = rng.choice([-1, -7, 0, qb, qb + 3, ex[b, max(j - 1, 0)]])
            elif qb >= 2:
                ex[b, j] = rng.integers(1, qb)
    return torch.as_tensor(ex, device="cuda")


def run(lens, extra, H_q=128, seed=0, n_sink=1, n_local=7, rows=None):
    q, kv, pt, sl = synth.decode_inputs(lens, H_q, D_QK, seed=seed, device="cuda")
    o, lse = loza_ssa_decode_selected(q, kv, pt, sl, extra, D_V, n_sink=n_sink, n_local=n_local,
                                      scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    kv_h, pt_h, sl_h, ex_h = compact_for_oracle(kv, pt, sl, extra)
    o_ref, lse_ref = orc.decode_selected(synth.bf16_bits(q), kv_h, pt_h, sl_h, ex_h, D_V, 128,
                                         n_sink, n_local, SCALE, rows=rows)
    if rows is not None:
        r = torch.as_tensor(rows, device="cuda")
        return q, kv, pt, sl, o.reshape(-1, D_V)[r], lse.reshape(-1)[r], o_ref, lse_ref
    return q, kv, pt, sl, o, lse, o_ref, lse_ref


@pytest.mark.parametrize("lens,max_extra", [([1, 129, 1000], 3), ([5000, 2048, 20000], 8),
                                            ([131072, 4096, 777, 3000], 5)])
def test_selected_pages_match_oracle(lens, max_extra):
    extra = random_extra(lens, max_extra, seed=max_extra)
    *_, o, lse, o_ref, lse_ref = run(lens, extra, seed=len(lens))
    assert_parity(o, lse, o_ref, lse_ref, f"selected {lens} x {max_extra}")


def test_every_page_listed_is_full_attention():
    """Listing every page between the sink and the window: the oracle's key set
    is then all keys j <= t (pinned on the CPU against causal attention)."""
    lens = [3000, 1700]
    n_pages = [(n + 127) // 128 for n in lens]
    ex = np.full((2, max(n_pages)), -1, np.int32)
    for b, npg in enumerate(n_pages):
        ex[b, :npg] = np.arange(npg)
    *_, o, lse, o_ref, lse_ref = run(lens, torch.as_tensor(ex, device="cuda"), H_q=64, seed=5)
    assert_parity(o, lse, o_ref, lse_ref, "every page")


def test_no_extra_pages_is_plain_decode_bitwise():
    lens = [5000, 300, 2049]
    q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=6, device="cuda")
    extra = torch.full((3, 6), -1, dtype=torch.int32, device="cuda")
    extra[0, 0] = 0            # a sink page: already in the window
    a = loza_ssa_decode_selected(q, kv, pt, sl, extra, D_V, scale=SCALE)
    b = loza_ssa_decode(q, kv, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_window_shapes_with_selected_pages():
    lens = [4000, 900]
    extra = random_extra(lens, 4, seed=9)
    for n_sink, n_local in ((0, 1), (2, 3)):
        *_, o, lse, o_ref, lse_ref = run(lens, extra, H_q=64, seed=9, n_sink=n_sink,
                                         n_local=n_local)
        assert_parity(o, lse, o_ref, lse_ref, f"sink={n_sink} local={n_local}")


def test_selected_full_size_sampled():
    """The 32-sequence decode workload with 8 chosen pages per sequence (24
    pages per sequence attended at most), sampled heads against the oracle."""
    s = synth.DECODE
    lens = synth.decode_seq_lens(0, s.B, s.len_lo, s.len_hi)
    extra = random_extra(lens, 8, seed=0, junk=False)
    rows = np.sort(np.random.default_rng(0).choice(s.B * s.H_q, size=256, replace=False))
    *_, o, lse, o_ref, lse_ref = run(lens, extra, H_q=s.H_q, seed=0, rows=rows)
    assert_parity(o, lse, o_ref, lse_ref, "selected full size")
