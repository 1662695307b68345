"""Paged SSA decode on the GPU against the CPU oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (LOZA_SSA_DEV_BAD_PAGE,
                                                      LOZA_SSA_DEV_BAD_SEQLEN, loza_ssa_decode,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu

D_QK, D_V = 576, 512
SCALE = 1 / 24.0


def compact_for_oracle(kv, page_table, seq_lens, n_sink=1, n_local=7):
    """Copy only the pages the windows can reach to the host and renumber the
    table (host bookkeeping: which pages to copy; the oracle still walks the
    table itself)."""
    pt = page_table.cpu().numpy()
    sl = seq_lens.cpu().numpy()
    needed = set()
    for b, n in enumerate(sl):
        last = (int(n) - 1) // 128
        for p in range(last + 1):
            if p < n_sink or p > last - n_local:
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


def run(seq_lens, H_q=128, seed=0, permute=True, n_sink=1, n_local=7, rows=None):
    q, kv, pt, sl = synth.decode_inputs(seq_lens, H_q, D_QK, seed=seed, device="cuda",
                                        permute=permute)
    o, lse = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=n_sink, n_local=n_local, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    kv_h, pt_h, sl_h = compact_for_oracle(kv, pt, sl, n_sink, n_local)
    o_ref, lse_ref = orc.decode(synth.bf16_bits(q), kv_h, pt_h, sl_h, D_V, 128, n_sink, n_local,
                                SCALE, rows=rows)
    if rows is not None:
        r = torch.as_tensor(rows, device="cuda")
        return q, kv, pt, sl, o.reshape(-1, D_V)[r], lse.reshape(-1)[r], o_ref, lse_ref
    return q, kv, pt, sl, o, lse, o_ref, lse_ref


@pytest.mark.parametrize("seq_lens", [[1], [128], [129], [1000], [1024, 1025], [5000, 1, 777],
                                      [131072, 4096, 12345]])
def test_small_batches(seq_lens):
    *_, o, lse, o_ref, lse_ref = run(seq_lens, seed=len(seq_lens))
    assert_parity(o, lse, o_ref, lse_ref, f"decode {seq_lens}")


@pytest.mark.parametrize("H_q", [1, 16, 100, 200])
def test_head_counts(H_q):
    *_, o, lse, o_ref, lse_ref = run([3000, 640], H_q=H_q, seed=H_q)
    assert_parity(o, lse, o_ref, lse_ref, f"H_q={H_q}")


@pytest.mark.parametrize("n_sink,n_local", [(0, 1), (2, 3), (1, 12)])
def test_window_shapes(n_sink, n_local):
    *_, o, lse, o_ref, lse_ref = run([4000, 300, 2049], H_q=64, seed=3, n_sink=n_sink,
                                     n_local=n_local)
    assert_parity(o, lse, o_ref, lse_ref, f"decode sink={n_sink} local={n_local}")


def test_page_permutation_is_bitwise_invisible():
    """Moving every page to another physical slot (and rewriting the table to
    match) leaves the result bit-for-bit unchanged."""
    lens = [6000, 2000, 900]
    q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=4, device="cuda", permute=False)
    perm = torch.randperm(kv.shape[0], generator=torch.Generator().manual_seed(7)).cuda()
    kv_b = torch.empty_like(kv)
    kv_b[perm] = kv
    pt_b = torch.where(pt >= 0, perm[pt.clamp(min=0).long()].int(), pt)
    o_a, l_a = loza_ssa_decode(q, kv, pt, sl, D_V, scale=SCALE)
    o_b, l_b = loza_ssa_decode(q, kv_b, pt_b, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    assert torch.equal(o_a, o_b) and torch.equal(l_a, l_b)


def test_decode_equals_gpu_prefill_last_row():
    """decode at seq_len = t+1 == prefill row t with the latent row broadcast
    to every head (q/k = the 576-wide rows, v = their first 512 entries is not
    a prefill head-dim, so compare both against the oracle's prefill row)."""
    lens = [1500]
    q, kv, pt, sl, o, lse, _, _ = run(lens, H_q=4, seed=6)
    n = lens[0]
    logical = torch.arange(n, device="cuda")
    phys = pt[0, logical // 128].long() * 128 + logical % 128
    rows = kv.reshape(-1, D_QK)[phys]
    for h in range(4):
        qq = torch.zeros((1, 1, n, D_QK), dtype=torch.bfloat16, device="cuda")
        qq[0, 0, n - 1] = q[0, h]
        o_p, l_p = orc.prefill(synth.bf16_bits(qq), synth.bf16_bits(rows[None, None]),
                               synth.bf16_bits(rows[None, None, :, :D_V]), 128, 1, 7, SCALE,
                               rows=np.array([n - 1]))
        assert_parity(o[0, h][None], lse[0, h][None], o_p, l_p, f"head {h}")


def test_bad_pages_and_lengths_are_flagged():
    q, kv, pt, sl = synth.decode_inputs([2000, 3000], 128, D_QK, seed=8, device="cuda")
    loza_ssa_get_last_device_status()
    bad = pt.clone()
    bad[1, 0] = kv.shape[0] + 5                       # sink page outside the pool
    loza_ssa_decode(q, kv, bad, sl, D_V, scale=SCALE)
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_PAGE
    long_len = torch.tensor([2000, pt.shape[1] * 128 + 1], dtype=torch.int32, device="cuda")
    o, _ = loza_ssa_decode(q, kv, pt, long_len, D_V, scale=SCALE)
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_SEQLEN
    # the valid sequence is still computed correctly
    good, _ = loza_ssa_decode(q, kv, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(o[0], good[0])


def test_decode_full_size():
    """32 sequences, lengths U[4096, 1048576], 128 heads, 576/512, random page
    permutation over the whole ~20 GB pool: every head of every sequence."""
    s = synth.DECODE
    lens = synth.decode_seq_lens(0, s.B, s.len_lo, s.len_hi)
    *_, o, lse, o_ref, lse_ref = run(lens, H_q=s.H_q, seed=0)
    assert_parity(o, lse, o_ref, lse_ref, "decode full")
