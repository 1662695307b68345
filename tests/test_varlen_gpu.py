"""Packed variable-length SSA prefill on the GPU against the CPU oracle."""
import math

import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (LOZA_SSA_DEV_BAD_CU_SEQLENS,
                                                      loza_ssa_get_last_device_status,
                                                      loza_ssa_prefill_varlen)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def run(lengths, H=2, d=128, seed=0, n_sink=1, n_local=7, dv=None, rows=None):
    dv = d if dv is None else dv
    q, k, v, cu = synth.varlen_inputs(lengths, H, d, dv, seed=seed, device="cuda")
    o, lse = loza_ssa_prefill_varlen(q, k, v, cu, max(lengths), n_sink=n_sink, n_local=n_local)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    o_ref, lse_ref = orc.prefill_varlen(*(synth.bf16_bits(t) for t in (q, k, v)),
                                        cu.cpu().numpy(), 128, n_sink, n_local, 1 / math.sqrt(d),
                                        rows=rows)
    return q, k, v, cu, o, lse, o_ref, lse_ref


@pytest.mark.parametrize("lengths", [[1], [1, 1, 1], [129, 1, 1300, 127, 128],
                                     [2048, 5, 1100, 300], [1024, 1025]])
def test_ragged_packs(lengths):
    *_, o, lse, o_ref, lse_ref = run(lengths, seed=len(lengths))
    assert_parity(o, lse, o_ref, lse_ref, f"varlen {lengths}")


def test_window_shapes_varlen():
    *_, o, lse, o_ref, lse_ref = run([900, 1700, 64], d=64, seed=3, n_sink=2, n_local=3)
    assert_parity(o, lse, o_ref, lse_ref, "varlen 2/3")


def test_sequences_up_to_1024_equal_causal():
    lengths = [1024, 700, 1, 333]
    q, k, v, cu, o, lse, _, _ = run(lengths, seed=11)
    cu_h = cu.cpu().numpy()
    for s in range(len(lengths)):
        a, b = cu_h[s], cu_h[s + 1]
        o_c, l_c = orc.causal_attention(*(synth.bf16_bits(t[:, a:b]) for t in (q, k, v)),
                                        scale=1 / math.sqrt(128))
        assert_parity(o[:, a:b], lse[:, a:b], o_c, l_c, f"seq {s} causal")


def test_varlen_equals_dense_per_sequence():
    lengths = [1500, 260]
    q, k, v, cu, o, lse, _, _ = run(lengths, seed=12)
    from block_sparse_streaming_ssa_b200.loza_ssa import loza_ssa_prefill
    cu_h = cu.cpu().numpy()
    for s in range(len(lengths)):
        a, b = cu_h[s], cu_h[s + 1]
        od, ld = loza_ssa_prefill(*(t[:, a:b].unsqueeze(0).contiguous() for t in (q, k, v)))
        torch.cuda.synchronize()
        assert torch.equal(od[0], o[:, a:b]) and torch.equal(ld[0], lse[:, a:b])


def test_bad_cu_seqlens_flagged_not_computed():
    lengths = [300, 200]
    q, k, v, cu = synth.varlen_inputs(lengths, 2, 64, 64, seed=1, device="cuda")
    bad = torch.tensor([0, 350, 300], dtype=torch.int32, device="cuda")   # decreasing
    loza_ssa_get_last_device_status()
    loza_ssa_prefill_varlen(q, k, v, bad, 350)
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_CU_SEQLENS
    short = torch.tensor([0, 300, 499], dtype=torch.int32, device="cuda")  # != total
    loza_ssa_prefill_varlen(q, k, v, short, 300)
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_CU_SEQLENS


def test_varlen_full_size_sampled():
    """8 sequences (seed-0 lengths, 360,448 tokens), H=32, d=128: whole launch on
    the GPU, oracle on sampled rows of 3 heads covering every sequence."""
    sp = synth.VARLEN
    lengths = synth.varlen_lengths(0, sp.n_seqs, sp.len_lo, sp.len_hi, sp.total_cap)
    q, k, v, cu = synth.varlen_inputs(lengths, sp.H, sp.d_qk, sp.d_v, seed=0, device="cuda")
    o, lse = loza_ssa_prefill_varlen(q, k, v, cu, max(lengths))
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    total = int(sum(lengths))
    heads = [0, 17, 31]
    cu_h = cu.cpu().numpy()
    rng = np.random.default_rng(5)
    picks = set()
    for hi in range(len(heads)):
        for s in range(len(lengths)):
            a, b = int(cu_h[s]), int(cu_h[s + 1])
            for i in (0, 127, 128, 1023, 1024, b - a - 1):
                if i < b - a:
                    picks.add(hi * total + a + i)
            picks.update((hi * total + rng.integers(a, b, size=40)).tolist())
    rows = np.array(sorted(picks), dtype=np.int64)
    hsel = torch.as_tensor(heads, device="cuda")
    o_ref, lse_ref = orc.prefill_varlen(*(synth.bf16_bits(t[hsel]) for t in (q, k, v)), cu_h,
                                        rows=rows, scale=sp.scale)
    r = torch.as_tensor(rows, device="cuda")
    assert_parity(o[hsel].reshape(-1, sp.d_v)[r], lse[hsel].reshape(-1)[r], o_ref, lse_ref,
                  "varlen sampled")


def test_most_sequences_at_mla_dims():
    """3000 packed sequences at d_qk = 192, d_v = 128 (the limit for these dims:
    the kernel keeps one work-item prefix per sequence in shared memory beside
    the 192-wide rings), lengths 1 .. 300 (one or three blocks each), every row
    of one head and a sample of the other checked against the oracle."""
    rng = np.random.default_rng(21)
    lengths = rng.integers(1, 301, size=3000).tolist()
    total = sum(lengths)
    rows = np.concatenate([np.arange(total), total + rng.choice(total, 2000, replace=False)])
    q, k, v, cu, o, lse, o_ref, lse_ref = run(lengths, H=2, d=192, dv=128, seed=21,
                                               rows=np.sort(rows))
    r = torch.as_tensor(np.sort(rows), device="cuda")
    assert_parity(o.reshape(-1, 128)[r], lse.reshape(-1)[r], o_ref, lse_ref,
                  "3000 sequences, d=192/128")
