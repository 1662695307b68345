"""Paged SSA decode over an FP8 latent cache (e4m3 codes, one fp32 scale per
token) on the GPU against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (LOZA_SSA_DEV_BAD_PAGE,
                                                      LOZA_SSA_DEV_BAD_SEQLEN, loza_ssa_decode,
                                                      loza_ssa_decode_fp8,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc
from tests.parity import LSE_MAX_ABS, O_REL_L2, assert_parity, errors

pytestmark = pytest.mark.gpu

D_QK, D_V = 576, 512
SCALE = 1 / 24.0


def compact_for_oracle(kv8, kv_scale, page_table, seq_lens, n_sink, n_local):
    """Host copies of the pages the windows can reach, with the table
    renumbered to match (host bookkeeping; the oracle walks the table itself)."""
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
    idx = torch.as_tensor(order, device=kv8.device, dtype=torch.long)
    return kv8[idx].cpu().numpy(), kv_scale[idx].cpu().numpy(), small, sl


def run(lens, H_q=128, seed=0, n_sink=1, n_local=7, spread=0.0, rows=None):
    q, kv8, ksc, pt, sl = synth.decode_inputs_fp8(lens, H_q, D_QK, seed=seed, device="cuda",
                                                  scale_spread=spread)
    o, lse = loza_ssa_decode_fp8(q, kv8, ksc, pt, sl, D_V, n_sink=n_sink, n_local=n_local,
                                 scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    kv8_h, ksc_h, pt_h, sl_h = compact_for_oracle(kv8, ksc, pt, sl, n_sink, n_local)
    o_ref, lse_ref = orc.decode_fp8(synth.bf16_bits(q), kv8_h, ksc_h, pt_h, sl_h, D_V, 128,
                                    n_sink, n_local, SCALE, rows=rows)
    if rows is not None:
        r = torch.as_tensor(rows, device="cuda")
        return o.reshape(-1, D_V)[r], lse.reshape(-1)[r], o_ref, lse_ref
    return o, lse, o_ref, lse_ref


@pytest.mark.parametrize("lens", [[1, 129, 1000, 5000, 20000], [128, 256, 1024, 1025, 7]])
def test_fp8_matches_oracle(lens):
    """One-token sequences, page boundaries, exactly the window, one past it,
    long contexts."""
    o, lse, o_ref, lse_ref = run(lens, seed=len(lens))
    assert_parity(o, lse, o_ref, lse_ref, f"fp8 {lens}")


@pytest.mark.parametrize("lens", [[1, 129, 1000, 5000, 20000]])
def test_fp8_wide_scale_range(lens):
    """Token scales spread over e^-3 .. e^3, so |O| reaches ~90, where one bf16
    step of the output alone is 0.5: the max-abs error is taken relative to
    the largest |O| (1e-2 of it), the relative L2 and LSE bars are unchanged."""
    o, lse, o_ref, lse_ref = run(lens, seed=len(lens), spread=3.0)
    max_abs, rel, lse_abs = errors(o, lse, o_ref, lse_ref)
    top = float(np.abs(o_ref).max())
    msg = f"O max-abs {max_abs:.3e} (max |O| {top:.1f}), rel-L2 {rel:.3e}, LSE {lse_abs:.3e}"
    assert max_abs <= 1e-2 * top and rel <= O_REL_L2 and lse_abs <= LSE_MAX_ABS, msg


@pytest.mark.parametrize("H_q,n_sink,n_local", [(16, 1, 7), (200, 1, 7), (128, 0, 3),
                                                (64, 2, 12)])
def test_fp8_heads_and_windows(H_q, n_sink, n_local):
    o, lse, o_ref, lse_ref = run([3000, 640, 20000], H_q=H_q, seed=H_q, n_sink=n_sink,
                                 n_local=n_local)
    assert_parity(o, lse, o_ref, lse_ref, f"fp8 H_q={H_q} sink={n_sink} local={n_local}")


def test_fp8_unit_scales_bit_identical_to_bf16_cache():
    """Scales of 1: the bf16 cache holding the same (exactly representable)
    values gives the same bits through loza_ssa_decode."""
    lens = [5000, 700, 129]
    q, kv8, _, pt, sl = synth.decode_inputs_fp8(lens, 128, D_QK, seed=5, device="cuda")
    ones = torch.ones(kv8.shape[:2], dtype=torch.float32, device="cuda")
    kv_bf16 = kv8.view(torch.float8_e4m3fn).to(torch.bfloat16)
    o8, l8 = loza_ssa_decode_fp8(q, kv8, ones, pt, sl, D_V, scale=SCALE)
    o16, l16 = loza_ssa_decode(q, kv_bf16, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(o8, o16) and torch.equal(l8, l16)


def test_fp8_subnormal_codes():
    """A cache of subnormal codes only (exponent field 0: the values m/8 2^-6,
    m = 0 .. 7, both signs) with scales of 2^6, so every key is -0.875 .. 0.875:
    a conversion that flushed subnormals would give O = 0."""
    lens = [1000, 300, 5]
    q, kv8, ksc, pt, sl = synth.decode_inputs_fp8(lens, 128, D_QK, seed=8, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(8)
    sub = torch.tensor([c for c in range(256) if (c & 0x78) == 0], dtype=torch.uint8,
                       device="cuda")
    kv8.copy_(sub[torch.randint(0, sub.numel(), kv8.shape, generator=g, device="cuda")])
    ksc.fill_(2.0 ** 6)
    o, lse = loza_ssa_decode_fp8(q, kv8, ksc, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    kv8_h, ksc_h, pt_h, sl_h = compact_for_oracle(kv8, ksc, pt, sl, 1, 7)
    o_ref, lse_ref = orc.decode_fp8(synth.bf16_bits(q), kv8_h, ksc_h, pt_h, sl_h, D_V, 128, 1,
                                    7, SCALE)
    assert_parity(o, lse, o_ref, lse_ref, "fp8 subnormal codes")


def test_fp8_every_code_bit_identical_to_bf16_cache():
    """Every non-NaN code, unit scales: bit-identical to the bf16 cache holding
    the same values (torch's exact e4m3 -> bf16 conversion)."""
    lens = [1000, 300, 5]
    q, kv8, _, pt, sl = synth.decode_inputs_fp8(lens, 128, D_QK, seed=9, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(9)
    codes = torch.tensor([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=torch.uint8,
                         device="cuda")
    kv8.copy_(codes[torch.randint(0, codes.numel(), kv8.shape, generator=g, device="cuda")])
    ones = torch.ones(kv8.shape[:2], dtype=torch.float32, device="cuda")
    o8, l8 = loza_ssa_decode_fp8(q, kv8, ones, pt, sl, D_V, scale=SCALE)
    o16, l16 = loza_ssa_decode(q, kv8.view(torch.float8_e4m3fn).to(torch.bfloat16), pt, sl, D_V,
                               scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(o8, o16) and torch.equal(l8, l16)


def test_fp8_full_workload_sampled():
    """The 32-sequence workload (contexts U[4096, 1M], random page permutation
    over the whole pool) in FP8, 256 sampled head rows."""
    s = synth.DECODE
    lens = synth.decode_seq_lens(0, s.B, s.len_lo, s.len_hi)
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(s.B * s.H_q, 256, replace=False))
    o, lse, o_ref, lse_ref = run(lens, seed=0, spread=0.0, rows=rows)
    assert_parity(o, lse, o_ref, lse_ref, "fp8 full workload")


def test_fp8_bad_pages_and_lengths_are_flagged():
    """A page id outside the pool and a length past the table set their status
    bits; the other sequence's rows are unchanged."""
    q, kv8, ksc, pt, sl = synth.decode_inputs_fp8([2000, 700], 128, D_QK, seed=4, device="cuda")
    good, _ = loza_ssa_decode_fp8(q, kv8, ksc, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    bad = pt.clone()
    bad[1, 0] = kv8.shape[0] + 5                       # sink page outside the pool
    o, _ = loza_ssa_decode_fp8(q, kv8, ksc, bad, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_PAGE
    assert torch.equal(o[0], good[0])
    long_len = torch.tensor([2000, pt.shape[1] * 128 + 1], dtype=torch.int32, device="cuda")
    o, _ = loza_ssa_decode_fp8(q, kv8, ksc, pt, long_len, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_SEQLEN
    assert torch.equal(o[0], good[0])
