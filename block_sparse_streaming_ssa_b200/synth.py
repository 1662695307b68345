"""Seeded synthetic inputs for the SSA workloads.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the CUDA path (tests, benchmark) and the CPU oracle
(tests) take their inputs from here, so the two sides see identical bf16 values.

Workloads (all synthetic: the pages publish no dataset for this kernel):

* ``tiny``   B=1, H=2, L=2048, d=64, N(0,1) fp32 -> bf16, scale 1/8.
* ``mha``    B=1, H=32, L=32768, d=128, 0.5*N(0,1) -> bf16, scale 1/sqrt(128).
* ``mla``    B=1, H=64, L=131072, d_qk=192, d_v=128, N(0,1) -> bf16, with +2.0
             added to key channel 0 of the first two 128-token blocks (a strong
             sink), scale 1/sqrt(192).
* ``decode`` 32 sequences, 128 query heads sharing one latent KV row of 576
             (512 latent + 64 rope), d_v=512, context lengths uniform integers
             in [4096, 1048576], 128-token pages placed by a random permutation
             of the whole pool, N(0,1) -> bf16, scale 1/sqrt(576).
* ``decode`` over an FP8 cache: the same shapes; each token row N(0,1),
             quantised to e4m3 codes with one fp32 scale max|x| / 440.
* ``varlen`` 8 sequences, lengths uniform in [1024, 131072] rounded to the
             nearest multiple of 128, redrawn until the total is <= 524288,
             H=32, d=128, N(0,1) -> bf16, scale 1/sqrt(128).

fp32 draws are rounded to bf16 once (round-to-nearest-even, torch ``.to``).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

BLOCK = 128


@dataclass(frozen=True)
class PrefillSpec:
    name: str
    B: int
    H: int
    L: int
    d_qk: int
    d_v: int
    std: float = 1.0
    sink_boost: float = 0.0      # added to key channel 0 of the first sink_tokens tokens
    sink_tokens: int = 256

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)


@dataclass(frozen=True)
class DecodeSpec:
    name: str
    B: int
    H_q: int
    d_qk: int
    d_v: int
    len_lo: int
    len_hi: int
    page_size: int = BLOCK

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)


@dataclass(frozen=True)
class VarlenSpec:
    name: str
    n_seqs: int
    H: int
    d_qk: int
    d_v: int
    len_lo: int
    len_hi: int
    total_cap: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)


TINY = PrefillSpec("tiny", B=1, H=2, L=2048, d_qk=64, d_v=64)
MHA = PrefillSpec("mha", B=1, H=32, L=32768, d_qk=128, d_v=128, std=0.5)
MLA = PrefillSpec("mla", B=1, H=64, L=131072, d_qk=192, d_v=128, sink_boost=2.0)
DECODE = DecodeSpec("decode", B=32, H_q=128, d_qk=576, d_v=512, len_lo=4096, len_hi=1048576)
VARLEN = VarlenSpec("varlen", n_seqs=8, H=32, d_qk=128, d_v=128, len_lo=1024, len_hi=131072,
                    total_cap=524288)

SPECS = {s.name: s for s in (TINY, MHA, MLA, DECODE, VARLEN)}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn_bf16(shape, g, device, std=1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def prefill_inputs(B, H, L, d_qk, d_v, seed=0, device="cpu", std=1.0, sink_boost=0.0,
                   sink_tokens=256):
    """q, k: [B,H,L,d_qk] bf16; v: [B,H,L,d_v] bf16 (contiguous)."""
    g = _gen(seed, device)
    q = _randn_bf16((B, H, L, d_qk), g, device, std)
    kf = torch.randn((B, H, L, d_qk), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        kf.mul_(std)
    if sink_boost:
        kf[:, :, : min(sink_tokens, L), 0] += sink_boost
    k = kf.to(torch.bfloat16)
    del kf
    v = _randn_bf16((B, H, L, d_v), g, device, std)
    return q, k, v


def prefill_spec_inputs(spec: PrefillSpec, seed=0, device="cpu"):
    return prefill_inputs(spec.B, spec.H, spec.L, spec.d_qk, spec.d_v, seed, device, spec.std,
                          spec.sink_boost, spec.sink_tokens)


def varlen_lengths(seed=0, n_seqs=8, lo=1024, hi=131072, total_cap=524288, round_to=BLOCK):
    """Sequence lengths: uniform integers in [lo, hi], rounded to the nearest
    multiple of ``round_to`` and clipped to [lo, hi]; the whole set is redrawn
    until its sum is <= total_cap."""
    rng = np.random.default_rng(seed)
    while True:
        raw = rng.integers(lo, hi, size=n_seqs, endpoint=True)
        lens = np.clip(np.rint(raw / round_to).astype(np.int64) * round_to, lo, hi)
        if lens.sum() <= total_cap:
            return [int(x) for x in lens]


def varlen_inputs(lengths, H, d_qk, d_v, seed=0, device="cpu", std=1.0):
    """Packed tensors q, k: [H,total,d_qk]; v: [H,total,d_v]; cu_seqlens int32 [n+1]."""
    total = int(sum(lengths))
    g = _gen(seed, device)
    q = _randn_bf16((H, total, d_qk), g, device, std)
    k = _randn_bf16((H, total, d_qk), g, device, std)
    v = _randn_bf16((H, total, d_v), g, device, std)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), device=device)
    return q, k, v, cu


def decode_seq_lens(seed=0, B=32, lo=4096, hi=1048576):
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi, size=B, endpoint=True)]


def decode_page_table(seq_lens, page_size=BLOCK, seed=0, max_pages=None, permute=True):
    """Page table [B, max_pages] int32 placing every logical page of every
    sequence at a distinct physical page, by a seeded random permutation of the
    whole pool (identity order if ``permute`` is False).  Unused entries are -1.
    Returns (page_table ndarray, n_pages)."""
    pages_per = [-(-int(n) // page_size) for n in seq_lens]
    n_pages = int(sum(pages_per))
    if max_pages is None:
        max_pages = max(pages_per)
    if permute:
        perm = np.random.default_rng(seed + 1).permutation(n_pages).astype(np.int32)
    else:
        perm = np.arange(n_pages, dtype=np.int32)
    table = np.full((len(seq_lens), max_pages), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(pages_per):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, n_pages


def decode_inputs(seq_lens, H_q, d_qk, seed=0, device="cpu", page_size=BLOCK, permute=True,
                  max_pages=None, q_len=None):
    """q [B,H_q,d_qk] bf16 ([B,q_len,H_q,d_qk] when q_len is given: several
    query tokens per sequence); paged kv [n_pages,page_size,d_qk] bf16;
    page_table [B,max_pages] int32 (device tensor); seq_lens [B] int32 (device
    tensor)."""
    table, n_pages = decode_page_table(seq_lens, page_size, seed, max_pages, permute)
    g = _gen(seed, device)
    B = len(seq_lens)
    q = _randn_bf16((B, H_q, d_qk) if q_len is None else (B, q_len, H_q, d_qk), g, device)
    kv = _randn_bf16((n_pages, page_size, d_qk), g, device)
    pt = torch.from_numpy(table).to(device)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device=device)
    return q, kv, pt, sl


def decode_inputs_fp8(seq_lens, H_q, d_qk, seed=0, device="cpu", page_size=BLOCK, permute=True,
                      max_pages=None, scale_spread=0.0, chunk_pages=2048):
    """q [B,H_q,d_qk] bf16 and an FP8 page pool: kv8 [n_pages,page_size,d_qk]
    uint8 e4m3 codes with kv_scale [n_pages,page_size] fp32 per token; page
    table and seq_lens as decode_inputs.  Each token's row is drawn N(0,1)
    (times exp(U(-spread, spread)) per token when scale_spread > 0), its scale
    is max|x| / 440 and its codes are torch's round-to-nearest float8_e4m3fn
    cast of x / scale (generated ``chunk_pages`` pages at a time)."""
    table, n_pages = decode_page_table(seq_lens, page_size, seed, max_pages, permute)
    g = _gen(seed, device)
    B = len(seq_lens)
    q = _randn_bf16((B, H_q, d_qk), g, device)
    kv8 = torch.empty((n_pages, page_size, d_qk), dtype=torch.uint8, device=device)
    kv_scale = torch.empty((n_pages, page_size), dtype=torch.float32, device=device)
    for p0 in range(0, n_pages, chunk_pages):
        p1 = min(n_pages, p0 + chunk_pages)
        x = torch.randn((p1 - p0, page_size, d_qk), generator=g, device=device,
                        dtype=torch.float32)
        if scale_spread:
            u = torch.rand((p1 - p0, page_size, 1), generator=g, device=device)
            x.mul_(torch.exp((2 * u - 1) * scale_spread))
        sc = x.abs().amax(dim=-1).clamp_min(1e-30) / 440.0
        kv8[p0:p1] = (x / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
        kv_scale[p0:p1] = sc
        del x
    pt = torch.from_numpy(table).to(device)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device=device)
    return q, kv8, kv_scale, pt, sl


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host copy of a bf16 tensor's bit patterns as uint16 (for the oracle)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
