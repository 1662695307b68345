"""Dense SSA prefill on the GPU against the CPU oracle (through the C ABI)."""
import math

import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_get_last_device_status,
                                                      loza_ssa_prefill)
from oracle import ssa_oracle as orc
from tests.parity import LSE_MAX_ABS, O_MAX_ABS, O_REL_L2, assert_parity

pytestmark = pytest.mark.gpu


def run_case(B, H, L, dqk, dv, n_sink=1, n_local=7, seed=0, std=1.0, sink_boost=0.0,
             rows=None, scale=None):
    q, k, v = synth.prefill_inputs(B, H, L, dqk, dv, seed=seed, device="cuda", std=std,
                                   sink_boost=sink_boost)
    scale = 1.0 / math.sqrt(dqk) if scale is None else scale
    o, lse = loza_ssa_prefill(q, k, v, n_sink=n_sink, n_local=n_local, scale=scale)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    qb, kb, vb = (synth.bf16_bits(t) for t in (q, k, v))
    if rows is None:
        o_ref, lse_ref = orc.prefill(qb, kb, vb, 128, n_sink, n_local, scale)
        return o, lse, o_ref, lse_ref
    o_ref, lse_ref = orc.prefill(qb, kb, vb, 128, n_sink, n_local, scale, rows=rows)
    return (o.reshape(-1, dv)[torch.as_tensor(rows, device="cuda")],
            lse.reshape(-1)[torch.as_tensor(rows, device="cuda")], o_ref, lse_ref)


def test_tiny_config_full():
    """B=1, H=2, L=2048, d=64, scale 1/8 (the small correctness workload), every row."""
    s = synth.TINY
    o, lse, o_ref, lse_ref = run_case(s.B, s.H, s.L, s.d_qk, s.d_v, scale=s.scale)
    assert_parity(o, lse, o_ref, lse_ref, "tiny")


@pytest.mark.parametrize("L", [1, 7, 127, 128, 129, 1000, 1024, 1025, 1300, 2200])
def test_ragged_lengths_d128(L):
    o, lse, o_ref, lse_ref = run_case(2, 3, L, 128, 128, seed=L)
    assert_parity(o, lse, o_ref, lse_ref, f"L={L}")


@pytest.mark.parametrize("dqk,dv", [(64, 64), (128, 128), (192, 128)])
def test_head_dims(dqk, dv):
    o, lse, o_ref, lse_ref = run_case(1, 2, 1500, dqk, dv, seed=dqk)
    assert_parity(o, lse, o_ref, lse_ref, f"d={dqk}/{dv}")


@pytest.mark.parametrize("n_sink,n_local", [(0, 1), (1, 1), (2, 3), (0, 8), (3, 5), (1, 16)])
def test_window_shapes(n_sink, n_local):
    o, lse, o_ref, lse_ref = run_case(1, 2, 2400, 64, 64, n_sink, n_local, seed=7)
    assert_parity(o, lse, o_ref, lse_ref, f"sink={n_sink} local={n_local}")


def test_short_sequences_equal_causal():
    """L <= 1024: the window covers the whole prefix, so SSA is causal attention."""
    q, k, v = synth.prefill_inputs(1, 2, 1000, 128, 128, seed=3, device="cuda")
    o, lse = loza_ssa_prefill(q, k, v)
    o_c, lse_c = orc.causal_attention(*(synth.bf16_bits(t) for t in (q, k, v)),
                                      scale=1 / math.sqrt(128))
    assert_parity(o, lse, o_c, lse_c, "causal")


@pytest.mark.parametrize("L,dqk,dv,n_local", [(3000, 128, 128, 24), (5000, 192, 128, 40),
                                               (2049, 64, 64, 100000)])
def test_full_attention_layer_is_causal(L, dqk, dv, n_local):
    """A full-attention layer of the ZigZag stack: no sink and a window of at
    least every block (n_local >= ceil(L/128), far more in the last case) is
    textbook causal attention over the whole prefix."""
    q, k, v = synth.prefill_inputs(1, 2, L, dqk, dv, seed=L, device="cuda")
    o, lse = loza_ssa_prefill(q, k, v, n_sink=0, n_local=n_local, scale=1 / math.sqrt(dqk))
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    o_c, lse_c = orc.causal_attention(*(synth.bf16_bits(t) for t in (q, k, v)),
                                      scale=1 / math.sqrt(dqk))
    assert_parity(o, lse, o_c, lse_c, f"full attention L={L} d={dqk}/{dv}")


def test_full_attention_layer_long_sampled():
    """Full attention at L = 32768 (256 key tiles for the last query block),
    sampled rows against the C oracle with the same all-covering window."""
    rng = np.random.default_rng(4)
    rows = np.sort(np.concatenate([rng.choice(2 * 32768, 600, replace=False),
                                   [0, 32767, 32768, 65535]]))
    o, lse, o_ref, lse_ref = run_case(1, 2, 32768, 128, 128, n_sink=0, n_local=256, seed=9,
                                      std=0.5, rows=rows)
    assert_parity(o, lse, o_ref, lse_ref, "full attention L=32768 sampled")


def test_strong_sink_and_large_scores():
    """Keys with a +2 mean on one channel in the first two blocks, and a large
    scale, push the running max around (exercises the O rescale path)."""
    o, lse, o_ref, lse_ref = run_case(1, 2, 2048, 192, 128, seed=5, sink_boost=2.0, scale=0.5)
    assert_parity(o, lse, o_ref, lse_ref, "sink/rescale")


def test_rescale_path_extreme_max_jump():
    """A later tile whose scores exceed the earlier max by far more than the
    lazy-rescale threshold forces every row through the O correction."""
    q, k, v = synth.prefill_inputs(1, 1, 1024, 64, 64, seed=9, device="cuda")
    k[:, :, 900:, :] *= 8          # keys of the last blocks dominate
    q = q * 2
    o, lse = loza_ssa_prefill(q.contiguous(), k.contiguous(), v, scale=0.3)
    o_ref, lse_ref = orc.prefill(*(synth.bf16_bits(t) for t in (q, k, v)), scale=0.3)
    assert_parity(o, lse, o_ref, lse_ref, "max jump")


def test_outputs_do_not_touch_neighbours():
    """Rows past L in the last block are never written (ragged tail)."""
    B, H, L, d = 1, 2, 200, 64
    q, k, v = synth.prefill_inputs(B, H, L, d, d, seed=2, device="cuda")
    o = torch.full((B * H * L + 64, d), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B * H * L + 64,), 7.0, dtype=torch.float32, device="cuda")
    loza_ssa_prefill(q, k, v, o=o[: B * H * L].view(B, H, L, d), lse=lse[: B * H * L].view(B, H, L))
    torch.cuda.synchronize()
    assert torch.all(o[B * H * L:] == 7.0) and torch.all(lse[B * H * L:] == 7.0)


def test_repeatable_bitwise():
    q, k, v = synth.prefill_inputs(1, 4, 3000, 128, 128, seed=4, device="cuda")
    o1, l1 = loza_ssa_prefill(q, k, v)
    o2, l2 = loza_ssa_prefill(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def run_full_size_sampled(spec, heads, n_rows, seed):
    """Whole workload on the GPU in the benchmark's launch; the oracle checks
    sampled rows of a few heads (random rows plus every block boundary the
    window geometry cares about, and the last rows)."""
    q, k, v = synth.prefill_spec_inputs(spec, seed=0, device="cuda")
    o, lse = loza_ssa_prefill(q, k, v, scale=spec.scale)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    L = spec.L
    rng = np.random.default_rng(seed)
    picks = set(rng.integers(0, len(heads) * L, size=n_rows).tolist())
    for hi in range(len(heads)):
        for i in (0, 127, 128, 895, 896, 1023, 1024, 1151, L - 129, L - 128, L - 1):
            picks.add(hi * L + i)
    rows = np.array(sorted(picks), dtype=np.int64)
    hsel = torch.as_tensor(heads, device="cuda")
    sub = [synth.bf16_bits(t[:, hsel]) for t in (q, k, v)]
    o_ref, lse_ref = orc.prefill(*sub, 128, 1, 7, spec.scale, rows=rows)
    r = torch.as_tensor(rows, device="cuda")
    o_s = o[:, hsel].reshape(-1, spec.d_v)[r]
    lse_s = lse[:, hsel].reshape(-1)[r]
    return o_s, lse_s, o_ref, lse_ref


def test_mha_full_size_every_row():
    """B=1, H=32, L=32768, d=128, 0.5*N(0,1): the benchmark's launch, every row of
    every head against the oracle (0.51 TFLOP of float64, computed four heads at
    a time; the error measures are taken over the whole output)."""
    spec = synth.MHA
    q, k, v = synth.prefill_spec_inputs(spec, seed=0, device="cuda")
    o, lse = loza_ssa_prefill(q, k, v, scale=spec.scale)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    max_abs = lse_abs = 0.0
    err2 = ref2 = 0.0
    for h0 in range(0, spec.H, 4):
        sub = [synth.bf16_bits(t[:, h0:h0 + 4]) for t in (q, k, v)]
        o_ref, lse_ref = orc.prefill(*sub, 128, 1, 7, spec.scale)
        got = o[:, h0:h0 + 4].float().cpu().numpy().astype(np.float64)
        got_lse = lse[:, h0:h0 + 4].cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all() and np.isfinite(got_lse).all()
        d = got - o_ref
        max_abs = max(max_abs, float(np.abs(d).max()))
        err2 += float((d * d).sum())
        ref2 += float((o_ref * o_ref).sum())
        lse_abs = max(lse_abs, float(np.abs(got_lse - lse_ref).max()))
    rel = (err2 / ref2) ** 0.5
    msg = f"mha every row: O max-abs {max_abs:.3e}, O rel-L2 {rel:.3e}, LSE max-abs {lse_abs:.3e}"
    assert max_abs <= O_MAX_ABS and rel <= O_REL_L2 and lse_abs <= LSE_MAX_ABS, msg


def test_mha_full_size_sampled():
    """B=1, H=32, L=32768, d=128, 0.5*N(0,1): the benchmark's launch, sampled rows."""
    o, lse, o_ref, lse_ref = run_full_size_sampled(synth.MHA, [0, 13, 31], 1500, 1)
    assert_parity(o, lse, o_ref, lse_ref, "mha sampled")


def test_mla_full_size_sampled():
    """B=1, H=64, L=131072, d_qk=192, d_v=128 with a +2 sink channel, sampled rows."""
    o, lse, o_ref, lse_ref = run_full_size_sampled(synth.MLA, [0, 37, 63], 1000, 2)
    assert_parity(o, lse, o_ref, lse_ref, "mla sampled")
