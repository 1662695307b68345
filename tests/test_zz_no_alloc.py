"""The decode entry point that allocates nothing (loza_ssa_decode_static_scratch).

Some callers cannot give the library device memory when they launch -- a
plugin's enqueue step inside a framework that owns every allocation, or
latency-critical code that must not call cudaMalloc for scratch space.  For
them the library keeps the decode split partials in a scratch array compiled
into the library.  These tests run that entry point through the C ABI and
check it against loza_ssa_decode (caller-provided workspace) on two calls in a
row, with the same tolerance as every parity test here; the second call sees
the scratch exactly as the first call left it.  This file is named to be
collected last.
"""
import ctypes

import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (LOZA_SSA_ERR_SCRATCH_LIMIT,
                                                      LOZA_SSA_STATIC_SCRATCH_SLOTS, lib,
                                                      loza_ssa_decode,
                                                      loza_ssa_decode_static_scratch,
                                                      loza_ssa_get_last_device_status)
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu

D_QK, D_V = 576, 512


def test_matches_workspace_decode_on_two_calls_in_a_row():
    scale = 1 / 24.0
    # first call: 32 sequences x 4 splits (8 window pages) = all 128 built-in slots
    lens_a = [4096 + 3000 * i for i in range(31)] + [100]
    # second call: fewer, shorter sequences (most slots keep the first call's data)
    lens_b = [129, 2000, 1, 777]
    for lens, seed in ((lens_a, 1), (lens_b, 2)):
        q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=seed, device="cuda")
        o_ref, lse_ref = loza_ssa_decode(q, kv, pt, sl, D_V, scale=scale)
        o, lse = loza_ssa_decode_static_scratch(q, kv, pt, sl, D_V, scale=scale)
        torch.cuda.synchronize()
        assert loza_ssa_get_last_device_status() == 0
        assert_parity(o, lse, o_ref.double().cpu().numpy(), lse_ref.double().cpu().numpy(),
                      f"static scratch, {len(lens)} sequences")


def test_rejects_more_than_the_scratch_holds():
    n = 33
    q, kv, pt, sl = synth.decode_inputs([300] * n, 128, D_QK, seed=3, device="cuda")
    o = torch.empty((n, 128, D_V), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((n, 128), dtype=torch.float32, device="cuda")
    assert n * 4 > LOZA_SSA_STATIC_SCRATCH_SLOTS
    vp = ctypes.c_void_p
    rc = lib().loza_ssa_decode_static_scratch(
        vp(q.data_ptr()), vp(kv.data_ptr()), vp(pt.data_ptr()), vp(sl.data_ptr()),
        vp(o.data_ptr()), vp(lse.data_ptr()), n, 128, D_QK, D_V, 128, pt.shape[1], kv.shape[0],
        1, 7, ctypes.c_float(1 / 24.0), vp(torch.cuda.current_stream().cuda_stream))
    assert rc == LOZA_SSA_ERR_SCRATCH_LIMIT
    assert b"split slots" in lib().loza_ssa_last_error_string()


def test_wide_window_stays_on_the_split_kernel():
    """A window of more than 16 pages: loza_ssa_decode takes the long-window
    kernel, the static-scratch call keeps the split kernel its scratch is
    sized for (2 sequences x 10 splits = 20 of the 128 slots); both match the
    oracle."""
    import numpy as np
    from oracle import ssa_oracle as orc
    from tests.test_decode_gpu import compact_for_oracle
    scale = 1 / 24.0
    lens = [5000, 20000]
    q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=4, device="cuda")
    o_s, lse_s = loza_ssa_decode_static_scratch(q, kv, pt, sl, D_V, n_sink=1, n_local=19,
                                                scale=scale)
    o_w, lse_w = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=1, n_local=19, scale=scale)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    kv_h, pt_h, sl_h = compact_for_oracle(kv, pt, sl, 1, 19)
    o_r, l_r = orc.decode(synth.bf16_bits(q), kv_h, pt_h, sl_h, D_V, 128, 1, 19, scale)
    assert_parity(o_s, lse_s, o_r, l_r, "static scratch, 20-page window")
    assert_parity(o_w, lse_w, o_r, l_r, "workspace call, 20-page window")
    assert np.isfinite(o_s.float().cpu().numpy()).all()
