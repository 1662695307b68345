"""The pipelines' bounded wait, made to run out on the GPU.

Every mbarrier wait in the kernels is bounded: past its limit it sets the
CTA's abort flag and LOZA_SSA_DEV_WAIT_TIMEOUT in the device status word and
returns, so a stuck pipeline ends its CTA instead of hanging the GPU.  The
debug export runs that same wait routine with a 1 ms limit on a barrier that
nothing arrives on (no named barrier is involved: those have no limit).  The
test checks that the call returns, that the status bit is set and read back
once, that the CTA's other waits give up on the abort flag, and that a normal
call afterwards runs clean."""
import math
import time

import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_debug_wait_timeout,
                                                      loza_ssa_decode,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu

WAIT_TIMEOUT_BIT = 1


def test_wait_runs_out_and_reports():
    assert loza_ssa_get_last_device_status() == 0
    # one untimed call first: the events below bracket the launch on the host
    # too, and a first call also loads the kernel and allocates its result
    loza_ssa_debug_wait_timeout(1000)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == WAIT_TIMEOUT_BIT
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    result = loza_ssa_debug_wait_timeout(1000)
    end.record()
    t0 = time.perf_counter()
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert result.tolist() == [1, 31]
    # the kernel lasted at least the limit, and nowhere near the others' 10 ms
    assert 0.9 <= start.elapsed_time(end) < 8.0, start.elapsed_time(end)
    assert loza_ssa_get_last_device_status() == WAIT_TIMEOUT_BIT
    assert loza_ssa_get_last_device_status() == 0   # reading it cleared it


def test_normal_call_after_a_timeout_is_clean():
    loza_ssa_debug_wait_timeout(200)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == WAIT_TIMEOUT_BIT
    lens = [1500, 200]
    q, kv, pt, sl = synth.decode_inputs(lens, 128, 576, seed=3, device="cuda")
    o, lse = loza_ssa_decode(q, kv, pt, sl, 512, scale=1 / math.sqrt(576))
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    o_ref, lse_ref = orc.decode(synth.bf16_bits(q), synth.bf16_bits(kv), pt.cpu().numpy(),
                                sl.cpu().numpy(), 512, scale=1 / math.sqrt(576))
    assert_parity(o, lse, o_ref, lse_ref, "decode after a timed-out wait")
