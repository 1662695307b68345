"""Dense prefill from host buffers (copies inside the C call, chunked and
overlapped) against the device call and the CPU oracle, through the C ABI."""
import math

import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_get_last_device_status,
                                                      loza_ssa_prefill, loza_ssa_prefill_host)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,L,dqk,dv,n_chunks", [(2, 3, 1300, 128, 128, 4), (1, 5, 2049, 64, 64, 1),
                                                    (1, 4, 3000, 192, 128, 100)])
def test_host_call_equals_device_call(B, H, L, dqk, dv, n_chunks):
    """Each chunk is whole (batch, head) planes, so the bits match the device call."""
    q, k, v = synth.prefill_inputs(B, H, L, dqk, dv, seed=L, device="cuda")
    o_d, lse_d = loza_ssa_prefill(q, k, v, scale=1 / math.sqrt(dqk))
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    o_h, lse_h = loza_ssa_prefill_host(hq, hk, hv, scale=1 / math.sqrt(dqk), n_chunks=n_chunks)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(lse_h, lse_d.cpu())


def test_host_call_matches_oracle_and_reuses_workspace():
    """Two calls back to back on one stream with one workspace (the second
    call's uploads wait for the first call's downloads), checked against the
    oracle."""
    s = synth.TINY
    ins = [synth.prefill_inputs(s.B, s.H, s.L, s.d_qk, s.d_v, seed=sd) for sd in (0, 1)]
    from block_sparse_streaming_ssa_b200.loza_ssa import loza_ssa_prefill_host_workspace_size
    ws = torch.empty(loza_ssa_prefill_host_workspace_size(s.B, s.H, s.L, s.d_qk, s.d_v),
                     dtype=torch.uint8, device="cuda")
    outs = []
    for q, k, v in ins:
        hq, hk, hv = (t.pin_memory() for t in (q, k, v))
        outs.append(loza_ssa_prefill_host(hq, hk, hv, scale=s.scale, n_chunks=2, workspace=ws))
    torch.cuda.synchronize()
    for (q, k, v), (o, lse) in zip(ins, outs):
        o_ref, lse_ref = orc.prefill(*(synth.bf16_bits(t) for t in (q, k, v)), 128, 1, 7, s.scale)
        assert_parity(o, lse, o_ref, lse_ref, "host prefill")
