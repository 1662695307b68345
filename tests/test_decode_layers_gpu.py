"""Decode through a stack of layers (the ZigZag layout of the QbitAI LoZA
article: full-attention MLA layers kept, the others SSA) on the GPU against
the CPU oracle, through the C ABI.  Full-attention layers attend to every key
of the sequence; SSA layers to the sink page plus the local pages."""
import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (LOZA_SSA_DEV_BAD_PAGE, loza_ssa_decode,
                                                      loza_ssa_decode_layers,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu

D_QK, D_V = 576, 512
SCALE = 1 / 24.0


def stack_inputs(lens, pattern, H_q=128, seed=0, max_pages=None):
    """One page table for the stack, and per layer its own query and pool."""
    q0, kv0, pt, sl = synth.decode_inputs(lens, H_q, D_QK, seed=seed, device="cuda",
                                          max_pages=max_pages)
    layers = [(q0, kv0, pattern[0])]
    for i, full in enumerate(pattern[1:], 1):
        q, kv, _, _ = synth.decode_inputs(lens, H_q, D_QK, seed=seed + 100 * i, device="cuda",
                                          max_pages=max_pages)
        layers.append((q, kv, full))
    return layers, pt, sl


def oracle_stack(layers, pt, sl, rows=None):
    host = [(synth.bf16_bits(q), synth.bf16_bits(kv), full) for q, kv, full in layers]
    return orc.decode_layers(host, pt.cpu().numpy(), sl.cpu().numpy(), D_V, 128, 1, 7, SCALE,
                             rows=rows)


@pytest.mark.parametrize("lens,pattern", [
    ([1, 129, 1000, 5000], (True, False)),
    ([20000, 777, 1025], (False, True, True, False)),
    ([128, 256, 1024, 1152, 3], (True,)),
])
def test_layer_stack_matches_oracle(lens, pattern):
    """Sequences inside one page, on page boundaries, exactly the window
    (1024 tokens), one token past it, and far beyond it."""
    layers, pt, sl = stack_inputs(lens, pattern, seed=len(lens))
    outs = loza_ssa_decode_layers(layers, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    refs = oracle_stack(layers, pt, sl)
    for i, ((o, lse), (o_r, l_r)) in enumerate(zip(outs, refs)):
        assert_parity(o, lse, o_r, l_r, f"layer {i} ({'full' if pattern[i] else 'ssa'}) {lens}")


def test_ssa_layer_in_stack_is_plain_decode():
    """An SSA layer of the stack gives exactly loza_ssa_decode's bits."""
    layers, pt, sl = stack_inputs([3000, 40000], (True, False), seed=7)
    outs = loza_ssa_decode_layers(layers, pt, sl, D_V, scale=SCALE)
    o, lse = loza_ssa_decode(layers[1][0], layers[1][1], pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(outs[1][0], o) and torch.equal(outs[1][1], lse)


def test_full_layer_long_table_sampled_rows():
    """The widest full-attention window (a 4096-page table, 2048 split CTAs
    per sequence, most of them past the sequence's end) on a 100K-token and
    a short sequence; rows sampled across both."""
    lens = [100000, 300]
    layers, pt, sl = stack_inputs(lens, (True,), H_q=128, seed=11, max_pages=4096)
    (o, lse), = loza_ssa_decode_layers(layers, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    rows = np.array([0, 1, 63, 127, 128, 200, 255])
    (o_r, l_r), = oracle_stack(layers, pt, sl, rows=rows)
    r = torch.as_tensor(rows, device="cuda")
    assert_parity(o.reshape(-1, D_V)[r], lse.reshape(-1)[r], o_r, l_r, "full, 4096-page table")


def test_full_layer_with_fewer_heads():
    """H_q = 16 (a partly filled head group) through a full layer."""
    layers, pt, sl = stack_inputs([2500, 130], (True, False), H_q=16, seed=3)
    outs = loza_ssa_decode_layers(layers, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    refs = oracle_stack(layers, pt, sl)
    for i, ((o, lse), (o_r, l_r)) in enumerate(zip(outs, refs)):
        assert_parity(o, lse, o_r, l_r, f"H_q=16 layer {i}")


def test_bad_page_in_full_layer_is_flagged():
    """A table entry outside the pool that only the full-attention layer reads
    (a middle page, outside the SSA window) flags the full layer; the SSA
    layer of the same stack and the other sequence are unaffected."""
    layers, pt, sl = stack_inputs([5000, 3000], (True, False), seed=21)
    good = loza_ssa_decode_layers(layers, pt, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    bad = pt.clone()
    bad[0, 10] = layers[0][1].shape[0] + 3            # page 10 of 40: full layer only
    outs = loza_ssa_decode_layers(layers, bad, sl, D_V, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_PAGE
    assert torch.equal(outs[0][0][1], good[0][0][1])   # full layer, other sequence
    assert torch.equal(outs[1][0], good[1][0])         # SSA layer, both sequences
