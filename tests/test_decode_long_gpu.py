"""Decode over long windows on the GPU against the CPU oracle, through the C
ABI.  Windows of more than 16 listed pages -- wide SSA windows, and the
full-attention layers of the ZigZag stack (every page up to the query's) --
run through the long-window kernel: CTA pairs that each keep half of O in
tensor memory across many pages, the pages shared out evenly over the pairs
(a pair's run may cross from one sequence into the next), one partial per
run, merged by LSE."""
import numpy as np
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (LOZA_SSA_DEV_BAD_PAGE,
                                                      LOZA_SSA_DEV_BAD_SEQLEN, loza_ssa_decode,
                                                      loza_ssa_decode_mtp,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc
from tests.parity import assert_parity
from tests.test_decode_gpu import compact_for_oracle

pytestmark = pytest.mark.gpu

D_QK, D_V = 576, 512
SCALE = 1 / 24.0


def full_window(pt):
    """(n_sink, n_local) of a full-attention layer over this page table."""
    return 0, pt.shape[1]


def run_full(lens, H_q=128, seed=0, rows=None, max_pages=None, kv_hook=None):
    q, kv, pt, sl = synth.decode_inputs(lens, H_q, D_QK, seed=seed, device="cuda",
                                        max_pages=max_pages)
    if kv_hook is not None:
        kv_hook(kv, pt, sl)
    ns, nl = full_window(pt)
    o, lse = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=ns, n_local=nl, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    o_r, l_r = orc.decode_full(synth.bf16_bits(q), synth.bf16_bits(kv), pt.cpu().numpy(),
                               sl.cpu().numpy(), D_V, 128, SCALE, rows=rows)
    if rows is not None:
        r = torch.as_tensor(rows, device="cuda")
        return o.reshape(-1, D_V)[r], lse.reshape(-1)[r], o_r, l_r
    return o, lse, o_r, l_r


@pytest.mark.parametrize("lens", [
    [2200],                        # 18 pages: fewer pages than CTA pairs
    [1, 128, 129, 2049],           # one page, page boundary, tiny units
    [5000, 16385, 40000, 777],     # runs that cross from one sequence to the next
])
def test_full_attention_matches_oracle(lens):
    o, lse, o_r, l_r = run_full(lens, seed=len(lens))
    assert_parity(o, lse, o_r, l_r, f"full attention {lens}")


@pytest.mark.parametrize("H_q", [16, 200])
def test_full_attention_head_counts(H_q):
    """A partial head group (16 heads: the Q box's rows past H_q are zero
    fill) and two groups (200 heads: two units per sequence)."""
    o, lse, o_r, l_r = run_full([9000, 3000], H_q=H_q, seed=H_q)
    assert_parity(o, lse, o_r, l_r, f"full attention H_q={H_q}")


@pytest.mark.parametrize("n_sink,n_local", [(1, 16), (2, 30), (0, 40)])
def test_wide_ssa_windows(n_sink, n_local):
    lens = [100000, 3000, 129, 7777]
    q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=n_local, device="cuda")
    o, lse = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=n_sink, n_local=n_local, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    kv_h, pt_h, sl_h = compact_for_oracle(kv, pt, sl, n_sink, n_local)
    o_r, l_r = orc.decode(synth.bf16_bits(q), kv_h, pt_h, sl_h, D_V, 128, n_sink, n_local, SCALE)
    assert_parity(o, lse, o_r, l_r, f"window sink={n_sink} local={n_local}")


def test_many_short_sequences():
    """150 sequences of 1 to 25 pages under a 40-page window: the pairs' page
    runs cross many sequence boundaries, and some sequences fit inside one
    pair's run.  Rows sampled over all of them."""
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(1, 25 * 128, size=150)]
    rows = np.sort(rng.choice(150 * 32, size=400, replace=False))
    q, kv, pt, sl = synth.decode_inputs(lens, 32, D_QK, seed=5, device="cuda")
    o, lse = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=0, n_local=40, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    o_r, l_r = orc.decode_full(synth.bf16_bits(q), synth.bf16_bits(kv), pt.cpu().numpy(),
                               sl.cpu().numpy(), D_V, 128, SCALE, rows=rows)
    r = torch.as_tensor(rows, device="cuda")
    assert_parity(o.reshape(-1, D_V)[r], lse.reshape(-1)[r], o_r, l_r, "150 short sequences")


def test_rising_scores_rescale_the_output():
    """The rope columns of the key rows (512..575, not part of V) scaled up
    page by page, so the running max of a row keeps rising far past the
    rescale threshold (2^8) within a run: O and the row sum are rescaled in
    tensor memory many times."""
    def ramp(kv, pt, sl):
        for b in range(pt.shape[0]):
            n_pages = (int(sl[b]) + 127) // 128
            for j in range(n_pages):
                kv[int(pt[b, j]), :, D_V:] *= 1.0 + 0.5 * j
    o, lse, o_r, l_r = run_full([20000, 9000], seed=9, kv_hook=ramp)
    assert_parity(o, lse, o_r, l_r, "rising scores")


def test_multi_token_long_window():
    """Three query tokens per sequence (rows = (sequence, token)) under a
    20-page window, tokens straddling a page boundary."""
    lens = [6000, 385, 12000]
    q_len = 3
    q, kv, pt, sl = synth.decode_inputs(lens, 64, D_QK, seed=13, device="cuda")
    qm = torch.randn(len(lens), q_len, 64, D_QK, generator=torch.Generator().manual_seed(13)
                     ).to(torch.bfloat16).cuda()
    o, lse = loza_ssa_decode_mtp(qm, kv, pt, sl, D_V, n_sink=1, n_local=19, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    kv_h, pt_h, sl_h = compact_for_oracle(kv, pt, sl, 1, 19)
    o_r, l_r = orc.decode_mtp(synth.bf16_bits(qm), kv_h, pt_h, sl_h, D_V, 128, 1, 19, SCALE)
    assert_parity(o, lse, o_r, l_r, "three tokens, 20-page window")


def test_repeat_calls_are_bitwise_equal():
    q, kv, pt, sl = synth.decode_inputs([30000, 5000, 60000], 128, D_QK, seed=21, device="cuda")
    ns, nl = full_window(pt)
    a = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=ns, n_local=nl, scale=SCALE)
    b = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=ns, n_local=nl, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def compact_sequences(q, kv, pt, sl, seqs):
    """The given sequences alone, their pages copied to a small pool and the
    table renumbered (host bookkeeping for the oracle's sake)."""
    pt_h, sl_h = pt.cpu().numpy(), sl.cpu().numpy()
    pages, table = [], np.full((len(seqs), pt_h.shape[1]), -1, np.int32)
    for i, b in enumerate(seqs):
        n = (int(sl_h[b]) + 127) // 128
        table[i, :n] = np.arange(len(pages), len(pages) + n)
        pages.extend(int(x) for x in pt_h[b, :n])
    idx = torch.as_tensor(pages, device=kv.device, dtype=torch.long)
    return (synth.bf16_bits(q[list(seqs)]), synth.bf16_bits(kv[idx]), table,
            sl_h[list(seqs)])


def test_bad_pages_and_lengths_are_flagged():
    """A table entry outside the pool is flagged and its page left out (as
    the split kernel does): for full attention that is the same as a table
    without the page and a sequence 128 tokens shorter.  A seq_len past the
    table gives that sequence no keys (O = 0, LSE = -inf) and leaves the
    others untouched."""
    lens = [5000, 3000]
    q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=8, device="cuda")
    ns, nl = full_window(pt)
    loza_ssa_get_last_device_status()
    bad = pt.clone()
    bad[1, 3] = kv.shape[0] + 5
    o, lse = loza_ssa_decode(q, kv, bad, sl, D_V, n_sink=ns, n_local=nl, scale=SCALE)
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_PAGE
    pt_h, sl_h = pt.cpu().numpy(), sl.cpu().numpy()
    o_r, l_r = orc.decode_full(synth.bf16_bits(q), synth.bf16_bits(kv), pt_h, sl_h, D_V, 128,
                               SCALE, rows=np.arange(128))
    assert_parity(o[0], lse[0], o_r, l_r, "good sequence beside a bad page")
    pt_gap = pt_h.copy()
    n1 = (lens[1] + 127) // 128
    pt_gap[1, 3:n1 - 1] = pt_h[1, 4:n1]
    pt_gap[1, n1 - 1:] = -1
    sl_gap = sl_h.copy()
    sl_gap[1] -= 128
    o_r, l_r = orc.decode_full(synth.bf16_bits(q), synth.bf16_bits(kv), pt_gap, sl_gap, D_V, 128,
                               SCALE, rows=np.arange(128, 256))
    assert_parity(o[1], lse[1], o_r, l_r, "sequence with its page 3 left out")
    long_len = torch.tensor([5000, pt.shape[1] * 128 + 1], dtype=torch.int32, device="cuda")
    o2, l2 = loza_ssa_decode(q, kv, pt, long_len, D_V, n_sink=ns, n_local=nl, scale=SCALE)
    assert loza_ssa_get_last_device_status() & LOZA_SSA_DEV_BAD_SEQLEN
    good, _ = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=ns, n_local=nl, scale=SCALE)
    torch.cuda.synchronize()
    assert torch.equal(o2[0], good[0])
    assert torch.all(o2[1] == 0) and torch.all(torch.isneginf(l2[1]))


def test_full_attention_context_workload_sampled():
    """The 128K-token full-attention layer of the layer-stack workload: 32
    sequences of 131072 tokens, 128 heads, random page permutation, in the
    launch the benchmark times; 24 heads each of the first and the last
    sequence against the oracle."""
    lens = [131072] * 32
    q, kv, pt, sl = synth.decode_inputs(lens, 128, D_QK, seed=1, device="cuda")
    ns, nl = full_window(pt)
    o, lse = loza_ssa_decode(q, kv, pt, sl, D_V, n_sink=ns, n_local=nl, scale=SCALE)
    torch.cuda.synchronize()
    assert loza_ssa_get_last_device_status() == 0
    seqs = (0, 31)
    heads = np.sort(np.random.default_rng(1).choice(128, size=24, replace=False))
    q_h, kv_h, pt_h, sl_h = compact_sequences(q, kv, pt, sl, seqs)
    del kv
    rows = np.concatenate([i * 128 + heads for i in range(len(seqs))])
    o_r, l_r = orc.decode_full(q_h, kv_h, pt_h, sl_h, D_V, 128, SCALE, rows=rows)
    got_o = torch.cat([o[b, torch.as_tensor(heads, device="cuda")] for b in seqs])
    got_l = torch.cat([lse[b, torch.as_tensor(heads, device="cuda")] for b in seqs])
    assert_parity(got_o, got_l, o_r, l_r, "128K full attention, sampled heads")


@pytest.mark.parametrize("lens,max_extra,n_local", [
    ([5000, 2048, 20000, 131072], 12, 7),   # 8 window pages + 12 chosen: 20 listed
    ([3000, 70000, 129], 10, 12),
])
def test_chosen_pages_on_the_long_path(lens, max_extra, n_local):
    """The window plus chosen pages (LongCat sparse-attention article, 机制 1
    and 机制 3) past 16 listed pages: the chosen pages that count (between the
    sink and the local run, each once; junk entries skipped) follow the
    window's in each row's list."""
    from tests.test_decode_selected_gpu import random_extra, run as selected_run
    extra = random_extra(lens, max_extra, seed=max_extra + n_local)
    *_, o, lse, o_ref, lse_ref = selected_run(lens, extra, seed=len(lens), n_local=n_local)
    assert_parity(o, lse, o_ref, lse_ref, f"chosen pages {lens} x {max_extra}, local {n_local}")
