"""Bit-exact checks of the kernels' own index work, run on the device through
the debug exports: the tile scheduler's key-block lists and the decode
kernel's (logical -> physical) page selection, against lists the oracle reads
off the mask."""
import pytest
import torch

from block_sparse_streaming_ssa_b200 import synth
from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_debug_decode_pages,
                                                      loza_ssa_debug_enumerate_tiles,
                                                      loza_ssa_get_last_device_status)
from oracle import ssa_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_sink,n_local", [(1, 7), (0, 1), (2, 3), (3, 5), (1, 1), (0, 8),
                                            (4, 4), (1, 20)])
def test_tile_lists_bit_exact(n_sink, n_local):
    nq = 48
    tiles, counts = loza_ssa_debug_enumerate_tiles(nq, n_sink, n_local)
    tiles, counts = tiles.cpu().numpy(), counts.cpu().numpy()
    blk = 8   # the block lists do not depend on the block size; 8 keeps the mask scan small
    for qb in range(nq):
        want = orc.key_blocks(qb, seq_len=nq * blk, blk=blk, n_sink=n_sink, n_local=n_local)
        assert counts[qb] == len(want), qb
        assert tiles[qb, : counts[qb]].tolist() == want, qb


def test_tile_lists_large_block_index():
    # the window for query blocks far into a 1M-token sequence
    qbs = 8192
    tiles, counts = loza_ssa_debug_enumerate_tiles(qbs)
    t = tiles.cpu().numpy()
    for qb in (7, 8, 100, 4095, 8191):
        assert t[qb].tolist() == [0] + list(range(qb - 6, qb + 1))
    assert int(counts.min()) == 1 and int(counts.max()) == 8


def test_decode_pages_bit_exact():
    s = synth.DECODE
    lens = synth.decode_seq_lens(0, s.B, s.len_lo, s.len_hi) + [1, 128, 129, 1000]
    table, n_pages = synth.decode_page_table(lens, seed=0)
    pt = torch.from_numpy(table).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    pages, counts = loza_ssa_debug_decode_pages(pt, sl, n_pages)
    assert loza_ssa_get_last_device_status() == 0
    pages, counts = pages.cpu().numpy(), counts.cpu().numpy()
    for b, n in enumerate(lens):
        last = (n - 1) // 128
        logical = orc.key_blocks(last, seq_len=n, blk=128)
        want = [int(table[b, p]) for p in logical]
        assert counts[b] == len(want)
        assert pages[b, : counts[b]].tolist() == want, b


def test_decode_pages_flag_out_of_range():
    lens = [1000, 3000]
    table, n_pages = synth.decode_page_table(lens, seed=1)
    table[1, 0] = n_pages         # the sink page of sequence 1 is outside the pool
    pt = torch.from_numpy(table).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    loza_ssa_get_last_device_status()
    pages, _ = loza_ssa_debug_decode_pages(pt, sl, n_pages)
    assert loza_ssa_get_last_device_status() & 2
    assert pages[1, 0].item() == -1
