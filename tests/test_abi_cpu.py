"""The C ABI on a machine without a GPU: the library loads, exports every
entry point include/loza_ssa.h declares, and rejects bad arguments with the
documented status codes before touching CUDA (no compute calls here)."""
import ctypes
import os
import re
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "loza_ssa.h")

pytestmark = pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists(
    os.path.join(ROOT, "block_sparse_streaming_ssa_b200", "libloza_ssa.so")),
    reason="neither nvcc nor a built library is available")


@pytest.fixture(scope="module")
def L():
    from block_sparse_streaming_ssa_b200 import build, loza_ssa
    build.build()
    return loza_ssa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(loza_ssa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("loza_ssa_prefill", "loza_ssa_prefill_varlen", "loza_ssa_decode",
                     "loza_ssa_decode_workspace_size", "loza_ssa_status_string",
                     "loza_ssa_get_last_device_status", "loza_ssa_debug_enumerate_tiles",
                     "loza_ssa_debug_decode_pages"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    for code in range(0, -9, -1):
        s = api.loza_ssa_status_string(code)
        assert s and s != "unknown status", code
    assert api.loza_ssa_status_string(-99) == "unknown status"
    assert api.loza_ssa_version() >= 10000


def test_decode_workspace_size(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    # one split per two window pages: B * ceil(H_q/128) * ceil((n_sink+n_local)/2) * 128
    # rows of 512 fp16 (+1 fp32 LSE), each part rounded up to 256 bytes
    rows = 32 * 1 * 4 * 128
    want = -(-rows * 512 * 2 // 256) * 256 + -(-rows * 4 // 256) * 256
    assert api.loza_ssa_decode_workspace_size(32, 128, 512, 1, 7) == want
    assert api.loza_ssa_decode_workspace_size(2, 200, 512, 1, 7) == \
        -(-2 * 2 * 4 * 128 * 1024 // 256) * 256 + -(-2 * 2 * 4 * 128 * 4 // 256) * 256
    assert api.loza_ssa_decode_workspace_size(2, 128, 512, 1, 6) == \
        api.loza_ssa_decode_workspace_size(2, 128, 512, 1, 7)        # 7 pages: 4 splits
    assert api.loza_ssa_decode_workspace_size(32, 128, 256, 1, 7) == 0      # d_v unsupported
    assert api.loza_ssa_decode_workspace_size(32, 128, 512, 1, 0) == 0      # n_local < 1


def test_decode_workspace_size_long_window(L):
    """Windows of more than 16 pages run through the long-window kernel for a
    bf16 cache and the split kernel for an FP8 one (same size query): the
    size covers both.  Long-window kernel: one partial slot per (row, head
    group) unit plus one per CTA pair (at most 128 pairs), 128 rows of 512
    fp16 and 128 fp32 LSEs each, and the plan's 3 * units + 1 ints; each part
    rounded up to 256 bytes."""
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    up = lambda x: -(-x // 256) * 256

    def split(B, hg, window):
        rows = B * hg * -(-window // 2) * 128
        return up(rows * 1024) + up(rows * 4)

    def long(B, hg):
        units = B * hg
        slots = units + 128
        return up(slots * 128 * 1024) + up(slots * 128 * 4) + up((3 * units + 1) * 4)

    # a short sequence batch: the long kernel's slots dominate
    assert api.loza_ssa_decode_workspace_size(1, 128, 512, 0, 20) == max(split(1, 1, 20), long(1, 1))
    assert api.loza_ssa_decode_workspace_size(1, 128, 512, 0, 20) == 16974592
    # a full-attention layer at 128K: the FP8 split kernel's 512 splits dominate
    assert api.loza_ssa_decode_workspace_size(32, 128, 512, 0, 1024) == split(32, 1, 1024)
    assert api.loza_ssa_decode_workspace_size(3, 200, 512, 2, 30) == \
        max(split(3, 2, 32), long(3, 2))
    # 16 pages: the split kernel alone
    assert api.loza_ssa_decode_workspace_size(1, 128, 512, 1, 15) == split(1, 1, 16)


def test_decode_selected_workspace_size(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    # one split per two listed pages: window 8 + 8 chosen pages -> 8 splits
    rows = 32 * 1 * 8 * 128
    want = -(-rows * 512 * 2 // 256) * 256 + -(-rows * 4 // 256) * 256
    assert api.loza_ssa_decode_selected_workspace_size(32, 128, 512, 1, 7, 8) == want
    assert api.loza_ssa_decode_selected_workspace_size(32, 128, 512, 1, 7, 0) == \
        api.loza_ssa_decode_workspace_size(32, 128, 512, 1, 7)
    assert api.loza_ssa_decode_selected_workspace_size(32, 128, 512, 1, 7, -1) == 0
    assert api.loza_ssa_decode_selected_workspace_size(32, 128, 512, 1, 7, 4089) == 0


def test_decode_mtp_workspace_size(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    # q_len tokens per sequence: the workspace of B * q_len one-token rows
    assert api.loza_ssa_decode_mtp_workspace_size(32, 2, 128, 512, 1, 7) == \
        api.loza_ssa_decode_workspace_size(64, 128, 512, 1, 7)
    assert api.loza_ssa_decode_mtp_workspace_size(32, 1, 128, 512, 1, 7) == \
        api.loza_ssa_decode_workspace_size(32, 128, 512, 1, 7)
    assert api.loza_ssa_decode_mtp_workspace_size(32, 0, 128, 512, 1, 7) == 0
    assert api.loza_ssa_decode_mtp_workspace_size(40000, 2, 128, 512, 1, 7) == 0


def test_decode_mtp_rejects_bad_q_len(L):
    vp = ctypes.c_void_p
    for q_len, B in ((0, 2), (2, 40000)):
        rc = L.loza_ssa_decode_mtp(vp(0x1000), vp(0x1000), vp(0x1000), vp(0x1000), q_len,
                                   vp(0x1000), vp(0x1000), B, 128, 576, 512, 128, 8, 16, 1, 7,
                                   ctypes.c_float(0.04), vp(0x1000), 1 << 30, None)
        assert rc == -2   # LOZA_SSA_ERR_SHAPE


def test_prefill_bwd_workspace_size(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    # fp32 D per row (256-byte aligned) + fp32 partial dK and dV of every sink
    # chunk: key block 0 of a 32-block sequence is seen by 32 query blocks,
    # cut into chunks of 8
    B, H, L, d = 1, 2, 4096, 128
    rows = B * H * L
    d_bytes = -(-rows * 4 // 256) * 256
    part = B * H * 4 * 128 * (d + d) * 4
    assert api.loza_ssa_prefill_bwd_workspace_size(B, H, L, d, d, 1, 7) == d_bytes + part
    # no sink blocks: no partials
    assert api.loza_ssa_prefill_bwd_workspace_size(B, H, L, d, d, 0, 7) == d_bytes
    # two sink blocks: 32 - 0 and 32 - 1 query blocks -> 4 + 4 chunks
    assert api.loza_ssa_prefill_bwd_workspace_size(B, H, L, d, d, 2, 7) == d_bytes + 2 * part
    # the MLA head dims: a partial holds dK (192 columns) and dV (128 columns)
    assert api.loza_ssa_prefill_bwd_workspace_size(B, H, L, 192, 128, 1, 7) == \
        d_bytes + B * H * 4 * 128 * (192 + 128) * 4
    # unsupported head dims / windows
    assert api.loza_ssa_prefill_bwd_workspace_size(B, H, L, 192, 192, 1, 7) == 0
    assert api.loza_ssa_prefill_bwd_workspace_size(B, H, L, 128, 64, 1, 7) == 0
    assert api.loza_ssa_prefill_bwd_workspace_size(B, H, L, 128, 128, 1, 0) == 0


def test_prefill_bwd_rejects_bad_arguments(L):
    vp = ctypes.c_void_p
    a = vp(0x1000)

    def call(B=1, H=2, Lq=1024, dqk=128, dv=128, block=128, n_sink=1, n_local=7, ptr=a,
             ws_bytes=1 << 30):
        return L.loza_ssa_prefill_bwd(ptr, a, a, a, a, a, a, a, a, B, H, Lq, dqk, dv, block, n_sink,
                                      n_local, ctypes.c_float(0.08), a, ws_bytes, None)
    assert call(ptr=None) == -1           # LOZA_SSA_ERR_NULL
    assert call(B=0) == -2                # LOZA_SSA_ERR_SHAPE
    assert call(dqk=192, dv=192) == -3    # LOZA_SSA_ERR_HEAD_DIM
    assert call(dqk=64, dv=128) == -3
    assert call(block=64) == -4           # LOZA_SSA_ERR_BLOCK
    assert call(n_local=0) == -5          # LOZA_SSA_ERR_WINDOW
    assert call(ptr=vp(0x1002)) == -6     # LOZA_SSA_ERR_ALIGN
    assert call(ws_bytes=16) == -7        # LOZA_SSA_ERR_WORKSPACE


def test_prefill_varlen_bwd_workspace_size(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    # D per row + 3 prefixes of n_seqs + 1 ints + an upper bound on the sink
    # slots: H * n_sink * ((total/128 + n_seqs + 7 n_seqs) / 8 + n_seqs)
    n, total, H, d = 3, 5000, 2, 64
    d_bytes = -(-H * total * 4 // 256) * 256
    pfx = -(-3 * (n + 1) * 4 // 256) * 256
    slots = H * 1 * ((total // 128 + n + 7 * n) // 8 + n)
    want = d_bytes + pfx + slots * 128 * (d + d) * 4
    assert api.loza_ssa_prefill_varlen_bwd_workspace_size(n, total, 4000, H, d, d, 1, 7) == want
    assert api.loza_ssa_prefill_varlen_bwd_workspace_size(n, total, 4000, H, d, d, 0, 7) == \
        d_bytes + pfx
    assert api.loza_ssa_prefill_varlen_bwd_workspace_size(4001, total, 10, H, d, d, 1, 7) == 0
    assert api.loza_ssa_prefill_varlen_bwd_workspace_size(n, total, 4000, H, 192, 128, 1, 7) == \
        d_bytes + pfx + slots * 128 * (192 + 128) * 4
    assert api.loza_ssa_prefill_varlen_bwd_workspace_size(n, total, 4000, H, 192, 192, 1, 7) == 0


def test_prefill_varlen_bwd_rejects_bad_arguments(L):
    vp = ctypes.c_void_p
    a = vp(0x1000)

    def call(n=2, total=300, H=2, d=64, dv=None, cu=a, ws_bytes=1 << 30):
        return L.loza_ssa_prefill_varlen_bwd(a, a, a, a, a, a, a, a, a, cu, n, total, 200, H, d,
                                             d if dv is None else dv, 128, 1, 7,
                                             ctypes.c_float(0.1), a, ws_bytes, None)
    assert call(cu=None) == -1            # LOZA_SSA_ERR_NULL
    assert call(n=0) == -2                # LOZA_SSA_ERR_SHAPE
    assert call(d=192) == -3              # LOZA_SSA_ERR_HEAD_DIM (192 / 192)
    assert call(d=128, dv=64) == -3
    assert call(cu=vp(0x1002)) == -6      # LOZA_SSA_ERR_ALIGN
    assert call(ws_bytes=8) == -7         # LOZA_SSA_ERR_WORKSPACE


def test_decode_selected_rejects_missing_list(L):
    vp = ctypes.c_void_p
    rc = L.loza_ssa_decode_selected(vp(0x1000), vp(0x1000), vp(0x1000), vp(0x1000), None, 4,
                                    vp(0x1000), vp(0x1000), 2, 128, 576, 512, 128, 8, 16, 1, 7,
                                    ctypes.c_float(0.04), vp(0x1000), 1 << 20, None)
    assert rc == -1   # LOZA_SSA_ERR_NULL: max_extra > 0 without a list


def _prefill(L, q=0x1000, k=0x1000, v=0x1000, o=0x1000, lse=0x1000, B=1, H=2, Ln=256, dqk=64,
             dv=64, block=128, ns=1, nl=7, scale=0.125):
    vp = ctypes.c_void_p
    return L.loza_ssa_prefill(vp(q), vp(k), vp(v), vp(o), vp(lse), B, H, Ln, dqk, dv, block, ns,
                              nl, ctypes.c_float(scale), None)


def test_prefill_argument_errors(L):
    assert _prefill(L, q=0) == -1
    assert _prefill(L, lse=0) == -1
    assert _prefill(L, Ln=0) == -2
    assert _prefill(L, B=0) == -2
    assert _prefill(L, scale=float("nan")) == -2
    assert _prefill(L, scale=float("inf")) == -2
    assert _prefill(L, dqk=96, dv=96) == -3
    assert _prefill(L, dqk=128, dv=64) == -3
    assert _prefill(L, block=64) == -4
    assert _prefill(L, ns=-1) == -5
    assert _prefill(L, nl=0) == -5
    assert _prefill(L, q=0x1008) == -6
    assert _prefill(L, lse=0x1002) == -6
    assert _prefill(L, o=0x1010) == -6      # o is written with 32-byte stores


def test_backward_outputs_need_32_byte_alignment(L):
    vp = ctypes.c_void_p
    a = vp(0x1000)
    for pos in (6, 7, 8):                   # dq, dk, dv
        ptrs = [a] * 9
        ptrs[pos] = vp(0x1010)
        assert L.loza_ssa_prefill_bwd(*ptrs, 1, 2, 1024, 128, 128, 128, 1, 7,
                                      ctypes.c_float(0.08), a, 1 << 30, None) == -6


def _decode(L, B=2, Hq=128, dqk=576, dv=512, ps=128, max_pages=16, n_pages=32, ns=1, nl=7,
            ws=0x10000, ws_bytes=1 << 30, q=0x1000, pt=0x1000):
    vp = ctypes.c_void_p
    return L.loza_ssa_decode(vp(q), vp(0x1000), vp(pt), vp(0x1000), vp(0x1000), vp(0x1000), B,
                             Hq, dqk, dv, ps, max_pages, n_pages, ns, nl, ctypes.c_float(0.04),
                             vp(ws), ws_bytes, None)


def test_decode_argument_errors(L):
    assert _decode(L, q=0) == -1
    assert _decode(L, B=0) == -2
    assert _decode(L, n_pages=0) == -2
    assert _decode(L, dqk=512) == -3
    assert _decode(L, dv=256) == -3
    assert _decode(L, ps=64) == -4
    assert _decode(L, nl=0) == -5
    assert _decode(L, ns=-1) == -5
    assert _decode(L, q=0x1004) == -6
    assert _decode(L, pt=0x1002) == -6
    assert _decode(L, ws=0) == -7
    assert _decode(L, ws_bytes=1024) == -7
    assert _decode(L, ws=0x10010) == -6


def test_prefill_host_workspace_and_errors(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    up = lambda x: -(-x // 256) * 256
    B, H, Lq = 2, 3, 1000
    want = 2 * up(B * H * Lq * 128 * 2) + 2 * up(B * H * Lq * 128 * 2) + up(B * H * Lq * 4)
    assert api.loza_ssa_prefill_host_workspace_size(B, H, Lq, 128, 128) == want
    assert api.loza_ssa_prefill_host_workspace_size(B, H, Lq, 96, 96) == 0
    vp = ctypes.c_void_p

    def call(q=0x1000, chunks=4, ws=0x10000, ws_bytes=1 << 30, dqk=128):
        return L.loza_ssa_prefill_host(vp(q), vp(0x1000), vp(0x1000), vp(0x1000), vp(0x1000),
                                       B, H, Lq, dqk, 128, 128, 1, 7, ctypes.c_float(0.09),
                                       chunks, vp(ws), ws_bytes, None)
    assert call(q=0) == -1
    assert call(ws=0) == -1
    assert call(chunks=0) == -2
    assert call(dqk=96) == -3
    assert call(ws_bytes=want - 1) == -7
    assert call(ws=0x10010) == -6


def test_decode_fp8_argument_errors(L):
    vp = ctypes.c_void_p

    def call(ksc=0x1000, kv=0x1000, dqk=576):
        return L.loza_ssa_decode_fp8(vp(0x1000), vp(kv), vp(ksc), vp(0x1000), vp(0x1000),
                                     vp(0x1000), vp(0x1000), 2, 128, dqk, 512, 128, 16, 32, 1, 7,
                                     ctypes.c_float(0.04), vp(0x10000), 1 << 30, None)

    assert call(ksc=0) == -1            # no scales
    assert call(kv=0) == -1
    assert call(dqk=512) == -3
    assert call(ksc=0x1002) == -6       # scales not 4-byte aligned
    assert call(kv=0x1008) == -6        # codes not 16-byte aligned


def test_decode_layers_workspace_size(L):
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    # SSA layers only: the SSA decode's workspace; with a full-attention layer,
    # the larger of that and a window of all max_pages pages
    assert api.loza_ssa_decode_layers_workspace_size(32, 128, 512, 1024, 1, 7, False) == \
        api.loza_ssa_decode_workspace_size(32, 128, 512, 1, 7)
    assert api.loza_ssa_decode_layers_workspace_size(32, 128, 512, 1024, 1, 7, True) == \
        api.loza_ssa_decode_workspace_size(32, 128, 512, 0, 1024)
    assert api.loza_ssa_decode_layers_workspace_size(32, 128, 512, 3, 1, 7, True) == \
        api.loza_ssa_decode_workspace_size(32, 128, 512, 1, 7)
    assert api.loza_ssa_decode_layers_workspace_size(32, 128, 512, 4097, 1, 7, True) == 0


def test_decode_layers_argument_errors(L):
    from block_sparse_streaming_ssa_b200.loza_ssa import LozaSsaDecodeLayer
    vp = ctypes.c_void_p

    def call(layers, n, max_pages=16):
        arr = (LozaSsaDecodeLayer * max(len(layers), 1))(*layers) if layers else None
        return L.loza_ssa_decode_layers(arr, n, vp(0x1000), vp(0x1000), 2, 128, 576, 512, 128,
                                        max_pages, 32, 1, 7, ctypes.c_float(0.04), vp(0x10000),
                                        1 << 30, None)

    ok = LozaSsaDecodeLayer(0x1000, 0x1000, 0x1000, 0x1000, 1)
    assert call([], 1) == -1                                              # no layer array
    assert call([ok], 0) == -2                                            # empty stack
    assert call([LozaSsaDecodeLayer(0, 0x1000, 0x1000, 0x1000, 0)], 1) == -1   # layer 0: no q
    assert call([ok], 1, max_pages=5000) == -5      # full attention over more than 4096 pages


def test_varlen_argument_errors(L):
    vp = ctypes.c_void_p
    f = ctypes.c_float(0.1)
    args = dict(n_seqs=2, total=300, maxlen=200, H=2, dqk=128, dv=128, block=128, ns=1, nl=7)

    def call(cu=0x1000, **kw):
        a = {**args, **kw}
        return L.loza_ssa_prefill_varlen(vp(0x1000), vp(0x1000), vp(0x1000), vp(0x1000),
                                          vp(0x1000), vp(cu), a["n_seqs"], a["total"],
                                          a["maxlen"], a["H"], a["dqk"], a["dv"], a["block"],
                                          a["ns"], a["nl"], f, None)
    assert call(cu=0) == -1
    assert call(n_seqs=0) == -2
    assert call(n_seqs=5000) == -2
    # d_qk = 192 keeps fewer sequence prefixes in shared memory
    assert call(n_seqs=3001, total=400000, dqk=192, dv=128) == -2
    assert call(n_seqs=3001, total=400000, dqk=192, dv=128, cu=0x1002) == -2
    assert call(n_seqs=3000, total=400000, dqk=192, dv=128, cu=0x1002) == -6
    assert call(n_seqs=4000, total=600000, cu=0x1002) == -6
    assert call(total=0) == -2
    assert call(dqk=192, dv=192) == -3
    assert call(block=256) == -4
    assert call(nl=0) == -5
    assert call(cu=0x1002) == -6


def test_debug_argument_errors(L):
    vp = ctypes.c_void_p
    assert L.loza_ssa_debug_enumerate_tiles(4, 1, 7, vp(0), vp(0x1000), 8, None) == -1
    assert L.loza_ssa_debug_enumerate_tiles(0, 1, 7, vp(0x1000), vp(0x1000), 8, None) == -2
    assert L.loza_ssa_debug_enumerate_tiles(4, 1, 0, vp(0x1000), vp(0x1000), 8, None) == -5
    assert L.loza_ssa_debug_decode_pages(vp(0x1000), vp(0x1000), 2, 8, 8, 64, 1, 7, vp(0x1000),
                                         vp(0x1000), 8, None) == -4


def test_static_scratch_limit_and_argument_order(L):
    """The workspace-free decode rejects a call that needs more split slots than
    its built-in array holds before touching CUDA, and reports argument errors
    with loza_ssa_decode's codes first (dummy non-null pointers; nothing runs)."""
    vp = ctypes.c_void_p
    a = vp(0x1000)

    def call(B=2, Hq=128, dqk=576, dv=512, ps=128, ns=1, nl=7, q=a):
        return L.loza_ssa_decode_static_scratch(q, a, a, a, a, a, B, Hq, dqk, dv, ps, 16, 64,
                                                ns, nl, ctypes.c_float(0.04), None)
    # 33 sequences x 4 splits = 132 slots > 128
    assert call(B=33) == -9                       # LOZA_SSA_ERR_SCRATCH_LIMIT
    assert call(B=2, Hq=129 * 128) == -9          # 2 x 129 head groups x 4 splits
    assert call(B=1, nl=300) == -9                # 1 x ceil(301 / 2) splits
    # over the limit and invalid as well: the argument error wins
    assert call(B=33, dv=256) == -3               # LOZA_SSA_ERR_HEAD_DIM
    assert call(B=33, dqk=512) == -3
    assert call(B=33, ps=64) == -4                # LOZA_SSA_ERR_BLOCK
    assert call(B=33, nl=0) == -5                 # LOZA_SSA_ERR_WINDOW
    assert call(B=33, q=None) == -1               # LOZA_SSA_ERR_NULL
    assert call(B=33, q=vp(0x1004)) == -6         # LOZA_SSA_ERR_ALIGN
    assert call(B=0) == -2                        # LOZA_SSA_ERR_SHAPE


def test_debug_wait_timeout_argument_errors(L):
    vp = ctypes.c_void_p
    assert L.loza_ssa_debug_wait_timeout(1000, None, None) == -1
    assert L.loza_ssa_debug_wait_timeout(0, vp(0x1000), None) == -2
    assert L.loza_ssa_debug_wait_timeout(100001, vp(0x1000), None) == -2
    assert L.loza_ssa_debug_wait_timeout(1000, vp(0x1002), None) == -6


def test_long_partition_arithmetic(L):
    """The long-window decode's split of all listed pages over CTA pairs (the
    library's own host/device arithmetic, run on the host): every pair used
    gets a non-empty run and the runs tile the page list; a unit's partial
    slots are exactly the pairs whose runs reach its pages, each slot written
    by one (unit, pair) run, inside the workspace's units + pairs slots.
    Checked against brute force: each page's owning pair by scanning the runs.
    Fewer pages than pairs, units without pages and all-empty lists included."""
    import numpy as np
    from block_sparse_streaming_ssa_b200 import loza_ssa as api
    rng = np.random.default_rng(0)
    cases = [([18], 74), ([0, 0, 0], 5), ([1, 1, 2, 17], 74), ([1024] * 32, 74),
             ([3, 0, 5, 100], 4)]
    for _ in range(300):
        n = int(rng.integers(1, 40))
        pages = [int(x) for x in rng.choice([0, 1, 2, 7, 16, 64, int(rng.integers(0, 600))], n)]
        cases.append((pages, int(rng.choice([1, 2, 3, 74, 128]))))
    for pages, launched in cases:
        start, first, count = api.loza_ssa_debug_long_partition(pages, launched)
        T = sum(pages)
        used = min(launched, max(T, 1))
        assert start[0] == 0 and start[used] == T and np.all(np.diff(start) >= 0)
        assert np.all(start[used:] == T)
        if T > 0:
            assert np.all(np.diff(start[:used + 1]) >= 1), (pages, launched)
        owner = np.searchsorted(start[:used + 1], np.arange(T), side="right") - 1
        off = np.concatenate([[0], np.cumsum(pages)])
        seen = set()
        for u, nu in enumerate(pages):
            if nu == 0:
                assert count[u] == 0
                continue
            ks = sorted(set(owner[off[u]:off[u + 1]].tolist()))
            assert ks == list(range(ks[0], ks[-1] + 1))
            assert first[u] == u + ks[0] and count[u] == len(ks), (pages, launched, u)
            for k in ks:
                slot = u + k
                assert slot not in seen and slot < len(pages) + launched
                seen.add(slot)
    assert api.lib().loza_ssa_debug_long_partition(None, 1, 1, None, None, None) == -1
    bad = np.array([-1], dtype=np.int32)
    out = np.zeros(2, dtype=np.int64)
    s = np.zeros(1, dtype=np.int32)
    assert api.lib().loza_ssa_debug_long_partition(bad.ctypes.data, 1, 1, out.ctypes.data,
                                                   s.ctypes.data, s.ctypes.data) == -2
