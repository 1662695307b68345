"""Thin Python binding of libloza_ssa.so (argument marshalling only).

Every function here has the name of the C entry point it calls (see
include/loza_ssa.h) and does nothing but check that tensors are CUDA,
contiguous and of the right dtype, allocate outputs the caller did not pass,
and hand raw pointers, sizes and the current CUDA stream to the library.
All attention work runs in the library's sm_100a kernels; if the library is
missing this module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libloza_ssa.so")
_lib = None

LOZA_SSA_DEV_WAIT_TIMEOUT = 1
LOZA_SSA_DEV_BAD_PAGE = 2
LOZA_SSA_DEV_BAD_SEQLEN = 4
LOZA_SSA_DEV_BAD_CU_SEQLENS = 8
LOZA_SSA_ERR_SCRATCH_LIMIT = -9
LOZA_SSA_STATIC_SCRATCH_SLOTS = 128


class LozaSsaDecodeLayer(ctypes.Structure):
    """struct loza_ssa_decode_layer of the C header."""
    _fields_ = [("q", ctypes.c_void_p), ("paged_kv", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("lse", ctypes.c_void_p), ("full_attention", ctypes.c_int)]


class LozaSsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m block_sparse_streaming_ssa_b200.build`"
                " (there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.loza_ssa_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                       f32, vp]
        L.loza_ssa_prefill.restype = i32
        L.loza_ssa_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                              i32, i32, i32, f32, vp]
        L.loza_ssa_prefill_varlen.restype = i32
        L.loza_ssa_decode.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                      i32, i32, f32, vp, sz, vp]
        L.loza_ssa_decode.restype = i32
        L.loza_ssa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.loza_ssa_decode_workspace_size.restype = sz
        L.loza_ssa_decode_selected.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32,
                                               i32, i32, i32, i32, i32, i32, f32, vp, sz, vp]
        L.loza_ssa_decode_selected.restype = i32
        L.loza_ssa_decode_selected_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.loza_ssa_decode_selected_workspace_size.restype = sz
        L.loza_ssa_decode_mtp.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32,
                                          i32, i32, i32, i32, f32, vp, sz, vp]
        L.loza_ssa_decode_mtp.restype = i32
        L.loza_ssa_decode_mtp_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.loza_ssa_decode_mtp_workspace_size.restype = sz
        L.loza_ssa_prefill_host.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                            i32, i32, f32, i32, vp, sz, vp]
        L.loza_ssa_prefill_host.restype = i32
        L.loza_ssa_prefill_host_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.loza_ssa_prefill_host_workspace_size.restype = sz
        L.loza_ssa_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                          i32, i32, i32, i32, f32, vp, sz, vp]
        L.loza_ssa_decode_fp8.restype = i32
        L.loza_ssa_decode_layers.argtypes = [ctypes.POINTER(LozaSsaDecodeLayer), i32, vp, vp,
                                             i32, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                             vp, sz, vp]
        L.loza_ssa_decode_layers.restype = i32
        L.loza_ssa_decode_layers_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32]
        L.loza_ssa_decode_layers_workspace_size.restype = sz
        L.loza_ssa_prefill_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                           i32, i32, i32, i32, f32, vp, sz, vp]
        L.loza_ssa_prefill_bwd.restype = i32
        L.loza_ssa_prefill_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32]
        L.loza_ssa_prefill_bwd_workspace_size.restype = sz
        L.loza_ssa_prefill_varlen_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32,
                                                  i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                                  vp, sz, vp]
        L.loza_ssa_prefill_varlen_bwd.restype = i32
        L.loza_ssa_prefill_varlen_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32,
                                                                 i32, i32]
        L.loza_ssa_prefill_varlen_bwd_workspace_size.restype = sz
        L.loza_ssa_status_string.argtypes = [i32]
        L.loza_ssa_status_string.restype = ctypes.c_char_p
        L.loza_ssa_last_error_string.argtypes = []
        L.loza_ssa_last_error_string.restype = ctypes.c_char_p
        L.loza_ssa_get_last_device_status.argtypes = [vp]
        L.loza_ssa_get_last_device_status.restype = i32
        L.loza_ssa_debug_enumerate_tiles.argtypes = [i32, i32, i32, vp, vp, i32, vp]
        L.loza_ssa_debug_enumerate_tiles.restype = i32
        L.loza_ssa_debug_decode_pages.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp,
                                                  i32, vp]
        L.loza_ssa_debug_decode_pages.restype = i32
        L.loza_ssa_debug_wait_timeout.argtypes = [i32, vp, vp]
        L.loza_ssa_debug_wait_timeout.restype = i32
        L.loza_ssa_debug_long_partition.argtypes = [vp, i32, i32, vp, vp, vp]
        L.loza_ssa_debug_long_partition.restype = i32
        L.loza_ssa_decode_static_scratch.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                                     i32, i32, i32, i32, i32, f32, vp]
        L.loza_ssa_decode_static_scratch.restype = i32
        L.loza_ssa_version.argtypes = []
        L.loza_ssa_version.restype = i32
        _lib = L
    return _lib


def loza_ssa_status_string(status: int) -> str:
    return lib().loza_ssa_status_string(status).decode()


def loza_ssa_last_error_string() -> str:
    return lib().loza_ssa_last_error_string().decode()


def loza_ssa_version() -> int:
    return lib().loza_ssa_version()


def _check(rc: int) -> None:
    if rc != 0:
        detail = loza_ssa_last_error_string() if rc == -8 else ""
        raise LozaSsaError(rc, f"libloza_ssa: {loza_ssa_status_string(rc)} ({rc}) {detail}".strip())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def loza_ssa_prefill(q, k, v, o=None, lse=None, block=128, n_sink=1, n_local=7, scale=None,
                     stream=None):
    """Dense SSA prefill.  q, k: bf16 [B,H,L,d_qk]; v: bf16 [B,H,L,d_v].
    Returns (o bf16 [B,H,L,d_v], lse fp32 [B,H,L])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, H, L, d_qk = q.shape
    d_v = v.shape[-1]
    if tuple(k.shape) != (B, H, L, d_qk) or tuple(v.shape[:3]) != (B, H, L):
        raise ValueError("q, k, v shapes disagree")
    if o is None:
        o = torch.empty((B, H, L, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    _check(lib().loza_ssa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, L, d_qk,
                                  d_v, block, n_sink, n_local, float(scale), _stream(stream)))
    return o, lse


def _need_host(t: torch.Tensor, dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def loza_ssa_prefill_host_workspace_size(B, H, L, d_qk, d_v) -> int:
    return int(lib().loza_ssa_prefill_host_workspace_size(B, H, L, d_qk, d_v))


def loza_ssa_prefill_host(q, k, v, o=None, lse=None, block=128, n_sink=1, n_local=7, scale=None,
                          n_chunks=8, workspace=None, stream=None):
    """Dense SSA prefill from host tensors (copies inside the call, overlapped
    across chunks of (batch, head) planes).  q, k, v: CPU bf16 [B,H,L,d]
    (pinned for overlap); o, lse: CPU outputs, allocated pinned if not given;
    workspace: uint8 CUDA tensor of loza_ssa_prefill_host_workspace_size bytes.
    The outputs are complete once `stream` (default: the current one) has
    passed the call.  Returns (o, lse)."""
    _need_host(q, torch.bfloat16, "q")
    _need_host(k, torch.bfloat16, "k")
    _need_host(v, torch.bfloat16, "v")
    B, H, L, d_qk = q.shape
    d_v = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, L, d_v), dtype=torch.bfloat16).pin_memory()
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32).pin_memory()
    _need_host(o, torch.bfloat16, "o")
    _need_host(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    need = loza_ssa_prefill_host_workspace_size(B, H, L, d_qk, d_v)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_prefill_host(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, L, d_qk, d_v, block, n_sink,
        n_local, float(scale), int(n_chunks), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return o, lse


def loza_ssa_prefill_varlen(q, k, v, cu_seqlens, max_seqlen, o=None, lse=None, block=128,
                            n_sink=1, n_local=7, scale=None, stream=None):
    """Packed varlen SSA prefill.  q, k: bf16 [H,total,d_qk]; v: bf16 [H,total,d_v];
    cu_seqlens: int32 CUDA [n_seqs+1].  Returns (o [H,total,d_v], lse [H,total])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    _need(cu_seqlens, torch.int32, "cu_seqlens")
    H, total, d_qk = q.shape
    d_v = v.shape[-1]
    if o is None:
        o = torch.empty((H, total, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    n_seqs = cu_seqlens.numel() - 1
    _check(lib().loza_ssa_prefill_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens), n_seqs, total,
        int(max_seqlen), H, d_qk, d_v, block, n_sink, n_local, float(scale), _stream(stream)))
    return o, lse


def loza_ssa_prefill_bwd_workspace_size(B, H, L, d_qk, d_v, n_sink=1, n_local=7) -> int:
    return int(lib().loza_ssa_prefill_bwd_workspace_size(B, H, L, d_qk, d_v, n_sink, n_local))


def loza_ssa_prefill_bwd(q, k, v, o, lse, dout, dq=None, dk=None, dv=None, block=128, n_sink=1,
                         n_local=7, scale=None, workspace=None, stream=None):
    """Gradients of loza_ssa_prefill.  q, k: bf16 [B,H,L,d]; v, o, dout: bf16
    [B,H,L,d]; lse: fp32 [B,H,L] from the forward pass.  Returns (dq, dk, dv)."""
    for t, dt, name in ((q, torch.bfloat16, "q"), (k, torch.bfloat16, "k"),
                        (v, torch.bfloat16, "v"), (o, torch.bfloat16, "o"),
                        (lse, torch.float32, "lse"), (dout, torch.bfloat16, "dout")):
        _need(t, dt, name)
    B, H, L, d_qk = q.shape
    d_v = v.shape[-1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, torch.bfloat16, name)
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    need = loza_ssa_prefill_bwd_workspace_size(B, H, L, d_qk, d_v, n_sink, n_local)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_prefill_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, L, d_qk, d_v, block, n_sink, n_local, float(scale), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return dq, dk, dv


def loza_ssa_prefill_varlen_bwd_workspace_size(n_seqs, total, max_seqlen, H, d_qk, d_v,
                                               n_sink=1, n_local=7) -> int:
    return int(lib().loza_ssa_prefill_varlen_bwd_workspace_size(n_seqs, total, max_seqlen, H,
                                                                d_qk, d_v, n_sink, n_local))


def loza_ssa_prefill_varlen_bwd(q, k, v, o, lse, dout, cu_seqlens, max_seqlen, dq=None, dk=None,
                                dv=None, block=128, n_sink=1, n_local=7, scale=None,
                                workspace=None, stream=None):
    """Gradients of loza_ssa_prefill_varlen.  q, k: bf16 [H,total,d]; v, o,
    dout: bf16 [H,total,d]; lse: fp32 [H,total]; cu_seqlens: int32 CUDA
    [n_seqs+1].  Returns (dq, dk, dv)."""
    for t, dt, name in ((q, torch.bfloat16, "q"), (k, torch.bfloat16, "k"),
                        (v, torch.bfloat16, "v"), (o, torch.bfloat16, "o"),
                        (lse, torch.float32, "lse"), (dout, torch.bfloat16, "dout"),
                        (cu_seqlens, torch.int32, "cu_seqlens")):
        _need(t, dt, name)
    H, total, d_qk = q.shape
    d_v = v.shape[-1]
    n_seqs = cu_seqlens.numel() - 1
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, torch.bfloat16, name)
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    need = loza_ssa_prefill_varlen_bwd_workspace_size(n_seqs, total, int(max_seqlen), H, d_qk,
                                                      d_v, n_sink, n_local)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_prefill_varlen_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(cu_seqlens), n_seqs, total, int(max_seqlen), H, d_qk, d_v, block, n_sink, n_local,
        float(scale), _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def loza_ssa_decode_workspace_size(B, H_q, d_v=512, n_sink=1, n_local=7) -> int:
    return int(lib().loza_ssa_decode_workspace_size(B, H_q, d_v, n_sink, n_local))


def loza_ssa_decode(q, paged_kv, page_table, seq_lens, d_v=512, o=None, lse=None, page_size=128,
                    n_sink=1, n_local=7, scale=None, workspace=None, stream=None):
    """Paged SSA decode.  q: bf16 [B,H_q,d_qk]; paged_kv: bf16 [n_pages,page_size,d_qk];
    page_table: int32 [B,max_pages]; seq_lens: int32 [B] (including the new token).
    Returns (o bf16 [B,H_q,d_v], lse fp32 [B,H_q])."""
    _need(q, torch.bfloat16, "q")
    _need(paged_kv, torch.bfloat16, "paged_kv")
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    B, H_q, d_qk = q.shape
    n_pages = paged_kv.shape[0]
    max_pages = page_table.shape[1]
    if o is None:
        o = torch.empty((B, H_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    need = loza_ssa_decode_workspace_size(B, H_q, d_v, n_sink, n_local)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_decode(
        _ptr(q), _ptr(paged_kv), _ptr(page_table), _ptr(seq_lens), _ptr(o), _ptr(lse), B, H_q,
        d_qk, d_v, page_size, max_pages, n_pages, n_sink, n_local, float(scale), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return o, lse


def loza_ssa_decode_fp8(q, paged_kv_fp8, kv_scale, page_table, seq_lens, d_v=512, o=None,
                        lse=None, page_size=128, n_sink=1, n_local=7, scale=None, workspace=None,
                        stream=None):
    """Paged SSA decode over an FP8 cache.  paged_kv_fp8: uint8 [n_pages,page_size,576]
    e4m3 codes; kv_scale: fp32 [n_pages,page_size] per-token scales (K = scale * code).
    Other arguments and the result as loza_ssa_decode."""
    _need(q, torch.bfloat16, "q")
    _need(paged_kv_fp8, torch.uint8, "paged_kv_fp8")
    _need(kv_scale, torch.float32, "kv_scale")
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    B, H_q, d_qk = q.shape
    n_pages = paged_kv_fp8.shape[0]
    if tuple(kv_scale.shape) != tuple(paged_kv_fp8.shape[:2]):
        raise ValueError("kv_scale must be [n_pages, page_size]")
    max_pages = page_table.shape[1]
    if o is None:
        o = torch.empty((B, H_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    need = loza_ssa_decode_workspace_size(B, H_q, d_v, n_sink, n_local)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_decode_fp8(
        _ptr(q), _ptr(paged_kv_fp8), _ptr(kv_scale), _ptr(page_table), _ptr(seq_lens), _ptr(o),
        _ptr(lse), B, H_q, d_qk, d_v, page_size, max_pages, n_pages, n_sink, n_local,
        float(scale), _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, lse


def loza_ssa_decode_selected_workspace_size(B, H_q, d_v=512, n_sink=1, n_local=7,
                                            max_extra=0) -> int:
    return int(lib().loza_ssa_decode_selected_workspace_size(B, H_q, d_v, n_sink, n_local,
                                                             max_extra))


def loza_ssa_decode_selected(q, paged_kv, page_table, seq_lens, extra_pages, d_v=512, o=None,
                             lse=None, page_size=128, n_sink=1, n_local=7, scale=None,
                             workspace=None, stream=None):
    """Paged decode over the SSA window plus per-sequence chosen pages.
    extra_pages: int32 CUDA [B, max_extra] logical page ids (entries that are
    negative, in the window or after it add nothing; duplicates count once).
    Other arguments and the result as loza_ssa_decode."""
    _need(q, torch.bfloat16, "q")
    _need(paged_kv, torch.bfloat16, "paged_kv")
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    _need(extra_pages, torch.int32, "extra_pages")
    B, H_q, d_qk = q.shape
    if extra_pages.dim() != 2 or extra_pages.shape[0] != B:
        raise ValueError("extra_pages must be [B, max_extra]")
    max_extra = extra_pages.shape[1]
    n_pages = paged_kv.shape[0]
    max_pages = page_table.shape[1]
    if o is None:
        o = torch.empty((B, H_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    need = loza_ssa_decode_selected_workspace_size(B, H_q, d_v, n_sink, n_local, max_extra)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_decode_selected(
        _ptr(q), _ptr(paged_kv), _ptr(page_table), _ptr(seq_lens), _ptr(extra_pages), max_extra,
        _ptr(o), _ptr(lse), B, H_q, d_qk, d_v, page_size, max_pages, n_pages, n_sink, n_local,
        float(scale), _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, lse


def loza_ssa_decode_mtp_workspace_size(B, q_len, H_q, d_v=512, n_sink=1, n_local=7) -> int:
    return int(lib().loza_ssa_decode_mtp_workspace_size(B, q_len, H_q, d_v, n_sink, n_local))


def loza_ssa_decode_mtp(q, paged_kv, page_table, seq_lens, d_v=512, o=None, lse=None,
                        page_size=128, n_sink=1, n_local=7, scale=None, workspace=None,
                        stream=None):
    """Paged SSA decode with q_len query tokens per sequence (positions
    seq_len-q_len .. seq_len-1).  q: bf16 [B,q_len,H_q,d_qk]; other inputs as
    loza_ssa_decode.  Returns (o bf16 [B,q_len,H_q,d_v], lse fp32 [B,q_len,H_q])."""
    _need(q, torch.bfloat16, "q")
    _need(paged_kv, torch.bfloat16, "paged_kv")
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    B, q_len, H_q, d_qk = q.shape
    n_pages = paged_kv.shape[0]
    max_pages = page_table.shape[1]
    if o is None:
        o = torch.empty((B, q_len, H_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, q_len, H_q), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    need = loza_ssa_decode_mtp_workspace_size(B, q_len, H_q, d_v, n_sink, n_local)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_decode_mtp(
        _ptr(q), _ptr(paged_kv), _ptr(page_table), _ptr(seq_lens), q_len, _ptr(o), _ptr(lse), B,
        H_q, d_qk, d_v, page_size, max_pages, n_pages, n_sink, n_local, float(scale),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, lse


def loza_ssa_decode_layers_workspace_size(B, H_q, d_v=512, max_pages=1, n_sink=1, n_local=7,
                                          any_full=True) -> int:
    return int(lib().loza_ssa_decode_layers_workspace_size(B, H_q, d_v, max_pages, n_sink,
                                                           n_local, int(bool(any_full))))


def loza_ssa_decode_layers(layers, page_table, seq_lens, d_v=512, page_size=128, n_sink=1,
                           n_local=7, scale=None, workspace=None, stream=None):
    """One decode step through a stack of layers sharing a page table.
    layers: sequence of (q bf16 [B,H_q,d_qk], paged_kv bf16 [n_pages,page_size,d_qk],
    full_attention bool).  Returns a list of (o bf16 [B,H_q,d_v], lse fp32 [B,H_q])."""
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    if len(layers) == 0:
        raise ValueError("at least one layer")
    q0, kv0, _ = layers[0]
    B, H_q, d_qk = q0.shape
    n_pages = kv0.shape[0]
    max_pages = page_table.shape[1]
    descs = (LozaSsaDecodeLayer * len(layers))()
    outs = []
    for i, (q, kv, is_full) in enumerate(layers):
        _need(q, torch.bfloat16, "q")
        _need(kv, torch.bfloat16, "paged_kv")
        if tuple(q.shape) != (B, H_q, d_qk) or kv.shape[0] != n_pages:
            raise ValueError("every layer needs the same q shape and page-pool size")
        o = torch.empty((B, H_q, d_v), dtype=torch.bfloat16, device=q.device)
        lse = torch.empty((B, H_q), dtype=torch.float32, device=q.device)
        descs[i] = LozaSsaDecodeLayer(q.data_ptr(), kv.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                      int(bool(is_full)))
        outs.append((o, lse))
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    any_full = any(bool(f) for _, _, f in layers)
    need = loza_ssa_decode_layers_workspace_size(B, H_q, d_v, max_pages, n_sink, n_local,
                                                 any_full)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q0.device)
    _need(workspace, torch.uint8, "workspace")
    _check(lib().loza_ssa_decode_layers(
        descs, len(layers), _ptr(page_table), _ptr(seq_lens), B, H_q, d_qk, d_v, page_size,
        max_pages, n_pages, n_sink, n_local, float(scale), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return outs


def loza_ssa_decode_static_scratch(q, paged_kv, page_table, seq_lens, d_v=512, o=None, lse=None,
                                   page_size=128, n_sink=1, n_local=7, scale=None, stream=None):
    """loza_ssa_decode without a workspace: the library uses its built-in
    scratch array instead, so nothing is allocated for the split partials (for
    callers that cannot provide device memory when they launch).  Limited to
    B * ceil(H_q/128) * ceil((n_sink + n_local)/2) <= LOZA_SSA_STATIC_SCRATCH_SLOTS;
    calls whose kernels overlap on the GPU share that scratch and must not run
    concurrently.  Returns (o bf16 [B,H_q,d_v], lse fp32 [B,H_q])."""
    _need(q, torch.bfloat16, "q")
    _need(paged_kv, torch.bfloat16, "paged_kv")
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    B, H_q, d_qk = q.shape
    if o is None:
        o = torch.empty((B, H_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    _check(lib().loza_ssa_decode_static_scratch(
        _ptr(q), _ptr(paged_kv), _ptr(page_table), _ptr(seq_lens), _ptr(o), _ptr(lse), B, H_q,
        d_qk, d_v, page_size, page_table.shape[1], paged_kv.shape[0], n_sink, n_local,
        float(scale), _stream(stream)))
    return o, lse


def loza_ssa_get_last_device_status(stream=None) -> int:
    rc = lib().loza_ssa_get_last_device_status(_stream(stream))
    if rc < 0:
        _check(rc)
    return rc


def loza_ssa_debug_enumerate_tiles(n_qblocks, n_sink=1, n_local=7, max_tiles=None, device="cuda",
                                   stream=None):
    """The kernels' tile scheduler run on the device: (tiles [n_qblocks,max_tiles], counts)."""
    if max_tiles is None:
        max_tiles = n_sink + n_local
    tiles = torch.full((n_qblocks, max_tiles), -1, dtype=torch.int32, device=device)
    counts = torch.zeros(n_qblocks, dtype=torch.int32, device=device)
    _check(lib().loza_ssa_debug_enumerate_tiles(n_qblocks, n_sink, n_local, _ptr(tiles),
                                                _ptr(counts), max_tiles, _stream(stream)))
    return tiles, counts


def loza_ssa_debug_decode_pages(page_table, seq_lens, n_pages, page_size=128, n_sink=1, n_local=7,
                                max_tiles=None, stream=None):
    """The decode kernel's page selection run on the device: (pages [B,max_tiles], counts)."""
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    B, max_pages = page_table.shape
    if max_tiles is None:
        max_tiles = n_sink + n_local
    pages = torch.full((B, max_tiles), -2, dtype=torch.int32, device=page_table.device)
    counts = torch.zeros(B, dtype=torch.int32, device=page_table.device)
    _check(lib().loza_ssa_debug_decode_pages(
        _ptr(page_table), _ptr(seq_lens), B, max_pages, n_pages, page_size, n_sink, n_local,
        _ptr(pages), _ptr(counts), max_tiles, _stream(stream)))
    return pages, counts


def loza_ssa_debug_wait_timeout(timeout_us, device="cuda", stream=None):
    """The kernels' bounded wait on a barrier nothing arrives on, with a limit of
    timeout_us: returns the device int32[2] result (1 if the waiting thread gave
    up, and how many of the 31 other threads gave up on its abort flag)."""
    result = torch.full((2,), -1, dtype=torch.int32, device=device)
    _check(lib().loza_ssa_debug_wait_timeout(int(timeout_us), _ptr(result), _stream(stream)))
    return result


def loza_ssa_debug_long_partition(unit_pages, pairs_launched):
    """Host arithmetic of the long-window decode's page split (no device
    work): for the pages each (row, head group) unit lists, returns
    (pair_start int64 [pairs_launched + 1], slot_first int32 [units],
    slot_count int32 [units])."""
    import numpy as np
    pages = np.ascontiguousarray(unit_pages, dtype=np.int32)
    start = np.zeros(int(pairs_launched) + 1, dtype=np.int64)
    first = np.zeros(pages.size, dtype=np.int32)
    count = np.zeros(pages.size, dtype=np.int32)
    _check(lib().loza_ssa_debug_long_partition(
        pages.ctypes.data, int(pages.size), int(pairs_launched), start.ctypes.data,
        first.ctypes.data, count.ctypes.data))
    return start, first, count
