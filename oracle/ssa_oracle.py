"""TEST INFRASTRUCTURE ONLY: the CPU oracle for LoZA streaming sparse attention.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this module.  The product path (the CUDA library and
its binding) never does, and the two share no code.

Two independent implementations live here:

* ``prefill`` / ``prefill_varlen`` / ``decode`` call the plain C oracle
  (``ssa_oracle.c``): double precision, one query row at a time, sums over the
  exact key set J(i) enumerated by window membership.
* ``brute_force_prefill`` / ``brute_force_decode`` materialise the boolean
  mask M as an n x n array (the idiom "LoZA：ZigZag稀疏注意力机制" §4.1 uses to
  build its own mask) and run a dense masked softmax in numpy float64.  They
  are for tiny inputs and cross-check the C oracle.

``causal_attention`` is textbook causal softmax attention ("LoZA：ZigZag稀疏注意力机制"
§2.1, first formula, restricted to j <= i); SSA reduces to it when the window
covers the whole prefix.

The mask (QbitAI LoZA article, paragraph on the 1024-token sparse window:
one global block plus seven local blocks of 128 tokens)::

    J(i) = { j <= i : floor(j/blk) in W(floor(i/blk)) }
    W(b) = {0 .. n_sink-1}  U  {max(n_sink, b-n_local+1) .. b}

Inputs are float64 arrays or bfloat16 bit patterns held in uint16 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libssa_oracle.so")
_lib = None

ELT_F64 = 0
ELT_BF16 = 1


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libssa_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.oracle_ssa_block_in_window.argtypes = [i64, i64, i64, i64]
        lib.oracle_ssa_block_in_window.restype = i32
        lib.oracle_ssa_mask.argtypes = [i64, i64, i64, i64, i64]
        lib.oracle_ssa_mask.restype = i32
        lib.oracle_ssa_row_count.argtypes = [i64, i64, i64, i64]
        lib.oracle_ssa_row_count.restype = i64
        lib.oracle_ssa_key_blocks.argtypes = [i64, i64, i64, i64, i64, vp, i64]
        lib.oracle_ssa_key_blocks.restype = i64
        lib.oracle_ssa_prefill_rows.argtypes = [
            vp, vp, vp, i32, i64, i64, i64, i32, i32, i64, i64, i64, dbl, vp, i64, vp, vp]
        lib.oracle_ssa_prefill_rows.restype = i32
        lib.oracle_ssa_prefill_varlen_rows.argtypes = [
            vp, vp, vp, i32, vp, i64, i64, i64, i32, i32, i64, i64, i64, dbl, vp, i64, vp, vp]
        lib.oracle_ssa_prefill_varlen_rows.restype = i32
        lib.oracle_ssa_decode_rows.argtypes = [
            vp, vp, i32, vp, vp, i64, i64, i32, i32, i64, i64, i64, i64, i64, dbl, vp, i64, vp, vp]
        lib.oracle_ssa_decode_rows.restype = i32
        lib.oracle_ssa_decode_sel_rows.argtypes = [
            vp, vp, i32, vp, vp, vp, i64, i64, i64, i32, i32, i64, i64, i64, i64, i64, ctypes.c_double,
            vp, i64, vp, vp]
        lib.oracle_ssa_decode_sel_rows.restype = i32
        lib.oracle_ssa_decode_mtp_rows.argtypes = [
            vp, vp, i32, vp, vp, i64, i64, i64, i32, i32, i64, i64, i64, i64, i64, dbl, vp, i64,
            vp, vp]
        lib.oracle_ssa_decode_mtp_rows.restype = i32
        lib.oracle_ssa_prefill_bwd.argtypes = [
            vp, vp, vp, vp, i32, i64, i64, i64, i32, i32, i64, i64, i64, dbl, vp, vp, vp]
        lib.oracle_ssa_prefill_bwd.restype = i32
        lib.oracle_ssa_num_threads.argtypes = []
        lib.oracle_ssa_num_threads.restype = i32
        _lib = lib
    return _lib


def _elt(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return ELT_F64
    if a.dtype == np.uint16:
        return ELT_BF16
    raise TypeError(f"oracle inputs must be float64 or bf16 bits in uint16, got {a.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_ssa_num_threads())


def block_in_window(qb, kb, n_sink=1, n_local=7) -> bool:
    return bool(_load().oracle_ssa_block_in_window(qb, kb, n_sink, n_local))


def mask(i, j, blk=128, n_sink=1, n_local=7) -> bool:
    return bool(_load().oracle_ssa_mask(i, j, blk, n_sink, n_local))


def row_count(i, blk=128, n_sink=1, n_local=7) -> int:
    return int(_load().oracle_ssa_row_count(i, blk, n_sink, n_local))


def key_blocks(qb, seq_len, blk=128, n_sink=1, n_local=7) -> list[int]:
    """Key blocks query block ``qb`` touches, read off the mask (ascending)."""
    cap = qb + 1
    out = np.zeros(cap, dtype=np.int64)
    n = _load().oracle_ssa_key_blocks(qb, blk, seq_len, n_sink, n_local, _ptr(out), cap)
    assert n >= 0
    return out[:n].tolist()


def prefill(q, k, v, blk=128, n_sink=1, n_local=7, scale=None, rows=None):
    """Dense SSA prefill.  q, k: [B,H,L,dqk]; v: [B,H,L,dv].

    ``rows``: optional flat indices (b*H + h)*L + i; returns (o [n,dv], lse [n]).
    Without ``rows`` returns (o [B,H,L,dv], lse [B,H,L]).
    """
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    B, H, L, dqk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, L, dqk) and v.shape == (B, H, L, dv)
    elt = _elt(q)
    assert _elt(k) == elt and _elt(v) == elt
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    full = rows is None
    rows = np.arange(B * H * L, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.empty((rows.size, dv), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    rc = _load().oracle_ssa_prefill_rows(
        _ptr(q), _ptr(k), _ptr(v), elt, B, H, L, dqk, dv, blk, n_sink, n_local, float(scale),
        _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError(f"oracle prefill failed ({rc})")
    if full:
        return o.reshape(B, H, L, dv), lse.reshape(B, H, L)
    return o, lse


def prefill_varlen(q, k, v, cu_seqlens, blk=128, n_sink=1, n_local=7, scale=None, rows=None):
    """Packed varlen SSA prefill.  q, k: [H,total,dqk]; v: [H,total,dv].

    ``rows``: optional flat indices h*total + token.
    """
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    H, total, dqk = q.shape
    dv = v.shape[-1]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    elt = _elt(q)
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    full = rows is None
    rows = np.arange(H * total, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.empty((rows.size, dv), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    rc = _load().oracle_ssa_prefill_varlen_rows(
        _ptr(q), _ptr(k), _ptr(v), elt, _ptr(cu), cu.size - 1, total, H, dqk, dv, blk, n_sink,
        n_local, float(scale), _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError(f"oracle varlen prefill failed ({rc})")
    if full:
        return o.reshape(H, total, dv), lse.reshape(H, total)
    return o, lse


def decode(q, kv, page_table, seq_lens, dv, page_size=128, n_sink=1, n_local=7, scale=None,
           rows=None):
    """Paged SSA decode.  q: [B,Hq,dqk]; kv: [n_pages,page_size,dqk];
    page_table: [B,max_pages] int32; seq_lens: [B] int32 (including the new token).
    ``rows``: optional flat indices b*Hq + h.
    """
    q = np.ascontiguousarray(q)
    kv = np.ascontiguousarray(kv)
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, dqk = q.shape
    n_pages = kv.shape[0]
    assert kv.shape[1] == page_size and kv.shape[2] == dqk
    elt = _elt(q)
    assert _elt(kv) == elt
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    full = rows is None
    rows = np.arange(B * Hq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.empty((rows.size, dv), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    rc = _load().oracle_ssa_decode_rows(
        _ptr(q), _ptr(kv), elt, _ptr(pt), _ptr(sl), B, Hq, dqk, dv, page_size, pt.shape[1],
        n_pages, n_sink, n_local, float(scale), _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError(f"oracle decode failed ({rc})")
    if full:
        return o.reshape(B, Hq, dv), lse.reshape(B, Hq)
    return o, lse


def decode_selected(q, kv, page_table, seq_lens, extra_pages, dv, page_size=128, n_sink=1,
                    n_local=7, scale=None, rows=None):
    """Paged decode over the SSA window plus selected pages (LongCat
    sparse-attention article, 机制 1 and 机制 3: a fixed sink + sliding-window
    budget plus pages of P = 128 tokens chosen by a page-level indexer).
    extra_pages: [B, max_extra] int32 logical page ids per sequence; an entry
    that is negative, past the query's page or already in the window adds
    nothing, and a page listed twice counts once.  Other arguments as decode().
    """
    q = np.ascontiguousarray(q)
    kv = np.ascontiguousarray(kv)
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    ex = np.ascontiguousarray(extra_pages, dtype=np.int32)
    B, Hq, dqk = q.shape
    assert ex.ndim == 2 and ex.shape[0] == B
    n_pages = kv.shape[0]
    assert kv.shape[1] == page_size and kv.shape[2] == dqk
    elt = _elt(q)
    assert _elt(kv) == elt
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    full = rows is None
    rows = np.arange(B * Hq, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.empty((rows.size, dv), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    rc = _load().oracle_ssa_decode_sel_rows(
        _ptr(q), _ptr(kv), elt, _ptr(pt), _ptr(sl), _ptr(ex), ex.shape[1], B, Hq, dqk, dv,
        page_size, pt.shape[1], n_pages, n_sink, n_local, float(scale), _ptr(rows), rows.size,
        _ptr(o), _ptr(lse))
    if rc:
        raise ValueError(f"oracle decode (selected pages) failed ({rc})")
    if full:
        return o.reshape(B, Hq, dv), lse.reshape(B, Hq)
    return o, lse


def prefill_bwd(q, k, v, dout, blk=128, n_sink=1, n_local=7, scale=None):
    """Gradients (dq, dk, dv) of the dense SSA prefill for upstream gradient
    dout = dL/dO, float64.  q, k: [B,H,L,dqk]; v, dout: [B,H,L,dv] (float64 or
    bf16 bit patterns, all the same kind)."""
    q, k, v, dout = (np.ascontiguousarray(a) for a in (q, k, v, dout))
    B, H, L, dqk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape == (B, H, L, dv) and dout.shape == v.shape
    elt = _elt(q)
    assert _elt(k) == elt and _elt(v) == elt and _elt(dout) == elt
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    dq = np.empty((B, H, L, dqk))
    dk = np.empty((B, H, L, dqk))
    dvv = np.empty((B, H, L, dv))
    rc = _load().oracle_ssa_prefill_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), elt, B, H, L, dqk,
                                        dv, blk, n_sink, n_local, float(scale), _ptr(dq), _ptr(dk),
                                        _ptr(dvv))
    if rc:
        raise ValueError(f"oracle prefill backward failed ({rc})")
    return dq, dk, dvv


def prefill_varlen_bwd(q, k, v, dout, cu_seqlens, blk=128, n_sink=1, n_local=7, scale=None):
    """Gradients of the packed varlen prefill: q, k: [H,total,dqk]; v, dout:
    [H,total,dv].  Every sequence is its own attention problem (its block
    indices count from its first token and no key crosses its boundary), so
    its gradients are those of the dense prefill over its slice; keys and
    queries of different sequences never meet."""
    q, k, v, dout = (np.ascontiguousarray(a) for a in (q, k, v, dout))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    dq = np.empty(q.shape)
    dk = np.empty(k.shape)
    dvv = np.empty(v.shape)
    for a, b in zip(cu[:-1], cu[1:]):
        if b <= a:
            continue
        g = prefill_bwd(q[None, :, a:b], k[None, :, a:b], v[None, :, a:b], dout[None, :, a:b],
                        blk, n_sink, n_local, scale)
        dq[:, a:b], dk[:, a:b], dvv[:, a:b] = (x[0] for x in g)
    return dq, dk, dvv


def decode_mtp(q, kv, page_table, seq_lens, dv, page_size=128, n_sink=1, n_local=7, scale=None,
               rows=None):
    """Paged decode with q_len query tokens per sequence: q [B, q_len, Hq, dqk];
    token k of sequence b is the query at position seq_lens[b] - q_len + k and
    attends J(t) of the SSA mask (QbitAI LoZA article, 1024-token window
    paragraph) at its own position.  ``rows``: optional flat indices
    (b*q_len + k)*Hq + h.  Returns o [B, q_len, Hq, dv], lse [B, q_len, Hq]."""
    q = np.ascontiguousarray(q)
    kv = np.ascontiguousarray(kv)
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, q_len, Hq, dqk = q.shape
    n_pages = kv.shape[0]
    assert kv.shape[1] == page_size and kv.shape[2] == dqk
    elt = _elt(q)
    assert _elt(kv) == elt
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    full = rows is None
    n_all = B * q_len * Hq
    rows = np.arange(n_all, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.empty((rows.size, dv), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    rc = _load().oracle_ssa_decode_mtp_rows(
        _ptr(q), _ptr(kv), elt, _ptr(pt), _ptr(sl), q_len, B, Hq, dqk, dv, page_size, pt.shape[1],
        n_pages, n_sink, n_local, float(scale), _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError(f"oracle decode (q_len tokens) failed ({rc})")
    if full:
        return o.reshape(B, q_len, Hq, dv), lse.reshape(B, q_len, Hq)
    return o, lse


# ---------------------------------------------------------------------------
# Independent numpy implementations (tiny inputs only)
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def mask_matrix(n: int, blk=128, n_sink=1, n_local=7) -> np.ndarray:
    """The SSA mask as a dense boolean [n, n] array, filled one entry at a time
    from the block rule (j <= i, and j's block is a sink block or one of the
    n_local most recent blocks up to and including i's own)."""
    m = np.zeros((n, n), dtype=bool)
    for i in range(n):
        bi = i // blk
        for j in range(i + 1):
            bj = j // blk
            m[i, j] = (bj < n_sink) or (bi - bj < n_local)
    return m


def _as_f64(a):
    return bf16_bits_to_f64(a) if a.dtype == np.uint16 else np.asarray(a, dtype=np.float64)


def brute_force_prefill(q, k, v, blk=128, n_sink=1, n_local=7, scale=None):
    """Dense masked softmax attention with a materialised mask, numpy float64.
    q, k: [..., L, dqk]; v: [..., L, dv]."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    L, dqk = q.shape[-2:]
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    m = mask_matrix(L, blk, n_sink, n_local)
    s = scale * np.einsum("...ic,...jc->...ij", q, k)
    s = np.where(m, s, -np.inf)
    smax = s.max(axis=-1, keepdims=True)
    p = np.where(m, np.exp(s - smax), 0.0)
    den = p.sum(axis=-1, keepdims=True)
    o = np.einsum("...ij,...jc->...ic", p, v) / den
    lse = smax[..., 0] + np.log(den[..., 0])
    return o, lse


def brute_force_prefill_bwd(q, k, v, dout, blk=128, n_sink=1, n_local=7, scale=None):
    """Backward of brute_force_prefill with the materialised mask, numpy
    float64, written as matrix products: P = softmax(masked S), dP = dO V^T,
    dS = P * (dP - rowsum(P * dP)), dQ = scale dS K, dK = scale dS^T Q,
    dV = P^T dO."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    L, dqk = q.shape[-2:]
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    m = mask_matrix(L, blk, n_sink, n_local)
    s = np.where(m, scale * np.einsum("...ic,...jc->...ij", q, k), -np.inf)
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    p = np.where(m, p, 0.0)
    p /= p.sum(axis=-1, keepdims=True)
    dp = np.einsum("...ic,...jc->...ij", dout, v)
    ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
    dq = scale * np.einsum("...ij,...jc->...ic", ds, k)
    dk = scale * np.einsum("...ij,...ic->...jc", ds, q)
    dvv = np.einsum("...ij,...ic->...jc", p, dout)
    return dq, dk, dvv


def brute_force_decode(q, kv, page_table, seq_lens, dv, page_size=128, n_sink=1, n_local=7,
                       scale=None):
    """Decode via an explicit gather of each sequence's logical key rows, then
    the last row of a materialised-mask attention.  q: [B,Hq,dqk]."""
    q, kv = _as_f64(q), _as_f64(kv)
    B, Hq, dqk = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    o = np.zeros((B, Hq, dv))
    lse = np.zeros((B, Hq))
    for b in range(B):
        n = int(seq_lens[b])
        logical = np.arange(n)
        phys = np.asarray(page_table[b])[logical // page_size] * page_size + logical % page_size
        keys = kv.reshape(-1, dqk)[phys]                      # [n, dqk]
        allowed = mask_matrix(n, page_size, n_sink, n_local)[n - 1]
        s = scale * q[b] @ keys.T                             # [Hq, n]
        s = np.where(allowed[None, :], s, -np.inf)
        smax = s.max(axis=-1, keepdims=True)
        p = np.where(allowed[None, :], np.exp(s - smax), 0.0)
        den = p.sum(axis=-1, keepdims=True)
        o[b] = p @ keys[:, :dv] / den
        lse[b] = smax[:, 0] + np.log(den[:, 0])
    return o, lse


def brute_force_decode_selected(q, kv, page_table, seq_lens, extra_pages, dv, page_size=128,
                                n_sink=1, n_local=7, scale=None):
    """Decode over an explicitly built key set: the window's keys (read off the
    materialised mask) plus every key of each listed page that lies at or
    before the query, gathered through the page table.  q: [B,Hq,dqk]."""
    q, kv = _as_f64(q), _as_f64(kv)
    B, Hq, dqk = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    o = np.zeros((B, Hq, dv))
    lse = np.zeros((B, Hq))
    for b in range(B):
        n = int(seq_lens[b])
        allowed = mask_matrix(n, page_size, n_sink, n_local)[n - 1].copy()
        for e in np.asarray(extra_pages[b]):
            if e >= 0:
                allowed[e * page_size:(e + 1) * page_size] = True   # keys past n are cut below
        allowed = allowed[:n]
        logical = np.nonzero(allowed)[0]
        phys = np.asarray(page_table[b])[logical // page_size] * page_size + logical % page_size
        keys = kv.reshape(-1, dqk)[phys]
        s = scale * q[b] @ keys.T
        smax = s.max(axis=-1, keepdims=True)
        p = np.exp(s - smax)
        den = p.sum(axis=-1, keepdims=True)
        o[b] = p @ keys[:, :dv] / den
        lse[b] = smax[:, 0] + np.log(den[:, 0])
    return o, lse


def e4m3_to_f64(codes) -> np.ndarray:
    """Values of OCP FP8 E4M3 codes (uint8), from the format's definition: bit
    7 sign, bits 3..6 exponent e with bias 7, bits 0..2 mantissa m; e = 0 is
    subnormal (m/8 * 2^-6), otherwise (1 + m/8) * 2^(e-7); e = 15 with m = 7
    is NaN (there are no infinities)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def dequant_fp8_cache(kv8, kv_scale) -> np.ndarray:
    """K_j = s_j * k8_j, float64: kv8 [n_pages, page_size, d] e4m3 codes,
    kv_scale [n_pages, page_size]."""
    k = e4m3_to_f64(kv8)
    if np.isnan(k).any():
        raise ValueError("NaN code in the FP8 cache")
    return k * np.asarray(kv_scale, dtype=np.float64)[..., None]


def decode_fp8(q, kv8, kv_scale, page_table, seq_lens, dv, page_size=128, n_sink=1, n_local=7,
               scale=None, rows=None):
    """Paged SSA decode over an FP8 latent cache: every token's row is e4m3
    codes times one fp32 scale.  The cache is dequantized exactly to float64
    and decode() runs on it (the decode-workload variant with an FP8 KV cache;
    the per-token scale layout is this library's reading, the pages fix none)."""
    q64 = _as_f64(q)
    kv = dequant_fp8_cache(kv8, kv_scale)
    return decode(q64, kv, page_table, seq_lens, dv, page_size, n_sink, n_local, scale, rows)


def decode_full(q, kv, page_table, seq_lens, dv, page_size=128, scale=None, rows=None):
    """Full-attention decode (the MLA layers that LoZA keeps, "LoZA：ZigZag稀疏注意力机制"
    §2.1, first formula, for the newest query token): softmax over every key
    0 .. seq_len-1 of the sequence, gathered through the page table, float64.
    q: [B,Hq,dqk]; kv: [n_pages,page_size,dqk]; the value is the first dv
    entries of the key row.  ``rows``: optional flat indices b*Hq + h.
    Returns (o, lse) shaped like decode()."""
    q, kv = _as_f64(q), _as_f64(kv)
    B, Hq, dqk = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    full = rows is None
    rows = np.arange(B * Hq, dtype=np.int64) if full else np.asarray(rows, dtype=np.int64)
    o = np.empty((rows.size, dv))
    lse = np.empty(rows.size)
    flat_kv = kv.reshape(-1, dqk)
    for b in np.unique(rows // Hq):
        sel = np.nonzero(rows // Hq == b)[0]
        heads = rows[sel] % Hq
        n = int(seq_lens[b])
        logical = np.arange(n)
        phys = np.asarray(page_table[b])[logical // page_size].astype(np.int64) * page_size \
            + logical % page_size
        keys = flat_kv[phys]                                  # [n, dqk]
        s = scale * q[b, heads] @ keys.T                      # [heads, n]
        smax = s.max(axis=-1, keepdims=True)
        p = np.exp(s - smax)
        den = p.sum(axis=-1, keepdims=True)
        o[sel] = p @ keys[:, :dv] / den
        lse[sel] = smax[:, 0] + np.log(den[:, 0])
    if full:
        return o.reshape(B, Hq, dv), lse.reshape(B, Hq)
    return o, lse


def decode_layers(layers, page_table, seq_lens, dv, page_size=128, n_sink=1, n_local=7,
                  scale=None, rows=None):
    """One decode step through a stack of attention layers (the ZigZag layout
    of the QbitAI LoZA article: some layers keep full MLA attention, the others
    are SSA).  ``layers``: sequence of (q, kv, full_attention) sharing one page
    table and seq_lens; each layer is decode_full() or decode() on its own
    inputs.  Returns a list of (o, lse), one per layer."""
    out = []
    for q, kv, is_full in layers:
        if is_full:
            out.append(decode_full(q, kv, page_table, seq_lens, dv, page_size, scale, rows))
        else:
            out.append(decode(q, kv, page_table, seq_lens, dv, page_size, n_sink, n_local, scale,
                              rows))
    return out


def causal_attention(q, k, v, scale=None):
    """Textbook causal softmax attention in float64 (keys j <= i)."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    L, dqk = q.shape[-2:]
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    s = scale * np.einsum("...ic,...jc->...ij", q, k)
    tri = np.tril(np.ones((L, L), dtype=bool))
    s = np.where(tri, s, -np.inf)
    lse = np.logaddexp.reduce(s, axis=-1)
    o = np.einsum("...ij,...jc->...ic", np.exp(s - lse[..., None]), v)
    return o, lse
