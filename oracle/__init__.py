"""fp64 CPU oracle for causal grouped-query attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its Python binding) never imports, links or calls it,
and it shares no code with that path.

The arithmetic lives in ``attn_ref.c`` (plain C, fp64, one query row at a
time); this module compiles it with gcc and marshals numpy arrays through
ctypes.  What it computes is the scaled-dot-product attention that the Tessera
pages name ("a FlashAttention forward kernel with online softmax, causal
masking, grouped-query attention" -- hysenlabs.com Tessera review, "The kernel
set and its torch fallback"), written out as its definition:

    s_ij = scale * <Q[b,h,i], K[b,h//G,j]>,  j <= i when causal
    O[b,h,i] = sum_j softmax_j(s_i) V[b,h//G,j]
    LSE[b,h,i] = logsumexp_j(s_ij)            (natural log)

and its exact gradient with respect to Q, K and V given dO (the chain rule
through the row softmax; see the backward section of ``attn_ref.c``), one
decoding step over a paged key/value cache (the paged-decode section), and
the attention block's prologue: RMSNorm and the rotary embedding of the
projected queries and keys (the prologue section).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "attn_ref.c")
LIB = os.path.join(_HERE, "liboracle_attn.so")

_lock = threading.Lock()
_lib = None


def build(src_path: str = SRC, out_path: str = LIB) -> str:
    """Compile the C oracle into a shared library (gcc, -O2, strict IEEE fp64).

    -ffp-contract=off keeps every multiply and add separately rounded, as the
    source is written; no -ffast-math.
    """
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
           "-o", out_path, src_path, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


def _stale(lib_path: str, src_path: str) -> bool:
    return (not os.path.exists(lib_path)
            or os.path.getmtime(lib_path) < os.path.getmtime(src_path))


def load(lib_path: str | None = None) -> ctypes.CDLL:
    """Load the oracle library, building it first when missing or stale.

    With ``lib_path`` given, load that file as is (used to test planted
    mistakes in a modified copy of the source).
    """
    global _lib
    if lib_path is not None:
        return _bind(ctypes.CDLL(lib_path))
    with _lock:
        if _lib is None:
            if _stale(LIB, SRC):
                build()
            _lib = _bind(ctypes.CDLL(LIB))
    return _lib


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    dp = ctypes.POINTER(ctypes.c_double)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    i64p = ctypes.POINTER(ctypes.c_int64)
    ci = ctypes.c_int
    lib.oracle_attn_fwd_f64.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci, ci,
                                        ci, ctypes.c_double]
    lib.oracle_attn_fwd_f64.restype = ci
    lib.oracle_attn_rows_bf16.argtypes = [u16p, u16p, u16p, ci, ci, ci, ci, ci,
                                          ci, ctypes.c_double, i64p,
                                          ctypes.c_int64, dp, dp]
    lib.oracle_attn_rows_bf16.restype = ci
    lib.oracle_attn_bwd_f64.argtypes = [dp, dp, dp, dp, dp, dp, dp, ci, ci, ci, ci, ci,
                                        ci, ctypes.c_double]
    lib.oracle_attn_bwd_f64.restype = ci
    lib.oracle_attn_bwd_dq_rows_bf16.argtypes = [u16p, u16p, u16p, u16p, ci, ci, ci, ci,
                                                 ci, ci, ctypes.c_double, i64p,
                                                 ctypes.c_int64, dp]
    lib.oracle_attn_bwd_dq_rows_bf16.restype = ci
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.oracle_paged_decode_f64.argtypes = [dp, dp, dp, i32p, i32p, ci, ci, ci, ci, ci, ci, ci,
                                            ctypes.c_double, dp, dp]
    lib.oracle_paged_decode_f64.restype = ci
    lib.oracle_rmsnorm_f64.argtypes = [dp, dp, ci, ci, ctypes.c_double, dp]
    lib.oracle_rmsnorm_f64.restype = ci
    lib.oracle_rope_qkv_f64.argtypes = [dp, i32p, ci, ci, ci, ci, ci, ctypes.c_double, dp, dp, dp]
    lib.oracle_rope_qkv_f64.restype = ci
    return lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def attn_fwd_f64(q, k, v, causal: bool = True, scale: float | None = None,
                 lib: ctypes.CDLL | None = None):
    """Full attention in fp64.

    q: [B,Hq,T,d], k and v: [B,Hkv,T,d] (anything numpy can view as float64).
    Returns (O [B,Hq,T,d] float64, LSE [B,Hq,T] float64).  ``scale`` defaults
    to 1/sqrt(d).
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B,Hkv,T,d] matching q")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, T, d), dtype=np.float64)
    lse = np.zeros((B, Hq, T), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_fwd_f64(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                                 _ptr(v, ctypes.c_double), _ptr(o, ctypes.c_double),
                                 _ptr(lse, ctypes.c_double), B, Hq, Hkv, T, d,
                                 int(bool(causal)), float(scale))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_f64 failed with code {rc}")
    return o, lse


def attn_rows_bf16(q_bits, k_bits, v_bits, rows, causal: bool = True,
                   scale: float | None = None, lib: ctypes.CDLL | None = None):
    """Selected output rows, reading bf16 inputs given as uint16 bit patterns.

    q_bits: uint16 [B,Hq,T,d]; k_bits, v_bits: uint16 [B,Hkv,T,d];
    rows: int64 [n,3] of (b, h, i).  Rows sorted by (b, h // G) reuse the
    widened key/value head.  Returns (O rows [n,d], LSE rows [n]) in fp64.
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    B, Hq, T, d = q_bits.shape
    Hkv = k_bits.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    n = rows.shape[0]
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_rows_bf16(_ptr(q_bits, ctypes.c_uint16),
                                   _ptr(k_bits, ctypes.c_uint16),
                                   _ptr(v_bits, ctypes.c_uint16), B, Hq, Hkv, T,
                                   d, int(bool(causal)), float(scale),
                                   _ptr(rows, ctypes.c_int64), n,
                                   _ptr(o, ctypes.c_double),
                                   _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_attn_rows_bf16 failed with code {rc}")
    return o, lse


def host_threads() -> int:
    """Host cores this process may run on (its CPU affinity), at least 1."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def fwd_runs(B: int, Hq: int, T: int, causal: bool, run_rows: int = 256):
    """The work units of attn_fwd_bf16_threaded: runs (b, h, i0, i1) of up to
    ``run_rows`` consecutive query rows of one head, longest causal extent
    first (a stable sort, so equal extents keep (b, h) order)."""
    runs = [(b, h, i0, min(i0 + run_rows, T)) for b in range(B) for h in range(Hq)
            for i0 in range(0, T, run_rows)]
    if causal:
        runs.sort(key=lambda r: -r[3])
    return runs


def run_flops(run, d: int, T: int, causal: bool) -> float:
    """Multiply-add work of one run: 4*d flops per visible key per row (the
    QK^T dot product and the PV accumulation), as the metric counts them."""
    _, _, i0, i1 = run
    if causal:
        keys = (i1 * (i1 + 1) - i0 * (i0 + 1)) // 2
    else:
        keys = (i1 - i0) * T
    return 4.0 * d * keys


def attn_fwd_bf16_threaded(q_bits, k_bits, v_bits, causal: bool = True,
                           scale: float | None = None, threads: int | None = None,
                           run_rows: int = 256, runs=None, lib: ctypes.CDLL | None = None):
    """Every output row of attention on bf16 inputs, on all host cores.

    q_bits: uint16 [B,Hq,T,d]; k_bits, v_bits: uint16 [B,Hkv,T,d] (bf16 bit
    patterns).  The rows are cut into runs of up to ``run_rows`` consecutive
    rows of one (b, h) (``fwd_runs``); each run is one call of the C row entry
    ``oracle_attn_rows_bf16``, writing straight into its slice of the outputs.
    ctypes releases the GIL during the call, so ``threads`` host threads
    (default: every core this process may use) work on runs at once.  A row's
    arithmetic is ``attend_one_row``'s whichever thread runs it, so the result
    is bit for bit that of one call over all rows.  ``runs`` restricts the work
    to the given runs (rows outside them are left as NaN).
    Returns (O [B,Hq,T,d], LSE [B,Hq,T]) in fp64.
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    B, Hq, T, d = q_bits.shape
    Hkv = k_bits.shape[1]
    if k_bits.shape != (B, Hkv, T, d) or v_bits.shape != k_bits.shape:
        raise ValueError("k and v must be [B,Hkv,T,d] matching q")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.full((B, Hq, T, d), np.nan)
    lse = np.full((B, Hq, T), np.nan)
    lib = lib or load()
    if runs is None:
        runs = fwd_runs(B, Hq, T, causal, run_rows)
    qp, kp, vp = (_ptr(a, ctypes.c_uint16) for a in (q_bits, k_bits, v_bits))

    def one(run):
        b, h, i0, i1 = run
        rows = np.empty((i1 - i0, 3), dtype=np.int64)
        rows[:, 0] = b
        rows[:, 1] = h
        rows[:, 2] = np.arange(i0, i1)
        rc = lib.oracle_attn_rows_bf16(qp, kp, vp, B, Hq, Hkv, T, d, int(bool(causal)),
                                       float(scale), _ptr(rows, ctypes.c_int64), i1 - i0,
                                       _ptr(o[b, h, i0:i1], ctypes.c_double),
                                       _ptr(lse[b, h, i0:i1], ctypes.c_double))
        if rc != 0:
            raise ValueError(f"oracle_attn_rows_bf16 failed with code {rc} on run {run}")

    with ThreadPoolExecutor(max_workers=threads or host_threads()) as pool:
        for f in [pool.submit(one, r) for r in runs]:
            f.result()
    return o, lse


def attn_bwd_threaded(q, k, v, dout, causal: bool = True, scale: float | None = None,
                      threads: int | None = None, lib: ctypes.CDLL | None = None):
    """attn_bwd_f64 with its (b, key/value head) slices on all host cores.

    Each slice -- its G query heads, their dO rows, one K/V head -- is one
    call of ``oracle_attn_bwd_f64`` on contiguous views (B = 1, Hkv = 1).  A
    slice's dK/dV sums run over the same heads and rows in the same order as
    in one call over the whole problem, and a dQ row depends only on its own
    slice, so the result is bit for bit that call's.
    Returns (dQ, dK, dV) in fp64.
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape or dout.shape != q.shape:
        raise ValueError("k, v must be [B,Hkv,T,d] and dout [B,Hq,T,d] matching q")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    G = Hq // Hkv
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(k.shape)
    lib = lib or load()
    dp = ctypes.c_double

    def one(bg):
        b, g = bg
        hs = slice(g * G, (g + 1) * G)
        rc = lib.oracle_attn_bwd_f64(_ptr(q[b, hs], dp), _ptr(k[b, g], dp), _ptr(v[b, g], dp),
                                     _ptr(dout[b, hs], dp), _ptr(dq[b, hs], dp),
                                     _ptr(dk[b, g], dp), _ptr(dv[b, g], dp), 1, G, 1, T, d,
                                     int(bool(causal)), float(scale))
        if rc != 0:
            raise ValueError(f"oracle_attn_bwd_f64 failed with code {rc} on slice {bg}")

    with ThreadPoolExecutor(max_workers=threads or host_threads()) as pool:
        for f in [pool.submit(one, (b, g)) for b in range(B) for g in range(Hkv)]:
            f.result()
    return dq, dk, dv


def attn_bwd_f64(q, k, v, dout, causal: bool = True, scale: float | None = None,
                 lib: ctypes.CDLL | None = None):
    """Gradients of the attention forward in fp64.

    q, dout: [B,Hq,T,d]; k, v: [B,Hkv,T,d].  Returns (dQ [B,Hq,T,d],
    dK [B,Hkv,T,d], dV [B,Hkv,T,d]) in float64; dK and dV sum over the query
    heads of each group.
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape or dout.shape != q.shape:
        raise ValueError("k, v must be [B,Hkv,T,d] and dout [B,Hq,T,d] matching q")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(k.shape, dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_bwd_f64(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                                 _ptr(v, ctypes.c_double), _ptr(dout, ctypes.c_double),
                                 _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                                 _ptr(dv, ctypes.c_double), B, Hq, Hkv, T, d,
                                 int(bool(causal)), float(scale))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd_f64 failed with code {rc}")
    return dq, dk, dv


def attn_bwd_dq_rows_bf16(q_bits, k_bits, v_bits, dout_bits, rows, causal: bool = True,
                          scale: float | None = None, lib: ctypes.CDLL | None = None):
    """Selected rows of dQ from bf16 inputs given as uint16 bit patterns.

    rows: int64 [n,3] of (b, h, i).  Returns dQ rows [n,d] in fp64.
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    dout_bits = np.ascontiguousarray(dout_bits, dtype=np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    B, Hq, T, d = q_bits.shape
    Hkv = k_bits.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    n = rows.shape[0]
    dq = np.zeros((n, d), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_bwd_dq_rows_bf16(_ptr(q_bits, ctypes.c_uint16),
                                          _ptr(k_bits, ctypes.c_uint16),
                                          _ptr(v_bits, ctypes.c_uint16),
                                          _ptr(dout_bits, ctypes.c_uint16), B, Hq, Hkv, T,
                                          d, int(bool(causal)), float(scale),
                                          _ptr(rows, ctypes.c_int64), n,
                                          _ptr(dq, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd_dq_rows_bf16 failed with code {rc}")
    return dq


def paged_decode_f64(q, k_cache, v_cache, block_table, seq_lens, scale: float | None = None,
                     lib: ctypes.CDLL | None = None):
    """One decode step over a paged K/V cache, in fp64.

    q: [B,Hq,d]; k_cache, v_cache: [num_blocks,Hkv,bs,d]; block_table: int32
    [B,max_blocks]; seq_lens: int32 [B].  Returns (O [B,Hq,d], LSE [B,Hq]).
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.float64)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.float64)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, d = q.shape
    num_blocks, Hkv, bs, _ = k_cache.shape
    max_blocks = block_table.shape[1] if block_table.ndim == 2 else 0
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, d), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_paged_decode_f64(_ptr(q, ctypes.c_double), _ptr(k_cache, ctypes.c_double),
                                     _ptr(v_cache, ctypes.c_double),
                                     _ptr(block_table, ctypes.c_int32),
                                     _ptr(seq_lens, ctypes.c_int32), B, Hq, Hkv, d, bs,
                                     max_blocks, num_blocks, float(scale),
                                     _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode_f64 failed with code {rc}")
    return o, lse


def rmsnorm_f64(x, w, eps: float = 1e-6, lib: ctypes.CDLL | None = None):
    """RMSNorm over the last dimension in fp64: x [..., dim], w [dim]."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    dim = x.shape[-1]
    if w.shape != (dim,):
        raise ValueError("w must be [dim]")
    rows = x.size // dim if dim else 0
    y = np.zeros_like(x)
    lib = lib or load()
    rc = lib.oracle_rmsnorm_f64(_ptr(x, ctypes.c_double), _ptr(w, ctypes.c_double), rows, dim,
                                float(eps), _ptr(y, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_rmsnorm_f64 failed with code {rc}")
    return y


def rope_qkv_f64(qkv, Hq: int, Hkv: int, positions=None, base: float = 10000.0,
                 lib: ctypes.CDLL | None = None):
    """Rotary embedding and head split in fp64.

    qkv: [B, T, (Hq + 2 Hkv) * d]; positions: int32 [B, T] or None (p = t).
    Returns (q [B,Hq,T,d], k [B,Hkv,T,d], v [B,Hkv,T,d]).
    """
    qkv = np.ascontiguousarray(qkv, dtype=np.float64)
    B, T, width = qkv.shape
    if width % (Hq + 2 * Hkv) != 0:
        raise ValueError("qkv width must be (Hq + 2 Hkv) * d")
    d = width // (Hq + 2 * Hkv)
    pos = None
    if positions is not None:
        pos = np.ascontiguousarray(positions, dtype=np.int32)
        if pos.shape != (B, T):
            raise ValueError("positions must be [B, T]")
    q = np.zeros((B, Hq, T, d))
    k = np.zeros((B, Hkv, T, d))
    v = np.zeros((B, Hkv, T, d))
    lib = lib or load()
    rc = lib.oracle_rope_qkv_f64(_ptr(qkv, ctypes.c_double),
                                 _ptr(pos, ctypes.c_int32) if pos is not None else None,
                                 B, T, Hq, Hkv, d, float(base), _ptr(q, ctypes.c_double),
                                 _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_rope_qkv_f64 failed with code {rc}")
    return q, k, v


def attn_fwd_varlen_f64(q, k, v, cu_seqlens, causal: bool = True, scale: float | None = None,
                        lib: ctypes.CDLL | None = None):
    """Packed variable-length attention in fp64: each sequence attends to
    itself only, with attn_fwd_f64's definition.

    q: [total, Hq, d]; k, v: [total, Hkv, d]; cu_seqlens: [B+1] offsets.
    Returns (O [total, Hq, d], LSE [Hq, total]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    cu = [int(x) for x in np.asarray(cu_seqlens)]
    total, Hq, d = q.shape
    o = np.zeros((total, Hq, d))
    lse = np.zeros((Hq, total))
    for b in range(len(cu) - 1):
        s, e = cu[b], cu[b + 1]
        if e < s or s < 0 or e > total:
            raise ValueError("cu_seqlens out of order or past total")
        if e == s:
            continue
        ob, lb = attn_fwd_f64(q[s:e].transpose(1, 0, 2)[None], k[s:e].transpose(1, 0, 2)[None],
                              v[s:e].transpose(1, 0, 2)[None], causal=causal, scale=scale,
                              lib=lib)
        o[s:e] = ob[0].transpose(1, 0, 2)
        lse[:, s:e] = lb[0]
    return o, lse
