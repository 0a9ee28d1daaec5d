"""Causal grouped-query FlashAttention forward for B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/tessera_attn.h``; every
step of the computation runs in the CUDA library ``libtessera_attn.so``
built in this directory (``python -m causal_gqa_attention_03_b200.build``).
There is no fallback: if the library is missing, every call raises.

Raw C-ABI names (integer pointers, sizes, stream handle):
    tessera_attn_fwd, tessera_attn_fwd_host, tessera_attn_fwd_host_plan,
    tessera_attn_device_error,
    tessera_status_str, tessera_attn_last_launch_count,
    tessera_attn_selftest_timeout, tessera_attn_bwd, tessera_attn_bwd_workspace_bytes,
    tessera_attn_bwd_workspace_bytes_kv,
    tessera_attn_bwd_noalloc, tessera_attn_bwd_noalloc_max_workspace_bytes,
    tessera_attn_decode, tessera_attn_decode_workspace_bytes, tessera_rmsnorm,
    tessera_rope_qkv, tessera_attn_fwd_varlen
Tensor convenience wrappers (PyTorch used only for memory and streams):
    attn_fwd(q, k, v, causal=True, scale=None, out=None, lse=None, stream=None)
    attn_fwd_host(q, k, v, causal=True, scale=None, out=None, lse=None,
                  staging=None, chunks=0, stream=None)
    attn_bwd(q, k, v, o, lse, dout, causal=True, scale=None, stream=None)
    attn_bwd_noalloc(q, k, v, o, lse, dout, causal=True, scale=None, stream=None)
    attn_decode(q, k_cache, v_cache, block_table, seq_lens, max_seq_len=None,
                scale=None, stream=None)
    rmsnorm(x, w, eps=1e-6, out=None, stream=None)
    rope_qkv(qkv, Hq, Hkv, positions=None, base=10000.0, stream=None)
    attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, causal=True, scale=None, stream=None)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtessera_attn.so")

# Symbols declared in include/tessera_attn.h.
EXPORTED = ("tessera_attn_fwd", "tessera_attn_fwd_host", "tessera_attn_fwd_host_plan",
            "tessera_attn_bwd",
            "tessera_attn_bwd_workspace_bytes", "tessera_attn_bwd_workspace_bytes_kv",
            "tessera_attn_bwd_noalloc",
            "tessera_attn_bwd_noalloc_max_workspace_bytes", "tessera_attn_device_error",
            "tessera_status_str", "tessera_attn_last_launch_count",
            "tessera_attn_selftest_timeout", "tessera_attn_decode",
            "tessera_attn_decode_workspace_bytes", "tessera_rmsnorm", "tessera_rope_qkv",
            "tessera_attn_fwd_varlen")

# Device error code recorded by tessera_attn_selftest_timeout.
DEVICE_ERR_SELFTEST = 9
# Device error code of a decode step given a sequence length or block id out of range.
DEVICE_ERR_DECODE_INPUT = 20
# Device error code of a packed forward given sequence offsets out of range.
DEVICE_ERR_VARLEN_INPUT = 10

STATUS = {0: "TESSERA_OK", 1: "TESSERA_ERR_INVALID_ARG", 2: "TESSERA_ERR_UNSUPPORTED",
          3: "TESSERA_ERR_MISALIGNED", 4: "TESSERA_ERR_CUDA", 5: "TESSERA_ERR_TIMEOUT",
          6: "TESSERA_ERR_TOO_LARGE"}

_lock = threading.Lock()
_lib = None


class TesseraError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({tessera_status_str(status)})")
        self.status = status


def load_library() -> ctypes.CDLL:
    """Load libtessera_attn.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"CUDA library not built: {LIB_PATH} is missing "
                    "(run python -m causal_gqa_attention_03_b200.build)")
            lib = ctypes.CDLL(LIB_PATH)
            vp = ctypes.c_void_p
            ci = ctypes.c_int
            lib.tessera_attn_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci,
                                             ctypes.c_float, vp]
            lib.tessera_attn_fwd.restype = ci
            lib.tessera_attn_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci,
                                                  ci, ci, ci, ci, ctypes.c_float, ci, vp]
            lib.tessera_attn_fwd_host.restype = ci
            lib.tessera_attn_fwd_host_plan.argtypes = [ci, ci, ci, ci, ctypes.POINTER(ci), ci]
            lib.tessera_attn_fwd_host_plan.restype = ci
            lib.tessera_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                             ctypes.c_size_t, ci, ci, ci, ci, ci, ci,
                                             ctypes.c_float, vp]
            lib.tessera_attn_bwd.restype = ci
            lib.tessera_attn_bwd_workspace_bytes.argtypes = [ci, ci, ci, ci]
            lib.tessera_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
            lib.tessera_attn_bwd_workspace_bytes_kv.argtypes = [ci, ci, ci, ci, ci]
            lib.tessera_attn_bwd_workspace_bytes_kv.restype = ctypes.c_size_t
            lib.tessera_attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci,
                                                     ci, ci, ci, ci, ctypes.c_float, vp]
            lib.tessera_attn_bwd_noalloc.restype = ci
            lib.tessera_attn_bwd_noalloc_max_workspace_bytes.argtypes = []
            lib.tessera_attn_bwd_noalloc_max_workspace_bytes.restype = ctypes.c_size_t
            lib.tessera_attn_device_error.argtypes = [ctypes.POINTER(ci)]
            lib.tessera_attn_device_error.restype = ci
            lib.tessera_status_str.argtypes = [ci]
            lib.tessera_status_str.restype = ctypes.c_char_p
            lib.tessera_attn_last_launch_count.argtypes = []
            lib.tessera_attn_last_launch_count.restype = ci
            lib.tessera_attn_selftest_timeout.argtypes = [ctypes.c_uint, vp]
            lib.tessera_attn_selftest_timeout.restype = ci
            lib.tessera_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                                ci, ci, ci, ci, ci, ci, ci, ci, ctypes.c_float, vp]
            lib.tessera_attn_decode.restype = ci
            lib.tessera_attn_decode_workspace_bytes.argtypes = [ci, ci, ci, ci]
            lib.tessera_attn_decode_workspace_bytes.restype = ctypes.c_size_t
            lib.tessera_attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci,
                                                    ci, ci, ctypes.c_float, vp]
            lib.tessera_attn_fwd_varlen.restype = ci
            lib.tessera_rmsnorm.argtypes = [vp, vp, vp, ci, ci, ctypes.c_float, vp]
            lib.tessera_rmsnorm.restype = ci
            lib.tessera_rope_qkv.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci,
                                             ctypes.c_float, vp]
            lib.tessera_rope_qkv.restype = ci
            _lib = lib
    return _lib


def tessera_attn_fwd(q: int, k: int, v: int, o: int, lse: int | None, B: int, Hq: int,
                     Hkv: int, T: int, d: int, causal: int, scale: float,
                     stream: int | None) -> int:
    """The C entry point with integer device pointers; returns the status code."""
    return load_library().tessera_attn_fwd(q, k, v, o, lse or None, B, Hq, Hkv, T, d,
                                           int(causal), float(scale), stream or None)


def tessera_attn_fwd_host(q_h: int, k_h: int, v_h: int, o_h: int, lse_h: int | None, q_d: int,
                          k_d: int, v_d: int, o_d: int, lse_d: int | None, B: int, Hq: int,
                          Hkv: int, T: int, d: int, causal: int, scale: float, chunks: int,
                          stream: int | None) -> int:
    """The pipelined host-buffer C entry point; returns the status code."""
    return load_library().tessera_attn_fwd_host(
        q_h, k_h, v_h, o_h, lse_h or None, q_d, k_d, v_d, o_d, lse_d or None, B, Hq, Hkv, T, d,
        int(causal), float(scale), int(chunks), stream or None)


def tessera_attn_fwd_host_plan(B: int, Hq: int, Hkv: int, chunks: int) -> list:
    """The pieces (s0, s1, h0, h1) tessera_attn_fwd_host cuts a problem into.

    Host only (no CUDA call); raises TesseraError on invalid sizes.
    """
    lib = load_library()
    n = lib.tessera_attn_fwd_host_plan(B, Hq, Hkv, chunks, None, 0)
    if n < 0:
        raise TesseraError(-n, "tessera_attn_fwd_host_plan")
    buf = (ctypes.c_int * (4 * max(n, 1)))()
    lib.tessera_attn_fwd_host_plan(B, Hq, Hkv, chunks, buf, n)
    return [tuple(buf[4 * i:4 * i + 4]) for i in range(n)]


def tessera_attn_bwd(q: int, k: int, v: int, o: int, lse: int, dout: int, dq: int, dk: int,
                     dv: int, workspace: int, workspace_bytes: int, B: int, Hq: int, Hkv: int,
                     T: int, d: int, causal: int, scale: float, stream: int | None) -> int:
    """The backward C entry point with integer device pointers; returns the status."""
    return load_library().tessera_attn_bwd(q, k, v, o, lse or None, dout or None, dq or None,
                                           dk or None, dv or None, workspace or None,
                                           int(workspace_bytes), B, Hq, Hkv, T, d,
                                           int(causal), float(scale), stream or None)


def tessera_attn_bwd_workspace_bytes(B: int, Hq: int, T: int, d: int) -> int:
    return load_library().tessera_attn_bwd_workspace_bytes(B, Hq, T, d)


def tessera_attn_bwd_workspace_bytes_kv(B: int, Hq: int, Hkv: int, T: int, d: int) -> int:
    return load_library().tessera_attn_bwd_workspace_bytes_kv(B, Hq, Hkv, T, d)


def tessera_attn_bwd_noalloc(q: int, k: int, v: int, o: int, lse: int, dout: int, dq: int,
                             dk: int, dv: int, B: int, Hq: int, Hkv: int, T: int, d: int,
                             causal: int, scale: float, stream: int | None) -> int:
    """The backward entry point with the library's own scratch; returns the status."""
    return load_library().tessera_attn_bwd_noalloc(q, k, v, o, lse or None, dout or None,
                                                   dq or None, dk or None, dv or None, B, Hq,
                                                   Hkv, T, d, int(causal), float(scale),
                                                   stream or None)


def tessera_attn_bwd_noalloc_max_workspace_bytes() -> int:
    return load_library().tessera_attn_bwd_noalloc_max_workspace_bytes()


def tessera_attn_decode(q: int, k_cache: int, v_cache: int, block_table: int, seq_lens: int,
                        o: int, lse: int | None, workspace: int | None, workspace_bytes: int,
                        B: int, Hq: int, Hkv: int, d: int, block_size: int, max_blocks: int,
                        num_blocks: int, max_seq_len: int, scale: float,
                        stream: int | None) -> int:
    """The paged-KV decode C entry point with integer device pointers; returns the status."""
    return load_library().tessera_attn_decode(
        q, k_cache, v_cache, block_table, seq_lens, o, lse or None, workspace or None,
        int(workspace_bytes), B, Hq, Hkv, d, block_size, max_blocks, num_blocks, max_seq_len,
        float(scale), stream or None)


def tessera_attn_decode_workspace_bytes(B: int, Hq: int, max_seq_len: int, d: int) -> int:
    return load_library().tessera_attn_decode_workspace_bytes(B, Hq, max_seq_len, d)


def tessera_attn_fwd_varlen(q: int, k: int, v: int, o: int, lse: int | None, cu_seqlens: int,
                            B: int, total: int, max_seqlen: int, Hq: int, Hkv: int, d: int,
                            causal: int, scale: float, stream: int | None) -> int:
    """The packed variable-length forward with integer device pointers; returns the status."""
    return load_library().tessera_attn_fwd_varlen(q or None, k or None, v or None, o or None,
                                                  lse or None, cu_seqlens or None, B, total,
                                                  max_seqlen, Hq, Hkv, d, int(causal),
                                                  float(scale), stream or None)


def tessera_rmsnorm(x: int, w: int, y: int, rows: int, dim: int, eps: float,
                    stream: int | None) -> int:
    """The RMSNorm C entry point with integer device pointers; returns the status."""
    return load_library().tessera_rmsnorm(x or None, w or None, y or None, rows, dim,
                                          float(eps), stream or None)


def tessera_rope_qkv(qkv: int, positions: int | None, q: int, k: int, v: int, B: int, T: int,
                     Hq: int, Hkv: int, d: int, base: float, stream: int | None) -> int:
    """The rotary-embedding C entry point with integer device pointers; returns the status."""
    return load_library().tessera_rope_qkv(qkv or None, positions or None, q or None, k or None,
                                           v or None, B, T, Hq, Hkv, d, float(base),
                                           stream or None)


def tessera_attn_device_error() -> int:
    """Read and clear the device-side error word (synchronises the device)."""
    code = ctypes.c_int(0)
    st = load_library().tessera_attn_device_error(ctypes.byref(code))
    if st != 0:
        raise TesseraError(st, "tessera_attn_device_error")
    return code.value


def tessera_status_str(status: int) -> str:
    return load_library().tessera_status_str(int(status)).decode()


def tessera_attn_last_launch_count() -> int:
    return load_library().tessera_attn_last_launch_count()


def tessera_attn_selftest_timeout(limit_us: int, stream: int | None = None) -> int:
    """Queue the bounded-wait diagnostic (see include/tessera_attn.h); returns the status."""
    return load_library().tessera_attn_selftest_timeout(int(limit_us), stream or None)


def attn_fwd(q, k, v, causal: bool = True, scale: float | None = None, out=None, lse=None,
             stream=None, want_lse: bool = True):
    """Attention forward on CUDA bf16 tensors q [B,Hq,T,d], k/v [B,Hkv,T,d].

    Returns (o, lse): o bf16 [B,Hq,T,d]; lse fp32 [B,Hq,T] (None when
    want_lse is False and no lse buffer is given).  Outputs are allocated with
    torch unless given.  The kernel is queued on ``stream`` (default: torch's
    current stream) and the call does not synchronise.
    """
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA bf16 tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-D tensor [B,H,T,d]")
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (B, Hkv, T, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B,Hkv,T,d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    st = tessera_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          lse.data_ptr() if lse is not None else None, B, Hq, Hkv, T, d,
                          int(bool(causal)), float(scale), stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_attn_fwd")
    return out, lse


def attn_fwd_host(q, k, v, causal: bool = True, scale: float | None = None, out=None, lse=None,
                  staging=None, chunks: int = 0, stream=None, want_lse: bool = True,
                  device=None):
    """Attention forward on host (CPU) bf16 tensors q [B,Hq,T,d], k/v [B,Hkv,T,d].

    The copies to and from the GPU are pipelined with the kernels by the C
    entry point tessera_attn_fwd_host; pinned (page-locked) tensors let them
    overlap.  Returns (o, lse) as host tensors (allocated pinned unless given).
    ``staging`` is a dict with device tensors 'q', 'k', 'v', 'o' and 'lse' of
    the full sizes (allocated with torch when None).  The call synchronises
    ``stream`` (default: torch's current stream) before returning.
    """
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.is_cuda:
            raise TypeError(f"{name} must be a host bf16 tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-D tensor [B,H,T,d]")
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (B, Hkv, T, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B,Hkv,T,d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, pin_memory=True)
    if staging is None:
        staging = {"q": torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                   "k": torch.empty(k.shape, dtype=torch.bfloat16, device=dev),
                   "v": torch.empty(k.shape, dtype=torch.bfloat16, device=dev),
                   "o": torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                   "lse": torch.empty((B, Hq, T), dtype=torch.float32, device=dev)}
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    lse_d = staging["lse"].data_ptr() if lse is not None else None
    st = tessera_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr() if lse is not None else None,
                               staging["q"].data_ptr(), staging["k"].data_ptr(),
                               staging["v"].data_ptr(), staging["o"].data_ptr(), lse_d, B, Hq, Hkv,
                               T, d, int(bool(causal)), float(scale), chunks, stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_attn_fwd_host")
    stream.synchronize()
    return out, lse


def attn_bwd(q, k, v, o, lse, dout, causal: bool = True, scale: float | None = None,
             dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of attn_fwd on CUDA tensors.

    q, o, dout: bf16 [B,Hq,T,d]; k, v: bf16 [B,Hkv,T,d]; lse: fp32 [B,Hq,T]
    from attn_fwd with the same arguments.  Outputs are bf16 and allocated
    with torch unless given; the fp32 workspace likewise (sized by
    tessera_attn_bwd_workspace_bytes_kv, so shapes with few key/value units
    get the balanced dK/dV form).  Queued on ``stream`` (default: torch's
    current stream); does not synchronise.
    """
    import torch

    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA bf16 tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-D tensor [B,H,T,d]")
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (B, Hkv, T, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B,Hkv,T,d] matching q")
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must match q")
    if (not isinstance(lse, torch.Tensor) or lse.dtype != torch.float32 or not lse.is_cuda
            or tuple(lse.shape) != (B, Hq, T) or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous CUDA fp32 tensor [B,Hq,T]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = tessera_attn_bwd_workspace_bytes_kv(B, Hq, Hkv, T, d)
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16) + 3) // 4, dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    st = tessera_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size(), B,
                          Hq, Hkv, T, d, int(bool(causal)), float(scale), stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_attn_bwd")
    return dq, dk, dv


def attn_bwd_noalloc(q, k, v, o, lse, dout, causal: bool = True, scale: float | None = None,
                     dq=None, dk=None, dv=None, stream=None):
    """As attn_bwd, through tessera_attn_bwd_noalloc (no workspace argument)."""
    import torch

    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    st = tessera_attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                  dv.data_ptr(), B, Hq, Hkv, T, d, int(bool(causal)),
                                  float(scale), stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_attn_bwd_noalloc")
    return dq, dk, dv


def attn_decode(q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int | None = None,
                scale: float | None = None, out=None, lse=None, workspace=None, stream=None,
                want_lse: bool = True):
    """One decode step over a paged K/V cache, on CUDA tensors.

    q: bf16 [B,Hq,d]; k_cache, v_cache: bf16 [num_blocks,Hkv,bs,d];
    block_table: int32 [B,max_blocks]; seq_lens: int32 [B] (device);
    max_seq_len: a host-side bound on seq_lens (default: the table's
    capacity max_blocks * bs).  Returns (o bf16 [B,Hq,d], lse fp32 [B,Hq]).
    Queued on ``stream`` (default: torch's current stream); does not synchronise.
    """
    import torch

    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA bf16 tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    for name, t in (("block_table", block_table), ("seq_lens", seq_lens)):
        if (not isinstance(t, torch.Tensor) or t.dtype != torch.int32 or not t.is_cuda
                or not t.is_contiguous()):
            raise TypeError(f"{name} must be a contiguous CUDA int32 tensor")
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B,Hq,d] and the caches [num_blocks,Hkv,bs,d]")
    B, Hq, d = q.shape
    num_blocks, Hkv, bs, dk = k_cache.shape
    if dk != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache must be [num_blocks,Hkv,bs,d] matching q")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table must be [B,max_blocks] and seq_lens [B]")
    max_blocks = block_table.shape[1]
    if max_seq_len is None:
        max_seq_len = max_blocks * bs
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    nbytes = tessera_attn_decode_workspace_bytes(B, Hq, max_seq_len, d)
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16) + 3) // 4, dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    st = tessera_attn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                             block_table.data_ptr(), seq_lens.data_ptr(), out.data_ptr(),
                             lse.data_ptr() if lse is not None else None, workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), B, Hq, Hkv, d, bs,
                             max_blocks, num_blocks, int(max_seq_len), float(scale),
                             stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_attn_decode")
    return out, lse


def rmsnorm(x, w, eps: float = 1e-6, out=None, stream=None):
    """RMSNorm over the last dimension of a CUDA bf16 tensor x with weight w
    (bf16 [dim]).  Returns out (allocated unless given; may be x itself)."""
    import torch

    for name, t in (("x", x), ("w", w)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA bf16 tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    dim = x.shape[-1]
    if tuple(w.shape) != (dim,):
        raise ValueError("w must be [dim]")
    if out is None:
        out = torch.empty_like(x)
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    st = tessera_rmsnorm(x.data_ptr(), w.data_ptr(), out.data_ptr(), x.numel() // dim, dim,
                         float(eps), stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_rmsnorm")
    return out


def rope_qkv(qkv, Hq: int, Hkv: int, positions=None, base: float = 10000.0, q=None, k=None,
             v=None, stream=None):
    """Rotary embedding and head split of a CUDA bf16 projection output
    qkv [B, T, (Hq + 2 Hkv) d]; positions int32 [B, T] or None (p = t).
    Returns (q [B,Hq,T,d], k [B,Hkv,T,d], v [B,Hkv,T,d])."""
    import torch

    if not isinstance(qkv, torch.Tensor) or qkv.dtype != torch.bfloat16 or not qkv.is_cuda:
        raise TypeError("qkv must be a CUDA bf16 tensor")
    if qkv.dim() != 3 or not qkv.is_contiguous():
        raise ValueError("qkv must be a contiguous [B, T, (Hq + 2 Hkv) d] tensor")
    B, T, width = qkv.shape
    if width % (Hq + 2 * Hkv) != 0:
        raise ValueError("qkv width must be (Hq + 2 Hkv) * d")
    d = width // (Hq + 2 * Hkv)
    if positions is not None:
        if (not isinstance(positions, torch.Tensor) or positions.dtype != torch.int32
                or not positions.is_cuda or tuple(positions.shape) != (B, T)
                or not positions.is_contiguous()):
            raise ValueError("positions must be a contiguous CUDA int32 [B, T] tensor")
    dev = qkv.device
    q = torch.empty((B, Hq, T, d), dtype=torch.bfloat16, device=dev) if q is None else q
    k = torch.empty((B, Hkv, T, d), dtype=torch.bfloat16, device=dev) if k is None else k
    v = torch.empty((B, Hkv, T, d), dtype=torch.bfloat16, device=dev) if v is None else v
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    st = tessera_rope_qkv(qkv.data_ptr(), positions.data_ptr() if positions is not None else None,
                          q.data_ptr(), k.data_ptr(), v.data_ptr(), B, T, Hq, Hkv, d,
                          float(base), stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_rope_qkv")
    return q, k, v


def attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen: int, causal: bool = True,
                    scale: float | None = None, out=None, lse=None, stream=None,
                    want_lse: bool = True):
    """Forward over packed sequences: q [total, Hq, d], k/v [total, Hkv, d]
    (CUDA bf16), cu_seqlens CUDA int32 [B+1], max_seqlen a host bound on the
    lengths.  Returns (o [total, Hq, d], lse [Hq, total] fp32 or None)."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA bf16 tensor")
        if t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [total, H, d] tensor")
    if (not isinstance(cu_seqlens, torch.Tensor) or cu_seqlens.dtype != torch.int32
            or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous()):
        raise TypeError("cu_seqlens must be a contiguous CUDA int32 [B+1] tensor")
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (total, Hkv, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [total, Hkv, d] matching q")
    B = cu_seqlens.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    st = tessera_attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr() if lse is not None else None,
                                 cu_seqlens.data_ptr(), B, total, int(max_seqlen), Hq, Hkv, d,
                                 int(bool(causal)), float(scale), stream.cuda_stream)
    if st != 0:
        raise TesseraError(st, "tessera_attn_fwd_varlen")
    return out, lse
