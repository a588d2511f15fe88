"""Exact IO-aware attention for NVIDIA B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI in include/fa.h (libfa_b200.so, built
in-tree by `python exact_io_aware_44_b200/build.py`). It only marshals
arguments: it checks shapes and dtypes, allocates outputs with torch, and
passes raw device pointers and the current CUDA stream. Every step of the
attention path runs in the library's CUDA kernels. There is no CPU fallback:
importing this package fails if the library is missing.

    o, lse = fwd(q, k, v, causal=True)           # bf16 (tensor cores) or fp32
    dq, dk, dv = bwd(q, k, v, o, lse, do, causal=True)

Layouts: q, o, do: [B, Hq, N, d]; k, v: [B, Hkv, N, d]; lse: [B, Hq, N] float32.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = ["head_shard", "fwd", "fwd_fp8", "decode", "decode_raw", "decode_workspace_bytes", "bwd", "fwd_raw", "fwd_fp8_raw", "bwd_raw", "bwd_phases_raw", "workspace_bytes", "get_status", "set_wait_budget_ns",
           "selftest_wait_timeout", "get_progress", "FAError", "LIB_PATH", "lib", "STATUS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")

STATUS = {0: "FA_OK", -1: "FA_ERR_INVALID_ARG", -2: "FA_ERR_UNSUPPORTED", -3: "FA_ERR_ALIGNMENT",
          -4: "FA_ERR_LAUNCH", -5: "FA_ERR_DEVICE_TIMEOUT", -6: "FA_ERR_NO_DEVICE"}

# exported symbols and their C signatures (must match include/fa.h)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_fwd_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _F, _F, _F, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_fwd_e5m2": (_I, [_P, _P, _P, _F, _F, _F, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_bwd_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "fa_decode_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "fa_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_bwd_preprocess": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "fa_bwd_main": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_bwd_convert": (_I, [_P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "fa_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_get_status": (_I, [_P]),
    "fa_get_progress": (_I, [_P, _I, _P]),
    "fa_set_wait_budget_ns": (None, [ctypes.c_uint64]),
    "fa_selftest_wait_timeout": (_I, [ctypes.c_uint64, _P]),
    "fa_error_string": (ctypes.c_char_p, [_I]),
    "fa_version": (_I, []),
}


class FAError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = lib.fa_error_string(code).decode() if lib is not None else STATUS.get(code, "?")
        super().__init__(f"{where}: {STATUS.get(code, code)} ({msg})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python exact_io_aware_44_b200/build.py` "
                          "(there is no CPU fallback)")
    so = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(so, name)
        fn.restype = res
        fn.argtypes = args
    return so


lib = _load()


def _check(code: int, where: str):
    if code != 0:
        raise FAError(code, where)


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _dims(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d):
        raise ValueError(f"k shape {tuple(k.shape)} does not match q shape {tuple(q.shape)}")
    return B, Hq, Hkv, N, d


def _require(t, name, dtype, device):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fwd_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, Hq, Hkv, N, d, causal, scale, stream_ptr, f32=False):
    """The C call itself on raw device pointers (ints); returns the status code."""
    fn = lib.fa_fwd_f32 if f32 else lib.fa_fwd
    return fn(_P(q_ptr), _P(k_ptr), _P(v_ptr), _P(o_ptr), _P(lse_ptr), B, Hq, Hkv, N, d, int(bool(causal)),
              float(scale), _P(stream_ptr))


def fwd(q, k, v, causal: bool = True, scale: float | None = None, out=None, lse=None, stream=None):
    """Forward pass. bf16 inputs run on the tensor cores (d in {64, 128, 256});
    float32 inputs run the fp32 CUDA-core kernel. Returns (o, lse)."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    dtype = q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("q, k, v must be bfloat16 or float32")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, dtype, q.device)
    if v.shape != k.shape:
        raise ValueError("v must have the shape of k")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _require(out, "out", dtype, q.device)
    _require(lse, "lse", torch.float32, q.device)
    fn = lib.fa_fwd_f32 if dtype == torch.float32 else lib.fa_fwd
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d, int(bool(causal)), scale,
              _stream_ptr(stream)), "fa_fwd")
    return out, lse


def fwd_fp8_raw(q_ptr, k_ptr, v_ptr, descale_q, descale_k, descale_v, o_ptr, lse_ptr, B, Hq, Hkv, N, d, causal,
                scale, stream_ptr, e5m2=False):
    """fa_fwd_fp8 (or fa_fwd_e5m2) on raw device pointers (ints); returns the status code."""
    fn = lib.fa_fwd_e5m2 if e5m2 else lib.fa_fwd_fp8
    return fn(_P(q_ptr), _P(k_ptr), _P(v_ptr), float(descale_q), float(descale_k), float(descale_v),
              _P(o_ptr), _P(lse_ptr), B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _P(stream_ptr))


def fwd_fp8(q, k, v, descale_q: float, descale_k: float, descale_v: float, causal: bool = True,
            scale: float | None = None, out=None, lse=None, stream=None):
    """Forward pass on FP8 inputs (torch.float8_e4m3fn or torch.float8_e5m2, all
    three the same, d = 128) with one descale per tensor: the real inputs are
    descale_q * q, descale_k * k, descale_v * v. Returns (o, lse) with o in bf16.
    `scale` defaults to 1/sqrt(d)."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    if q.dtype not in (torch.float8_e4m3fn, torch.float8_e5m2):
        raise TypeError("q, k, v must be torch.float8_e4m3fn or torch.float8_e5m2")
    e5m2 = q.dtype == torch.float8_e5m2
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, q.dtype, q.device)
    if v.shape != k.shape:
        raise ValueError("v must have the shape of k")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.bfloat16, q.device)
    _require(lse, "lse", torch.float32, q.device)
    fn = lib.fa_fwd_e5m2 if e5m2 else lib.fa_fwd_fp8
    _check(fn(_ptr(q), _ptr(k), _ptr(v), float(descale_q), float(descale_k), float(descale_v), _ptr(out),
              _ptr(lse), B, Hq, Hkv, N, d, int(bool(causal)), scale, _stream_ptr(stream)), "fa_fwd_fp8")
    return out, lse


def head_shard(B: int, Hq: int, Hkv: int, rank: int, world: int):
    """The query and key/value heads one rank computes when a problem is split
    across `world` GPUs by heads (no exchange between ranks: every (batch, kv head)
    group is independent in the forward and the backward).

    Heads are counted on the flattened [B * H] axis of the [B, H, N, d] layout, so
    a rank's share is one contiguous slice: query heads [q0, q1) and kv heads
    [k0, k1), cut at GQA group boundaries, with group counts differing by at most
    one between ranks. The slice is a valid problem of its own with B = 1,
    Hq = q1 - q0, Hkv = k1 - k0 (query head i of the slice reads kv head
    i // (Hq / Hkv) of its slice). Returns (q0, q1, k0, k1); an empty slice when
    world exceeds the number of groups."""
    if world < 1 or not 0 <= rank < world or Hkv < 1 or Hq % Hkv:
        raise ValueError("invalid shard request")
    groups, g = B * Hkv, Hq // Hkv
    base, extra = divmod(groups, world)
    k0 = rank * base + min(rank, extra)
    k1 = k0 + base + (1 if rank < extra else 0)
    return k0 * g, k1 * g, k0, k1


def decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_splits=0) -> int:
    return int(lib.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, int(num_splits)))


def decode_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, ws_ptr, B, Hq, Hkv, Nq, Nk, d, causal, scale, num_splits,
               stream_ptr):
    """fa_decode on raw device pointers (ints); returns the status code."""
    return lib.fa_decode(_P(q_ptr), _P(k_ptr), _P(v_ptr), _P(o_ptr), _P(lse_ptr), _P(ws_ptr), B, Hq, Hkv, Nq, Nk,
                         d, int(bool(causal)), float(scale), int(num_splits), _P(stream_ptr))


def decode(q, k, v, causal: bool = True, scale: float | None = None, num_splits: int = 0, out=None, lse=None,
           workspace=None, stream=None):
    """Attention of q [B, Hq, Nq, d] (the last Nq positions) against a key/value
    cache k, v [B, Hkv, Nk, d], all bf16, split along the keys; d = 64 or 128. At
    d = 128 a GQA group's (Hq / Hkv) * Nq query rows form one unit up to 32 rows,
    else blocks of 128 rows (always at d = 64). num_splits = 0: one CTA per SM, each an equal slice of all units'
    128-key chunks; > 0: units * num_splits CTAs. Returns (o, lse)."""
    import torch
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, dk) != (B, d) or v.shape != k.shape:
        raise ValueError("k, v must be [B, Hkv, Nk, d] with q's B and d")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, torch.bfloat16, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_splits)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    _check(lib.fa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(workspace), B, Hq, Hkv, Nq, Nk, d,
                         int(bool(causal)), scale, int(num_splits), _stream_ptr(stream)), "fa_decode")
    return out, lse


def workspace_bytes(B, Hq, Hkv, N, d) -> int:
    return int(lib.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d))


def bwd_raw(q, k, v, o, lse, do, dq, dk, dv, ws, B, Hq, Hkv, N, d, causal, scale, stream_ptr):
    """The C call itself on raw device pointers (ints); returns the status code."""
    return lib.fa_bwd(_P(q), _P(k), _P(v), _P(o), _P(lse), _P(do), _P(dq), _P(dk), _P(dv), _P(ws), B, Hq, Hkv, N,
                      d, int(bool(causal)), float(scale), _P(stream_ptr))


def bwd_phases_raw(q, k, v, o, lse, do, dq, dk, dv, ws, B, Hq, Hkv, N, d, causal, scale, stream_ptr,
                   between=None):
    """fa_bwd as its three C calls (preprocess, main, convert) on raw pointers.
    `between(i)` (optional) is called before phase i = 0, 1, 2 and after the
    last (i = 3), e.g. to record CUDA events on the same stream. Returns the
    first nonzero status code, else 0."""
    c = int(bool(causal))
    st = _P(stream_ptr)
    calls = (lambda: lib.fa_bwd_preprocess(_P(o), _P(do), _P(ws), B, Hq, Hkv, N, d, st),
             lambda: lib.fa_bwd_main(_P(q), _P(k), _P(v), _P(lse), _P(do), _P(dk), _P(dv), _P(ws), B, Hq, Hkv, N, d,
                                     c, float(scale), st),
             lambda: lib.fa_bwd_convert(_P(dq), _P(ws), B, Hq, Hkv, N, d, float(scale), st))
    for i, call in enumerate(calls):
        if between is not None:
            between(i)
        rc = call()
        if rc != 0:
            return rc
    if between is not None:
        between(3)
    return 0


def bwd(q, k, v, o, lse, do, causal: bool = True, scale: float | None = None, workspace=None, out=None,
        stream=None):
    """Backward pass (bf16). Returns (dq, dk, dv)."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _require(t, n, torch.bfloat16, q.device)
    _require(lse, "lse", torch.float32, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nbytes = workspace_bytes(B, Hq, Hkv, N, d)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    elif workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace needs {nbytes} bytes")
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = out
    _check(lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                      _ptr(workspace), B, Hq, Hkv, N, d, int(bool(causal)), scale, _stream_ptr(stream)), "fa_bwd")
    return dq, dk, dv


def get_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(lib.fa_get_status(_stream_ptr(stream)))


def get_progress(n: int, stream=None):
    """Per-CTA progress words of the last forward / backward main-kernel launch
    (see fa_get_progress in include/fa.h), as a list of n ints."""
    buf = (ctypes.c_uint * max(int(n), 0))()
    rc = lib.fa_get_progress(ctypes.cast(buf, ctypes.c_void_p), int(n), _stream_ptr(stream))
    if rc < 0:
        raise FAError(rc, "fa_get_progress")
    return list(buf)[:rc]


def set_wait_budget_ns(ns: int):
    lib.fa_set_wait_budget_ns(int(ns))


def selftest_wait_timeout(budget_ns: int = 10_000_000, stream=None) -> int:
    return int(lib.fa_selftest_wait_timeout(int(budget_ns), _stream_ptr(stream)))
