"""token_sparse_attention_sm_b200: shared-routing token-sparse decode
attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libsparse_decode.so`` (declared in
``include/sparse_decode.h``).  It only marshals arguments: every step of the
path -- scoring, selection, gather attention, split merge -- runs in the
library's CUDA kernels.  PyTorch provides device memory and the current
stream.  There is no CPU or PyTorch fallback: if the library is missing,
every call raises.

What is computed (CLSA article, sections 研究の背景と課題 and CLSAの仕組み;
Louver summary, sections 問題定義 and 1. 半空間範囲検索への帰着): one routing
pass scores every cached key with the GQA-group-summed q.k/sqrt(d), keeps the
top-k (ties to the lower index) or every key with score >= tau, and every
layer then attends over only that one shared set.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

__all__ = ["SparseDecodeError", "lib_path", "load", "score", "select_topk",
           "select_threshold", "route_topk", "route_threshold", "attn_gather",
           "decode_step", "read_device_status", "workspace_bytes",
           "Workspace", "STATUS_NAMES", "EXPORTED_SYMBOLS", "decode_step_grouped",
           "kv_append", "LouverIndex", "louver_build", "louver_route_threshold",
           "DecodeStepGraph", "selftest_bounded_wait", "louver_decode_step",
           "device_usable", "read_device_flags", "FLAG_SLOW_SELECT"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_FILE = os.path.join(_PKG, "libsparse_decode.so")

STATUS_NAMES = {
    0: "SPARSE_OK", 1: "SPARSE_ERR_INVALID_ARG", 2: "SPARSE_ERR_UNSUPPORTED",
    3: "SPARSE_ERR_WORKSPACE", 4: "SPARSE_ERR_CAPACITY",
    5: "SPARSE_ERR_NONFINITE", 6: "SPARSE_ERR_CUDA", 7: "SPARSE_ERR_TIMEOUT",
    8: "SPARSE_ERR_INDEX", 9: "SPARSE_ERR_INTERNAL",
}

EXPORTED_SYMBOLS = (
    "sparse_status_string", "sparse_version", "sparse_workspace_size",
    "sparse_workspace_init", "sparse_score", "sparse_select_topk",
    "sparse_select_threshold", "sparse_route_topk", "sparse_route_threshold",
    "sparse_attn_gather", "sparse_decode_step", "sparse_read_device_status",
    "sparse_route_topk_static", "sparse_decode_step_grouped", "sparse_kv_append",
    "sparse_louver_sizes", "sparse_louver_build", "sparse_louver_route_threshold",
    "sparse_selftest_bounded_wait", "sparse_louver_decode_step",
    "sparse_pointer_device_usable", "sparse_graph_launch", "sparse_decode_step_join",
    "sparse_decode_step_fused", "sparse_graph_upload",
)

DTYPE_CODES = {torch.float32: 0, torch.bfloat16: 1}


class SparseDecodeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("N", ctypes.c_int32),
                ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("n_cap", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def lib_path() -> str:
    return _LIB_FILE


def load():
    """Load libsparse_decode.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_FILE):
            raise RuntimeError(
                f"CUDA library not built: {_LIB_FILE} is missing "
                "(run `python -m token_sparse_attention_sm_b200.build`)")
        lib = ctypes.CDLL(_LIB_FILE)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        SH = ctypes.POINTER(_Shape)
        sigs = {
            "sparse_status_string": (ctypes.c_char_p, [I32]),
            "sparse_version": (I32, []),
            "sparse_workspace_size": (I32, [SH, I32, I32, ctypes.POINTER(SZ)]),
            "sparse_workspace_init": (I32, [P, SZ, P]),
            "sparse_score": (I32, [SH, P, P, P, P, SZ, P]),
            "sparse_select_topk": (I32, [SH, P, I32, P, P, SZ, P]),
            "sparse_select_threshold": (I32, [SH, P, P, I32, P, P, P, SZ, P]),
            "sparse_route_topk": (I32, [SH, P, P, I32, P, P, SZ, P]),
            "sparse_route_threshold": (I32, [SH, P, P, P, I32, P, P, P, SZ, P]),
            "sparse_attn_gather": (I32, [SH, I32, P, P, P, P, I32, P, P, P, P,
                                         SZ, P]),
            "sparse_decode_step": (I32, [SH, I32, P, P, P, P, I32, P, I32, P, P,
                                         P, P, P, SZ, P]),
            "sparse_decode_step_join": (I32, [SH, I32, P, P, P, P, I32, P, I32, P, P,
                                              P, P, P, SZ, P, P]),
            "sparse_decode_step_fused": (I32, [SH, I32, I32, I32, ctypes.POINTER(I32)]),
            "sparse_read_device_status": (I32, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
            "sparse_route_topk_static": (I32, [SH, P, P, I32, P, P]),
            "sparse_decode_step_grouped": (I32, [SH, I32, I32, P, P, P, P, I32, P, I32,
                                                 P, P, P, P, P, SZ, P]),
            "sparse_kv_append": (I32, [SH, P, P, P, P, P]),
            "sparse_louver_sizes": (I32, [SH, I32, ctypes.POINTER(SZ), ctypes.POINTER(SZ)]),
            "sparse_selftest_bounded_wait": (I32, [P, SZ, ctypes.c_uint64, P]),
            "sparse_louver_decode_step": (I32, [SH, I32, P, P, P, P, P, SZ, I32, P, I32, P, P,
                                                P, P, P, SZ, P, SZ, P]),
            "sparse_louver_build": (I32, [SH, P, I32, P, SZ, P, SZ, P]),
            "sparse_louver_route_threshold": (I32, [SH, P, P, SZ, I32, P, I32, P, P, P, P,
                                                    SZ, P]),
            "sparse_pointer_device_usable": (I32, [P, ctypes.POINTER(I32)]),
            "sparse_graph_launch": (I32, [P, P]),
            "sparse_graph_upload": (I32, [P, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _check(rc: int, what: str):
    if rc != 0:
        raise SparseDecodeError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _shape(B, N, Hq, Hkv, d, dtype, n_cap: int = 0) -> _Shape:
    if dtype not in DTYPE_CODES:
        raise TypeError(f"unsupported dtype {dtype}")
    return _Shape(B, N, Hq, Hkv, d, DTYPE_CODES[dtype], int(n_cap))


def _length(n_cap: int, n: int | None) -> int:
    """Cache length in use: n (1 <= n <= rows allocated) or all rows."""
    if n is None:
        return n_cap
    n = int(n)
    if not 1 <= n <= n_cap:
        raise ValueError(f"cache length n={n} outside [1, {n_cap}]")
    return n


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")


def device_usable(t) -> bool:
    """True when kernels can write t at its own address: a CUDA tensor, or a
    pinned host tensor mapped into the device's address space."""
    if t.is_cuda:
        return True
    if not t.is_pinned():
        return False
    ok = ctypes.c_int32(0)
    _check(load().sparse_pointer_device_usable(_ptr(t), ctypes.byref(ok)),
           "pointer_device_usable")
    return bool(ok.value)


def _need_result(t, shape, dtype, name: str, host_ok: bool = False):
    """A caller-given result tensor (if any) must have exactly this shape and
    dtype, be contiguous, and be device memory -- or, where host_ok, pinned
    host memory mapped into the device's address space -- since the kernels
    write all of it."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.is_cuda or (host_ok and device_usable(t)):
        return
    raise ValueError(f"{name} must be a CUDA tensor" +
                     (" or pinned host memory the device can reach at its own address"
                      if host_ok else ""))


def _need_tau(tau, shape):
    """tau holds one threshold per row of the sets: exactly this shape, real."""
    if tuple(tau.shape) != tuple(shape) or not tau.is_floating_point():
        raise ValueError(f"tau must be a float tensor of shape {tuple(shape)}, "
                         f"got {tau.dtype} {tuple(tau.shape)}")


def _need_out(out, like):
    """out (if given) must have like's shape and dtype, be contiguous, and be
    device memory or mapped pinned host memory (the attention then writes the
    results straight to the host)."""
    _need_result(out, like.shape, like.dtype, "out", host_ok=True)


def workspace_bytes(B, N, Hq, Hkv, d, dtype, k_or_cap: int, L: int) -> int:
    n = ctypes.c_size_t(0)
    sh = _shape(B, N, Hq, Hkv, d, dtype)
    _check(load().sparse_workspace_size(ctypes.byref(sh), int(k_or_cap), int(L),
                                        ctypes.byref(n)), "workspace_size")
    return int(n.value)


class Workspace:
    """A zero-initialised device workspace that grows on demand.  Calls that
    share one must be ordered on the same stream.  Growing replaces the
    buffer: a CUDA graph captured earlier keeps using the old one, so whoever
    holds such a graph also holds a reference to the buffer it captured
    (DecodeStepGraph does)."""

    def __init__(self, device=None):
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8,
                                   device=self.device)
        return self.buf


_default_ws = {}


def _ws(ws: Workspace | None, device) -> Workspace:
    if ws is not None:
        return ws
    key = torch.device(device).index
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


FLAG_SLOW_SELECT = 1 << 8  # informational: a top-k select took its exact streaming path


def read_device_flags(ws: Workspace) -> int:
    """Synchronise the current stream, read (and reset) the device status
    word of ``ws`` and return its raw bits without raising: the error flags
    (NONFINITE 1, CAPACITY 2, TIMEOUT 4, INDEX 8, INTERNAL 16) and the
    informational FLAG_SLOW_SELECT."""
    flags = ctypes.c_uint32(0)
    load().sparse_read_device_status(_ptr(ws.buf), _stream(), ctypes.byref(flags))
    return int(flags.value)


def read_device_status(ws: Workspace, raise_on_error: bool = True) -> int:
    """Synchronise the current stream and read (and reset) the device status
    word of ``ws``; raises SparseDecodeError unless it is SPARSE_OK."""
    flags = ctypes.c_uint32(0)
    rc = load().sparse_read_device_status(_ptr(ws.buf), _stream(), ctypes.byref(flags))
    if raise_on_error:
        _check(rc, f"device status (flags=0x{flags.value:x})")
    return rc


def selftest_bounded_wait(ws: Workspace, limit_ns: int = 50_000_000) -> int:
    """Run the bounded-wait self-test on ws (a wait nothing satisfies, given
    up after limit_ns) and return the device status it leaves: expected
    SPARSE_ERR_TIMEOUT (7).  Resets the status word."""
    buf = ws.get(1 << 20)
    _check(load().sparse_selftest_bounded_wait(_ptr(buf), buf.numel(), int(limit_ns),
                                               _stream()), "selftest_bounded_wait")
    return read_device_status(ws, raise_on_error=False)


def _dims_qk(q, K):
    if q.dim() != 3 or K.dim() != 4:
        raise ValueError("q must be [B,Hq,d] and K [B,Hkv,N,d]")
    B, Hq, d = q.shape
    Bk, Hkv, N, dk = K.shape
    if Bk != B or dk != d:
        raise ValueError("q and K disagree on B or d")
    if q.dtype != K.dtype:
        raise ValueError("q and K must share a dtype")
    return B, N, Hq, Hkv, d


def score(q, K, ws: Workspace | None = None, check: bool = True, out=None,
          n: int | None = None):
    """Routing scores S [B,Hkv,N] fp32 (written into ``out`` if given).  K may
    hold more rows than the cache length n (default: all rows)."""
    _need_cuda(q, K, out)
    B, Ncap, Hq, Hkv, d = _dims_qk(q, K)
    N = _length(Ncap, n)
    _need_result(out, (B, Hkv, N), torch.float32, "out")
    w = _ws(ws, q.device)
    sh = _shape(B, N, Hq, Hkv, d, q.dtype, Ncap)
    buf = w.get(workspace_bytes(B, N, Hq, Hkv, d, q.dtype, 1, 1))
    S = torch.empty((B, Hkv, N), dtype=torch.float32, device=q.device) if out is None else out
    _check(load().sparse_score(ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(S),
                               _ptr(buf), buf.numel(), _stream()), "score")
    if check:
        read_device_status(w)
    return S


def select_topk(S, k: int, ws: Workspace | None = None, check: bool = True,
                idx=None):
    """Top-k of S [B,Hkv,N] fp32 -> idx [B,Hkv,k] int32 ascending."""
    _need_cuda(S, idx)
    B, Hkv, N = S.shape
    _need_result(idx, (B, Hkv, k), torch.int32, "idx")
    w = _ws(ws, S.device)
    sh = _shape(B, N, Hkv, Hkv, 64, torch.float32)
    buf = w.get(workspace_bytes(B, N, Hkv, Hkv, 64, torch.float32, k, 1))
    if idx is None:
        idx = torch.empty((B, Hkv, k), dtype=torch.int32, device=S.device)
    _check(load().sparse_select_topk(ctypes.byref(sh), _ptr(S), int(k), _ptr(idx),
                                     _ptr(buf), buf.numel(), _stream()),
           "select_topk")
    if check:
        read_device_status(w)
    return idx


def _threshold_outputs(idx, count, B, Hkv, cap, device):
    """idx [B,Hkv,cap] and count [B,Hkv] int32: the given ones (checked) or
    new ones."""
    if idx is None:
        idx = torch.empty((B, Hkv, cap), dtype=torch.int32, device=device)
    if count is None:
        count = torch.empty((B, Hkv), dtype=torch.int32, device=device)
    _need_cuda(idx, count)
    if (idx.shape != (B, Hkv, cap) or count.shape != (B, Hkv) or idx.dtype != torch.int32
            or count.dtype != torch.int32):
        raise ValueError("idx must be int32 [B,Hkv,cap] and count int32 [B,Hkv]")
    return idx, count


def select_threshold(S, tau, cap: int, ws: Workspace | None = None,
                     check: bool = True, idx=None, count=None):
    """Threshold sets of S: (idx [B,Hkv,cap], count [B,Hkv])."""
    _need_cuda(S, tau)
    B, Hkv, N = S.shape
    _need_tau(tau, (B, Hkv))
    w = _ws(ws, S.device)
    sh = _shape(B, N, Hkv, Hkv, 64, torch.float32)
    buf = w.get(workspace_bytes(B, N, Hkv, Hkv, 64, torch.float32, cap, 1))
    idx, count = _threshold_outputs(idx, count, B, Hkv, cap, S.device)
    _check(load().sparse_select_threshold(
        ctypes.byref(sh), _ptr(S), _ptr(tau.float().contiguous()), int(cap),
        _ptr(idx), _ptr(count), _ptr(buf), buf.numel(), _stream()),
        "select_threshold")
    if check:
        read_device_status(w)
    return idx, count


def route_topk(q, K, k: int, ws: Workspace | None = None, check: bool = True,
               idx=None, n: int | None = None):
    """Shared routing (top-k): idx [B,Hkv,k] int32 ascending, over the first n
    cache rows (default: all rows of K)."""
    _need_cuda(q, K, idx)
    B, Ncap, Hq, Hkv, d = _dims_qk(q, K)
    N = _length(Ncap, n)
    _need_result(idx, (B, Hkv, k), torch.int32, "idx")
    w = _ws(ws, q.device)
    sh = _shape(B, N, Hq, Hkv, d, q.dtype, Ncap)
    buf = w.get(workspace_bytes(B, N, Hq, Hkv, d, q.dtype, k, 1))
    if idx is None:
        idx = torch.empty((B, Hkv, k), dtype=torch.int32, device=q.device)
    _check(load().sparse_route_topk(ctypes.byref(sh), _ptr(q), _ptr(K), int(k),
                                    _ptr(idx), _ptr(buf), buf.numel(), _stream()),
           "route_topk")
    if check:
        read_device_status(w)
    return idx


def route_threshold(q, K, tau, cap: int, ws: Workspace | None = None,
                    check: bool = True, n: int | None = None, idx=None, count=None):
    """Shared routing (threshold): (idx [B,Hkv,cap], count [B,Hkv]), over the
    first n cache rows (default: all rows of K)."""
    _need_cuda(q, K, tau)
    B, Ncap, Hq, Hkv, d = _dims_qk(q, K)
    N = _length(Ncap, n)
    w = _ws(ws, q.device)
    sh = _shape(B, N, Hq, Hkv, d, q.dtype, Ncap)
    buf = w.get(workspace_bytes(B, N, Hq, Hkv, d, q.dtype, cap, 1))
    idx, count = _threshold_outputs(idx, count, B, Hkv, cap, q.device)
    _need_tau(tau, (B, Hkv))
    tau = tau.float().contiguous()
    _check(load().sparse_route_threshold(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(tau), int(cap), _ptr(idx),
        _ptr(count), _ptr(buf), buf.numel(), _stream()), "route_threshold")
    if check:
        read_device_status(w)
    return idx, count


def attn_gather(q, K, V, idx, count=None, ws: Workspace | None = None,
                check: bool = True, return_lse: bool = True, out=None, lse=None,
                n: int | None = None):
    """Attention of q ([B,Hq,d] or [L,B,Hq,d]) over the idx rows
    [B,Hkv,stride] (first count[b,h] of each row if count is given).
    Returns (out, lse) with out shaped like q."""
    _need_cuda(q, K, V, idx, count)
    _need_out(out, q)
    _need_result(lse, q.shape[:-1], torch.float32, "lse", host_ok=True)
    single = q.dim() == 3
    q4 = q.unsqueeze(0) if single else q
    L, B, Hq, d = q4.shape
    Bk, Hkv, Ncap, dk = K.shape
    N = _length(Ncap, n)
    if V.shape != K.shape or Bk != B or dk != d:
        raise ValueError("shape mismatch between q, K and V")
    if idx.dtype != torch.int32 or idx.dim() != 3 or idx.shape[:2] != (B, Hkv):
        raise ValueError("idx must be int32 [B,Hkv,stride]")
    _need_result(count, (B, Hkv), torch.int32, "count")
    stride = idx.shape[2]
    w = _ws(ws, q.device)
    sh = _shape(B, N, Hq, Hkv, d, q.dtype, Ncap)
    buf = w.get(workspace_bytes(B, N, Hq, Hkv, d, q.dtype, stride, L))
    if out is None:
        out = torch.empty_like(q4)
    elif single:
        out = out.unsqueeze(0)
    if lse is None and return_lse:
        lse = torch.empty((L, B, Hq), dtype=torch.float32, device=q.device)
    elif lse is not None and single:
        lse = lse.unsqueeze(0)
    _check(load().sparse_attn_gather(
        ctypes.byref(sh), L, _ptr(q4), _ptr(K), _ptr(V), _ptr(idx), stride,
        _ptr(count), _ptr(out), _ptr(lse), _ptr(buf), buf.numel(), _stream()),
        "attn_gather")
    if check:
        read_device_status(w)
    if single:
        return out[0], (lse[0] if lse is not None else None)
    return out, lse


def decode_step_fused(B: int, N: int, Hq: int, Hkv: int, d: int, dtype, L: int,
                      k: int | None = None, cap: int | None = None) -> bool:
    """Whether decode_step on this shape (top-k with ``k``, threshold with
    ``cap``) runs on the fused kernels (the routing scan, then one kernel
    that selects and attends), where idx, count and out are write-only."""
    topk = k is not None
    sh = _shape(B, N, Hq, Hkv, d, dtype)
    f = ctypes.c_int32(0)
    _check(load().sparse_decode_step_fused(ctypes.byref(sh), int(L), int(k) if topk else 0,
                                           0 if topk else int(cap), ctypes.byref(f)),
           "decode_step_fused")
    return bool(f.value)


def decode_step(q_route, q_layers, K, V, k: int | None = None, tau=None,
                cap: int | None = None, ws: Workspace | None = None,
                check: bool = True, out=None, idx=None, count=None, lse=None,
                return_lse: bool = True, n: int | None = None, layers_ready=None):
    """One fused decode step: route once, attend L layers over that set.

    Top-k mode with ``k``; threshold mode with ``tau`` [B,Hkv] and ``cap``.
    The cache is the first n rows of K and V (default: all rows).
    Returns dict(idx, count, out, lse).  Preallocated outputs may be passed
    to keep a timing loop free of allocations.  ``layers_ready`` (a
    torch.cuda.Event): the attention waits for it, the routing does not --
    for q_layers still being copied on another stream.  When the step runs
    on the fused kernels (decode_step_fused), idx and count may also be
    mapped pinned host memory (they are only written)."""
    _need_cuda(q_route, q_layers, K, V, tau)
    B, Ncap, Hq, Hkv, d = _dims_qk(q_route, K)
    N = _length(Ncap, n)
    L = q_layers.shape[0]
    if q_layers.shape != (L, B, Hq, d) or V.shape != K.shape:
        raise ValueError("q_layers must be [L,B,Hq,d] and V like K")
    _need_out(out, q_layers)
    topk = k is not None
    if topk == (tau is not None):
        raise ValueError("give exactly one of k or tau")
    stride = int(k) if topk else int(cap)
    fused = decode_step_fused(B, N, Hq, Hkv, d, q_route.dtype, L, k=k if topk else None,
                              cap=None if topk else cap)
    _need_result(idx, (B, Hkv, stride), torch.int32, "idx", host_ok=fused)
    if not topk:
        _need_result(count, (B, Hkv), torch.int32, "count", host_ok=fused)
    _need_result(lse, (L, B, Hq), torch.float32, "lse", host_ok=True)
    if not topk:
        _need_tau(tau, (B, Hkv))
    dev = q_route.device
    w = _ws(ws, dev)
    sh = _shape(B, N, Hq, Hkv, d, q_route.dtype, Ncap)
    buf = w.get(workspace_bytes(B, N, Hq, Hkv, d, q_route.dtype, stride, L))
    if idx is None:
        idx = torch.empty((B, Hkv, stride), dtype=torch.int32, device=dev)
    if count is None and not topk:
        count = torch.empty((B, Hkv), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty_like(q_layers)
    if lse is None and return_lse:
        lse = torch.empty((L, B, Hq), dtype=torch.float32, device=dev)
    tau_t = None if topk else tau.float().contiguous()
    ev = None if layers_ready is None else ctypes.c_void_p(layers_ready.cuda_event)
    _check(load().sparse_decode_step_join(
        ctypes.byref(sh), L, _ptr(q_route), _ptr(q_layers), _ptr(K), _ptr(V),
        int(k) if topk else 0, _ptr(tau_t), 0 if topk else int(cap), _ptr(idx),
        _ptr(count), _ptr(out), _ptr(lse), _ptr(buf), buf.numel(), _stream(), ev),
        "decode_step")
    if check:
        read_device_status(w)
    return {"idx": idx, "count": count, "out": out, "lse": lse}


def decode_step_grouped(q_routes, q_layers, K, V, R: int, k: int | None = None, tau=None,
                        cap: int | None = None, ws: Workspace | None = None,
                        check: bool = True, out=None, idx=None, count=None, lse=None,
                        return_lse: bool = True, n: int | None = None):
    """Decode step re-routing every R layers (sparse_decode_step_grouped).

    q_routes [ceil(L/R),B,Hq,d]: group g of R consecutive layers routes with
    q_routes[g].  Top-k mode with ``k``; threshold mode with ``tau``
    [ceil(L/R),B,Hkv] and ``cap``.  Returns dict(idx [ngroups,B,Hkv,stride],
    count, out [L,B,Hq,d], lse [L,B,Hq])."""
    _need_cuda(q_routes, q_layers, K, V, tau)
    if q_routes.dim() != 4 or K.dim() != 4:
        raise ValueError("q_routes must be [ngroups,B,Hq,d] and K [B,Hkv,N,d]")
    B, Ncap, Hq, Hkv, d = _dims_qk(q_routes[0], K)
    N = _length(Ncap, n)
    L = q_layers.shape[0]
    R = int(R)
    if R < 1:
        raise ValueError("R must be >= 1")
    ng = (L + R - 1) // R
    if q_routes.shape[0] != ng or q_layers.shape != (L, B, Hq, d) or V.shape != K.shape:
        raise ValueError("q_routes must be [ceil(L/R),B,Hq,d], q_layers [L,B,Hq,d], V like K")
    _need_out(out, q_layers)
    topk = k is not None
    if topk == (tau is not None):
        raise ValueError("give exactly one of k or tau")
    stride = int(k) if topk else int(cap)
    _need_result(idx, (ng, B, Hkv, stride), torch.int32, "idx")
    if not topk:
        _need_result(count, (ng, B, Hkv), torch.int32, "count")
    _need_result(lse, (L, B, Hq), torch.float32, "lse", host_ok=True)
    if not topk:
        _need_tau(tau, (ng, B, Hkv))
    dev = q_routes.device
    w = _ws(ws, dev)
    sh = _shape(B, N, Hq, Hkv, d, q_routes.dtype, Ncap)
    buf = w.get(workspace_bytes(B, N, Hq, Hkv, d, q_routes.dtype, stride, min(R, L)))
    if idx is None:
        idx = torch.empty((ng, B, Hkv, stride), dtype=torch.int32, device=dev)
    if count is None and not topk:
        count = torch.empty((ng, B, Hkv), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty_like(q_layers)
    if lse is None and return_lse:
        lse = torch.empty((L, B, Hq), dtype=torch.float32, device=dev)
    tau_t = None if topk else tau.float().contiguous()
    _check(load().sparse_decode_step_grouped(
        ctypes.byref(sh), L, R, _ptr(q_routes), _ptr(q_layers), _ptr(K), _ptr(V),
        int(k) if topk else 0, _ptr(tau_t), 0 if topk else int(cap), _ptr(idx),
        _ptr(count), _ptr(out), _ptr(lse), _ptr(buf), buf.numel(), _stream()),
        "decode_step_grouped")
    if check:
        read_device_status(w)
    return {"idx": idx, "count": count, "out": out, "lse": lse}


def kv_append(K, V, k_new, v_new, n: int):
    """Write the new token's key and value rows k_new, v_new [B,Hkv,d] as row
    n-1 of every (sequence, KV head) of K and V [B,Hkv,n_cap,d] (n <= n_cap:
    the cache length including the new token), on the current stream."""
    _need_cuda(K, V, k_new, v_new)
    if K.dim() != 4 or V.shape != K.shape:
        raise ValueError("K and V must be [B,Hkv,n_cap,d] of one shape")
    B, Hkv, Ncap, d = K.shape
    N = _length(Ncap, n)
    if k_new.shape != (B, Hkv, d) or v_new.shape != (B, Hkv, d):
        raise ValueError("k_new and v_new must be [B,Hkv,d]")
    if not (k_new.dtype == v_new.dtype == K.dtype == V.dtype):
        raise ValueError("K, V, k_new and v_new must share a dtype")
    sh = _shape(B, N, Hkv, Hkv, d, K.dtype, Ncap)
    _check(load().sparse_kv_append(ctypes.byref(sh), _ptr(K), _ptr(V), _ptr(k_new),
                                   _ptr(v_new), _stream()), "kv_append")


class LouverIndex:
    """A Louver index over the first n rows of one K cache [B,Hkv,n_cap,d]:
    the device index buffer and the index's own workspace (which no other
    call may share)."""

    def __init__(self, K, r: int, n: int):
        B, Hkv, Ncap, d = K.shape
        self.B, self.Hkv, self.N, self.Ncap, self.d = B, Hkv, n, Ncap, d
        self.dtype, self.r, self.device = K.dtype, int(r), K.device
        ib, wb = ctypes.c_size_t(0), ctypes.c_size_t(0)
        sh = _shape(B, n, Hkv, Hkv, d, K.dtype, Ncap)
        _check(load().sparse_louver_sizes(ctypes.byref(sh), self.r, ctypes.byref(ib),
                                          ctypes.byref(wb)), "louver_sizes")
        self.index = torch.empty(int(ib.value), dtype=torch.uint8, device=K.device)
        last = self._parts()["leaf_radii"]
        if last[0] + last[3] > self.index.numel():
            raise RuntimeError("index layout does not match the library's")
        self.ws = Workspace(K.device)
        self.ws_bytes = int(wb.value)
        self.ws.get(self.ws_bytes)

    def _parts(self):
        """(offset, dtype, shape) of each part of the index buffer, in the
        library's layout: each part at the next 256-byte boundary."""
        BH, N, d, nc = self.B * self.Hkv, self.N, self.d, self.N // self.r
        shapes = [("perm", torch.int32, (self.B, self.Hkv, N)),
                  ("centres", torch.float32, (self.B, self.Hkv, nc, d)),
                  ("radii", torch.float32, (self.B, self.Hkv, nc)),
                  ("keys", self.dtype, (self.B, self.Hkv, N, d)),
                  ("leaf_centres", torch.float32, (self.B, self.Hkv, N // 32, d)),
                  ("leaf_radii", torch.float32, (self.B, self.Hkv, N // 32))]
        parts, off = {}, 0
        for name, dt, shape in shapes:
            size = int(np.prod(shape)) * torch.tensor([], dtype=dt).element_size()
            parts[name] = (off, dt, shape, size)
            off += (size + 255) // 256 * 256
        return parts

    def _view(self, name):
        off, dt, shape, size = self._parts()[name]
        return self.index[off:off + size].view(dt).view(shape)

    def perm(self):
        """Key ids in cluster order, [B,Hkv,N] int32 (cluster c of head bh is
        perm[bh][c*r .. c*r+r), leaf l is perm[bh][32*l .. 32*l+32))."""
        return self._view("perm")

    def centres(self):
        """Cluster centres, [B,Hkv,N/r,d] fp32."""
        return self._view("centres")

    def radii(self):
        """Cluster radii, [B,Hkv,N/r] fp32."""
        return self._view("radii")

    def keys(self):
        """Cluster-ordered key rows, [B,Hkv,N,d] (row p of head bh is key
        perm[bh][p])."""
        return self._view("keys")

    def leaf_centres(self):
        """Centres of the 32-key leaves, [B,Hkv,N/32,d] fp32."""
        return self._view("leaf_centres")

    def leaf_radii(self):
        """Radii of the 32-key leaves, [B,Hkv,N/32] fp32."""
        return self._view("leaf_radii")


def louver_build(K, r: int, n: int | None = None, check: bool = True) -> LouverIndex:
    """Build the Louver index (balanced PCA tree, clusters of r keys, bounding
    balls) over the first n rows of K [B,Hkv,n_cap,d] on the current stream."""
    _need_cuda(K)
    if K.dim() != 4:
        raise ValueError("K must be [B,Hkv,n_cap,d]")
    N = _length(K.shape[2], n)
    ix = LouverIndex(K, r, N)
    sh = _shape(ix.B, N, ix.Hkv, ix.Hkv, ix.d, K.dtype, ix.Ncap)
    buf = ix.ws.get(ix.ws_bytes)
    _check(load().sparse_louver_build(ctypes.byref(sh), _ptr(K), ix.r, _ptr(ix.index),
                                      ix.index.numel(), _ptr(buf), buf.numel(), _stream()),
           "louver_build")
    if check:
        read_device_status(ix.ws)
    return ix


def louver_route_threshold(q, K, index: LouverIndex, tau, cap: int, check: bool = True,
                           return_survivors: bool = False, idx=None, count=None,
                           survivors=None):
    """Threshold routing through a Louver index: (idx [B,Hkv,cap], count [B,Hkv])
    -- the set route_threshold returns -- plus, if asked, survivors [B,Hkv,2]
    (clusters that passed the ball test, and the 32-key leaves of those that
    passed theirs: the keys checked exactly).  K only checks that the index was
    built for this cache: the index holds its own copy of the keys."""
    _need_cuda(q, K, tau)
    B, Ncap, Hq, Hkv, d = _dims_qk(q, K)
    if (B, Hkv, Ncap, d, K.dtype) != (index.B, index.Hkv, index.Ncap, index.d, index.dtype):
        raise ValueError("the index was built for another K")
    sh = _shape(B, index.N, Hq, Hkv, d, q.dtype, Ncap)
    idx, count = _threshold_outputs(idx, count, B, Hkv, cap, q.device)
    _need_result(survivors, (B, Hkv, 2), torch.int32, "survivors")
    surv = survivors
    if return_survivors and surv is None:
        surv = torch.empty((B, Hkv, 2), dtype=torch.int32, device=q.device)
    _need_tau(tau, (B, Hkv))
    tau = tau.float().contiguous()
    buf = index.ws.get(index.ws_bytes)
    _check(load().sparse_louver_route_threshold(
        ctypes.byref(sh), _ptr(q), _ptr(index.index), index.index.numel(), index.r,
        _ptr(tau), int(cap), _ptr(idx), _ptr(count), _ptr(surv), _ptr(buf), buf.numel(),
        _stream()), "louver_route_threshold")
    if check:
        read_device_status(index.ws)
    if return_survivors:
        return idx, count, surv
    return idx, count


class DecodeStepGraph:
    """A decode step with its host transfers, captured once as a CUDA graph.

    The object owns one pinned host buffer for the step's inputs and one for
    its results, with tensor views: ``q_route_host`` [B,Hq,d] and
    ``q_layers_host`` [L,B,Hq,d] (the cache dtype) to write the next step's
    queries into, ``out_host`` [L,B,Hq,d], ``idx_host`` [B,Hkv,k or cap] and,
    in threshold mode, ``count_host`` [B,Hkv] to read.  Each replay runs one
    decode step (top-k with ``k``, or threshold with a device ``tau`` [B,Hkv]
    and ``cap``) over the cache K, V as one graph launch: the routing query is
    copied in and routing starts while the layers' queries travel on a second
    stream (joined before the attention).  When the pinned buffer is mapped
    into the device's address space (``mapped_out``) the attention writes its
    outputs straight into ``out_host``; on the fused kernels (``fused``: the
    routing scan, then one select + attention kernel) it writes the set (and
    counts) there too (``results_direct``), so nothing is copied back; on
    separate routing and attention kernels the set travels back on the second
    stream while the attention runs.  Without a mapping (or with
    ``host_writes=False``), outputs and set are copied back together after
    the attention.  With ``index`` (a LouverIndex
    of K) and threshold mode the step routes through the index.  ``replay()`` enqueues a step on ``stream`` (a new stream by
    default; graphs that share a workspace must use one stream),
    ``synchronize()`` waits for it, calling the object does both.  The device
    status is checked once after the warm-up step (use
    ``read_device_status(self.ws)`` to check later ones)."""

    @staticmethod
    def _layout(parts):
        """Byte offsets of tensors packed at 256-byte boundaries."""
        offs, n = [], 0
        for shape, dtype in parts:
            offs.append(n)
            size = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
            n += (size + 255) // 256 * 256
        return offs, n

    def __init__(self, K, V, L: int, Hq: int, k: int | None = None, tau=None,
                 cap: int | None = None, ws: Workspace | None = None, n: int | None = None,
                 stream=None, index: "LouverIndex | None" = None,
                 host_writes: bool = True):
        _need_cuda(K, V, tau)
        dev = K.device
        B, Hkv, _, d = K.shape
        dt = K.dtype
        topk = k is not None
        stride = int(k) if topk else int(cap)
        self.ws = _ws(ws, dev)
        self.stream = stream if stream is not None else torch.cuda.Stream(device=dev)
        ins = [((B, Hq, d), dt), ((L, B, Hq, d), dt)]
        outs = [((L, B, Hq, d), dt), ((B, Hkv, stride), torch.int32)]
        if not topk:
            outs.append(((B, Hkv), torch.int32))
        in_offs, in_n = self._layout(ins)
        out_offs, out_n = self._layout(outs)
        self.host_in = torch.empty(in_n, dtype=torch.uint8).pin_memory()
        self.host_out = torch.empty(out_n, dtype=torch.uint8).pin_memory()
        self.dev_in = torch.empty(in_n, dtype=torch.uint8, device=dev)
        self.dev_out = torch.empty(out_n, dtype=torch.uint8, device=dev)

        def views(buf, offs, parts):
            res = []
            for o, (shape, dtype) in zip(offs, parts):
                size = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
                res.append(buf[o:o + size].view(dtype).view(shape))
            return res

        self.q_route_host, self.q_layers_host = views(self.host_in, in_offs, ins)
        q_route, q_layers = views(self.dev_in, in_offs, ins)
        hv = views(self.host_out, out_offs, outs)
        dv = views(self.dev_out, out_offs, outs)
        self.out_host, self.idx_host = hv[0], hv[1]
        self.count_host = None if topk else hv[2]
        out, idx = dv[0], dv[1]
        count = None if topk else dv[2]
        if index is not None:
            if topk:
                raise ValueError("routing through a Louver index needs tau and cap")
            n = index.N

            def route():
                louver_route_threshold(q_route, K, index, tau, cap, check=False, idx=idx,
                                       count=count)
        elif topk:
            def route():
                route_topk(q_route, K, k, ws=self.ws, check=False, idx=idx, n=n)
        else:
            def route():
                route_threshold(q_route, K, tau, cap, ws=self.ws, check=False, n=n, idx=idx,
                                count=count)

        # host_writes=False: kernels write only device memory, and every
        # result comes back by one copy after the step
        self.mapped_out = host_writes and device_usable(self.out_host)
        out_dst = self.out_host if self.mapped_out else out
        # on the fused kernels the step only writes its set, counts and
        # outputs: with mapped host buffers all of them go straight to the host
        self.fused = index is None and decode_step_fused(
            B, _length(K.shape[2], n), Hq, Hkv, d, dt, L, k=k if topk else None,
            cap=None if topk else cap)
        direct = self.fused and self.mapped_out
        self.results_direct = direct

        def attend():
            attn_gather(q_layers, K, V, idx, count=count, ws=self.ws, check=False,
                        return_lse=False, out=out_dst, n=n)

        def fused_step(layers_ready):
            decode_step(q_route, q_layers, K, V, k=k if topk else None,
                        tau=None if topk else tau, cap=None if topk else cap, ws=self.ws,
                        check=False, out=out_dst, idx=self.idx_host if direct else idx,
                        count=(self.count_host if direct else count) if not topk else None,
                        return_lse=False, n=n, layers_ready=layers_ready)

        # byte ranges of the packed buffers: [q_route | q_layers], [out | idx (| count)]
        qr_end = in_offs[1]
        back = out_offs[1] if self.mapped_out else 0
        self.side = torch.cuda.Stream(device=dev)
        ev = [torch.cuda.Event() for _ in range(4)]

        def body():
            main = torch.cuda.current_stream(dev)
            # the routing query first: the two uploads share one copy engine
            self.dev_in[:qr_end].copy_(self.host_in[:qr_end], non_blocking=True)
            ev[0].record(main)
            self.side.wait_event(ev[0])
            with torch.cuda.stream(self.side):
                self.dev_in[qr_end:].copy_(self.host_in[qr_end:], non_blocking=True)
                ev[1].record(self.side)
            if self.fused:
                # routing, then (once the layers' queries are in) the fused
                # select + attention; results back after it unless written
                # to the host directly
                fused_step(ev[1])
                if not direct:
                    self.host_out[back:].copy_(self.dev_out[back:], non_blocking=True)
                return
            route()
            if self.mapped_out:
                ev[2].record(main)
                self.side.wait_event(ev[2])
                with torch.cuda.stream(self.side):
                    self.host_out[back:].copy_(self.dev_out[back:], non_blocking=True)
                    ev[3].record(self.side)
            main.wait_event(ev[1])
            attend()
            if self.mapped_out:
                main.wait_event(ev[3])
            else:
                self.host_out.copy_(self.dev_out, non_blocking=True)

        self.q_route_host.zero_()
        self.q_layers_host.zero_()
        with torch.cuda.stream(self.stream):
            body()                       # warm-up: sizes the workspaces, loads the library
            self.stream.synchronize()
            read_device_status(self.ws)
            if index is not None:
                read_device_status(index.ws)
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph, stream=self.stream):
                body()
        # the graph holds raw addresses: keep every buffer it touches alive
        # (a later, larger call may replace a workspace's buffer)
        self._captured = (self.ws.buf, index.ws.buf if index is not None else None, index,
                          K, V, tau)
        self._exec = ctypes.c_void_p(self.graph.raw_cuda_graph_exec())
        self._st = ctypes.c_void_p(self.stream.cuda_stream)
        self._launch = load().sparse_graph_launch

    @property
    def h2d_bytes(self) -> int:
        return self.host_in.numel()

    @property
    def d2h_bytes(self) -> int:
        return self.host_out.numel()

    def replay(self):
        """Enqueue one step on the object's stream (inputs from, results to,
        the pinned host buffers): one C call launching the instantiated graph."""
        rc = self._launch(self._exec, self._st)
        if rc != 0:
            raise SparseDecodeError(rc, "graph_launch")

    def synchronize(self):
        self.stream.synchronize()

    def __call__(self):
        """One step, synchronised: returns (out_host, idx_host[, count_host])."""
        self.replay()
        self.synchronize()
        if self.count_host is None:
            return self.out_host, self.idx_host
        return self.out_host, self.idx_host, self.count_host


def graph_upload(graph, stream=None):
    """Upload a captured torch.cuda.CUDAGraph's work to the device before its
    first replay (sparse_graph_upload), on `stream` (default: current)."""
    st = stream if stream is not None else torch.cuda.current_stream()
    _check(load().sparse_graph_upload(ctypes.c_void_p(graph.raw_cuda_graph_exec()),
                                      ctypes.c_void_p(st.cuda_stream)), "graph_upload")


def louver_decode_step(q_route, q_layers, K, V, index: LouverIndex, tau, cap: int,
                       ws: Workspace | None = None, check: bool = True, out=None, idx=None,
                       count=None, lse=None, return_lse: bool = True):
    """One decode step with threshold routing through a Louver index, then
    every layer's attention over the set.  Returns dict(idx, count, out, lse)
    (as decode_step in threshold mode)."""
    _need_cuda(q_route, q_layers, K, V, tau)
    B, Ncap, Hq, Hkv, d = _dims_qk(q_route, K)
    if (B, Hkv, Ncap, d, K.dtype) != (index.B, index.Hkv, index.Ncap, index.d, index.dtype):
        raise ValueError("the index was built for another K")
    L = q_layers.shape[0]
    if q_layers.shape != (L, B, Hq, d) or V.shape != K.shape:
        raise ValueError("q_layers must be [L,B,Hq,d] and V like K")
    _need_out(out, q_layers)
    dev = q_route.device
    w = _ws(ws, dev)
    N = index.N
    sh = _shape(B, N, Hq, Hkv, d, q_route.dtype, Ncap)
    buf = w.get(workspace_bytes(B, N, Hq, Hkv, d, q_route.dtype, cap, L))
    idx, count = _threshold_outputs(idx, count, B, Hkv, cap, dev)
    _need_result(lse, (L, B, Hq), torch.float32, "lse", host_ok=True)
    _need_tau(tau, (B, Hkv))
    if out is None:
        out = torch.empty_like(q_layers)
    if lse is None and return_lse:
        lse = torch.empty((L, B, Hq), dtype=torch.float32, device=dev)
    tau = tau.float().contiguous()
    lbuf = index.ws.get(index.ws_bytes)
    _check(load().sparse_louver_decode_step(
        ctypes.byref(sh), L, _ptr(q_route), _ptr(q_layers), _ptr(K), _ptr(V),
        _ptr(index.index), index.index.numel(), index.r, _ptr(tau), int(cap), _ptr(idx),
        _ptr(count), _ptr(out), _ptr(lse), _ptr(lbuf), lbuf.numel(), _ptr(buf), buf.numel(),
        _stream()), "louver_decode_step")
    if check:
        read_device_status(w)
    return {"idx": idx, "count": count, "out": out, "lse": lse}

