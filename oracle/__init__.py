"""Plain CPU oracle for shared-routing token-sparse decode attention.

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product path (the
CUDA library and its Python binding) never imports this package, and this
package never imports the product path.

The arithmetic lives in ``oracle.c`` (plain C, no blocking or reordering
beyond what the definitions state).  This module only compiles it with gcc and
marshals numpy arrays through ctypes.  See the header of ``oracle.c`` for the
passages each function follows:

* CLSA article ("CLSAとは？ルーティング共有で128Kコンテキスト推論を17倍高速化する
  スパースアテンション"), sections 研究の背景と課題 and CLSAの仕組み: top-k routing
  computed once and shared by every cross-decoder layer;
* Louver summary ("技術サマリー：スパースアテンションを範囲検索問題として捉える"),
  sections 問題定義 and 1. 半空間範囲検索への帰着: the threshold set
  {j : score_j >= tau} with no false negatives.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

# -ffp-contract=off: no fused multiply-add, so every fp32 product and sum is
# rounded as written.  -O2 without -ffast-math keeps the summation order.
CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
          "-fno-fast-math", "-fopenmp"]

_lock = threading.Lock()
_lib = None

OK, BAD_ARG, NONFINITE, NOMEM = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I = ctypes.c_void_p, ctypes.c_int
            sigs = {
                "oracle_scores_f32": [I, I, I, I, I, P, P, P],
                "oracle_scores_f64": [I, I, I, I, I, P, P, P],
                "oracle_topk": [I, I, P, I, P],
                "oracle_threshold": [I, I, P, P, I, P, P],
                "oracle_percentile_tau": [I, I, P, I, I, P],
                "oracle_attn": [I, I, I, I, I, I, P, P, P, P, I, P, P, P],
                "oracle_decode_step": [I, I, I, I, I, I, P, P, P, P, I, P, I,
                                       P, P, P, P, P],
                "oracle_decode_step_grouped": [I, I, I, I, I, I, I, P, P, P, P, I, P,
                                               I, P, P, P, P, P],
                "oracle_num_threads": [],
            }
            for name, argtypes in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = argtypes
                fn.restype = I
            _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != OK:
        names = {BAD_ARG: "bad argument", NONFINITE: "non-finite value",
                 NOMEM: "out of memory"}
        raise OracleError(f"{what}: {names.get(rc, rc)}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def scores(q, K, dtype=np.float32) -> np.ndarray:
    """Routing scores S [B,Hkv,N] from q [B,Hq,d] and K [B,Hkv,N,d].

    ``dtype=np.float32`` follows the fixed fp32 summation order;
    ``np.float64`` is the double-precision arbiter."""
    q, K = _f32(q), _f32(K)
    B, Hq, d = q.shape
    Bk, Hkv, N, dk = K.shape
    if Bk != B or dk != d:
        raise OracleError("scores: shape mismatch")
    lib = _load()
    if np.dtype(dtype) == np.float64:
        S = np.empty((B, Hkv, N), np.float64)
        rc = lib.oracle_scores_f64(B, N, Hq, Hkv, d, _p(q), _p(K), _p(S))
    else:
        S = np.empty((B, Hkv, N), np.float32)
        rc = lib.oracle_scores_f32(B, N, Hq, Hkv, d, _p(q), _p(K), _p(S))
    _check(rc, "scores")
    return S


def topk(S, k: int) -> np.ndarray:
    """Top-k index sets [.., k] of S [.., N], ascending, ties to lower index."""
    S = _f32(S)
    lead, N = S.shape[:-1], S.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    idx = np.empty((BH, k), np.int32)
    _check(_load().oracle_topk(BH, N, _p(S), int(k), _p(idx)), "topk")
    return idx.reshape(*lead, k)


def threshold(S, tau, cap: int):
    """Threshold sets: (idx [.., cap] with -1 past the count, count [..])."""
    S = _f32(S)
    lead, N = S.shape[:-1], S.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    tau = _f32(tau).reshape(BH)
    idx = np.full((BH, cap), -1, np.int32)
    count = np.empty((BH,), np.int32)
    _check(_load().oracle_threshold(BH, N, _p(S), _p(tau), int(cap), _p(idx),
                                    _p(count)), "threshold")
    return idx.reshape(*lead, cap), count.reshape(lead)


def percentile_tau(S, num: int = 97, den: int = 100) -> np.ndarray:
    """Nearest-rank num/den percentile of each row of S (fp32)."""
    S = _f32(S)
    lead, N = S.shape[:-1], S.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    tau = np.empty((BH,), np.float32)
    _check(_load().oracle_percentile_tau(BH, N, _p(S), int(num), int(den),
                                         _p(tau)), "percentile_tau")
    return tau.reshape(lead)


def attn(q, K, V, idx, count=None):
    """Attention over the selected rows, in double precision.

    q [Lq,B,Hq,d] (or [B,Hq,d] for one layer); idx [B,Hkv,stride]; count
    [B,Hkv] or None.  Returns (out [Lq,B,Hq,d] f64, lse [Lq,B,Hq] f64) with the
    leading Lq dropped again when q had none."""
    q = _f32(q)
    single = q.ndim == 3
    if single:
        q = q[None]
    K, V, idx = _f32(K), _f32(V), _i32(idx)
    Lq, B, Hq, d = q.shape
    _, Hkv, N, _ = K.shape
    stride = idx.shape[-1]
    cnt = None if count is None else _i32(count)
    out = np.empty((Lq, B, Hq, d), np.float64)
    lse = np.empty((Lq, B, Hq), np.float64)
    rc = _load().oracle_attn(Lq, B, Hq, Hkv, d, N, _p(q), _p(K), _p(V), _p(idx),
                             stride, None if cnt is None else _p(cnt), _p(out),
                             _p(lse))
    _check(rc, "attn")
    if single:
        return out[0], lse[0]
    return out, lse


def decode_step(q_route, q_layers, K, V, k: int | None = None, tau=None,
                cap: int | None = None):
    """One shared-routing decode step.

    Returns dict(S, idx, count, out, lse); top-k mode when ``k`` is given,
    threshold mode when ``tau`` is given (with capacity ``cap``)."""
    q_route, q_layers, K, V = _f32(q_route), _f32(q_layers), _f32(K), _f32(V)
    L, B, Hq, d = q_layers.shape
    _, Hkv, N, _ = K.shape
    S = np.empty((B, Hkv, N), np.float32)
    if k is not None:
        stride, kk, tau_p, capv = int(k), int(k), None, 0
    else:
        if tau is None or cap is None:
            raise OracleError("decode_step: give k, or tau and cap")
        tau = _f32(tau).reshape(B * Hkv)
        stride, kk, tau_p, capv = int(cap), 0, _p(tau), int(cap)
    idx = np.full((B, Hkv, stride), -1, np.int32)
    count = np.full((B, Hkv), stride, np.int32)
    out = np.empty((L, B, Hq, d), np.float64)
    lse = np.empty((L, B, Hq), np.float64)
    rc = _load().oracle_decode_step(L, B, Hq, Hkv, d, N, _p(q_route),
                                    _p(q_layers), _p(K), _p(V), kk, tau_p, capv,
                                    _p(S), _p(idx), _p(count), _p(out), _p(lse))
    _check(rc, "decode_step")
    return {"S": S, "idx": idx, "count": count, "out": out, "lse": lse}


def decode_step_grouped(q_routes, q_layers, K, V, R: int, k: int | None = None,
                        tau=None, cap: int | None = None):
    """Decode step re-routing every R layers (``oracle_decode_step_grouped``).

    q_routes [ngroups,B,Hq,d] with ngroups = ceil(L/R); tau [ngroups,B,Hkv]
    in threshold mode.  Returns dict(S [ngroups,B,Hkv,N], idx [ngroups,B,Hkv,
    stride], count [ngroups,B,Hkv], out [L,B,Hq,d], lse [L,B,Hq])."""
    q_routes, q_layers, K, V = _f32(q_routes), _f32(q_layers), _f32(K), _f32(V)
    L, B, Hq, d = q_layers.shape
    _, Hkv, N, _ = K.shape
    ng = (L + R - 1) // R
    if q_routes.shape != (ng, B, Hq, d):
        raise OracleError("decode_step_grouped: q_routes must be [ceil(L/R),B,Hq,d]")
    if k is not None:
        stride, kk, tau_p, capv = int(k), int(k), None, 0
    else:
        if tau is None or cap is None:
            raise OracleError("decode_step_grouped: give k, or tau and cap")
        tau = _f32(tau).reshape(ng * B * Hkv)
        stride, kk, tau_p, capv = int(cap), 0, _p(tau), int(cap)
    S = np.empty((ng, B, Hkv, N), np.float32)
    idx = np.full((ng, B, Hkv, stride), -1, np.int32)
    count = np.full((ng, B, Hkv), stride, np.int32)
    out = np.empty((L, B, Hq, d), np.float64)
    lse = np.empty((L, B, Hq), np.float64)
    rc = _load().oracle_decode_step_grouped(L, int(R), B, Hq, Hkv, d, N, _p(q_routes),
                                            _p(q_layers), _p(K), _p(V), kk, tau_p, capv,
                                            _p(S), _p(idx), _p(count), _p(out), _p(lse))
    _check(rc, "decode_step_grouped")
    return {"S": S, "idx": idx, "count": count, "out": out, "lse": lse}
