"""Seeded synthetic decode workloads.

This module only draws inputs.  It holds none of the method's arithmetic (no
scoring, selection or attention), so that the CUDA path and the CPU oracle can
both be fed from it without sharing anything else.

The shapes and value distributions follow the workloads the CLSA article
("CLSAとは？ルーティング共有で128Kコンテキスト推論を17倍高速化するスパースアテンション",
sections 計算コストの削減効果 and 推論速度の改善結果) speaks of: 128K-token
contexts, k = 2048 selected tokens and 16 cross-decoder layers sharing one
routing set; and, for the threshold variant, the Louver summary
("技術サマリー：スパースアテンションを範囲検索問題として捉える", section 問題定義),
where the kept set size varies per query.  No dataset or trained weights are
used: q, K and V are Gaussian, with optional planted heavy-hitter keys and one
amplified outlier channel per head.  The Louver workload draws its keys
around a few centres instead (a low intrinsic dimension, the structure its
index prunes on; the summary's section 2. Louver インデックス groups keys
into compact clusters for that reason).

Draw order, per sequence b with ``numpy.random.default_rng(seeds[b])``, all as
float32 standard normals unless stated:
  1. q_route[b]             [Hq, d]
  2. q_layers[:, b]         [L, Hq, d]
  3. K[b, h] for h ascending [N, d] each; with ``blobs`` > 0 (clustered
     keys) instead, per h: centres 2 * N(0,1) [blobs, d], each key's centre
     as integers in [0, blobs) [N], then N(0,1) [N, d] noise scaled by
     ``blob_spread`` and added to the key's centre
  4. V[b, h] for h ascending [N, d] each
  5. outlier channel per h  integers in [0, d)        (only if ``outlier``)
  6. heavy-hitter positions per h, uniform without replacement (``heavy`` > 0)
  7. heavy-hitter noise per h, N(0, 0.1^2)             [heavy, d]
Each block is rounded to the workload dtype (bf16: round-to-nearest-even)
right after it is drawn.  The outlier channel is multiplied by 8 in both K
and V (exact in bf16).  Heavy-hitter rows are written after that scaling:
row = 4 * qbar / ||qbar|| + noise, where qbar is the mean of the rounded
q_route rows of the KV head's query group, computed in float32 and then
rounded to the dtype.  V rows at those positions are left as drawn.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

_TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    Hq: int
    Hkv: int
    d: int
    L: int
    k: int = 0                 # top-k size (top-k mode)
    dtype: str = "bf16"        # "f32" or "bf16"
    heavy: int = 0             # planted heavy-hitter keys per KV head
    outlier: bool = False      # one x8 channel per KV head in K and V
    seeds: tuple = (0,)        # one seed per sequence
    mode: str = "topk"         # "topk" or "threshold"
    cap: int = 0               # threshold capacity per head
    tau_pct: tuple = (97, 100)  # threshold: nearest-rank percentile of scores
    blobs: int = 0             # clustered keys: centres per KV head (0: i.i.d.)
    blob_spread: float = 0.1   # clustered keys: noise scale around a centre
    description: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self):
        return _TORCH_DTYPES[self.dtype]

    @property
    def esize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def stride(self) -> int:
        return self.k if self.mode == "topk" else self.cap

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32", B=1, N=4096, Hq=8, Hkv=2, d=64, L=2, k=256, dtype="f32",
        seeds=(0,),
        description="tiny fp32: B=1, N=4096, Hq=8, Hkv=2, d=64, k=256, L=2; "
                    "q,K,V i.i.d. N(0,1), seed 0"),
    "decode_32k": Workload(
        "decode_32k", B=1, N=32768, Hq=32, Hkv=8, d=128, L=16, k=2048,
        heavy=64, seeds=(0,),
        description="bf16 decode: B=1, N=32768, Hq=32, Hkv=8, d=128, k=2048, "
                    "L=16; 64 planted heavy hitters per KV head"),
    "decode_128k": Workload(
        "decode_128k", B=1, N=131072, Hq=32, Hkv=8, d=128, L=16, k=2048,
        heavy=256, outlier=True, seeds=(0,),
        description="headline bf16 decode: B=1, N=131072, Hq=32, Hkv=8, "
                    "d=128, k=2048, L=16; one x8 outlier channel per head; "
                    "256 planted heavy hitters per head"),
    "batched_16x64k": Workload(
        "batched_16x64k", B=16, N=65536, Hq=32, Hkv=8, d=128, L=16, k=2048,
        heavy=64, seeds=tuple(range(1, 17)),
        description="batched bf16 decode: 16 independent sequences of "
                    "N=65536, Hq=32, Hkv=8, d=128, k=2048, L=16; seeds 1..16"),
    "threshold_128k": Workload(
        "threshold_128k", B=1, N=131072, Hq=32, Hkv=8, d=128, L=16,
        mode="threshold", cap=8192, heavy=64, seeds=(0,),
        description="threshold bf16: B=1, N=131072, Hq=32, Hkv=8, d=128, "
                    "L=16; tau per head = nearest-rank 97th percentile score; "
                    "cap 8192; 64 planted heavy hitters per head"),
    "louver_128k": Workload(
        "louver_128k", B=1, N=131072, Hq=32, Hkv=8, d=128, L=16,
        mode="threshold", cap=8192, blobs=64, blob_spread=0.1, seeds=(0,),
        description="threshold bf16 over clustered keys: B=1, N=131072, Hq=32, "
                    "Hkv=8, d=128, L=16; keys = one of 64 centres 2*N(0,1) per "
                    "head + 0.1*N(0,1); tau per head = nearest-rank 97th "
                    "percentile score; cap 8192"),
}


def custom(B=1, N=1000, Hq=8, Hkv=2, d=64, L=2, k=16, dtype="bf16", heavy=0,
           outlier=False, seed=0, mode="topk", cap=0, blobs=0,
           blob_spread=0.1) -> Workload:
    """A small workload for tests; sequence b uses seed + b."""
    return Workload(f"custom_B{B}_N{N}_Hq{Hq}_Hkv{Hkv}_d{d}_L{L}_{dtype}",
                    B=B, N=N, Hq=Hq, Hkv=Hkv, d=d, L=L, k=k, dtype=dtype,
                    heavy=heavy, outlier=outlier,
                    seeds=tuple(seed + b for b in range(B)), mode=mode,
                    cap=cap, blobs=blobs, blob_spread=blob_spread)


def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(_TORCH_DTYPES[dtype])


def generate(w: Workload, batches=None) -> dict:
    """Draw the inputs of ``w`` as CPU tensors in the workload dtype.

    Returns dict(q_route [B,Hq,d], q_layers [L,B,Hq,d], K [B,Hkv,N,d],
    V [B,Hkv,N,d], outlier [B,Hkv] int64 (-1 if none), heavy_pos
    [B,Hkv,heavy] int64).  ``batches`` restricts the draw to a subset of
    sequence indices (each sequence has its own seed, so a subset is drawn
    exactly as in the full set); B then equals len(batches)."""
    bs = list(range(w.B)) if batches is None else list(batches)
    B, N, Hq, Hkv, d, L, G = len(bs), w.N, w.Hq, w.Hkv, w.d, w.L, w.G
    td = w.torch_dtype
    q_route = torch.empty((B, Hq, d), dtype=td)
    q_layers = torch.empty((L, B, Hq, d), dtype=td)
    K = torch.empty((B, Hkv, N, d), dtype=td)
    V = torch.empty((B, Hkv, N, d), dtype=td)
    outlier = torch.full((B, Hkv), -1, dtype=torch.int64)
    heavy_pos = torch.empty((B, Hkv, w.heavy), dtype=torch.int64)
    for bi, b in enumerate(bs):
        rng = np.random.default_rng(w.seeds[b])
        q_route[bi] = _round(rng.standard_normal((Hq, d), dtype=np.float32), w.dtype)
        q_layers[:, bi] = _round(rng.standard_normal((L, Hq, d), dtype=np.float32), w.dtype)
        for h in range(Hkv):
            if w.blobs > 0:
                cen = 2.0 * rng.standard_normal((w.blobs, d), dtype=np.float32)
                which = rng.integers(0, w.blobs, size=N)
                noise = rng.standard_normal((N, d), dtype=np.float32)
                K[bi, h] = _round(cen[which] + np.float32(w.blob_spread) * noise, w.dtype)
            else:
                K[bi, h] = _round(rng.standard_normal((N, d), dtype=np.float32), w.dtype)
        for h in range(Hkv):
            V[bi, h] = _round(rng.standard_normal((N, d), dtype=np.float32), w.dtype)
        if w.outlier:
            ch = rng.integers(0, d, size=Hkv)
            for h in range(Hkv):
                c = int(ch[h])
                outlier[bi, h] = c
                K[bi, h, :, c] *= 8
                V[bi, h, :, c] *= 8
        if w.heavy > 0:
            pos = [rng.choice(N, size=w.heavy, replace=False) for _ in range(Hkv)]
            qf = q_route[bi].float().numpy()
            for h in range(Hkv):
                qbar = qf[h * G:(h + 1) * G].mean(axis=0, dtype=np.float32)
                unit = (4.0 * qbar / np.linalg.norm(qbar)).astype(np.float32)
                noise = rng.normal(0.0, 0.1, size=(w.heavy, d)).astype(np.float32)
                rows = _round(unit[None, :] + noise, w.dtype)
                p = torch.from_numpy(np.asarray(pos[h], dtype=np.int64))
                K[bi, h, p] = rows
                heavy_pos[bi, h] = p
    return {"q_route": q_route, "q_layers": q_layers, "K": K, "V": V,
            "outlier": outlier, "heavy_pos": heavy_pos}


def f32(t: torch.Tensor) -> np.ndarray:
    """Exact float32 numpy view of a workload tensor (bf16 widens exactly)."""
    return np.ascontiguousarray(t.float().numpy())


def query_variants(w: Workload, x: dict, n: int, seed: int = 1000) -> list:
    """``n`` further decode queries for the same cache, for benchmarks that
    rotate queries so the selected rows change from step to step.

    Variant r (r >= 1) draws, per sequence, with default_rng(seed + r):
    q_route = x's q_route + 0.5 * N(0,1) (so the planted keys stay relevant)
    and fresh N(0,1) q_layers; both rounded to the dtype.  Variant 0 is x's
    own pair."""
    out = [(x["q_route"], x["q_layers"])]
    for r in range(1, n):
        rng = np.random.default_rng(seed + r)
        qr = x["q_route"].float().numpy()
        noise = rng.standard_normal(qr.shape, dtype=np.float32)
        q_route = _round(qr + 0.5 * noise, w.dtype)
        q_layers = _round(rng.standard_normal(tuple(x["q_layers"].shape),
                                              dtype=np.float32), w.dtype)
        out.append((q_route, q_layers))
    return out
