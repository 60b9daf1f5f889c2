"""Plain CPU oracle of the Louver index, one subspace.

TEST INFRASTRUCTURE ONLY (like the rest of this package): the tests and the
CPU-baseline leg of ``bench.py`` are the only callers; the product path never
imports it.

Louver summary ("技術サマリー：スパースアテンションを範囲検索問題として捉える"):

* section 1. 半空間範囲検索への帰着: the kept set of a query is every key in the
  halfspace {p : <q,p> >= tau}; no false negatives.
* section 2. Louver インデックス: keys are grouped into clusters of a fixed size
  r by a balanced PCA tree; each cluster is enclosed in a bounding ball
  (centre c, radius rho); a query first tests each ball against its halfspace
  and prunes the clusters whose ball does not meet it, then checks the keys
  of the surviving clusters exactly.

Readings (where the page is silent):

* Subspaces: the page splits d into S contiguous subspaces of d/S dimensions
  with an index each, and its first query algorithm keeps a key only if the
  key's cluster passes the ball test in every subspace, against a threshold
  tau_s per subspace whose rule it does not give.  Reading: the plainest rule
  that keeps every key scoring >= tau.  With U_s the largest ball bound of
  subspace s over the head's clusters, <q,k> = sum_s <q_s,k_s> >= tau forces
  <q_s,k_s> >= tau - sum_{s' != s} U_s' for every s, so
  tau_s = tau - sum_{s' != s} U_s'.  With S = 1 this is the plain ball test
  (tau_1 = tau), and the page's two query algorithms coincide.
* Balanced PCA tree: a node's keys are split at the median of their
  projections on the node's principal direction (the top eigenvector of the
  node's covariance) into two halves of equal size, recursively, down to
  nodes of r keys; N / r must be a power of two.  The larger half of the
  projections goes to the second child; equal projections go to the lower
  position first (the top-k tie rule).  The principal direction's sign and
  the exact split do not change the query result, only the pruning.
* The query vector is the routing query of the scores, qbar = (sum over the
  G query heads of the KV head) / sqrt(d), so <qbar, k_j> is the score S_j.
  A ball meets the halfspace iff <qbar, c> + |qbar| rho >= tau; a cluster is
  pruned only when that bound is below tau by more than a margin: the
  comparison band (1e-4 |tau| + 1e-6) plus 1e-5 |qbar| (|c| + rho).  The
  second term bounds the fp32 rounding of a member's score (at most a few
  1e-7 of |qbar| |k| for d <= 128, and |k| <= |c| + rho), which does not
  shrink with tau, so no fp32 rounding of the exact check can make a pruned
  key pass even when tau is near zero.  With S subspaces the norm bound of a
  member is (|c_s| + rho_s) + sum_{s' != s} R_s', R_s' the largest
  |c| + rho of subspace s', and the bound against tau_s uses it.
"""
from __future__ import annotations

import math

import numpy as np

from . import scores as _scores
from . import threshold as _threshold


def build_index(Kh, r: int) -> dict:
    """Balanced PCA tree over one head's keys Kh [N,d] (fp32).

    Returns dict(perm [N] int64: key ids in cluster order, cluster i holding
    perm[i*r:(i+1)*r]; centres [N/r,d] f64; radii [N/r] f64)."""
    X = np.asarray(Kh, np.float64)
    N, d = X.shape
    if N % r or (N // r) & (N // r - 1):
        raise ValueError("N / r must be a power of two")
    order = np.arange(N)
    n = N
    while n > r:
        new = np.empty_like(order)
        for s0 in range(0, N, n):
            seg = order[s0:s0 + n]
            Y = X[seg] - X[seg].mean(axis=0)
            _, vecs = np.linalg.eigh(Y.T @ Y)
            p = Y @ vecs[:, -1]
            # the n/2 largest projections, ties to the lower position
            top = np.sort(np.argsort(-p, kind="stable")[:n // 2])
            mask = np.zeros(n, bool)
            mask[top] = True
            new[s0:s0 + n] = np.concatenate([seg[~mask], seg[mask]])
        order = new
        n //= 2
    members = X[order].reshape(N // r, r, d)
    centres = members.mean(axis=1)
    radii = np.sqrt(((members - centres[:, None, :]) ** 2).sum(-1)).max(axis=1)
    return {"perm": order, "centres": centres, "radii": radii}


def ball_bounds(index: dict, qbar) -> np.ndarray:
    """Upper bound of <qbar, p> over each cluster's ball."""
    q = np.asarray(qbar, np.float64)
    return index["centres"] @ q + np.linalg.norm(q) * index["radii"]


def band(tau: float) -> float:
    return 1e-4 * abs(tau) + 1e-6


def keep_clusters(index: dict, qbar, tau: float) -> np.ndarray:
    """The ball test: True for every cluster that may hold a key with score
    >= tau (its bound is not below tau by more than the margin)."""
    q = np.asarray(qbar, np.float64)
    qn = np.linalg.norm(q)
    slack = 1e-5 * qn * (np.linalg.norm(index["centres"], axis=1) + index["radii"])
    return ball_bounds(index, q) >= tau - band(tau) - slack


def keep_clusters_subspaces(indexes: list, qbar, tau: float) -> list:
    """The all-subspace filter: for every subspace s (index s over dimensions
    s*d/S .. (s+1)*d/S), True for each cluster that passes its ball test
    against tau_s = tau - sum_{s' != s} U_s'."""
    q = np.asarray(qbar, np.float64)
    S = len(indexes)
    ds = q.shape[0] // S
    qs = [q[s * ds:(s + 1) * ds] for s in range(S)]
    bounds = [ball_bounds(ix, qs[s]) for s, ix in enumerate(indexes)]
    U = [float(b.max()) for b in bounds]
    R = [float((np.linalg.norm(ix["centres"], axis=1) + ix["radii"]).max()) for ix in indexes]
    qn = np.linalg.norm(q)
    keep = []
    for s, ix in enumerate(indexes):
        rest_U = sum(U) - U[s]
        rest_R = sum(R) - R[s]
        slack = 1e-5 * qn * (np.linalg.norm(ix["centres"], axis=1) + ix["radii"] + rest_R)
        keep.append(bounds[s] >= tau - rest_U - band(tau) - slack)
    return keep


def candidates(indexes: list, keep: list, N: int) -> np.ndarray:
    """Keys whose cluster passes in every subspace (bool [N])."""
    ok = np.ones(N, bool)
    for ix, kp in zip(indexes, keep):
        r = N // len(kp)
        member = np.zeros(N, bool)
        member[ix["perm"].reshape(-1, r)[kp].ravel()] = True
        ok &= member
    return ok


def route_threshold_subspaces(q, K, tau, cap: int, r: int, S: int):
    """Threshold routing through S subspace indexes (the all-subspace
    filter, then the exact check of the candidates), every (b, h).

    Returns (idx [B,Hkv,cap], count [B,Hkv], candidates [B,Hkv] = keys that
    passed the filter in every subspace).  The set equals the full-scan
    threshold set on the oracle's fp32 scores."""
    q = np.asarray(q, np.float32)
    K = np.asarray(K, np.float32)
    tau = np.asarray(tau, np.float32)
    B, Hq, d = q.shape
    _, Hkv, N, _ = K.shape
    if d % S:
        raise ValueError("S must divide d")
    ds = d // S
    G = Hq // Hkv
    Sc = _scores(q, K)
    idx = np.full((B, Hkv, cap), -1, np.int32)
    count = np.zeros((B, Hkv), np.int32)
    ncand = np.zeros((B, Hkv), np.int64)
    for b in range(B):
        for h in range(Hkv):
            indexes = [build_index(K[b, h][:, s * ds:(s + 1) * ds], r) for s in range(S)]
            qbar = q[b, h * G:(h + 1) * G].astype(np.float64).sum(0) / math.sqrt(d)
            keep = keep_clusters_subspaces(indexes, qbar, float(tau[b, h]))
            cand = np.nonzero(candidates(indexes, keep, N))[0]
            ncand[b, h] = len(cand)
            sel = cand[Sc[b, h, cand] >= tau[b, h]]
            count[b, h] = len(sel)
            m = min(len(sel), cap)
            idx[b, h, :m] = sel[:m]
    return idx, count, ncand


def route_threshold(q, K, tau, cap: int, r: int):
    """Threshold routing through the index, every (b, h).

    q [B,Hq,d], K [B,Hkv,N,d], tau [B,Hkv].  Returns (idx [B,Hkv,cap],
    count [B,Hkv], survivors [B,Hkv] = clusters that pass the ball test).
    The exact check uses the oracle's fp32 scores, so the set equals the
    full-scan threshold set."""
    q = np.asarray(q, np.float32)
    K = np.asarray(K, np.float32)
    tau = np.asarray(tau, np.float32)
    B, Hq, d = q.shape
    _, Hkv, N, _ = K.shape
    G = Hq // Hkv
    S = _scores(q, K)
    idx = np.full((B, Hkv, cap), -1, np.int32)
    count = np.zeros((B, Hkv), np.int32)
    surv = np.zeros((B, Hkv), np.int64)
    for b in range(B):
        for h in range(Hkv):
            index = build_index(K[b, h], r)
            qbar = q[b, h * G:(h + 1) * G].astype(np.float64).sum(0) / math.sqrt(d)
            t = float(tau[b, h])
            keep = keep_clusters(index, qbar, t)
            surv[b, h] = int(keep.sum())
            cand = index["perm"].reshape(-1, r)[keep].ravel()
            sel = np.sort(cand[S[b, h, cand] >= tau[b, h]])
            count[b, h] = len(sel)
            m = min(len(sel), cap)
            idx[b, h, :m] = sel[:m]
    return idx, count, surv


def full_scan_threshold(q, K, tau, cap: int):
    """The plain threshold set on the oracle's scores (for comparisons)."""
    return _threshold(_scores(q, K), tau, cap)
