"""Pins for the CPU oracle: each test checks it against something other than
itself -- a hand-worked example, a closed form, a library routine, brute force
or an invariant -- chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.

Passages: CLSA article, sections 研究の背景と課題 (top-k keeps the k
highest-scoring tokens; sparse attention attends only to them) and CLSAの仕組み
(one index set, computed once, reused by every cross-decoder layer); Louver
summary, sections 問題定義 and 1. 半空間範囲検索への帰着 (keep every key with
<q,k> >= tau, with no false negatives)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.attention

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# Hand-worked example (tests/golden/hand_worked_tiny.json)
# --------------------------------------------------------------------------

@pytest.fixture(scope="module")
def hand():
    with open(os.path.join(GOLDEN, "hand_worked_tiny.json")) as f:
        return json.load(f)


def test_hand_worked_scores_topk_threshold(hand):
    q = np.array(hand["q_route"], np.float32)
    K = np.array(hand["K"], np.float32)
    S = oracle.scores(q, K)
    np.testing.assert_array_equal(S, np.array(hand["expected_scores"], np.float32))
    for k, want in hand["expected_topk"].items():
        np.testing.assert_array_equal(oracle.topk(S, int(k)), np.array(want))
    for case in hand["expected_threshold"]:
        idx, cnt = oracle.threshold(S, np.array([[case["tau"]]], np.float32), cap=5)
        assert int(cnt[0, 0]) == len(case["idx"])
        assert list(idx[0, 0, :cnt[0, 0]]) == case["idx"]


def test_hand_worked_attention(hand):
    K = np.array(hand["K"], np.float32)
    V = np.array(hand["V"], np.float32)
    ql = np.zeros((1, 1, 2, 4), np.float32)
    ql[0, 0, 0, 0] = np.float32(2 * math.log(2))
    idx = np.array(hand["expected_topk"]["2"], np.int32)
    out, lse = oracle.attn(ql, K, V, idx)
    exp = hand["expected_attn_top2"]
    np.testing.assert_allclose(out[0, 0], np.array(exp["out"]), atol=exp["tol"])
    np.testing.assert_allclose(lse[0, 0], [math.log(12), math.log(2)], atol=exp["tol"])


# --------------------------------------------------------------------------
# Scores
# --------------------------------------------------------------------------

def _einsum_scores_f64(q, K, G):
    """Group-summed scores by library einsum in fp64 with the key heads
    repeated over their query groups (torch/numpy GQA convention)."""
    Krep = np.repeat(K.astype(np.float64), G, axis=1)          # [B,Hq,N,d]
    per_head = np.einsum("bgd,bgnd->bgn", q.astype(np.float64), Krep)
    B, Hq, N = per_head.shape
    return per_head.reshape(B, Hq // G, G, N).sum(axis=2) / math.sqrt(q.shape[-1])


@pytest.mark.parametrize("B,N,Hq,Hkv,d", [(2, 37, 6, 2, 16), (1, 200, 8, 2, 64),
                                          (3, 19, 4, 4, 8), (1, 50, 8, 1, 128)])
def test_scores_vs_library_einsum(B, N, Hq, Hkv, d):
    r = _rng(B * 1000 + N)
    q = r.standard_normal((B, Hq, d), dtype=np.float32)
    K = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    ref = _einsum_scores_f64(q, K, Hq // Hkv)
    S64 = oracle.scores(q, K, np.float64)
    np.testing.assert_allclose(S64, ref, rtol=1e-12, atol=1e-12)
    # fp32 summation error bound: n * u * sum|terms| with n = G*d + 2.
    Krep = np.repeat(np.abs(K.astype(np.float64)), Hq // Hkv, axis=1)
    mag = np.einsum("bgd,bgnd->bgn", np.abs(q.astype(np.float64)), Krep)
    mag = mag.reshape(B, Hkv, Hq // Hkv, N).sum(axis=2) / math.sqrt(d)
    bound = ((Hq // Hkv) * d + 2) * 2.0 ** -24 * mag + 1e-30
    S32 = oracle.scores(q, K)
    assert np.all(np.abs(S32 - ref) <= bound)


def test_scores_integer_inputs_exact():
    """Small integers: every product and partial sum is exact in fp32 and
    the scale 1/sqrt(64) = 1/8 is a power of two, so the result is exact."""
    r = _rng(7)
    q = r.integers(-3, 4, size=(2, 8, 64)).astype(np.float32)
    K = r.integers(-3, 4, size=(2, 2, 33, 64)).astype(np.float32)
    G = 4
    exact = np.einsum("bgd,bgnd->bgn", q.astype(np.int64),
                      np.repeat(K.astype(np.int64), G, axis=1))
    exact = exact.reshape(2, 2, G, 33).sum(axis=2)
    np.testing.assert_array_equal(oracle.scores(q, K), (exact / 8.0).astype(np.float32))


def test_scores_head_mapping_contiguous_groups():
    """Only query head 5 is non-zero; with G=4 it belongs to KV head 1, whose
    keys are one-hot, so S[:,1,j] = q[5, c_j] / sqrt(d) and KV head 0 is 0."""
    d, N = 16, 10
    q = np.zeros((1, 8, d), np.float32)
    q[0, 5] = np.arange(1, d + 1, dtype=np.float32)
    K = np.zeros((1, 2, N, d), np.float32)
    cols = (np.arange(N) * 3) % d
    K[0, 1, np.arange(N), cols] = 1.0
    K[0, 0] = 1.0
    S = oracle.scores(q, K)
    np.testing.assert_array_equal(S[0, 0], np.zeros(N, np.float32))
    np.testing.assert_array_equal(S[0, 1], ((cols + 1) / 4.0).astype(np.float32))


def test_scores_power_of_two_scaling_and_key_permutation():
    r = _rng(3)
    q = r.standard_normal((1, 4, 32), dtype=np.float32)
    K = r.standard_normal((1, 1, 64, 32), dtype=np.float32)
    S = oracle.scores(q, K)
    np.testing.assert_array_equal(oracle.scores(2 * q, K), 2 * S)
    perm = r.permutation(64)
    np.testing.assert_array_equal(oracle.scores(q, K[:, :, perm]), S[:, :, perm])


# --------------------------------------------------------------------------
# Top-k
# --------------------------------------------------------------------------

@pytest.mark.parametrize("N,k,levels", [(64, 7, None), (1000, 100, 17),
                                        (500, 499, 3), (300, 1, None)])
def test_topk_vs_stable_argsort(N, k, levels):
    r = _rng(N + k)
    S = r.standard_normal((3, N)).astype(np.float32)
    if levels:  # force many exact ties
        S = np.round(S * levels / 4).astype(np.float32)
    got = oracle.topk(S, k)
    for row in range(3):
        want = np.sort(np.argsort(-S[row], kind="stable")[:k])
        np.testing.assert_array_equal(got[row], want)


def test_topk_bruteforce_all_subsets():
    """Integer scores with ties, N <= 10: the set with the largest sum,
    ties between sets broken by the lexicographically smallest index tuple
    (which is the lower-index tie rule at the k-th score)."""
    r = _rng(11)
    for trial in range(30):
        N = int(r.integers(1, 11))
        S = r.integers(-2, 3, size=(1, N)).astype(np.float32)
        for k in range(1, N + 1):
            best = max(itertools.combinations(range(N), k),
                       key=lambda c: (S[0, list(c)].sum(), [-i for i in c]))
            np.testing.assert_array_equal(oracle.topk(S, k)[0], np.array(best))


def test_topk_special_cases():
    S = np.full((2, 50), 0.25, np.float32)
    np.testing.assert_array_equal(oracle.topk(S, 9), np.tile(np.arange(9), (2, 1)))
    r = _rng(5)
    S = r.standard_normal((2, 40)).astype(np.float32)
    np.testing.assert_array_equal(oracle.topk(S, 40), np.tile(np.arange(40), (2, 1)))
    # -0.0 and +0.0 are the same score: the lower index wins
    S = np.array([[-1.0, 0.0, -0.0, -0.0, 0.0]], np.float32)
    S[0, 2] = -0.0
    np.testing.assert_array_equal(oracle.topk(S, 2), [[1, 2]])
    # permutation of distinct scores permutes the set
    S = r.permutation(1000).astype(np.float32)[None]
    perm = r.permutation(1000)
    base = set(oracle.topk(S, 30)[0])
    got = set(oracle.topk(S[:, perm], 30)[0])
    assert {int(perm[j]) for j in got} == base


# --------------------------------------------------------------------------
# Threshold
# --------------------------------------------------------------------------

def test_threshold_special_cases():
    r = _rng(9)
    S = r.standard_normal((2, 300)).astype(np.float32)
    tau = S.max(axis=1) + 1
    idx, cnt = oracle.threshold(S, tau, cap=300)
    assert cnt.tolist() == [0, 0]
    idx, cnt = oracle.threshold(S, S.min(axis=1), cap=300)
    assert cnt.tolist() == [300, 300]
    np.testing.assert_array_equal(idx, np.tile(np.arange(300), (2, 1)))
    # tau = k-th largest of distinct scores -> exactly the top-k set
    k = 37
    kth = -np.sort(-S, axis=1)[:, k - 1]
    idx, cnt = oracle.threshold(S, kth, cap=300)
    assert cnt.tolist() == [k, k]
    np.testing.assert_array_equal(idx[:, :k], oracle.topk(S, k))
    # capacity overflow: true count, lowest indices written
    idx, cnt = oracle.threshold(S, S.min(axis=1), cap=10)
    assert cnt.tolist() == [300, 300]
    np.testing.assert_array_equal(idx, np.tile(np.arange(10), (2, 1)))


def test_threshold_no_false_negatives_against_fp64():
    r = _rng(21)
    q = r.standard_normal((1, 8, 64), dtype=np.float32)
    K = r.standard_normal((1, 2, 5000, 64), dtype=np.float32)
    S = oracle.scores(q, K)
    S64 = oracle.scores(q, K, np.float64)
    tau = oracle.percentile_tau(S, 97, 100)
    idx, cnt = oracle.threshold(S, tau, cap=5000)
    for h in range(2):
        band = 1e-4 * abs(float(tau[0, h])) + 1e-6
        sel = set(idx[0, h, :cnt[0, h]].tolist())
        must = set(np.nonzero(S64[0, h] >= tau[0, h] + band)[0].tolist())
        never = set(np.nonzero(S64[0, h] < tau[0, h] - band)[0].tolist())
        assert must <= sel and not (never & sel)


def test_percentile_tau_matches_numpy_inverted_cdf():
    r = _rng(4)
    S = r.standard_normal((3, 131)).astype(np.float32)
    tau = oracle.percentile_tau(S, 97, 100)
    for row in range(3):
        want = np.percentile(S[row], 97, method="inverted_cdf")
        assert tau[row] == np.float32(want)
    # nearest rank at the headline length: ceil(0.97 * 131072) = 127140, so
    # 131072 - 127139 = 3933 distinct scores are >= tau
    S = r.permutation(131072).astype(np.float32)[None]
    tau = oracle.percentile_tau(S, 97, 100)
    assert float(tau[0]) == 127139.0
    assert int(oracle.threshold(S, tau, cap=131072)[1][0]) == 3933


# --------------------------------------------------------------------------
# Attention over the selected set
# --------------------------------------------------------------------------

def _sdpa_f64(q, K, V):
    """torch scaled_dot_product_attention (math backend) in fp64 with GQA repetition.
    q [B,Hq,d] (one query per head), K,V [B,Hkv,n,d]."""
    qt = torch.from_numpy(q.astype(np.float64))[:, :, None, :]
    Kt = torch.from_numpy(K.astype(np.float64))
    Vt = torch.from_numpy(V.astype(np.float64))
    G = q.shape[1] // K.shape[1]
    Kt = Kt.repeat_interleave(G, dim=1)
    Vt = Vt.repeat_interleave(G, dim=1)
    # the plain math backend: one fixed evaluation order, whatever the thread pool
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)
    logits = (qt @ Kt.transpose(-1, -2))[:, :, 0, :] / math.sqrt(q.shape[-1])
    return o[:, :, 0, :].numpy(), torch.logsumexp(logits, dim=-1).numpy()


@pytest.mark.parametrize("B,N,Hq,Hkv,d", [(1, 300, 8, 2, 64), (2, 57, 4, 1, 32),
                                          (1, 129, 32, 8, 128)])
def test_attn_all_selected_equals_dense_sdpa(B, N, Hq, Hkv, d):
    r = _rng(N)
    q = r.standard_normal((B, Hq, d), dtype=np.float32)
    K = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    V = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    idx = np.tile(np.arange(N, dtype=np.int32), (B, Hkv, 1))
    out, lse = oracle.attn(q, K, V, idx)
    o_ref, lse_ref = _sdpa_f64(q, K, V)
    np.testing.assert_allclose(out, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_attn_subset_equals_dense_on_gathered_rows():
    r = _rng(77)
    B, Hq, Hkv, N, d, c = 2, 8, 2, 400, 64, 33
    q = r.standard_normal((B, Hq, d), dtype=np.float32)
    K = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    V = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    idx = np.stack([np.stack([np.sort(r.choice(N, c, replace=False))
                              for _ in range(Hkv)]) for _ in range(B)]).astype(np.int32)
    out, lse = oracle.attn(q, K, V, idx)
    Kg = np.take_along_axis(K, idx[..., None].astype(np.int64), axis=2)
    Vg = np.take_along_axis(V, idx[..., None].astype(np.int64), axis=2)
    o_ref, lse_ref = _sdpa_f64(q, Kg, Vg)
    np.testing.assert_allclose(out, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_attn_single_key_and_constant_values():
    r = _rng(8)
    q = r.standard_normal((1, 4, 16), dtype=np.float32)
    K = r.standard_normal((1, 1, 20, 16), dtype=np.float32)
    V = r.standard_normal((1, 1, 20, 16), dtype=np.float32)
    out, _ = oracle.attn(q, K, V, np.array([[[13]]], np.int32))
    np.testing.assert_array_equal(out[0], np.tile(V[0, 0, 13].astype(np.float64), (4, 1)))
    Vc = np.tile(np.linspace(-2, 2, 16, dtype=np.float32), (1, 1, 20, 1))
    idx = np.array([[[1, 4, 9, 16]]], np.int32)
    out, _ = oracle.attn(q, K, Vc, idx)
    np.testing.assert_allclose(out[0], np.tile(Vc[0, 0, 0], (4, 1)), atol=1e-14)


def test_attn_weights_are_softmax_and_sum_to_one():
    """V rows are one-hot (row t of the selection -> e_t), so o equals the
    softmax weights; compared with scipy's softmax of the logits."""
    r = _rng(12)
    d, c, N = 32, 20, 60
    q = r.standard_normal((1, 2, d), dtype=np.float32)
    K = r.standard_normal((1, 1, N, d), dtype=np.float32)
    sel = np.sort(r.choice(N, c, replace=False)).astype(np.int32)
    V = np.zeros((1, 1, N, d), np.float32)
    V[0, 0, sel, np.arange(c)] = 1.0
    out, lse = oracle.attn(q, K, V, sel[None, None])
    logits = (q[0].astype(np.float64) @ K[0, 0, sel].astype(np.float64).T) / math.sqrt(d)
    np.testing.assert_allclose(out[0][:, :c], scipy.special.softmax(logits, axis=1),
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out[0].sum(axis=1), 1.0, atol=1e-12)
    np.testing.assert_allclose(lse[0], scipy.special.logsumexp(logits, axis=1), atol=1e-12)


def test_attn_empty_and_partial_counts():
    r = _rng(13)
    q = r.standard_normal((1, 4, 8), dtype=np.float32)
    K = r.standard_normal((1, 2, 10, 8), dtype=np.float32)
    V = r.standard_normal((1, 2, 10, 8), dtype=np.float32)
    idx = np.array([[[0, 1, 2, 3], [5, 6, 7, 8]]], np.int32)
    out, lse = oracle.attn(q, K, V, idx, count=np.array([[0, 2]], np.int32))
    assert np.all(out[0, :2] == 0) and np.all(np.isneginf(lse[0, :2]))
    o2, l2 = oracle.attn(q[:, 2:], K[:, 1:], V[:, 1:], idx[:, 1:, :2])
    np.testing.assert_array_equal(out[0, 2:], o2[0])
    np.testing.assert_array_equal(lse[0, 2:], l2[0])


# --------------------------------------------------------------------------
# The decode step: one routing set shared by every layer
# --------------------------------------------------------------------------

def test_decode_step_routes_once_and_shares_the_set():
    r = _rng(31)
    B, N, Hq, Hkv, d, L, k = 1, 700, 8, 2, 64, 3, 50
    qr = r.standard_normal((B, Hq, d), dtype=np.float32)
    ql = r.standard_normal((L, B, Hq, d), dtype=np.float32)
    K = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    V = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    res = oracle.decode_step(qr, ql, K, V, k=k)
    np.testing.assert_array_equal(res["idx"], oracle.topk(oracle.scores(qr, K), k))
    for layer in range(L):
        Kg = np.take_along_axis(K, res["idx"][..., None].astype(np.int64), axis=2)
        Vg = np.take_along_axis(V, res["idx"][..., None].astype(np.int64), axis=2)
        o_ref, lse_ref = _sdpa_f64(ql[layer], Kg, Vg)
        np.testing.assert_allclose(res["out"][layer], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][layer], lse_ref, atol=1e-12)
    # nearest rank: tau is the ceil(0.9 * 700) = 630th smallest score, so
    # 700 - 630 + 1 = 71 distinct scores are kept per head
    tau = oracle.percentile_tau(res["S"], 90, 100)
    th = oracle.decode_step(qr, ql, K, V, tau=tau, cap=N)
    assert th["count"].tolist() == [[71, 71]]


# --------------------------------------------------------------------------
# Routing recomputed every R layers (CLSA article, sections 計算コストの削減効果
# and 推論速度の改善結果: per-layer routing vs one shared set vs sharing across
# a few layers)
# --------------------------------------------------------------------------

def test_grouped_step_per_layer_routing_vs_library():
    """R = 1: every layer routes with its own query.  Integer inputs make the
    scores exact, so each layer's set equals a stable argsort of the fp64
    library scores, and each layer's output equals dense attention over the
    gathered rows."""
    r = _rng(41)
    B, N, Hq, Hkv, d, L, k = 2, 90, 8, 2, 16, 3, 7
    G = Hq // Hkv
    qrs = r.integers(-3, 4, (L, B, Hq, d)).astype(np.float32)
    ql = r.standard_normal((L, B, Hq, d), dtype=np.float32)
    K = r.integers(-3, 4, (B, Hkv, N, d)).astype(np.float32)
    V = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    res = oracle.decode_step_grouped(qrs, ql, K, V, 1, k=k)
    for layer in range(L):
        qsum = qrs[layer].astype(np.float64).reshape(B, Hkv, G, d).sum(2)
        S64 = np.einsum("bhd,bhnd->bhn", qsum, K.astype(np.float64)) / math.sqrt(d)
        for b in range(B):
            for h in range(Hkv):
                ref = np.sort(np.argsort(-S64[b, h], kind="stable")[:k])
                np.testing.assert_array_equal(res["idx"][layer, b, h], ref)
        Kg = np.take_along_axis(K, res["idx"][layer][..., None].astype(np.int64), axis=2)
        Vg = np.take_along_axis(V, res["idx"][layer][..., None].astype(np.int64), axis=2)
        o_ref, lse_ref = _sdpa_f64(ql[layer], Kg, Vg)
        np.testing.assert_allclose(res["out"][layer], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][layer], lse_ref, atol=1e-12)


def test_grouped_step_group_boundaries_and_invariants():
    """Groups are R consecutive layers, the last one shorter when R does not
    divide L; R >= L is the shared-routing step; equal routing queries give
    equal sets in every group; threshold mode counts per group."""
    r = _rng(43)
    B, N, Hq, Hkv, d, L, k = 1, 300, 8, 2, 32, 5, 20
    ql = r.standard_normal((L, B, Hq, d), dtype=np.float32)
    K = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    V = r.standard_normal((B, Hkv, N, d), dtype=np.float32)
    qrs = r.standard_normal((3, B, Hq, d), dtype=np.float32)
    res = oracle.decode_step_grouped(qrs, ql, K, V, 2, k=k)       # layers {0,1} {2,3} {4}
    for g, layers in enumerate([[0, 1], [2, 3], [4]]):
        one = oracle.decode_step(qrs[g], ql[layers], K, V, k=k)
        np.testing.assert_array_equal(res["idx"][g], one["idx"])
        np.testing.assert_array_equal(res["out"][layers], one["out"])
    assert not np.array_equal(res["idx"][0], res["idx"][1])   # distinct queries route apart
    shared = oracle.decode_step_grouped(qrs[:1], ql, K, V, L, k=k)
    ref = oracle.decode_step(qrs[0], ql, K, V, k=k)
    np.testing.assert_array_equal(shared["idx"][0], ref["idx"])
    np.testing.assert_array_equal(shared["out"], ref["out"])
    same = oracle.decode_step_grouped(np.repeat(qrs[:1], 3, 0), ql, K, V, 2, k=k)
    for g in range(3):
        np.testing.assert_array_equal(same["idx"][g], ref["idx"])
    np.testing.assert_allclose(same["out"], ref["out"], rtol=0, atol=0)
    tau = np.stack([oracle.percentile_tau(res["S"][g], 95, 100) for g in range(3)])
    th = oracle.decode_step_grouped(qrs, ql, K, V, 2, tau=tau, cap=N)
    for g in range(3):
        S = oracle.scores(qrs[g], K)
        np.testing.assert_array_equal(th["count"][g], (S >= tau[g][..., None]).sum(-1))


# --------------------------------------------------------------------------
# Louver index, one subspace (Louver summary, section 2. Louver インデックス):
# balanced PCA tree clusters, bounding balls, ball test then exact check
# --------------------------------------------------------------------------

def _blobs(r, B, Hkv, N, d, nblob=16, spread=0.05):
    """Keys drawn around a few centres (low intrinsic dimension, like real
    attention keys), the structure the index prunes on."""
    centres = r.standard_normal((B, Hkv, nblob, d)).astype(np.float32) * 2
    which = r.integers(0, nblob, (B, Hkv, N))
    K = np.take_along_axis(centres, which[..., None], axis=2)
    return (K + spread * r.standard_normal((B, Hkv, N, d))).astype(np.float32)


def test_louver_tree_closed_form_split_and_balls():
    """Keys spread along one axis u (plus tiny noise): the root split of the
    balanced PCA tree puts the N/2 keys with the smallest coordinate along u
    on one side; clusters partition the keys; every ball holds its keys."""
    from oracle import louver
    r = _rng(51)
    N, d, rc = 256, 16, 16
    u = r.standard_normal(d)
    u /= np.linalg.norm(u)
    t = r.permutation(N).astype(np.float64)          # distinct coordinates
    Kh = (t[:, None] * u[None, :] + 1e-3 * r.standard_normal((N, d))).astype(np.float32)
    ix = louver.build_index(Kh, rc)
    perm = ix["perm"]
    assert sorted(perm.tolist()) == list(range(N))
    low = set(np.argsort(t)[:N // 2].tolist())
    halves = [set(perm[:N // 2].tolist()), set(perm[N // 2:].tolist())]
    assert low in halves
    X = Kh.astype(np.float64)[perm].reshape(N // rc, rc, d)
    dist = np.sqrt(((X - ix["centres"][:, None, :]) ** 2).sum(-1))
    assert np.all(dist <= ix["radii"][:, None] + 1e-12)
    np.testing.assert_allclose(ix["centres"], X.mean(1), rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", ["gaussian", "blobs"])
def test_louver_query_equals_full_scan_and_prunes_soundly(kind):
    """The index's threshold set equals the full-scan threshold set exactly
    (no false negatives, no extras) at several tau; every pruned cluster
    holds only keys scoring below tau; on clustered keys most clusters are
    pruned."""
    from oracle import louver
    r = _rng(53)
    B, Hq, Hkv, N, d, rc = 1, 8, 2, 1024, 32, 16
    q = r.standard_normal((B, Hq, d), dtype=np.float32)
    K = (r.standard_normal((B, Hkv, N, d), dtype=np.float32) if kind == "gaussian"
         else _blobs(r, B, Hkv, N, d))
    S = oracle.scores(q, K)
    S64 = oracle.scores(q, K, np.float64)
    for pct in (50, 97, 100):
        tau = oracle.percentile_tau(S, pct, 100)
        idx, cnt, surv = louver.route_threshold(q, K, tau, N, rc)
        ridx, rcnt = louver.full_scan_threshold(q, K, tau, N)
        np.testing.assert_array_equal(cnt, rcnt)
        np.testing.assert_array_equal(idx, ridx)
        G = Hq // Hkv
        for h in range(Hkv):
            ix = louver.build_index(K[0, h], rc)
            qbar = q[0, h * G:(h + 1) * G].astype(np.float64).sum(0) / math.sqrt(d)
            t = float(tau[0, h])
            pruned = ~louver.keep_clusters(ix, qbar, t)
            keys = ix["perm"].reshape(-1, rc)[pruned].ravel()
            assert np.all(S64[0, h, keys] < t)
        if kind == "blobs" and pct == 97:
            assert surv.sum() < 0.5 * Hkv * (N // rc)


@pytest.mark.parametrize("S", [2, 4])
@pytest.mark.parametrize("kind", ["gaussian", "blobs"])
def test_louver_subspaces_equal_full_scan_and_sound(S, kind):
    """The all-subspace filter with tau_s = tau - sum of the other subspaces'
    largest bounds: the set equals the full-scan threshold set; every key
    scoring >= tau in fp64 is a candidate (closed form: the sum of a key's
    subspace scores is its score, each bounded by its subspace's largest
    ball bound); with S = 1 the filter is the plain ball test."""
    from oracle import louver
    r = _rng(61 + S)
    B, Hq, Hkv, N, d, rc = 1, 8, 2, 1024, 32, 16
    q = r.standard_normal((B, Hq, d), dtype=np.float32)
    K = (r.standard_normal((B, Hkv, N, d), dtype=np.float32) if kind == "gaussian"
         else _blobs(r, B, Hkv, N, d))
    S32 = oracle.scores(q, K)
    S64 = oracle.scores(q, K, np.float64)
    G = Hq // Hkv
    for pct in (50, 97, 100):
        tau = oracle.percentile_tau(S32, pct, 100)
        idx, cnt, ncand = louver.route_threshold_subspaces(q, K, tau, N, rc, S)
        ridx, rcnt = louver.full_scan_threshold(q, K, tau, N)
        np.testing.assert_array_equal(cnt, rcnt)
        np.testing.assert_array_equal(idx, ridx)
        assert np.all(ncand >= cnt)
        ds = d // S
        for h in range(Hkv):
            Kh = K[0, h]
            indexes = [louver.build_index(Kh[:, s * ds:(s + 1) * ds], rc) for s in range(S)]
            qbar = q[0, h * G:(h + 1) * G].astype(np.float64).sum(0) / math.sqrt(d)
            t = float(tau[0, h])
            keep = louver.keep_clusters_subspaces(indexes, qbar, t)
            cand = louver.candidates(indexes, keep, N)
            assert np.all(cand[S64[0, h] >= t]), "a key scoring >= tau was filtered out"
            # the subspace scores of every key add up to its score
            part = sum(Kh[:, s * ds:(s + 1) * ds].astype(np.float64) @ qbar[s * ds:(s + 1) * ds]
                       for s in range(S))
            np.testing.assert_allclose(part, S64[0, h], rtol=1e-12, atol=1e-12)
    # S = 1 reduces to the plain ball test
    tau = oracle.percentile_tau(S32, 97, 100)
    for h in range(Hkv):
        ix = louver.build_index(K[0, h], rc)
        qbar = q[0, h * G:(h + 1) * G].astype(np.float64).sum(0) / math.sqrt(d)
        t = float(tau[0, h])
        np.testing.assert_array_equal(louver.keep_clusters_subspaces([ix], qbar, t)[0],
                                      louver.keep_clusters(ix, qbar, t))

