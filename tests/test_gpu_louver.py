"""GPU parity of the Louver index (Louver summary, section 2. Louver インデックス;
section 1. 半空間範囲検索への帰着 for the set it must return).

The index itself is not unique (the tree's directions come from fp32 power
iteration on the device, the oracle's from an exact eigendecomposition), so
the tests check what makes any index valid -- the permutation, the clusters'
balanced sizes, ball containment in fp64, centres equal to member means --
and what is unique: the returned set, which must equal the full-scan
threshold set on the same scores bit for bit (GPU route_threshold) and the
oracle's set within the comparison band; and zero false negatives.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import louver as olouver
import token_sparse_attention_sm_b200 as sd
from token_sparse_attention_sm_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    from token_sparse_attention_sm_b200 import build
    build.build()
    sd.load()
    return torch.device("cuda", 0)


def _band(s):
    return 1e-4 * abs(float(s)) + 1e-6


def _f(x):
    return synth.f32(x)


def _assert_same_set(a, b, cap):
    """(idx, count) pairs equal: the counts, and the first min(count, cap)
    entries of every row (entries beyond them are not written)."""
    ai, ac = a[0].cpu().numpy(), a[1].cpu().numpy()
    bi, bc = b[0].cpu().numpy(), b[1].cpu().numpy()
    np.testing.assert_array_equal(ac, bc)
    for bh in np.ndindex(ac.shape):
        n = min(int(ac[bh]), cap)
        np.testing.assert_array_equal(ai[bh][:n], bi[bh][:n])


def _check_index(ix, K32, r):
    """K32 [B,Hkv,N,d] fp32 (the keys the index covers)."""
    B, Hkv, N, d = K32.shape
    perm = ix.perm().cpu().numpy()
    keys = ix.keys().float().cpu().numpy()
    cen = ix.centres().cpu().numpy().astype(np.float64)
    rad = ix.radii().cpu().numpy().astype(np.float64)
    lcen = ix.leaf_centres().cpu().numpy().astype(np.float64)
    lrad = ix.leaf_radii().cpu().numpy().astype(np.float64)
    for b in range(B):
        for h in range(Hkv):
            p = perm[b, h]
            assert np.array_equal(np.sort(p), np.arange(N)), "not a permutation"
            np.testing.assert_array_equal(keys[b, h], K32[b, h][p])  # cluster-ordered copy
            members = K32[b, h][p].astype(np.float64).reshape(N // r, r, d)
            mean = members.mean(axis=1)
            np.testing.assert_allclose(cen[b, h], mean, rtol=1e-4, atol=1e-4)
            dist = np.sqrt(((members - cen[b, h][:, None, :]) ** 2).sum(-1)).max(axis=1)
            assert np.all(dist <= rad[b, h]), "a key lies outside its cluster's ball"
            # the 32-key leaves below the clusters
            leaves = K32[b, h][p].astype(np.float64).reshape(N // 32, 32, d)
            np.testing.assert_allclose(lcen[b, h], leaves.mean(axis=1), rtol=1e-4, atol=1e-4)
            ldist = np.sqrt(((leaves - lcen[b, h][:, None, :]) ** 2).sum(-1)).max(axis=1)
            assert np.all(ldist <= lrad[b, h]), "a key lies outside its leaf's ball"


def _check_set(gidx, gcnt, q32, K32, tau, cap):
    """The GPU set against the oracle: equal to the fp32 threshold set except
    for keys within the band of tau; every key >= tau + band present."""
    S = oracle.scores(q32, K32)
    S64 = oracle.scores(q32, K32, np.float64)
    ridx, rcnt = oracle.threshold(S, tau, cap)
    B, Hkv = gcnt.shape
    for b in range(B):
        for h in range(Hkv):
            t = tau[b, h]
            band = _band(t)
            g = set(gidx[b, h, :min(gcnt[b, h], cap)].tolist())
            if gcnt[b, h] <= cap:
                must = set(np.nonzero(S64[b, h] >= t + band)[0].tolist())
                never = set(np.nonzero(S64[b, h] < t - band)[0].tolist())
                assert must <= g, "false negative"
                assert not (g & never), "false positive"
            assert abs(int(gcnt[b, h]) - int(rcnt[b, h])) <= \
                int(np.sum(np.abs(S[b, h] - t) <= band))
    return rcnt


CASES = [
    dict(B=1, N=8192, Hq=8, Hkv=2, d=128, dtype="bf16", r=128, blobs=16, pct=97),
    dict(B=2, N=4096, Hq=4, Hkv=2, d=64, dtype="f32", r=64, blobs=8, pct=90),
    dict(B=1, N=16384, Hq=16, Hkv=4, d=128, dtype="bf16", r=256, blobs=0, pct=99),
    dict(B=1, N=2048, Hq=2, Hkv=1, d=64, dtype="bf16", r=32, blobs=4, pct=50),
    # more than 16 heads: each head's clusters owned by CTAs of that head only
    dict(B=3, N=2048, Hq=8, Hkv=8, d=64, dtype="bf16", r=64, blobs=4, pct=90),
    dict(B=5, N=4096, Hq=16, Hkv=4, d=128, dtype="f32", r=128, blobs=8, pct=97),
    # more heads than SMs: one CTA per head, the grid takes more than one wave
    dict(B=40, N=1024, Hq=8, Hkv=4, d=64, dtype="bf16", r=32, blobs=4, pct=90),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
def test_louver_index_and_set(dev, c):
    w = synth.custom(B=c["B"], N=c["N"], Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"], L=1,
                     dtype=c["dtype"], seed=11, mode="threshold", cap=c["N"],
                     blobs=c["blobs"], blob_spread=0.1)
    x = synth.generate(w)
    q32, K32 = _f(x["q_route"]), _f(x["K"])
    qd, Kd = x["q_route"].to(dev), x["K"].to(dev)
    ix = sd.louver_build(Kd, c["r"])
    _check_index(ix, K32, c["r"])
    S = oracle.scores(q32, K32)
    tau = oracle.percentile_tau(S, c["pct"], 100)
    taud = torch.from_numpy(tau).to(dev)
    cap = c["N"]
    gidx, gcnt, surv = sd.louver_route_threshold(qd, Kd, ix, taud, cap, return_survivors=True)
    # bit-identical to the full-scan threshold routing on the GPU
    _assert_same_set((gidx, gcnt), sd.route_threshold(qd, Kd, taud, cap), cap)
    gidx, gcnt = gidx.cpu().numpy(), gcnt.cpu().numpy()
    _check_set(gidx, gcnt, q32, K32, tau, cap)
    # every cluster, and every 32-key leaf, holding a selected key passed its
    # ball test
    perm = ix.perm().cpu().numpy()
    surv = surv.cpu().numpy()
    nc = c["N"] // c["r"]
    for b in range(c["B"]):
        for h in range(c["Hkv"]):
            pos = np.empty(c["N"], np.int64)
            pos[perm[b, h]] = np.arange(c["N"])
            sel = gidx[b, h, :gcnt[b, h]]
            held = len(set((pos[sel] // c["r"]).tolist()))
            held_leaves = len(set((pos[sel] // 32).tolist()))
            assert held <= surv[b, h, 0] <= nc
            assert held_leaves <= surv[b, h, 1] <= surv[b, h, 0] * (c["r"] // 32)


def test_louver_matches_oracle_louver(dev):
    """The oracle's own Louver route (its own index) returns the same set on
    the oracle's scores; the GPU set agrees with it within the band."""
    w = synth.custom(B=1, N=4096, Hq=8, Hkv=2, d=64, L=1, dtype="f32", seed=5,
                     mode="threshold", cap=4096, blobs=16, blob_spread=0.05)
    x = synth.generate(w)
    q32, K32 = _f(x["q_route"]), _f(x["K"])
    tau = oracle.percentile_tau(oracle.scores(q32, K32), 97, 100)
    oidx, ocnt, osurv = olouver.route_threshold(q32, K32, tau, 4096, 64)
    ix = sd.louver_build(x["K"].to(dev), 64)
    gidx, gcnt, gsurv = sd.louver_route_threshold(x["q_route"].to(dev), x["K"].to(dev), ix,
                                                  torch.from_numpy(tau).to(dev), 4096,
                                                  return_survivors=True)
    gidx, gcnt = gidx.cpu().numpy(), gcnt.cpu().numpy()
    rcnt = _check_set(gidx, gcnt, q32, K32, tau, 4096)
    np.testing.assert_array_equal(ocnt, rcnt)
    # both indexes prune most clusters on tightly clustered keys
    assert osurv.max() < 0.5 * (4096 // 64)
    assert gsurv.cpu().numpy()[..., 0].max() < 0.5 * (4096 // 64)


def test_louver_prunes_clustered_128k(dev):
    """The clustered 128K workload: zero false negatives and most clusters
    pruned, at the size the benchmark measures."""
    w = synth.WORKLOADS["louver_128k"]
    x = synth.generate(w)
    q32, K32 = _f(x["q_route"]), _f(x["K"])
    qd, Kd = x["q_route"].to(dev), x["K"].to(dev)
    tau = oracle.percentile_tau(oracle.scores(q32, K32), *w.tau_pct)
    taud = torch.from_numpy(tau).to(dev)
    ix = sd.louver_build(Kd, 128)
    gidx, gcnt, surv = sd.louver_route_threshold(qd, Kd, ix, taud, w.cap, return_survivors=True)
    _assert_same_set((gidx, gcnt), sd.route_threshold(qd, Kd, taud, w.cap), w.cap)
    _check_set(gidx.cpu().numpy(), gcnt.cpu().numpy(), q32, K32, tau, w.cap)
    surv = surv.cpu().numpy()
    assert surv[..., 0].max() < 0.5 * (w.N // 128)
    assert np.all(surv[..., 1] < surv[..., 0] * 4)   # the leaf balls prune inside clusters


def test_louver_cache_longer_than_length_and_rebuild(dev):
    """n < n_cap: the index covers the first n rows only; keys beyond are
    never returned.  A second build over the same keys gives a valid index
    and the same set."""
    w = synth.custom(B=1, N=6144, Hq=8, Hkv=2, d=128, L=1, dtype="bf16", seed=3,
                     mode="threshold", cap=4096, blobs=8)
    x = synth.generate(w)
    n = 4096
    Kd = x["K"].to(dev)
    qd = x["q_route"].to(dev)
    K32 = _f(x["K"])[:, :, :n]
    q32 = _f(x["q_route"])
    tau = oracle.percentile_tau(oracle.scores(q32, K32), 90, 100)
    taud = torch.from_numpy(tau).to(dev)
    ix = sd.louver_build(Kd, 64, n=n)
    _check_index(ix, K32, 64)
    a = sd.louver_route_threshold(qd, Kd, ix, taud, 4096)
    ix2 = sd.louver_build(Kd, 64, n=n)
    _check_index(ix2, K32, 64)
    b = sd.louver_route_threshold(qd, Kd, ix2, taud, 4096)
    f = sd.route_threshold(qd, Kd, taud, 4096, n=n)
    _assert_same_set(a, f, 4096)
    _assert_same_set(b, f, 4096)
    _check_set(a[0].cpu().numpy(), a[1].cpu().numpy(), q32, K32, tau, 4096)


def test_louver_empty_set_capacity_and_status_reset(dev):
    w = synth.custom(B=1, N=2048, Hq=4, Hkv=2, d=64, L=1, dtype="bf16", seed=8,
                     mode="threshold", cap=64, blobs=4)
    x = synth.generate(w)
    qd, Kd = x["q_route"].to(dev), x["K"].to(dev)
    ix = sd.louver_build(Kd, 64)
    tau = torch.tensor([[1e9, -1e9]], device=dev)
    gidx, gcnt = sd.louver_route_threshold(qd, Kd, ix, tau, 64, check=False)
    assert sd.read_device_status(ix.ws, raise_on_error=False) == 4   # capacity
    assert gcnt.cpu().tolist() == [[0, 2048]]
    assert gidx[0, 1].cpu().tolist() == list(range(64))
    tau = torch.full((1, 2), 1e9, device=dev)
    _, gcnt = sd.louver_route_threshold(qd, Kd, ix, tau, 64, check=False)
    assert sd.read_device_status(ix.ws, raise_on_error=False) == 0   # reset
    assert gcnt.cpu().tolist() == [[0, 0]]


def test_louver_repeated_queries_keep_workspace_clean(dev):
    """Many queries through one index: the bitmap and survivor counters the
    kernels keep zero between calls stay zero (every call equals the full
    scan)."""
    w = synth.custom(B=2, N=4096, Hq=8, Hkv=2, d=128, L=1, dtype="bf16", seed=21,
                     mode="threshold", cap=4096, blobs=16)
    x = synth.generate(w)
    Kd = x["K"].to(dev)
    ix = sd.louver_build(Kd, 128)
    variants = synth.query_variants(w, x, 6, seed=77)
    for i, (qr, _) in enumerate(variants):
        qd = qr.to(dev)
        S = oracle.scores(_f(qr), _f(x["K"]))
        tau = torch.from_numpy(oracle.percentile_tau(S, 80 + 3 * i, 100)).to(dev)
        a = sd.louver_route_threshold(qd, Kd, ix, tau, 4096)
        _assert_same_set(a, sd.route_threshold(qd, Kd, tau, 4096), 4096)


@pytest.mark.parametrize("cap", [262144, 100000])
def test_louver_large_sets_several_compaction_passes(dev, cap):
    """Half of 262,144 keys selected: the head's bitmap takes two compaction
    passes and each pass selects more indices than the staging buffer in
    shared memory holds (the rest go straight to memory); with cap below the
    count the first cap indices are kept and capacity is flagged."""
    w = synth.custom(B=1, N=262144, Hq=4, Hkv=1, d=64, L=1, dtype="bf16", seed=13,
                     mode="threshold", cap=cap)
    x = synth.generate(w)
    qd, Kd = x["q_route"].to(dev), x["K"].to(dev)
    q32, K32 = _f(x["q_route"]), _f(x["K"])
    tau = oracle.percentile_tau(oracle.scores(q32, K32), 50, 100)
    taud = torch.from_numpy(tau).to(dev)
    ix = sd.louver_build(Kd, 64)
    a = sd.louver_route_threshold(qd, Kd, ix, taud, cap, check=False)
    st_a = sd.read_device_status(ix.ws, raise_on_error=False)
    ws = sd.Workspace(dev)
    f = sd.route_threshold(qd, Kd, taud, cap, ws=ws, check=False)
    st_f = sd.read_device_status(ws, raise_on_error=False)
    _assert_same_set(a, f, cap)
    assert st_a == st_f == (4 if int(a[1][0, 0]) > cap else 0)
    assert int(a[1][0, 0]) > 65536


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_louver_decode_step_equals_route_then_gather(dev, dtype, d):
    """The fused Louver step returns exactly what routing through the index
    followed by the gather attention returns, and its attention matches the
    oracle on the oracle's threshold set."""
    w = synth.custom(B=1, N=8192, Hq=8, Hkv=2, d=d, L=4, dtype=dtype, seed=23,
                     mode="threshold", cap=2048, blobs=16)
    x = synth.generate(w)
    t = {n: x[n].to(dev) for n in ("q_route", "q_layers", "K", "V")}
    q32, K32 = _f(x["q_route"]), _f(x["K"])
    S = oracle.scores(q32, K32)
    tau = oracle.percentile_tau(S, 95, 100)
    taud = torch.from_numpy(tau).to(dev)
    ix = sd.louver_build(t["K"], 128)
    res = sd.louver_decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], ix, taud, w.cap)
    gidx, gcnt = sd.louver_route_threshold(t["q_route"], t["K"], ix, taud, w.cap)
    o, l = sd.attn_gather(t["q_layers"], t["K"], t["V"], gidx, count=gcnt)
    _assert_same_set((res["idx"], res["count"]), (gidx, gcnt), w.cap)
    assert torch.equal(res["out"], o) and torch.equal(res["lse"], l)
    ridx, rcnt = oracle.threshold(S, tau, w.cap)
    _check_set(res["idx"].cpu().numpy(), res["count"].cpu().numpy(), q32, K32, tau, w.cap)
    o_ref, l_ref = oracle.attn(_f(x["q_layers"]), K32, _f(x["V"]), ridx, rcnt)
    o_gpu, l_gpu = sd.attn_gather(t["q_layers"], t["K"], t["V"], torch.from_numpy(ridx).to(dev),
                                  count=torch.from_numpy(rcnt).to(dev))
    tol = 2e-2 if dtype == "bf16" else 1e-4
    assert np.abs(o_gpu.float().cpu().numpy() - o_ref).max() <= tol



@pytest.mark.parametrize("seed", range(24))
def test_louver_random_shapes(dev, seed):
    """Seeded random shapes (r 32..256, N = r * 2^j up to 32K, B, Hkv, G,
    d 64/128, fp32/bf16, clustered or Gaussian keys, tau from the median to
    beyond the maximum, cap below and above the set size): the set equals the
    full-scan threshold routing bitwise, with the same status."""
    rng = np.random.default_rng(20_000 + seed)
    r = int(rng.choice([32, 64, 128, 256]))
    N = r * int(2 ** rng.integers(0, 8))
    N = min(N, 32768)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4]))
    B = int(rng.integers(1, 3))
    d = int(rng.choice([64, 128]))
    dtype = str(rng.choice(["bf16", "f32"]))
    blobs = int(rng.choice([0, 4, 16]))
    pct = int(rng.choice([50, 90, 99, 100]))
    cap = int(rng.integers(1, N + 1))
    w = synth.custom(B=B, N=N, Hq=G * Hkv, Hkv=Hkv, d=d, L=1, dtype=dtype, seed=seed,
                     mode="threshold", cap=cap, blobs=blobs)
    x = synth.generate(w)
    qd, Kd = x["q_route"].to(dev), x["K"].to(dev)
    tau = oracle.percentile_tau(oracle.scores(_f(x["q_route"]), _f(x["K"])), pct, 100)
    if pct == 100:
        tau = tau + 1.0  # beyond every score: empty sets
    taud = torch.from_numpy(tau.astype(np.float32)).to(dev)
    ix = sd.louver_build(Kd, r)
    a = sd.louver_route_threshold(qd, Kd, ix, taud, cap, check=False)
    sa = sd.read_device_status(ix.ws, raise_on_error=False)
    ws = sd.Workspace(dev)
    f = sd.route_threshold(qd, Kd, taud, cap, ws=ws, check=False)
    sf = sd.read_device_status(ws, raise_on_error=False)
    _assert_same_set(a, f, cap)
    assert sa == sf


def test_louver_step_graph_equals_eager(dev):
    """DecodeStepGraph routing through a Louver index returns, for each query
    written into its pinned views, what the eager louver_decode_step returns."""
    w = synth.custom(B=1, N=8192, Hq=8, Hkv=2, d=128, L=3, dtype="bf16", seed=31,
                     mode="threshold", cap=2048, blobs=16)
    x = synth.generate(w)
    K, V = x["K"].to(dev), x["V"].to(dev)
    tau = oracle.percentile_tau(oracle.scores(_f(x["q_route"]), _f(x["K"])), 95, 100)
    taud = torch.from_numpy(tau).to(dev)
    ix = sd.louver_build(K, 128)
    g = sd.DecodeStepGraph(K, V, w.L, w.Hq, tau=taud, cap=w.cap, ws=sd.Workspace(dev), index=ix)
    for qr, ql in synth.query_variants(w, x, 3, seed=5):
        g.q_route_host.copy_(qr)
        g.q_layers_host.copy_(ql)
        out_h, idx_h, cnt_h = g()
        ref = sd.louver_decode_step(qr.to(dev), ql.to(dev), K, V, ix, taud, w.cap)
        assert torch.equal(out_h, ref["out"].cpu())
        _assert_same_set((idx_h, cnt_h), (ref["idx"].cpu(), ref["count"].cpu()), w.cap)


def test_louver_nonfinite_inputs_are_flagged(dev):
    """A NaN key makes the index build report SPARSE_ERR_NONFINITE; a NaN tau
    makes the query report it; neither faults, and a clean build and query on
    the same workspace afterwards work."""
    w = synth.custom(B=1, N=2048, Hq=4, Hkv=2, d=64, L=1, dtype="f32", seed=12,
                     mode="threshold", cap=2048, blobs=4)
    x = synth.generate(w)
    K = x["K"].clone()
    K[0, 1, 77, 5] = float("nan")
    Kd = K.to(dev)
    with pytest.raises(sd.SparseDecodeError) as ei:
        sd.louver_build(Kd, 64)
    assert ei.value.status == 5
    Kc = x["K"].to(dev)
    ix = sd.louver_build(Kc, 64)
    qd = x["q_route"].to(dev)
    tau = torch.tensor([[0.5, float("nan")]], device=dev)
    sd.louver_route_threshold(qd, Kc, ix, tau, 2048, check=False)
    assert sd.read_device_status(ix.ws, raise_on_error=False) == 5
    tau = torch.tensor([[0.5, 0.5]], device=dev)
    a = sd.louver_route_threshold(qd, Kc, ix, tau, 2048)
    _assert_same_set(a, sd.route_threshold(qd, Kc, tau, 2048), 2048)


def _keys_on_a_line(rng, N, d, torch_dtype):
    """Keys t_i * s (one head): t a permutation of N distinct values, s a
    fixed direction.  fp32: s a random unit vector plus 1e-3 noise per key;
    bf16: s with entries in {+-1, +-1/2, +-1/4} and t integers in [-N/2, N/2),
    so every key is exact in bf16 (N <= 256) and the keys are collinear."""
    t = rng.permutation(N).astype(np.float64) - N // 2
    if torch_dtype == torch.float32:
        s = rng.standard_normal(d)
        s /= np.linalg.norm(s)
        Kh = t[:, None] * s[None, :] + 1e-3 * rng.standard_normal((N, d))
    else:
        s = rng.choice([-1.0, -0.5, -0.25, 0.25, 0.5, 1.0], size=d)
        Kh = t[:, None] * s[None, :]
    return t, Kh.astype(np.float32)


@pytest.mark.parametrize("dtype,d,N,r", [("f32", 64, 4096, 64), ("bf16", 128, 256, 32),
                                         ("f32", 128, 2048, 256)])
def test_louver_tree_splits_keys_on_a_line_by_their_coordinate(dev, dtype, d, N, r):
    """Louver summary, section 2. Louver インデックス (balanced tree of
    principal-direction splits at the median): for keys spread along one
    direction the principal direction of every node is that direction, so
    every node of the tree -- each run of N / 2^L consecutive entries of the
    cluster order, down to the 32-key leaves -- holds the keys whose
    coordinates along it have ranks in one aligned block [j N/2^L, (j+1)
    N/2^L).  The GPU tree must have this form at every level, and its node
    sets must equal the oracle's (fp64 eigendecomposition) at every level.
    """
    torch_dtype = torch.float32 if dtype == "f32" else torch.bfloat16
    rng = np.random.default_rng(4242)
    B, Hkv = 1, 2
    ts, K32 = [], np.zeros((B, Hkv, N, d), np.float32)
    for h in range(Hkv):
        t, Kh = _keys_on_a_line(rng, N, d, torch_dtype)
        ts.append(t)
        K32[0, h] = Kh
    K = torch.from_numpy(K32).to(dev, torch_dtype)
    assert torch.equal(K.float().cpu(), torch.from_numpy(K32)), "keys not exact in this dtype"
    ix = sd.louver_build(K, r)
    torch.cuda.synchronize()
    _check_index(ix, K32, r)
    perm = ix.perm().cpu().numpy()
    for h in range(Hkv):
        rank = np.empty(N, np.int64)
        rank[np.argsort(ts[h], kind="stable")] = np.arange(N)
        oix = olouver.build_index(K32[0, h], r)
        operm = np.asarray(oix["perm"])
        size = N // 2
        while size >= 32:
            for j in range(N // size):
                blk = rank[perm[0, h, j * size:(j + 1) * size]]
                lo = blk.min()
                assert lo % size == 0 and blk.max() == lo + size - 1, \
                    f"head {h}: node of {size} keys is not one block of coordinate ranks"
            if size >= r:  # the oracle's tree stops at the clusters
                g = sorted(tuple(sorted(perm[0, h, j * size:(j + 1) * size].tolist()))
                           for j in range(N // size))
                o = sorted(tuple(sorted(operm[j * size:(j + 1) * size].tolist()))
                           for j in range(N // size))
                assert g == o, f"head {h}: nodes of {size} keys differ from the oracle's"
            size //= 2
