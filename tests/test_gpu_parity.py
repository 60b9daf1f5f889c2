"""Parity of the CUDA library (through its C ABI) with the CPU oracle.

Comparison rules (fixed before any kernel ran):
* Scores: |S_gpu - S_exact| within the fp32 rounding bound of the kernel's
  order of operations, gamma_{G+d+1} * sum|q_i k_i| / sqrt(d) with
  gamma_n = n 2^-24 / (1 - n 2^-24), S_exact in fp64.
* Selection on the SAME fp32 scores (the GPU's own, fed to the oracle):
  bit-exact index sets, ties included (the decision is taken in the same
  precision on both sides).
* Routing end to end (GPU scores vs oracle scores): the sets may differ only
  in keys whose oracle score lies within 1e-4*|s_k| + 1e-6 of the k-th score
  (or of tau); top-k sets keep exactly k members; threshold sets miss no key
  whose fp64 score is >= tau + band.
* Attention on the oracle's own index set: max |out - oracle| <= 1e-4 for
  fp32 and <= 2e-2 for bf16; lse within 1e-4 (fp32) / 1e-3 (bf16).
Passages: CLSA article, sections 研究の背景と課題 and CLSAの仕組み; Louver
summary, sections 問題定義 and 1. 半空間範囲検索への帰着."""
import numpy as np
import pytest
import torch

import oracle
import token_sparse_attention_sm_b200 as sd
from token_sparse_attention_sm_b200 import synth

pytestmark = pytest.mark.gpu

OUT_TOL = {"f32": 1e-4, "bf16": 2e-2}
LSE_TOL = {"f32": 1e-4, "bf16": 1e-3}


@pytest.fixture(scope="module")
def dev():
    from token_sparse_attention_sm_b200 import build
    build.build()
    sd.load()
    return torch.device("cuda", 0)


def _to(dev, x, names=("q_route", "q_layers", "K", "V")):
    return {n: x[n].to(dev) for n in names}


def _f(x):
    return synth.f32(x)


def _band(s):
    return 1e-4 * abs(float(s)) + 1e-6


def assert_topk_within_band(gidx, S_oracle, k):
    """gidx [B,Hkv,k] from the GPU; S_oracle [B,Hkv,N] fp32 oracle scores."""
    B, Hkv, _ = gidx.shape
    ref = oracle.topk(S_oracle, k)
    for b in range(B):
        for h in range(Hkv):
            g = gidx[b, h]
            assert len(set(g.tolist())) == k, "duplicate indices"
            assert np.all(np.diff(g) > 0), "not ascending"
            kth = np.sort(S_oracle[b, h])[-k]
            diff = set(g.tolist()) ^ set(ref[b, h].tolist())
            bad = [j for j in diff if abs(S_oracle[b, h, j] - kth) > _band(kth)]
            assert not bad, f"(b={b},h={h}) {len(bad)} indices outside the band"


def assert_attn_close(out_gpu, lse_gpu, out_ref, lse_ref, dtype):
    o = out_gpu.float().cpu().numpy()
    err = np.abs(o - out_ref).max()
    assert err <= OUT_TOL[dtype], f"max |out - oracle| = {err}"
    lg = lse_gpu.cpu().numpy().astype(np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lg), fin)
    if fin.any():
        lerr = np.abs(lg[fin] - lse_ref[fin]).max()
        assert lerr <= LSE_TOL[dtype], f"max |lse - oracle| = {lerr}"


# ---------------------------------------------------------------------------
# A1: scores
# ---------------------------------------------------------------------------

SCORE_CASES = [
    dict(B=1, N=4096, Hq=8, Hkv=2, d=64, dtype="f32"),
    dict(B=2, N=1000, Hq=8, Hkv=2, d=128, dtype="f32"),
    dict(B=1, N=4099, Hq=32, Hkv=8, d=128, dtype="bf16"),
    dict(B=3, N=777, Hq=8, Hkv=8, d=64, dtype="bf16"),
    dict(B=1, N=5, Hq=16, Hkv=1, d=128, dtype="bf16"),
    dict(B=2, N=300, Hq=16, Hkv=2, d=64, dtype="f32"),
]


@pytest.mark.parametrize("c", SCORE_CASES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
def test_scores_match_oracle(dev, c):
    w = synth.custom(L=1, k=1, heavy=0, seed=c["N"], **c)
    x = synth.generate(w)
    t = _to(dev, x)
    S = sd.score(t["q_route"], t["K"]).cpu().numpy()
    q, K = _f(x["q_route"]), _f(x["K"])
    S64 = oracle.scores(q, K, np.float64)
    G = w.G
    Krep = np.repeat(np.abs(K.astype(np.float64)), G, axis=1)
    mag = np.einsum("bgd,bgnd->bgn", np.abs(q.astype(np.float64)), Krep)
    mag = mag.reshape(w.B, w.Hkv, G, w.N).sum(axis=2) / np.sqrt(w.d)
    # The kernel sums the G query rows (G-1 fp32 additions), multiplies by
    # fl(1/sqrt(d)) (two roundings: the constant and the product), then takes
    # one d-long dot product with fused multiply-adds (at most d-1 rounded
    # additions in any order).  Every rounding is relative to a partial sum
    # bounded by the magnitudes above, so with u = 2^-24 and
    # gamma_n = n u / (1 - n u) the error is at most gamma_{G+d} * mag; one
    # more u covers the fp64 arbiter's own rounding (about 2^-53 * G d * mag).
    u = 2.0 ** -24
    n = G + w.d + 1
    bound = n * u / (1 - n * u) * mag + 1e-30
    assert np.all(np.abs(S - S64) <= bound)


# ---------------------------------------------------------------------------
# A2 / A2': selection on identical scores -> bit-exact
# ---------------------------------------------------------------------------

SEL_CASES = [(1, 4096, 256), (2, 32768, 2048), (1, 131072, 2048), (3, 1000, 1),
             (1, 1000, 1000), (2, 5, 3), (1, 70000, 4097), (4, 2048, 2047)]


@pytest.mark.parametrize("B,N,k", SEL_CASES)
def test_select_topk_bit_exact(dev, B, N, k):
    r = np.random.default_rng(N + k)
    S = (r.standard_normal((B, 2, N)) * 2).astype(np.float32)
    idx = sd.select_topk(torch.from_numpy(S).to(dev), k).cpu().numpy()
    np.testing.assert_array_equal(idx, oracle.topk(S, k))


@pytest.mark.parametrize("levels", [1, 3, 50, 4000])
def test_select_topk_ties_bit_exact(dev, levels):
    """Few distinct score values: the k-th value is shared by many keys and
    the lower indices must win; -0.0 and +0.0 are the same score."""
    r = np.random.default_rng(levels)
    N, k = 20000, 1500
    S = r.integers(0, levels, size=(2, 3, N)).astype(np.float32) - levels // 2
    S[0, 0, ::7] = -0.0
    idx = sd.select_topk(torch.from_numpy(S).to(dev), k).cpu().numpy()
    np.testing.assert_array_equal(idx, oracle.topk(S, k))


def test_select_topk_all_equal(dev):
    S = np.full((1, 2, 5000), 0.5, np.float32)
    idx = sd.select_topk(torch.from_numpy(S).to(dev), 100).cpu().numpy()
    np.testing.assert_array_equal(idx, np.tile(np.arange(100), (1, 2, 1)))


@pytest.mark.parametrize("B,N,cap,pct", [(1, 131072, 8192, 97), (2, 4096, 300, 90),
                                         (1, 1000, 1000, 0), (3, 77, 5, 50)])
def test_select_threshold_bit_exact(dev, B, N, cap, pct):
    r = np.random.default_rng(N)
    S = (r.standard_normal((B, 2, N)) * 2).astype(np.float32)
    tau = oracle.percentile_tau(S, pct, 100) if pct else S.min(axis=2)
    ws = sd.Workspace(dev)
    gidx, gcnt = sd.select_threshold(torch.from_numpy(S).to(dev),
                                     torch.from_numpy(tau).to(dev), cap, ws=ws,
                                     check=False)
    st = sd.read_device_status(ws, raise_on_error=False)
    ridx, rcnt = oracle.threshold(S, tau, cap)
    gcnt = gcnt.cpu().numpy()
    np.testing.assert_array_equal(gcnt, rcnt)
    gidx = gidx.cpu().numpy()
    for b in range(B):
        for h in range(2):
            n = min(rcnt[b, h], cap)
            np.testing.assert_array_equal(gidx[b, h, :n], ridx[b, h, :n])
    assert st == (4 if (rcnt > cap).any() else 0)


def test_select_threshold_empty_and_capacity(dev):
    S = np.random.default_rng(1).standard_normal((1, 2, 3000)).astype(np.float32)
    ws = sd.Workspace(dev)
    tau = np.array([[100.0, -100.0]], np.float32)
    gidx, gcnt = sd.select_threshold(torch.from_numpy(S).to(dev),
                                     torch.from_numpy(tau).to(dev), 64, ws=ws,
                                     check=False)
    assert sd.read_device_status(ws, raise_on_error=False) == 4   # capacity
    assert gcnt.cpu().tolist() == [[0, 3000]]
    assert gidx[0, 1].cpu().tolist() == list(range(64))
    sd.select_threshold(torch.from_numpy(S).to(dev),
                        torch.from_numpy(np.full((1, 2), 100.0, np.float32)).to(dev),
                        64, ws=ws, check=False)
    assert sd.read_device_status(ws, raise_on_error=False) == 0   # status was reset


# ---------------------------------------------------------------------------
# A3 / A4: attention on the oracle's index set
# ---------------------------------------------------------------------------

ATTN_CASES = [
    dict(B=1, N=4096, Hq=8, Hkv=2, d=64, L=2, k=256, dtype="f32"),
    dict(B=2, N=3000, Hq=32, Hkv=8, d=128, L=16, k=2048, dtype="bf16"),
    dict(B=1, N=999, Hq=8, Hkv=1, d=128, L=3, k=77, dtype="bf16"),
    dict(B=2, N=500, Hq=4, Hkv=4, d=64, L=1, k=1, dtype="bf16"),
    dict(B=1, N=700, Hq=16, Hkv=1, d=64, L=5, k=700, dtype="f32"),
    dict(B=1, N=129, Hq=32, Hkv=8, d=128, L=40, k=129, dtype="bf16"),
]


@pytest.mark.parametrize("c", ATTN_CASES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
def test_attn_gather_matches_oracle(dev, c):
    w = synth.custom(heavy=0, seed=c["N"] + c["L"], **c)
    x = synth.generate(w)
    t = _to(dev, x)
    S = oracle.scores(_f(x["q_route"]), _f(x["K"]))
    idx = oracle.topk(S, w.k)
    out, lse = sd.attn_gather(t["q_layers"], t["K"], t["V"], torch.from_numpy(idx).to(dev))
    o_ref, l_ref = oracle.attn(_f(x["q_layers"]), _f(x["K"]), _f(x["V"]), idx)
    assert_attn_close(out, lse, o_ref, l_ref, w.dtype)
    # a single layer through the 3-D form gives the same numbers
    o1, l1 = sd.attn_gather(t["q_layers"][0], t["K"], t["V"], torch.from_numpy(idx).to(dev))
    assert_attn_close(o1, l1, o_ref[0], l_ref[0], w.dtype)


def test_attn_gather_counts_and_empty_sets(dev):
    w = synth.custom(B=2, N=2000, Hq=8, Hkv=2, d=128, L=2, k=512, dtype="bf16", seed=3)
    x = synth.generate(w)
    t = _to(dev, x)
    r = np.random.default_rng(0)
    idx = np.stack([np.stack([np.sort(r.choice(2000, 512, replace=False))
                              for _ in range(2)]) for _ in range(2)]).astype(np.int32)
    count = np.array([[0, 5], [512, 300]], np.int32)
    out, lse = sd.attn_gather(t["q_layers"], t["K"], t["V"], torch.from_numpy(idx).to(dev),
                              count=torch.from_numpy(count).to(dev))
    o_ref, l_ref = oracle.attn(_f(x["q_layers"]), _f(x["K"]), _f(x["V"]), idx, count)
    assert_attn_close(out, lse, o_ref, l_ref, "bf16")
    assert torch.all(out[:, 0, :4] == 0)
    assert torch.all(torch.isneginf(lse[:, 0, :4]))


def test_attn_gather_bad_index_flags_without_fault(dev):
    w = synth.custom(B=1, N=100, Hq=4, Hkv=1, d=64, L=1, k=8, dtype="bf16", seed=1)
    x = synth.generate(w)
    t = _to(dev, x)
    idx = torch.tensor([[[0, 1, 2, 3, 4, 5, 6, 100]]], dtype=torch.int32, device=dev)
    ws = sd.Workspace(dev)
    sd.attn_gather(t["q_layers"], t["K"], t["V"], idx, ws=ws, check=False)
    assert sd.read_device_status(ws, raise_on_error=False) == 8   # SPARSE_ERR_INDEX


# ---------------------------------------------------------------------------
# Routing end to end and the fused step
# ---------------------------------------------------------------------------

@pytest.fixture(params=["select_kernel", "fused_step"])
def route_path(request):
    """Top-k routing ends in the select kernel (sparse_route_topk) or, in a
    decode step, inside the attention kernel; every routing test runs both
    ways and reads the index set either call returns."""
    return request.param


def _route(path, t, K, k, ws=None, L=1):
    """The top-k set of routing with t["q_route"] over K, by `path` (the
    device status is left for the caller to read)."""
    if path == "select_kernel":
        return sd.route_topk(t["q_route"], K, k, ws=ws, check=False)
    res = sd.decode_step(t["q_route"], t["q_layers"][:L], K, torch.zeros_like(K), k=k, ws=ws,
                         check=False)
    return res["idx"]


ROUTE_CASES = [
    dict(B=1, N=4096, Hq=8, Hkv=2, d=64, k=256, dtype="f32"),
    dict(B=2, N=10007, Hq=32, Hkv=8, d=128, k=333, dtype="bf16", heavy=16),
    dict(B=1, N=1, Hq=4, Hkv=1, d=128, k=1, dtype="bf16"),
    dict(B=1, N=6000, Hq=16, Hkv=1, d=64, k=6000, dtype="bf16"),
]


@pytest.mark.parametrize("c", ROUTE_CASES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
def test_route_topk_matches_oracle(dev, c, route_path):
    w = synth.custom(L=1, seed=c["N"], **c)
    x = synth.generate(w)
    t = _to(dev, x)
    gidx = _route(route_path, t, t["K"], w.k).cpu().numpy()
    S = oracle.scores(_f(x["q_route"]), _f(x["K"]))
    assert_topk_within_band(gidx, S, w.k)
    again = _route(route_path, t, t["K"], w.k).cpu().numpy()
    np.testing.assert_array_equal(gidx, again)   # deterministic


def test_nonfinite_key_is_flagged(dev):
    w = synth.custom(B=1, N=1000, Hq=8, Hkv=2, d=64, L=1, k=10, dtype="bf16", seed=2)
    x = synth.generate(w)
    t = _to(dev, x)
    t["K"][0, 1, 17, 3] = float("nan")
    ws = sd.Workspace(dev)
    sd.route_topk(t["q_route"], t["K"], 10, ws=ws, check=False)
    assert sd.read_device_status(ws, raise_on_error=False) == 5   # NONFINITE


def _check_decode(dev, w, x, batches_checked=None):
    t = _to(dev, x)
    res = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], k=w.k)
    gidx = res["idx"].cpu().numpy()
    bsel = list(range(w.B)) if batches_checked is None else list(batches_checked)
    q = _f(x["q_route"][bsel])
    K = _f(x["K"][bsel])
    S = oracle.scores(q, K)
    assert_topk_within_band(gidx[bsel], S, w.k)
    # shared routing: the fused step's set is the routing call's set, bitwise
    np.testing.assert_array_equal(gidx, sd.route_topk(t["q_route"], t["K"], w.k).cpu().numpy())
    # every layer's output equals the gather call on that set (both split the
    # set into the same equal shares), and matches the oracle on the oracle's
    # own set
    out2, lse2 = sd.attn_gather(t["q_layers"], t["K"], t["V"], res["idx"])
    assert torch.equal(out2, res["out"]) and torch.equal(lse2, res["lse"])
    ridx = oracle.topk(S, w.k)
    o_gpu, l_gpu = sd.attn_gather(t["q_layers"][:, bsel].contiguous(), t["K"][bsel].contiguous(),
                                  t["V"][bsel].contiguous(), torch.from_numpy(ridx).to(dev))
    o_ref, l_ref = oracle.attn(_f(x["q_layers"][:, bsel]), K, _f(x["V"][bsel]), ridx)
    assert_attn_close(o_gpu, l_gpu, o_ref, l_ref, w.dtype)
    return res


@pytest.mark.parametrize("name", ["tiny_f32", "decode_32k", "decode_128k"])
def test_decode_step_named_workloads(dev, name):
    w = synth.WORKLOADS[name]
    x = synth.generate(w)
    _check_decode(dev, w, x)


def test_decode_step_batched_16x64k(dev):
    """The batched workload, every one of its 16 sequences checked: index
    sets within the band of the oracle's, the step's set equal to the routing
    call's, and attention on the oracle's sets within tolerance."""
    w = synth.WORKLOADS["batched_16x64k"]
    x = synth.generate(w)
    _check_decode(dev, w, x)


@pytest.mark.parametrize("name,cap", [("threshold_128k", 8192), ("threshold_128k", 2000)])
def test_decode_step_threshold(dev, name, cap):
    w = synth.WORKLOADS[name]
    x = synth.generate(w)
    t = _to(dev, x)
    q, K = _f(x["q_route"]), _f(x["K"])
    S = oracle.scores(q, K)
    S64 = oracle.scores(q, K, np.float64)
    tau = oracle.percentile_tau(S, *w.tau_pct)
    ws = sd.Workspace(dev)
    res = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"],
                         tau=torch.from_numpy(tau).to(dev), cap=cap, ws=ws, check=False)
    st = sd.read_device_status(ws, raise_on_error=False)
    gidx, gcnt = res["idx"].cpu().numpy(), res["count"].cpu().numpy()
    ridx, rcnt = oracle.threshold(S, tau, cap)
    assert st == (4 if (rcnt > cap).any() else 0)
    for h in range(w.Hkv):
        band = _band(tau[0, h])
        g = set(gidx[0, h, :min(gcnt[0, h], cap)].tolist())
        if gcnt[0, h] <= cap:
            must = set(np.nonzero(S64[0, h] >= tau[0, h] + band)[0].tolist())
            never = set(np.nonzero(S64[0, h] < tau[0, h] - band)[0].tolist())
            assert must <= g and not (g & never), "false negative or positive"
        assert abs(int(gcnt[0, h]) - int(rcnt[0, h])) <= \
            int(np.sum(np.abs(S[0, h] - tau[0, h]) <= band))
    # attention with the oracle's set and counts
    o_gpu, l_gpu = sd.attn_gather(t["q_layers"], t["K"], t["V"], torch.from_numpy(ridx).to(dev),
                                  count=torch.from_numpy(np.minimum(rcnt, cap)).to(dev))
    o_ref, l_ref = oracle.attn(_f(x["q_layers"]), K, _f(x["V"]), ridx, np.minimum(rcnt, cap))
    assert_attn_close(o_gpu, l_gpu, o_ref, l_ref, w.dtype)


def test_decode_step_threshold_empty_set(dev):
    w = synth.custom(B=1, N=3000, Hq=8, Hkv=2, d=128, L=2, dtype="bf16", seed=9,
                     mode="threshold", cap=64)
    x = synth.generate(w)
    t = _to(dev, x)
    tau = torch.full((1, 2), 1e9, device=dev)
    res = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], tau=tau, cap=64)
    assert res["count"].cpu().tolist() == [[0, 0]]
    assert torch.all(res["out"] == 0) and torch.all(torch.isneginf(res["lse"]))


def test_route_topk_all_equal_keys_takes_lowest_indices(dev, route_path):
    """Every score equal: the boundary bin holds all N keys, more than the
    select lists on chip, so the select takes its streaming path."""
    w = synth.custom(B=1, N=20000, Hq=8, Hkv=2, d=128, L=1, k=300, dtype="bf16", seed=4)
    x = synth.generate(w)
    t = _to(dev, x)
    K = t["K"].clone()
    K[:] = K[:, :, :1, :]
    idx = _route(route_path, t, K, 300).cpu().numpy()
    np.testing.assert_array_equal(idx, np.tile(np.arange(300), (1, 2, 1)))


def test_route_topk_recovers_from_dirty_workspace(dev, route_path):
    """A workspace whose histogram area holds garbage (not zero-filled) is
    detected (the counts do not sum to N) and the result is still exact; the
    call leaves the area clean for the next one."""
    w = synth.custom(B=2, N=5000, Hq=8, Hkv=2, d=128, L=1, k=100, dtype="bf16", seed=6)
    x = synth.generate(w)
    t = _to(dev, x)
    S = oracle.scores(_f(x["q_route"]), _f(x["K"]))
    ws = sd.Workspace(dev)
    ws.get(sd.workspace_bytes(2, 5000, 8, 2, 128, torch.bfloat16, 100, 1))
    # header 4 KB | histogram [256][2048] | scores
    hist = 4096
    areas = [(hist, hist + 4 * 2048 * 4)]
    for a, b in areas:
        ws.buf[a:b] = 7
    for _ in range(2):
        gidx = _route(route_path, t, t["K"], 100, ws=ws).cpu().numpy()
        assert_topk_within_band(gidx, S, 100)
    for a, b in areas:
        assert int(ws.buf[a:b].sum()) == 0


def test_scan_claim_counters_left_zero(dev):
    """The routing scan claims its tiles through counters in the workspace
    header ([1024, 3072)); every scan, top-k or threshold marking, long or
    short, leaves them zero for the next call, and the next call still sees
    every tile (its scores equal a fresh workspace's)."""
    ws = sd.Workspace(dev)
    for N, B, Hkv in ((131072, 1, 8), (5000, 2, 2), (300, 3, 8), (70000, 1, 1)):
        w = synth.custom(B=B, N=N, Hq=4 * Hkv, Hkv=Hkv, d=128, L=1, k=min(100, N), dtype="bf16",
                         seed=N)
        x = synth.generate(w)
        t = _to(dev, x)
        idx = sd.route_topk(t["q_route"], t["K"], w.k, ws=ws)
        torch.cuda.synchronize()
        assert int(ws.buf[1024:3072].view(torch.int32).abs().sum()) == 0, N
        tau = torch.zeros((B, Hkv), device=dev)
        sd.route_threshold(t["q_route"], t["K"], tau, N, ws=ws)
        torch.cuda.synchronize()
        assert int(ws.buf[1024:3072].view(torch.int32).abs().sum()) == 0, N
        again = sd.route_topk(t["q_route"], t["K"], w.k, ws=ws)
        fresh = sd.route_topk(t["q_route"], t["K"], w.k, ws=sd.Workspace(dev))
        assert torch.equal(again, idx) and torch.equal(again, fresh)


@pytest.mark.parametrize("k,count", [(4096, None), (8192, [3933, 4100, 100, 0, 8192, 2, 3000, 7000])])
def test_attn_gather_many_keys_per_cta(dev, k, count):
    """More selected keys than one on-chip chunk per CTA: the running max is
    carried across chunks and the tensor-memory accumulator is rescaled."""
    w = synth.custom(B=1, N=30000, Hq=32, Hkv=8, d=128, L=16, k=k, dtype="bf16", seed=k)
    x = synth.generate(w)
    t = _to(dev, x)
    S = oracle.scores(_f(x["q_route"]), _f(x["K"]))
    idx = oracle.topk(S, k)
    c = None if count is None else np.array([count], np.int32)
    out, lse = sd.attn_gather(t["q_layers"], t["K"], t["V"], torch.from_numpy(idx).to(dev),
                              count=None if c is None else torch.from_numpy(c).to(dev))
    o_ref, l_ref = oracle.attn(_f(x["q_layers"]), _f(x["K"]), _f(x["V"]), idx, c)
    assert_attn_close(out, lse, o_ref, l_ref, "bf16")


@pytest.mark.parametrize("dtype,N", [("bf16", 20011), ("f32", 3001)])
def test_dense_attention_all_keys(dev, dtype, N):
    """k = N: the gather attention over every cached key is dense attention
    (the comparison the per-layer routing measurement uses), against the
    oracle on all keys."""
    w = synth.custom(B=1, N=N, Hq=8, Hkv=2, d=128, L=4, k=N, dtype=dtype, seed=29)
    x = synth.generate(w)
    t = _to(dev, x)
    idx = np.tile(np.arange(N, dtype=np.int32), (1, w.Hkv, 1))
    out, lse = sd.attn_gather(t["q_layers"], t["K"], t["V"], torch.from_numpy(idx).to(dev))
    o_ref, l_ref = oracle.attn(_f(x["q_layers"]), _f(x["K"]), _f(x["V"]), idx)
    assert_attn_close(out, lse, o_ref, l_ref, dtype)


@pytest.mark.parametrize("kind", ["random", "duplicated_rows", "few_values", "heavy"])
def test_route_topk_bit_exact_on_its_own_scores(dev, kind, route_path):
    """Routing (scan + exact select) against the oracle's top-k of the very
    scores the scan produced: identical fp32 scores, so the index sets must
    be identical, ties included."""
    w = synth.custom(B=2, N=40000, Hq=32, Hkv=8, d=128, L=1, k=2048, dtype="bf16",
                     heavy=64 if kind == "heavy" else 0, seed=17)
    x = synth.generate(w)
    t = _to(dev, x)
    K = t["K"]
    if kind == "duplicated_rows":       # groups of 3 identical rows: exact score ties
        K = K.clone()
        K[:, :, 1::3] = K[:, :, 0:-1:3][:, :, :K[:, :, 1::3].shape[2]]
        K[:, :, 2::3] = K[:, :, 0:-2:3][:, :, :K[:, :, 2::3].shape[2]]
    elif kind == "few_values":          # small integers: many exact ties
        K = torch.randint(-2, 3, K.shape, device=dev).to(K.dtype)
    ws = sd.Workspace(dev)
    S = sd.score(t["q_route"], K, ws=ws).cpu().numpy()
    idx = _route(route_path, t, K, w.k, ws=ws).cpu().numpy()
    np.testing.assert_array_equal(idx, oracle.topk(S, w.k))


@pytest.mark.parametrize("B,N,Hkv,k", [(1, 131072, 8, 2048), (3, 20000, 2, 1), (4, 8192, 4, 8000),
                                       (1, 65536, 1, 700), (2, 2048, 8, 64),
                                       (16, 65536, 8, 2048), (1, 262144, 2, 2048)])
def test_fused_select_equals_select_kernel(dev, B, N, Hkv, k):
    """The select inside the attention kernel (decode step) and the select
    kernel (routing call) give the same index sets, bit for bit, over shapes
    where scan CTAs span two heads, a head spans one CTA or many, k = 1, k
    close to N, the batched decode shape, and a cache too long for the fused
    select (the step then runs the select kernel itself)."""
    w = synth.custom(B=B, N=N, Hq=4 * Hkv, Hkv=Hkv, d=128, L=1, k=k, dtype="bf16", seed=N + k)
    x = synth.generate(w)
    t = _to(dev, x)
    ws = sd.Workspace(dev)
    a = _route("fused_step", t, t["K"], k, ws=ws).cpu().numpy()
    assert sd.read_device_flags(ws) & ~sd.FLAG_SLOW_SELECT == 0
    b = _route("select_kernel", t, t["K"], k, ws=ws).cpu().numpy()
    np.testing.assert_array_equal(a, b)
    S = oracle.scores(_f(x["q_route"]), _f(x["K"]))
    assert_topk_within_band(a, S, k)


def _plant(K, rows, v):
    """K [B,Hkv,N,d] with the given rows of every head set to the vector v."""
    K = K.clone()
    K[:, :, rows] = v.to(K.dtype)
    return K


def _qbar_dir(t, Hkv):
    """Unit vector along head 0's summed routing query (its keys' score
    direction)."""
    q = t["q_route"][0].float()
    qbar = q.reshape(Hkv, q.shape[0] // Hkv, -1).sum(1)[0]
    return qbar / qbar.norm()


@pytest.mark.parametrize("route", ["select_kernel", "fused_step"])
def test_select_ties_split_across_ctas(dev, route):
    """40 keys with one identical top score, spread over the runs of the
    head's CTAs, and k = 19: the k-th value is shared, so the set is the 19
    lowest-index keys of the 40 -- a run holding the 18th..20th takes only
    part of its tied keys.  The split select does this on its fast path."""
    B, N, Hkv, k = 1, 131072, 2, 19
    w = synth.custom(B=B, N=N, Hq=4 * Hkv, Hkv=Hkv, d=128, L=1, k=k, dtype="bf16", seed=77)
    x = synth.generate(w)
    t = _to(dev, x)
    rows = torch.arange(40) * 3000 + 7
    K = _plant(t["K"], rows, 8 * _qbar_dir(t, Hkv))
    ws = sd.Workspace(dev)
    S = sd.score(t["q_route"], K, ws=ws).cpu().numpy()
    a = _route(route, t, K, k, ws=ws).cpu().numpy()
    assert sd.read_device_flags(ws) == 0
    ref = oracle.topk(S, k)
    np.testing.assert_array_equal(a, ref)
    np.testing.assert_array_equal(ref[0, 0], rows[:k].numpy())


@pytest.mark.parametrize("route", ["select_kernel", "fused_step"])
def test_select_boundary_bin_over_capacity(dev, route):
    """4096 identical keys in one CTA's run score above every other key and
    k = 2048 of them are taken: the boundary bin overflows that CTA's list,
    so every CTA takes the exact streaming path (FLAG_SLOW_SELECT, not an
    error), which returns the 2048 lowest indices; the next call on the same
    workspace is back on the fast path."""
    B, N, Hkv, k = 1, 131072, 2, 2048
    w = synth.custom(B=B, N=N, Hq=4 * Hkv, Hkv=Hkv, d=128, L=1, k=k, dtype="bf16", seed=78)
    x = synth.generate(w)
    t = _to(dev, x)
    rows = torch.arange(4096) + 100
    K = _plant(t["K"], rows, 8 * _qbar_dir(t, Hkv))
    ws = sd.Workspace(dev)
    S = sd.score(t["q_route"], K, ws=ws).cpu().numpy()
    a = _route(route, t, K, k, ws=ws).cpu().numpy()
    assert sd.read_device_flags(ws) == sd.FLAG_SLOW_SELECT
    np.testing.assert_array_equal(a, oracle.topk(S, k))
    b = _route(route, t, t["K"], k, ws=ws).cpu().numpy()
    assert sd.read_device_flags(ws) == 0
    assert_topk_within_band(b, oracle.scores(_f(x["q_route"]), _f(x["K"])), k)


@pytest.mark.parametrize("route", ["select_kernel", "fused_step"])
def test_select_whole_set_in_one_run(dev, route):
    """Every key of head 0's top k lies in one CTA's run (a block of keys
    shifted along the head's query direction): the select kernel keeps its
    fast path with one CTA writing the whole set; the attention kernel,
    which holds at most 2048 keys per CTA on chip, takes the streaming path
    with equal shares once the run holds more.  Both return the exact set."""
    B, N, Hkv = 1, 131072, 2
    for k, slow in ((1500, False), (3000, True)):
        w = synth.custom(B=B, N=N, Hq=4 * Hkv, Hkv=Hkv, d=128, L=1, k=k, dtype="bf16",
                         seed=79)
        x = synth.generate(w)
        t = _to(dev, x)
        K = t["K"].clone()
        K[:, :, 300:300 + 4000] += (10 * _qbar_dir(t, Hkv)).to(K.dtype)
        ws = sd.Workspace(dev)
        S = sd.score(t["q_route"], K, ws=ws).cpu().numpy()
        a = _route(route, t, K, k, ws=ws).cpu().numpy()
        want = sd.FLAG_SLOW_SELECT if (slow and route == "fused_step") else 0
        assert sd.read_device_flags(ws) == want, (k, route)
        np.testing.assert_array_equal(a, oracle.topk(S, k))


@pytest.mark.parametrize("route", ["select_kernel", "fused_step"])
def test_select_fast_path_on_the_decode_workloads(dev, route):
    """On the decode workloads' distributions no head falls back to the
    streaming select."""
    for name in ("decode_32k", "decode_128k", "batched_16x64k"):
        w = synth.WORKLOADS[name]
        x = synth.generate(w)
        t = _to(dev, x)
        ws = sd.Workspace(dev)
        _route(route, t, t["K"], w.k, ws=ws, L=w.L)
        assert sd.read_device_flags(ws) == 0, name


# ---------------------------------------------------------------------------
# Routing recomputed every R layers (per-layer routing at R = 1, partial
# sharing in between, shared routing at R >= L)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L,R", [(7, 3), (16, 1), (16, 4), (4, 9)])
def test_decode_step_grouped_topk(dev, L, R):
    """Every group's set matches the oracle's top-k of that group's routing
    scores (within the rounding band) and equals the routing call on that
    query bitwise; every layer's output equals the gather call on its group's
    set and matches the oracle on the oracle's sets."""
    w = synth.custom(B=1, N=6000, Hq=16, Hkv=4, d=128, L=L, k=300, dtype="bf16", seed=10 * L + R)
    x = synth.generate(w)
    t = _to(dev, x)
    ng = -(-L // R)
    g = torch.Generator().manual_seed(R)
    qrs = torch.randn((ng, w.B, w.Hq, w.d), generator=g).to(torch.bfloat16)
    qrs_d = qrs.to(dev)
    res = sd.decode_step_grouped(qrs_d, t["q_layers"], t["K"], t["V"], R, k=w.k)
    ref = oracle.decode_step_grouped(_f(qrs), _f(x["q_layers"]), _f(x["K"]), _f(x["V"]), R,
                                     k=w.k)
    gidx = res["idx"].cpu().numpy()
    for grp in range(ng):
        layers = list(range(grp * R, min(L, (grp + 1) * R)))
        assert_topk_within_band(gidx[grp], ref["S"][grp], w.k)
        np.testing.assert_array_equal(
            gidx[grp], sd.route_topk(qrs_d[grp], t["K"], w.k).cpu().numpy())
        out2, lse2 = sd.attn_gather(t["q_layers"][layers].contiguous(), t["K"], t["V"],
                                    res["idx"][grp].contiguous())
        assert torch.equal(out2, res["out"][layers]) and torch.equal(lse2, res["lse"][layers])
    o_gpu = torch.empty_like(res["out"])
    l_gpu = torch.empty_like(res["lse"])
    for grp in range(ng):
        layers = list(range(grp * R, min(L, (grp + 1) * R)))
        o, l = sd.attn_gather(t["q_layers"][layers].contiguous(), t["K"], t["V"],
                              torch.from_numpy(ref["idx"][grp]).to(dev))
        o_gpu[layers], l_gpu[layers] = o, l
    assert_attn_close(o_gpu, l_gpu, ref["out"], ref["lse"], "bf16")


def test_decode_step_grouped_threshold(dev):
    """Threshold mode: each group keeps every key at or above its own tau
    (no false negatives against fp64 scores) and each layer attends over its
    group's set."""
    L, R = 5, 2
    w = synth.custom(B=1, N=8000, Hq=8, Hkv=2, d=128, L=L, k=1, dtype="bf16", seed=5)
    x = synth.generate(w)
    t = _to(dev, x)
    ng = -(-L // R)
    g = torch.Generator().manual_seed(99)
    qrs = torch.randn((ng, w.B, w.Hq, w.d), generator=g).to(torch.bfloat16)
    S = np.stack([oracle.scores(_f(qrs[i]), _f(x["K"])) for i in range(ng)])
    S64 = np.stack([oracle.scores(_f(qrs[i]), _f(x["K"]), np.float64) for i in range(ng)])
    tau = np.stack([oracle.percentile_tau(S[i], 97, 100) for i in range(ng)])
    cap = 512
    res = sd.decode_step_grouped(qrs.to(dev), t["q_layers"], t["K"], t["V"], R,
                                 tau=torch.from_numpy(tau).to(dev), cap=cap)
    gidx, gcnt = res["idx"].cpu().numpy(), res["count"].cpu().numpy()
    for grp in range(ng):
        for h in range(w.Hkv):
            band = _band(tau[grp, 0, h])
            got = set(gidx[grp, 0, h, :gcnt[grp, 0, h]].tolist())
            must = set(np.nonzero(S64[grp, 0, h] >= tau[grp, 0, h] + band)[0].tolist())
            never = set(np.nonzero(S64[grp, 0, h] < tau[grp, 0, h] - band)[0].tolist())
            assert must <= got and not (got & never)
        layers = list(range(grp * R, min(L, (grp + 1) * R)))
        out2, lse2 = sd.attn_gather(t["q_layers"][layers].contiguous(), t["K"], t["V"],
                                    res["idx"][grp].contiguous(),
                                    count=res["count"][grp].contiguous())
        assert torch.equal(out2, res["out"][layers]) and torch.equal(lse2, res["lse"][layers])


# ---------------------------------------------------------------------------
# Decode steps as a model runs them: append the new token's K/V row, then route
# and attend over a cache whose allocation is longer than its length
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_kv_append_then_decode(dev, dtype, d):
    """Three steps on a cache allocated for n_cap rows: each appends a row at
    the current length and decodes over exactly the first n rows.  Rows past n
    hold huge values that would dominate any score if read.  Results equal a
    dense copy of the first n rows bitwise, and the oracle on that cache."""
    B, n_cap, n0, Hq, Hkv, L, k = 1, 3000, 2500, 8, 2, 2, 100
    w = synth.custom(B=B, N=n_cap, Hq=Hq, Hkv=Hkv, d=d, L=L, k=k, dtype=dtype, seed=d)
    x = synth.generate(w)
    t = _to(dev, x)
    K, V = t["K"].clone(), t["V"].clone()
    K[:, :, n0:] = 100
    V[:, :, n0:] = 100
    g = torch.Generator().manual_seed(7)
    for step in range(3):
        n = n0 + 1 + step
        k_new = torch.randn((B, Hkv, d), generator=g).to(K.dtype).to(dev)
        v_new = torch.randn((B, Hkv, d), generator=g).to(K.dtype).to(dev)
        sd.kv_append(K, V, k_new, v_new, n)
        assert torch.equal(K[:, :, n - 1], k_new) and torch.equal(V[:, :, n - 1], v_new)
        assert torch.all(K[:, :, n:] == 100)
        res = sd.decode_step(t["q_route"], t["q_layers"], K, V, k=k, n=n)
        Kd, Vd = K[:, :, :n].contiguous(), V[:, :, :n].contiguous()
        dense = sd.decode_step(t["q_route"], t["q_layers"], Kd, Vd, k=k)
        np.testing.assert_array_equal(res["idx"].cpu().numpy(), dense["idx"].cpu().numpy())
        assert torch.equal(res["out"], dense["out"]) and torch.equal(res["lse"], dense["lse"])
        Kh, Vh = _f(Kd.cpu()), _f(Vd.cpu())
        S = oracle.scores(_f(x["q_route"]), Kh)
        assert_topk_within_band(res["idx"].cpu().numpy(), S, k)
        ridx = oracle.topk(S, k)
        o_gpu, l_gpu = sd.attn_gather(t["q_layers"], K, V, torch.from_numpy(ridx).to(dev), n=n)
        o_ref, l_ref = oracle.attn(_f(x["q_layers"]), Kh, Vh, ridx)
        assert_attn_close(o_gpu, l_gpu, o_ref, l_ref, dtype)


@pytest.mark.parametrize("mode,dtype", [("topk", "bf16"), ("threshold", "bf16"),
                                        ("topk", "f32")])
def test_decode_step_graph_equals_eager_step(dev, mode, dtype):
    """The captured step with its host transfers returns, for each new
    query written into its pinned input views, exactly what the eager step
    returns: on the fused kernels with every result written straight into
    the mapped host buffer (bf16), and on separate routing and attention
    kernels (fp32)."""
    w = synth.custom(B=2, N=5000, Hq=8, Hkv=2, d=128, L=3, k=100, dtype=dtype, seed=17,
                     heavy=8, mode=mode, cap=5000)
    x = synth.generate(w)
    K, V = x["K"].to(dev), x["V"].to(dev)
    variants = synth.query_variants(w, x, 3, seed=90)
    kw = dict(k=w.k) if mode == "topk" else dict(
        tau=torch.from_numpy(oracle.percentile_tau(oracle.scores(_f(x["q_route"]), _f(x["K"])),
                                                   90, 100)).to(dev), cap=w.cap)
    g = sd.DecodeStepGraph(K, V, w.L, w.Hq, ws=sd.Workspace(dev), **kw)
    assert g.mapped_out       # torch's pinned buffers are mapped under unified addressing
    assert g.fused == (dtype == "bf16") and g.results_direct == g.fused
    assert g.h2d_bytes >= (w.B * w.Hq * w.d + w.L * w.B * w.Hq * w.d) * 2
    for qr, ql in variants:
        g.q_route_host.copy_(qr)
        g.q_layers_host.copy_(ql)
        res = g()
        ref = sd.decode_step(qr.to(dev), ql.to(dev), K, V, **kw)
        assert torch.equal(res[0], ref["out"].cpu())
        if mode == "topk":
            assert torch.equal(res[1], ref["idx"].cpu())
        else:
            assert torch.equal(res[2], ref["count"].cpu())
            for b in range(w.B):
                for h in range(w.Hkv):
                    n = min(int(ref["count"][b, h]), w.cap)
                    assert torch.equal(res[1][b, h, :n], ref["idx"][b, h, :n].cpu())
    sd.read_device_status(g.ws)


def test_decode_step_graph_survives_workspace_growth(dev):
    """A later call that needs a larger workspace replaces the workspace's
    buffer; a graph captured before keeps the buffer it captured and still
    returns the eager step's results."""
    w = synth.custom(B=1, N=4000, Hq=8, Hkv=2, d=128, L=2, k=64, dtype="bf16", seed=41)
    x = synth.generate(w)
    K, V = x["K"].to(dev), x["V"].to(dev)
    ws = sd.Workspace(dev)
    g = sd.DecodeStepGraph(K, V, w.L, w.Hq, k=w.k, ws=ws)
    before = ws.buf.data_ptr()
    long_k = torch.zeros((1, w.Hkv, 400_000, w.d), dtype=torch.bfloat16, device=dev)
    sd.score(x["q_route"].to(dev), long_k, ws=ws)   # a longer cache: grows ws
    assert ws.buf.data_ptr() != before
    g.q_route_host.copy_(x["q_route"])
    g.q_layers_host.copy_(x["q_layers"])
    out, idx = g()
    ref = sd.decode_step(x["q_route"].to(dev), x["q_layers"].to(dev), K, V, k=w.k)
    assert torch.equal(out, ref["out"].cpu())
    assert torch.equal(idx, ref["idx"].cpu())


def test_outputs_written_straight_to_pinned_host_memory(dev):
    """attn_gather and decode_step given a pinned host out write there the
    same bytes they write to device memory."""
    w = synth.custom(B=1, N=3000, Hq=8, Hkv=2, d=128, L=2, k=64, dtype="bf16", seed=23)
    x = synth.generate(w)
    t = {n: x[n].to(dev) for n in ("q_route", "q_layers", "K", "V")}
    ref = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], k=w.k)
    host = torch.full(tuple(t["q_layers"].shape), float("nan"),
                      dtype=torch.bfloat16).pin_memory()
    assert sd.device_usable(host)
    res = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], k=w.k, out=host)
    torch.cuda.synchronize()
    assert res["out"].data_ptr() == host.data_ptr()
    assert torch.equal(host, ref["out"].cpu())
    host.fill_(float("nan"))
    sd.attn_gather(t["q_layers"], t["K"], t["V"], ref["idx"], out=host)
    torch.cuda.synchronize()
    assert torch.equal(host, ref["out"].cpu())


def test_bounded_wait_expires_and_context_stays_usable(dev):
    """Failure detection without a fault: the library's bounded wait, on a
    counter nothing increments, gives up after its limit, reports
    SPARSE_ERR_TIMEOUT through the status word, and the next calls on the
    same workspace and stream run normally."""
    import time
    ws = sd.Workspace(dev)
    t0 = time.perf_counter()
    assert sd.selftest_bounded_wait(ws, limit_ns=100_000_000) == 7   # TIMEOUT
    assert time.perf_counter() - t0 >= 0.09
    assert sd.read_device_status(ws, raise_on_error=False) == 0       # status was reset
    w = synth.custom(B=1, N=4096, Hq=8, Hkv=2, d=128, L=2, k=64, dtype="bf16", seed=3)
    x = synth.generate(w)
    t = _to(dev, x)
    res = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], k=w.k, ws=ws)
    ref = oracle.decode_step(_f(x["q_route"]), _f(x["q_layers"]), _f(x["K"]), _f(x["V"]), k=w.k)
    assert_topk_within_band(res["idx"].cpu().numpy(), ref["S"], w.k)


CANARY = -123456789


def _fenced(shape, dtype, dev, pad=4096):
    """A contiguous tensor of `shape` at the front of a larger buffer whose
    tail holds a canary pattern."""
    n = int(np.prod(shape))
    if dtype in (torch.int32,):
        buf = torch.full((n + pad,), CANARY, dtype=dtype, device=dev)
    else:
        buf = torch.full((n + pad,), -7.25, dtype=dtype, device=dev)
    return buf, buf[:n].view(*shape)


def _tail_intact(buf, n):
    tail = buf[n:]
    want = CANARY if buf.dtype == torch.int32 else -7.25
    return bool((tail == want).all())


def test_no_call_writes_past_its_outputs(dev):
    """Canary words after every output buffer (scores, index sets, counts,
    attention outputs and lse, the Louver set) stay untouched, including a
    threshold set that overflows its capacity."""
    w = synth.custom(B=2, N=8192, Hq=8, Hkv=2, d=128, L=3, k=100, dtype="bf16", seed=41,
                     heavy=4, blobs=0)
    x = synth.generate(w)
    t = _to(dev, x)
    B, Hkv, N, L, Hq, d, k = w.B, w.Hkv, w.N, w.L, w.Hq, w.d, w.k
    ws = sd.Workspace(dev)
    bS, S = _fenced((B, Hkv, N), torch.float32, dev)
    sd.score(t["q_route"], t["K"], ws=ws, out=S)
    assert _tail_intact(bS, S.numel())
    bi, idx = _fenced((B, Hkv, k), torch.int32, dev)
    sd.route_topk(t["q_route"], t["K"], k, ws=ws, idx=idx)
    assert _tail_intact(bi, idx.numel())
    bi2, idx2 = _fenced((B, Hkv, k), torch.int32, dev)
    sd.select_topk(S, k, ws=ws, idx=idx2)
    assert _tail_intact(bi2, idx2.numel())
    cap = 64   # far below the set size: capacity overflow
    tau = torch.zeros((B, Hkv), device=dev)
    for fn in (lambda i, c: sd.route_threshold(t["q_route"], t["K"], tau, cap, ws=ws,
                                               check=False, idx=i, count=c),
               lambda i, c: sd.select_threshold(S, tau, cap, ws=ws, check=False, idx=i,
                                                count=c)):
        bti, ti = _fenced((B, Hkv, cap), torch.int32, dev)
        btc, tc = _fenced((B, Hkv), torch.int32, dev)
        fn(ti, tc)
        assert sd.read_device_status(ws, raise_on_error=False) == 4
        assert _tail_intact(bti, ti.numel()) and _tail_intact(btc, tc.numel())
        assert int(tc.min()) > cap
    bo, out = _fenced((L, B, Hq, d), torch.bfloat16, dev)
    bl, lse = _fenced((L, B, Hq), torch.float32, dev)
    sd.attn_gather(t["q_layers"], t["K"], t["V"], idx, ws=ws, out=out, lse=lse)
    assert _tail_intact(bo, out.numel()) and _tail_intact(bl, lse.numel())
    bo2, out2 = _fenced((L, B, Hq, d), torch.bfloat16, dev)
    bl2, lse2 = _fenced((L, B, Hq), torch.float32, dev)
    bi3, idx3 = _fenced((B, Hkv, k), torch.int32, dev)
    sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], k=k, ws=ws, out=out2,
                   lse=lse2, idx=idx3)
    assert _tail_intact(bo2, out2.numel()) and _tail_intact(bl2, lse2.numel())
    assert _tail_intact(bi3, idx3.numel())
    ix = sd.louver_build(t["K"], 128)
    bli, li = _fenced((B, Hkv, cap), torch.int32, dev)
    blc, lc = _fenced((B, Hkv), torch.int32, dev)
    sd.louver_route_threshold(t["q_route"], t["K"], ix, tau, cap, check=False, idx=li, count=lc)
    assert sd.read_device_status(ix.ws, raise_on_error=False) == 4
    assert _tail_intact(bli, li.numel()) and _tail_intact(blc, lc.numel())


@pytest.mark.parametrize("B,N,Hkv,d,dtype,pct,cap", [(2, 5003, 2, 128, "bf16", 90, 600),
                                                     (1, 131072, 8, 128, "bf16", 97, 8192),
                                                     (3, 777, 4, 64, "f32", 50, 200),
                                                     (1, 4096, 2, 64, "bf16", 99, 5)])
def test_route_threshold_equals_select_on_its_scores(dev, B, N, Hkv, d, dtype, pct, cap):
    """The marking scan + bitmap compaction gives exactly the threshold select
    of the scan's own scores (same fp32 scores, same comparison): counts and
    index rows bitwise, capacity overflow included; and the oracle's set
    within the band."""
    w = synth.custom(B=B, N=N, Hq=4 * Hkv, Hkv=Hkv, d=d, L=1, dtype=dtype, seed=N + pct,
                     mode="threshold", cap=cap)
    x = synth.generate(w)
    t = _to(dev, x, ("q_route", "K"))
    q32, K32 = _f(x["q_route"]), _f(x["K"])
    S = oracle.scores(q32, K32)
    tau = oracle.percentile_tau(S, pct, 100)
    taud = torch.from_numpy(tau).to(dev)
    ws = sd.Workspace(dev)
    gi, gc = sd.route_threshold(t["q_route"], t["K"], taud, cap, ws=ws, check=False)
    st1 = sd.read_device_status(ws, raise_on_error=False)
    Sg = sd.score(t["q_route"], t["K"], ws=ws)
    si, sc = sd.select_threshold(Sg, taud, cap, ws=ws, check=False)
    st2 = sd.read_device_status(ws, raise_on_error=False)
    assert st1 == st2
    np.testing.assert_array_equal(gc.cpu().numpy(), sc.cpu().numpy())
    gi, si, gcn = gi.cpu().numpy(), si.cpu().numpy(), gc.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            n = min(int(gcn[b, h]), cap)
            np.testing.assert_array_equal(gi[b, h, :n], si[b, h, :n])
    S64 = oracle.scores(q32, K32, np.float64)
    ridx, rcnt = oracle.threshold(S, tau, cap)
    for b in range(B):
        for h in range(Hkv):
            band = _band(tau[b, h])
            assert abs(int(gcn[b, h]) - int(rcnt[b, h])) <= int(np.sum(np.abs(S[b, h] - tau[b, h]) <= band))
            if gcn[b, h] <= cap:
                g = set(gi[b, h, :gcn[b, h]].tolist())
                must = set(np.nonzero(S64[b, h] >= tau[b, h] + band)[0].tolist())
                never = set(np.nonzero(S64[b, h] < tau[b, h] - band)[0].tolist())
                assert must <= g and not (g & never)



def _random_case(seed):
    r = np.random.default_rng(10_000 + seed)
    d = int(r.choice([64, 128]))
    dtype = str(r.choice(["bf16", "f32"]))
    G = int(r.choice([1, 2, 4, 8, 16]))
    Hkv = int(r.choice([1, 2, 3, 4, 8]))
    B = int(r.integers(1, 4))
    N = int(r.choice([1, 2, 31, 33, 127, 500, 1000, 4097, 12345, 30001]))
    L = int(r.integers(1, 6))
    mode = str(r.choice(["topk", "threshold"]))
    k = int(r.integers(1, N + 1))
    cap = int(r.integers(1, N + 1))
    return dict(B=B, N=N, Hq=G * Hkv, Hkv=Hkv, d=d, L=L, k=k, dtype=dtype, mode=mode, cap=cap,
                heavy=int(min(N, r.integers(0, 5))), seed=seed)


@pytest.mark.parametrize("seed", range(64))
def test_random_shapes_fused_step(dev, seed):
    """Seeded random shapes (ragged N from 1, any k or cap, G 1..16, d 64/128,
    fp32/bf16, top-k and threshold with capacity overflow) through the fused
    step: the set within the band of the oracle's, the shared-routing
    property, and attention on the oracle's set within tolerance."""
    c = _random_case(seed)
    w = synth.custom(B=c["B"], N=c["N"], Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"], L=c["L"],
                     k=c["k"], dtype=c["dtype"], heavy=c["heavy"], seed=c["seed"],
                     mode=c["mode"], cap=c["cap"])
    x = synth.generate(w)
    t = _to(dev, x)
    q32, K32, V32 = _f(x["q_route"]), _f(x["K"]), _f(x["V"])
    S = oracle.scores(q32, K32)
    ws = sd.Workspace(dev)
    if c["mode"] == "topk":
        res = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], k=c["k"], ws=ws)
        gidx = res["idx"].cpu().numpy()
        assert_topk_within_band(gidx, S, c["k"])
        np.testing.assert_array_equal(gidx, sd.route_topk(t["q_route"], t["K"], c["k"],
                                                          ws=ws).cpu().numpy())
        ridx, rcnt = oracle.topk(S, c["k"]), None
    else:
        tau = oracle.percentile_tau(S, 90, 100)
        res = sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"],
                             tau=torch.from_numpy(tau).to(dev), cap=c["cap"], ws=ws, check=False)
        st = sd.read_device_status(ws, raise_on_error=False)
        ridx, rcnt = oracle.threshold(S, tau, c["cap"])
        gcnt = res["count"].cpu().numpy()
        gidx = res["idx"].cpu().numpy()
        S64 = oracle.scores(q32, K32, np.float64)
        for b in range(c["B"]):
            for h in range(c["Hkv"]):
                band = _band(tau[b, h])
                assert abs(int(gcnt[b, h]) - int(rcnt[b, h])) <= \
                    int(np.sum(np.abs(S[b, h] - tau[b, h]) <= band))
                if gcnt[b, h] <= c["cap"]:
                    g = set(gidx[b, h, :gcnt[b, h]].tolist())
                    must = set(np.nonzero(S64[b, h] >= tau[b, h] + band)[0].tolist())
                    never = set(np.nonzero(S64[b, h] < tau[b, h] - band)[0].tolist())
                    assert must <= g and not (g & never)
        assert (st == 4) == bool((gcnt > c["cap"]).any())
        rcnt = np.minimum(rcnt, c["cap"]).astype(np.int32)
    o_gpu, l_gpu = sd.attn_gather(t["q_layers"], t["K"], t["V"], torch.from_numpy(ridx).to(dev),
                                  count=None if rcnt is None else torch.from_numpy(rcnt).to(dev),
                                  ws=ws)
    o_ref, l_ref = oracle.attn(_f(x["q_layers"]), K32, V32, ridx, rcnt)
    assert_attn_close(o_gpu, l_gpu, o_ref, l_ref, c["dtype"])
