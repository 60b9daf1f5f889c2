"""Host checks of the seeded input generator (no method arithmetic in it)."""
import numpy as np
import torch

from token_sparse_attention_sm_b200 import synth


def test_deterministic_and_subset_consistent():
    w = synth.custom(B=3, N=300, Hq=8, Hkv=2, d=64, L=2, k=8, heavy=5,
                     outlier=True, seed=4)
    a = synth.generate(w)
    b = synth.generate(w)
    for key in a:
        assert torch.equal(a[key], b[key])
    sub = synth.generate(w, batches=[2])
    for key in ("q_route", "K", "V", "outlier", "heavy_pos"):
        assert torch.equal(sub[key][0], a[key][2])
    assert torch.equal(sub["q_layers"][:, 0], a["q_layers"][:, 2])


def test_heavy_hitters_and_outlier_channel():
    w = synth.custom(B=1, N=500, Hq=8, Hkv=2, d=64, L=1, k=8, heavy=7,
                     outlier=True, seed=0)
    x = synth.generate(w)
    qf = x["q_route"].float().numpy()[0]
    for h in range(2):
        pos = x["heavy_pos"][0, h].numpy()
        assert len(set(pos.tolist())) == 7 and pos.min() >= 0 and pos.max() < 500
        qbar = qf[4 * h:4 * h + 4].mean(axis=0)
        unit = 4 * qbar / np.linalg.norm(qbar)
        rows = x["K"][0, h, pos].float().numpy()
        assert np.abs(rows - unit).max() < 0.6          # 0.1-sigma noise
        c = int(x["outlier"][0, h])
        others = np.delete(np.arange(500), pos)
        kc = x["K"][0, h, others, c].float().numpy()
        assert 6 < kc.std() < 10                          # x8 channel
        assert 0.8 < np.delete(x["K"][0, h, others].float().numpy(), c, axis=1).std() < 1.2


def test_dtypes_and_rounding():
    w = synth.custom(B=1, N=64, Hq=4, Hkv=1, d=64, L=1, k=4, dtype="bf16")
    x = synth.generate(w)
    assert x["K"].dtype == torch.bfloat16
    f = synth.f32(x["K"])
    assert f.dtype == np.float32
    assert np.array_equal(torch.from_numpy(f).to(torch.bfloat16).float().numpy(), f)
    w32 = w.with_(dtype="f32")
    assert synth.generate(w32)["K"].dtype == torch.float32


def test_named_workloads_shapes():
    w = synth.WORKLOADS["decode_128k"]
    assert (w.B, w.N, w.Hq, w.Hkv, w.d, w.L, w.k) == (1, 131072, 32, 8, 128, 16, 2048)
    assert w.outlier and w.heavy == 256
    t = synth.WORKLOADS["threshold_128k"]
    assert t.mode == "threshold" and t.cap == 8192 and t.stride == 8192
    bt = synth.WORKLOADS["batched_16x64k"]
    assert bt.seeds == tuple(range(1, 17))


def test_clustered_keys_recipe():
    """blobs > 0: every key of a head is its centre (one of `blobs`, drawn
    2 * N(0,1)) plus blob_spread * N(0,1) noise, so keys lie close to their
    nearest centre, far from the others, with about blob_spread per axis."""
    w = synth.custom(B=1, N=2000, Hq=8, Hkv=2, d=64, L=1, dtype="f32", seed=3,
                     mode="threshold", cap=64, blobs=6, blob_spread=0.1)
    x = synth.generate(w)
    K = synth.f32(x["K"])[0].astype(np.float64)               # [Hkv, N, d]
    for h in range(2):
        X = K[h]
        # recover the centres: centres sit ~2*sqrt(2d) ~ 23 apart and keys
        # within ~0.1*sqrt(d) ~ 0.8 of theirs, so farthest-point picks give
        # one key per blob and one nearest-pick pass gives the groups
        pick = [0]
        for _ in range(5):
            dmin = np.min(((X[:, None, :] - X[pick][None]) ** 2).sum(-1), axis=1)
            pick.append(int(np.argmax(dmin)))
        lab = np.argmin(((X[:, None, :] - X[pick][None]) ** 2).sum(-1), axis=1)
        cent = np.stack([X[lab == c].mean(0) for c in range(6)])
        resid = X - cent[lab]
        assert 0.08 < resid.std() < 0.12                     # blob_spread per axis
        assert np.sqrt((resid ** 2).sum(1)).max() < 0.1 * 8 + 0.5
    lw = synth.WORKLOADS["louver_128k"]
    assert (lw.N, lw.Hq, lw.Hkv, lw.d, lw.L, lw.cap, lw.blobs) == (131072, 32, 8, 128, 16,
                                                                  8192, 64)
    assert lw.mode == "threshold" and lw.blob_spread == 0.1
