"""sparse_route_topk_static: routing for callers that cannot allocate device
memory (a plugin whose host framework owns every device allocation, or code
that must not call cudaMalloc once running).  Its scratch is a fixed array
inside the library, so this checks, through the C ABI, that two calls in a
row give the same index sets as sparse_route_topk with a caller workspace
(index work: bit-exact), and that shapes beyond the built-in limit are
rejected.  This file sorts last so a failure here leaves the rest of the
suite already run; it also passes on its own in a fresh process."""
import ctypes

import pytest
import torch

import token_sparse_attention_sm_b200 as sd
from token_sparse_attention_sm_b200 import synth

pytestmark = pytest.mark.gpu


def _call_static(lib, q, K, k):
    B, Hq, d = q.shape
    _, Hkv, N, _ = K.shape
    sh = sd._shape(B, N, Hq, Hkv, d, q.dtype)
    idx = torch.full((B, Hkv, k), -1, dtype=torch.int32, device=q.device)
    rc = lib.sparse_route_topk_static(ctypes.byref(sh), sd._ptr(q), sd._ptr(K), int(k),
                                      sd._ptr(idx), sd._stream())
    return rc, idx


def test_static_scratch_route_matches_workspace_route():
    from token_sparse_attention_sm_b200 import build
    build.build()
    lib = sd.load()
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS["decode_128k"]          # B*Hkv*N = 2^20: the limit
    x = synth.generate(w)
    K = x["K"].to(dev)
    queries = [qr.to(dev) for qr, _ in synth.query_variants(w, x, 2)]
    for qr in queries:                           # two calls in a row
        rc, idx_static = _call_static(lib, qr, K, w.k)
        assert rc == 0, sd.STATUS_NAMES.get(rc, rc)
        idx_ws = sd.route_topk(qr, K, w.k)
        torch.cuda.synchronize()
        assert torch.equal(idx_static, idx_ws)
    # a first call of the same shape again after a different query
    rc, again = _call_static(lib, queries[0], K, w.k)
    torch.cuda.synchronize()
    assert rc == 0 and torch.equal(again, sd.route_topk(queries[0], K, w.k))


def test_static_scratch_rejects_shapes_beyond_its_limit():
    """Rejected on the host before any device work, so the (small) buffers
    passed here are never read."""
    lib = sd.load()
    dev = torch.device("cuda", 0)
    q = torch.zeros(1, 8, 128, dtype=torch.bfloat16, device=dev)
    K = torch.zeros(1, 2, 16, 128, dtype=torch.bfloat16, device=dev)
    idx = torch.zeros(1, 2, 16, dtype=torch.int32, device=dev)
    for B, N, Hq, Hkv in [(1, 600000, 8, 2), (1, 16, 130, 65)]:   # 1.2M scores; 65 heads
        sh = sd._shape(B, N, Hq, Hkv, 128, torch.bfloat16)
        rc = lib.sparse_route_topk_static(ctypes.byref(sh), sd._ptr(q), sd._ptr(K), 16,
                                          sd._ptr(idx), sd._stream())
        assert rc == 3   # SPARSE_ERR_WORKSPACE
