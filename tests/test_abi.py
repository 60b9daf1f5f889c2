"""The C-ABI library loads on a machine without a GPU, exports every symbol
the header declares, and rejects bad arguments on the host before any device
work (so these checks need no GPU)."""
import ctypes
import os
import re

import pytest
import torch

import token_sparse_attention_sm_b200 as sd
from token_sparse_attention_sm_b200 import build as sd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_decode.h")


@pytest.fixture(scope="module")
def lib():
    sd_build.build()
    return sd.load()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(sparse_[a-z_]+)\s*\(", text)))


def test_header_symbols_are_exported(lib):
    declared = _declared()
    assert set(declared) == set(sd.EXPORTED_SYMBOLS)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in sd.STATUS_NAMES.items():
        assert lib.sparse_status_string(code).decode().startswith(name)
    assert lib.sparse_version() >= 100


def _shape(**kw):
    base = dict(B=1, N=4096, Hq=8, Hkv=2, d=64, dtype=1)
    base.update(kw)
    return sd._Shape(**base)


def _ws_size(lib, sh, k=16, L=2):
    n = ctypes.c_size_t(0)
    rc = lib.sparse_workspace_size(ctypes.byref(sh), k, L, ctypes.byref(n))
    return rc, n.value


def test_workspace_size_validation(lib):
    rc, n = _ws_size(lib, _shape())
    assert rc == 0 and n >= 256 + 2 * 4096 * 4
    assert _ws_size(lib, _shape(Hq=7))[0] == 1          # Hq % Hkv
    assert _ws_size(lib, _shape(d=96))[0] == 2          # unsupported d
    assert _ws_size(lib, _shape(dtype=7))[0] == 2
    assert _ws_size(lib, _shape(Hq=34, Hkv=2))[0] == 2  # G = 17 > 16
    assert _ws_size(lib, _shape(N=0))[0] == 1
    assert _ws_size(lib, _shape(), k=0)[0] == 1
    assert _ws_size(lib, _shape(), L=0)[0] == 1
    assert _ws_size(lib, _shape(Hq=16, Hkv=1), L=65)[0] == 2  # L*G > 1024


def test_bad_arguments_rejected_before_device_work(lib):
    sh = _shape()
    fake = ctypes.c_void_p(0x10000)      # never dereferenced: checks come first
    odd = ctypes.c_void_p(0x10008)       # not 16-byte aligned
    ws_ok = ctypes.c_void_p(0x100000)
    rc, need = _ws_size(lib, sh, k=16, L=1)
    # null pointers
    assert lib.sparse_route_topk(ctypes.byref(sh), None, fake, 16, fake, ws_ok,
                                 need, None) == 1
    # k out of range
    assert lib.sparse_route_topk(ctypes.byref(sh), fake, fake, 0, fake, ws_ok,
                                 need, None) == 1
    assert lib.sparse_route_topk(ctypes.byref(sh), fake, fake, 4097, fake, ws_ok,
                                 need, None) == 1
    # misaligned K
    assert lib.sparse_route_topk(ctypes.byref(sh), fake, odd, 16, fake, ws_ok,
                                 need, None) == 1
    # workspace too small
    assert lib.sparse_route_topk(ctypes.byref(sh), fake, fake, 16, fake, ws_ok,
                                 need - 1, None) == 3
    # unsupported head dim
    sh96 = _shape(d=96)
    assert lib.sparse_score(ctypes.byref(sh96), fake, fake, fake, ws_ok, 1 << 30,
                            None) == 2
    # decode step: both k and tau, or neither
    rc, need = _ws_size(lib, sh, k=16, L=2)
    assert lib.sparse_decode_step(ctypes.byref(sh), 2, fake, fake, fake, fake, 16,
                                  fake, 0, fake, fake, fake, None, ws_ok, need,
                                  None) == 1
    assert lib.sparse_decode_step(ctypes.byref(sh), 2, fake, fake, fake, fake, 0,
                                  None, 16, fake, fake, fake, None, ws_ok, need,
                                  None) == 1
    # threshold needs count and cap >= 1
    assert lib.sparse_route_threshold(ctypes.byref(sh), fake, fake, fake, 0, fake,
                                      fake, ws_ok, need, None) == 1
    assert lib.sparse_attn_gather(ctypes.byref(sh), 1, fake, fake, fake, fake, 0,
                                  None, fake, None, ws_ok, need, None) == 1
    assert lib.sparse_read_device_status(None, None, None) == 1
    # cache capacity below the cache length
    short = _shape(n_cap=100)
    assert lib.sparse_route_topk(ctypes.byref(short), fake, fake, 16, fake, ws_ok,
                                 1 << 30, None) == 1
    assert lib.sparse_kv_append(ctypes.byref(short), fake, fake, fake, fake, None) == 1
    # append: null or misaligned rows
    assert lib.sparse_kv_append(ctypes.byref(sh), fake, fake, None, fake, None) == 1
    assert lib.sparse_kv_append(ctypes.byref(sh), fake, fake, odd, fake, None) == 1
    # grouped step: R < 1
    rc, need = _ws_size(lib, sh, k=16, L=2)
    assert lib.sparse_decode_step_grouped(ctypes.byref(sh), 4, 0, fake, fake, fake, fake, 16,
                                          None, 0, fake, None, fake, None, ws_ok, need,
                                          None) == 1


def test_python_binding_refuses_cpu_tensors(lib):
    q = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    K = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sd.route_topk(q, K, 8)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(sd, "_LIB_FILE", str(tmp_path / "absent.so"))
    monkeypatch.setattr(sd, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        sd.load()


def test_louver_arguments_rejected_before_device_work(lib):
    """Louver index: r and N must give a balanced tree (r a power of two in
    [32, 256], N / r a power of two); undersized buffers, null or misaligned
    pointers are refused before any device work."""
    P = ctypes.c_size_t
    ib, wb = P(0), P(0)
    ok = _shape(N=8192)
    assert lib.sparse_louver_sizes(ctypes.byref(ok), 128, ctypes.byref(ib), ctypes.byref(wb)) == 0
    # the index holds perm, centres, radii and a copy of the keys
    BH, N, d, es = ok.B * ok.Hkv, ok.N, ok.d, 2 if ok.dtype == 1 else 4
    assert ib.value >= BH * N * 4 + BH * (N // 128) * (d + 1) * 4 + BH * N * d * es
    for r in (16, 48, 512):
        assert lib.sparse_louver_sizes(ctypes.byref(ok), r, ctypes.byref(ib),
                                       ctypes.byref(wb)) == 2
    for n in (8192 + 128, 96 * 128):           # N not a multiple / N/r not a power of two
        sh = _shape(N=n)
        assert lib.sparse_louver_sizes(ctypes.byref(sh), 128, ctypes.byref(ib),
                                       ctypes.byref(wb)) == 2
    assert lib.sparse_louver_sizes(ctypes.byref(ok), 128, None, ctypes.byref(wb)) == 1
    lib.sparse_louver_sizes(ctypes.byref(ok), 128, ctypes.byref(ib), ctypes.byref(wb))
    fake = ctypes.c_void_p(0x10000)
    big = ctypes.c_void_p(0x100000)
    odd = ctypes.c_void_p(0x10010)              # 16- but not 256-byte aligned
    # build: null K, misaligned index, index or workspace too small
    assert lib.sparse_louver_build(ctypes.byref(ok), None, 128, big, ib.value, big, wb.value,
                                   None) == 1
    assert lib.sparse_louver_build(ctypes.byref(ok), fake, 128, odd, ib.value, big, wb.value,
                                   None) == 1
    assert lib.sparse_louver_build(ctypes.byref(ok), fake, 128, big, ib.value - 1, big,
                                   wb.value, None) == 3
    assert lib.sparse_louver_build(ctypes.byref(ok), fake, 128, big, ib.value, big,
                                   wb.value - 1, None) == 3
    # query: cap < 1, null tau, unsupported r
    assert lib.sparse_louver_route_threshold(ctypes.byref(ok), fake, big, ib.value, 128, fake,
                                             0, fake, fake, None, big, wb.value, None) == 1
    assert lib.sparse_louver_route_threshold(ctypes.byref(ok), fake, big, ib.value, 128, None,
                                             8, fake, fake, None, big, wb.value, None) == 1
    assert lib.sparse_louver_route_threshold(ctypes.byref(ok), fake, big, ib.value, 100, fake,
                                             8, fake, fake, None, big, wb.value, None) == 2


def test_selftest_arguments_rejected(lib):
    fake = ctypes.c_void_p(0x100000)
    assert lib.sparse_selftest_bounded_wait(None, 1 << 20, 1000, None) == 1
    assert lib.sparse_selftest_bounded_wait(ctypes.c_void_p(0x100010), 1 << 20, 1000, None) == 1
    assert lib.sparse_selftest_bounded_wait(fake, 1024, 1000, None) == 1



def test_pointer_device_usable_on_host_memory(lib):
    """NULL arguments are rejected; ordinary (pageable) host memory is never
    reported usable by kernels."""
    ok = ctypes.c_int32(7)
    assert lib.sparse_pointer_device_usable(None, ctypes.byref(ok)) == 1
    buf = ctypes.create_string_buffer(4096)
    assert lib.sparse_pointer_device_usable(ctypes.addressof(buf), None) == 1
    assert lib.sparse_pointer_device_usable(ctypes.addressof(buf), ctypes.byref(ok)) == 0
    assert ok.value == 0


def test_python_binding_refuses_pageable_out(lib):
    """An out tensor in pageable host memory is refused before any launch."""
    t = torch.zeros(2, 1, 8, 64, dtype=torch.bfloat16)
    assert not sd.device_usable(t)
    with pytest.raises(ValueError):
        sd._need_out(t, t)
    with pytest.raises(ValueError):
        sd._need_out(torch.zeros(2, 1, 8, 32, dtype=torch.bfloat16), t)


def test_graph_launch_rejects_null(lib):
    assert lib.sparse_graph_launch(None, None) == 1


def test_graph_upload_rejects_null(lib):
    assert lib.sparse_graph_upload(None, None) == 1


def test_result_and_tau_checks_reject_bad_tensors(lib):
    """Caller-given results must match exactly and live where kernels can
    write them; tau needs one float per row of the sets.  All checked before
    anything is launched."""
    sd._need_result(None, (2, 3), torch.int32, "idx")          # nothing given: fine
    with pytest.raises(ValueError, match="idx"):
        sd._need_result(torch.zeros(2, 4, dtype=torch.int32), (2, 3), torch.int32, "idx")
    with pytest.raises(ValueError, match="idx"):
        sd._need_result(torch.zeros(2, 3, dtype=torch.int64), (2, 3), torch.int32, "idx")
    with pytest.raises(ValueError, match="contiguous"):
        sd._need_result(torch.zeros(3, 2, dtype=torch.int32).t(), (2, 3), torch.int32, "idx")
    with pytest.raises(ValueError, match="CUDA"):                # host memory, right shape
        sd._need_result(torch.zeros(2, 3, dtype=torch.int32), (2, 3), torch.int32, "idx")
    with pytest.raises(ValueError, match="pinned"):              # pageable host memory
        sd._need_result(torch.zeros(2, 3), (2, 3), torch.float32, "lse", host_ok=True)
    sd._need_tau(torch.zeros(2, 3), (2, 3))
    with pytest.raises(ValueError, match="tau"):
        sd._need_tau(torch.zeros(2, 4), (2, 3))
    with pytest.raises(ValueError, match="tau"):
        sd._need_tau(torch.zeros(2, 3, dtype=torch.int32), (2, 3))


def test_decode_step_fused_is_shape_logic(lib):
    """Which decode steps run on the fused select + attention kernel: bf16
    with at most 128 query rows per KV head over all layers and a cache the
    select's on-chip bitmap covers; the answer needs no device."""
    def fused(sh, L, k, cap=0):
        f = ctypes.c_int32(-1)
        rc = lib.sparse_decode_step_fused(ctypes.byref(sh), L, k, cap, ctypes.byref(f))
        return rc, f.value
    big = _shape(N=131072, Hq=32, Hkv=8, d=128)
    assert fused(big, 16, 2048) == (0, 1)
    assert fused(big, 16, 0, 8192) == (0, 1)                      # threshold
    assert fused(_shape(N=131072, Hq=32, Hkv=8, d=128, dtype=0), 16, 2048) == (0, 0)
    assert fused(_shape(N=262144, Hq=32, Hkv=8, d=128), 16, 2048) == (0, 0)
    assert fused(big, 64, 2048) == (0, 0)                         # 256 query rows
    assert fused(big, 0, 2048)[0] == 1
    assert fused(big, 16, 0, 0)[0] == 1
    assert lib.sparse_decode_step_fused(ctypes.byref(big), 16, 2048, 0, None) == 1
    assert lib.sparse_decode_step_fused(ctypes.byref(_shape(d=96)), 2, 16, 0,
                                        ctypes.byref(ctypes.c_int32())) == 2


def test_decode_step_join_checks_like_decode_step(lib):
    sh = _shape()
    fake = ctypes.c_void_p(1 << 20)
    ws_ok = ctypes.c_void_p(1 << 24)
    rc, need = _ws_size(lib, sh, k=16, L=2)
    # both k and tau; then a workspace one byte short
    assert lib.sparse_decode_step_join(ctypes.byref(sh), 2, fake, fake, fake, fake, 16, fake,
                                       0, fake, fake, fake, None, ws_ok, need, None,
                                       None) == 1
    assert lib.sparse_decode_step_join(ctypes.byref(sh), 2, fake, fake, fake, fake, 16, None,
                                       0, fake, None, fake, None, ws_ok, need - 1, None,
                                       None) == 3
