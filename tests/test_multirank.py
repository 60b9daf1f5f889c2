"""Multi-process host logic on CPU (gloo, world_size 2): the decode path
shards into independent sequences with no exchange step, so each rank runs
its own share and only the timing uses collectives (barrier, max over ranks).
The per-rank compute here is the CPU oracle, standing in for the GPU path."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import oracle
    from token_sparse_attention_sm_b200 import dist as sdist
    from token_sparse_attention_sm_b200 import synth

    assert sdist.init("gloo", timeout_s=60)
    r, w, lr = sdist.env_rank_world()
    assert (r, w, lr) == (rank, world, rank)
    wl = synth.custom(B=5, N=300, Hq=8, Hkv=2, d=64, L=2, k=20, dtype="bf16", seed=3)
    lo, hi = sdist.shard_range(wl.B, w, r)
    x = synth.generate(wl, batches=range(lo, hi))
    res = oracle.decode_step(synth.f32(x["q_route"]), synth.f32(x["q_layers"]),
                             synth.f32(x["K"]), synth.f32(x["V"]), k=wl.k)
    np.save(os.path.join(out_dir, f"idx{rank}.npy"), res["idx"])
    np.save(os.path.join(out_dir, f"out{rank}.npy"), res["out"])
    sdist.barrier()
    mx = sdist.max_over_ranks(10.0 + rank)
    tot = sdist.sum_over_ranks(hi - lo)
    with open(os.path.join(out_dir, f"stats{rank}.txt"), "w") as f:
        f.write(f"{lo} {hi} {mx} {tot}\n")
    dist.barrier()
    sdist.finalize()


def test_shard_range_covers_every_unit_once():
    from token_sparse_attention_sm_b200 import dist as sdist
    for n in (0, 1, 5, 16, 17):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                lo, hi = sdist.shard_range(n, world, r)
                assert 0 <= lo <= hi <= n
                seen.extend(range(lo, hi))
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        sdist.shard_range(4, 2, 2)


def test_two_rank_gloo_replicas_match_single_process(tmp_path):
    import oracle
    from token_sparse_attention_sm_b200 import synth

    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2,
                       start_method="spawn", join=True)
    stats = [open(tmp_path / f"stats{r}.txt").read().split() for r in range(2)]
    assert [s[:2] for s in stats] == [["0", "2"], ["2", "5"]]
    assert all(float(s[2]) == 11.0 for s in stats)      # max over ranks
    assert all(float(s[3]) == 5.0 for s in stats)       # every sequence once
    wl = synth.custom(B=5, N=300, Hq=8, Hkv=2, d=64, L=2, k=20, dtype="bf16", seed=3)
    x = synth.generate(wl)
    ref = oracle.decode_step(synth.f32(x["q_route"]), synth.f32(x["q_layers"]),
                             synth.f32(x["K"]), synth.f32(x["V"]), k=wl.k)
    idx = np.concatenate([np.load(tmp_path / f"idx{r}.npy") for r in range(2)], axis=0)
    out = np.concatenate([np.load(tmp_path / f"out{r}.npy") for r in range(2)], axis=1)
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_array_equal(out, ref["out"])
