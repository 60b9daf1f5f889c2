"""Run a few launches of one entry point on a named workload, for profilers.

    python -m token_sparse_attention_sm_b200.profile_case \
        --workload decode_128k --op decode --reps 3

--op is one of: score, route, attn, decode, threshold (full-scan threshold
routing, tau the 97th-percentile score of each head), louver (the same
threshold routing through a Louver index with clusters of --r keys).  Inputs come from the seeded
generator; nothing is checked or timed here (use bench.py for timing and the
tests for parity).  The process exits non-zero if the device reports any
condition."""
from __future__ import annotations

import argparse

import torch

import token_sparse_attention_sm_b200 as sd
from token_sparse_attention_sm_b200 import synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="decode_128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--op", default="decode",
                    choices=["score", "route", "attn", "decode", "threshold", "louver"])
    ap.add_argument("--r", type=int, default=128)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    w = synth.WORKLOADS[a.workload]
    x = synth.generate(w)
    dev = torch.device("cuda", 0)
    t = {n: x[n].to(dev) for n in ("q_route", "q_layers", "K", "V")}
    ws = sd.Workspace(dev)
    k = w.k if w.mode == "topk" else w.cap
    idx = sd.route_topk(t["q_route"], t["K"], k, ws=ws) if a.op == "attn" else None
    if a.op in ("louver", "threshold"):
        S = sd.score(t["q_route"], t["K"], ws=ws)
        tau = torch.kthvalue(S, -(-97 * w.N // 100), dim=-1).values.contiguous()
    if a.op == "louver":
        ix = sd.louver_build(t["K"], a.r)
    for _ in range(a.reps):
        if a.op == "louver":
            sd.louver_route_threshold(t["q_route"], t["K"], ix, tau, w.cap or w.N, check=False)
            continue
        if a.op == "threshold":
            sd.route_threshold(t["q_route"], t["K"], tau, w.cap or w.N, ws=ws, check=False)
            continue
        if a.op == "score":
            sd.score(t["q_route"], t["K"], ws=ws, check=False)
        elif a.op == "route":
            sd.route_topk(t["q_route"], t["K"], k, ws=ws, check=False)
        elif a.op == "attn":
            sd.attn_gather(t["q_layers"], t["K"], t["V"], idx, ws=ws, check=False)
        else:
            sd.decode_step(t["q_route"], t["q_layers"], t["K"], t["V"], k=k, ws=ws,
                           check=False)
    torch.cuda.synchronize()
    sd.read_device_status(ws)
    if a.op == "louver":
        sd.read_device_status(ix.ws)
    print(f"{a.op} x{a.reps} on {w.name}: ok")


if __name__ == "__main__":
    main()
