"""Times one stage of the layer alone, through its C-ABI entry point, on a synthetic layer's shapes.

    python -m mixture_experts_routing_gate_b200.stagebench --stage gate --workload v3_prefill
    python -m mixture_experts_routing_gate_b200.stagebench --stage experts --workload v3_prefill --experts 32 --tokens 512
    python -m mixture_experts_routing_gate_b200.stagebench --stage experts --workload v4_skew --swiglu-limit 10 --row-weights
    python -m mixture_experts_routing_gate_b200.stagebench --stage ngram_gate --workload hash

Only the inputs the stage needs are allocated (the router needs x and the router weight, not the
22 GB of expert weights), which keeps profiler captures of a single kernel small.  --experts and
--tokens shrink the layer while keeping its per-expert shape.  Prints one JSON line with the mean
time per call (CUDA events on the launching stream, after warm-up) and the stage's algorithmic
traffic per call.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import moe as M
from . import workloads as W


def _primes_above(m: int, k: int):
    """The k smallest primes greater than m (trial division)."""
    out, q = [], m + 1
    while len(out) < k:
        if q > 1 and all(q % f for f in range(2, int(q ** 0.5) + 1)):
            out.append(q)
        q += 1
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--stage", required=True, choices=["gate", "hash_gate", "ngram_gate", "dispatch", "experts", "combine",
                                                       "update_bias"])
    ap.add_argument("--workload", default="v3_prefill", choices=sorted(W.CONFIGS))
    ap.add_argument("--experts", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--swiglu-limit", type=float, default=None, help="experts stage: clamp limit")
    ap.add_argument("--row-weights", action="store_true", help="experts stage: gate weights inside the experts")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "mxfp4"], help="experts stage: weight format")
    ap.add_argument("--token-chunk", type=int, default=0, help="experts: desc.token_chunk (0: chosen from the shape)")
    ap.add_argument("--split-per-call", action="store_true",
                    help="gates: split the router weight into bf16 planes on every call (no moe_gate_prepare)")
    a = ap.parse_args()

    cfg = W.CONFIGS[a.workload]
    if a.experts:
        cfg = cfg.replace(n_experts=a.experts)
    if a.tokens:
        cfg = cfg.replace(T=a.tokens)
    if a.swiglu_limit is not None:
        cfg = cfg.replace(swiglu_limit=a.swiglu_limit)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, k, E, d, I = cfg.T, cfg.topk, cfg.n_experts, cfg.dim, cfg.inter_dim
    S = T * k
    desc = M.layer_desc(cfg, token_chunk=a.token_chunk)
    ws = M.Workspace(desc, T, device=dev)
    x, wg, bias, off = W.make_router_inputs(cfg, device=dev)
    planes = None if a.split_per_call else M.prepare_gate(desc, wg)   # once, outside the timed calls
    weights = torch.empty((T, k), dtype=torch.float32, device=dev)
    indices = torch.empty((T, k), dtype=torch.int32, device=dev)
    ids = table = None
    if cfg.is_hash:
        p = W.token_frequencies(cfg)
        tab, _ = M.moe_build_tid2eid(p, E, k)
        table = torch.from_numpy(tab).to(dev)
        ids = torch.from_numpy(W.sample_token_ids(cfg, p)).to(dev)

    def route():
        if cfg.is_hash:
            M.moe_hash_gate(desc, ids, table, x, wg, weights, indices, ws)
        else:
            M.moe_gate(desc, x, wg, bias, off, weights, indices, ws)

    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ros = torch.empty(S, dtype=torch.int32, device=dev)
    tor = torch.empty(S, dtype=torch.int32, device=dev)

    if a.stage in ("gate", "hash_gate"):
        fn = route
        # router weight: the fp32 matrix when split per call, else its prepared bf16 plane(s)
        wbytes = E * d * 4 if a.split_per_call else E * d * 2 * (3 if cfg.gate_general_fp32 else 1)
        nbytes = T * d * 2 + (wbytes if a.stage == "gate" else S * d * 4) + S * 8
        flops = 2.0 * T * d * (E if a.stage == "gate" else k)
    elif a.stage == "ngram_gate":
        if not cfg.is_hash:
            raise SystemExit("ngram_gate needs a hash workload")
        prev = torch.cat([torch.zeros(1, dtype=torch.int32, device=dev), ids[:-1]])
        primes = [int(q) for q in _primes_above(cfg.hash_vocab, k)]
        fn = lambda: M.moe_ngram_gate(desc, prev, ids, primes, cfg.hash_vocab, x, wg, weights, indices, ws)
        nbytes = T * d * 2 + S * d * 4 + S * 8 + T * 8
        flops = 2.0 * T * d * k
    elif a.stage == "update_bias":
        route()
        M.moe_dispatch(desc, indices, x, counts, offsets, ros, tor,
                       torch.empty((S, d), dtype=torch.bfloat16, device=dev), ws)
        b = torch.zeros(E, dtype=torch.float32, device=dev)
        fn = lambda: M.moe_update_bias(desc, T, counts, b, 0.001)
        nbytes = E * 12
        flops = 0.0
    else:
        route()
        x_perm = torch.empty((S, d), dtype=torch.bfloat16, device=dev)
        if a.stage == "dispatch":
            fn = lambda: M.moe_dispatch(desc, indices, x, counts, offsets, ros, tor, x_perm, ws)
            nbytes = S * 4 * 3 + S * d * 2 + T * d * 2
            flops = 0.0
        else:
            M.moe_dispatch(desc, indices, x, counts, offsets, ros, tor, x_perm, ws)
            out_perm = torch.empty((S, d), dtype=torch.bfloat16, device=dev)
            out_sh = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
            if a.stage == "combine":
                out_perm.copy_(W.normal_bf16((S, d), 0.1, cfg.seed, 90, device=dev))
                out_sh.copy_(W.normal_bf16((T, d), 0.1, cfg.seed, 91, device=dev))
                y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
                fn = lambda: M.moe_combine(desc, T, out_perm, ros, weights, out_sh, y)
                nbytes = (S + T) * d * 2 + S * 8 + T * d * 2
                flops = 0.0
            else:
                rw = W.uniform(S, cfg.seed, 92).to(dev, torch.float32) if a.row_weights else None
                if a.weights == "mxfp4":
                    w4 = W.make_mxfp4_weights(cfg, device=dev)
                    fn = lambda: M.moe_expert_ffn_mxfp4(desc, x_perm, offsets, x, w4, out_perm, out_sh, ws,
                                                        row_weights=rw)
                    per_weight = 0.5 + 1.0 / 32
                else:
                    li = W.make_layer(cfg, device=dev)
                    fn = lambda: M.moe_expert_ffn(desc, x_perm, offsets, x, li.w1, li.w3, li.w2, out_perm, out_sh,
                                                  ws, row_weights=rw)
                    per_weight = 2
                torch.cuda.synchronize()
                active = int((counts.cpu() > 0).sum())
                nbytes = int((active + 1) * 3 * d * I * per_weight) + (S + T) * d * 2 * 2
                flops = 6.0 * d * I * (S + T)
    for _ in range(a.warmup):
        fn()
    M.check_device_errors(ws, a.stage)
    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(a.iters + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(a.iters):
        fn()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    M.check_device_errors(ws, a.stage)
    ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(a.iters)]
    mean = sum(ms) / len(ms)
    print(json.dumps({"stage": a.stage, "workload": cfg.name, "T": T, "E": E, "d": d, "I": I,
                      "ms_mean": mean, "ms_min": min(ms), "GBps": nbytes / (mean * 1e-3) / 1e9,
                      "TFLOPs": flops / (mean * 1e-3) / 1e12, "bytes": nbytes}))


if __name__ == "__main__":
    main()
