"""Benchmark of the MoE layer forward on B200: tokens/s per layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3_prefill] [--impl ours|reference]

A step is one pass of the whole layer (gate, dispatch, grouped SwiGLU experts, combine) over one
batch of the seeded synthetic workload, with inputs resident in HBM.  The four stages are issued
through their C-ABI entry points (the same launch sequence as moe_forward) with CUDA events between
them on the launching stream, so the per-stage times come from the timed region itself.  The
expert weights (22.6 GB for the V3 prefill layer) exceed the 126 MB L2 many times over, so no L2
flush is needed between steps.  `e2e` times moe_forward itself with pinned host buffers: the copy
of x to the device, the layer, and the copy of y back, every step.

--impl reference times the CPU oracle (the only other implementation of the layer) on a bounded
sample of tokens of the same workload, on this host's cores.

Under torchrun (N > 1) every rank runs an independent replica of the layer on its own GPU (the
layer does not shard); value = tokens processed by all ranks / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s on 1 B200; % bf16 tensor peak (GEMM), % HBM BW (route/decode)"
# DRAM bytes read + written per forward by the expert-FFN unit's two GEMM launches, from one
# single-pass ncu capture of the full workload (profiles/moe_forward_v3_prefill_launches.md).  Valid
# only for the kernels it was measured on: set to None whenever those kernels change.
MEASURED_TRAFFIC = {"v3_prefill": 15.985e9 + 0.143e9 + 7.744e9 + 0.510e9}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------------------------------------
# distributed plumbing (replicas only: the only collectives are the barrier and the max of times)
# ------------------------------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, device_index: int):
        self.proc = None
        self.out = None
        self.index = str(device_index)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = ["--id=GPU-" + uuid if not uuid.startswith("GPU-") else "--id=" + uuid]
        except Exception:
            self.sel = ["--id=%d" % device_index]

    def __enter__(self):
        try:
            self.out = open(os.path.join("/tmp", f"moe_bench_clocks_{os.getpid()}.csv"), "w+")
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.5)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.out is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.out.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.out.read())) if len(r) >= 9]
        if rows and len({r[0].strip() for r in rows}) > 1:   # the selector was ignored: keep our GPU only
            rows = [r for r in rows if r[0].strip() == self.index] or rows
        self.out.close()
        try:
            os.unlink(self.out.name)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------------------
# the CPU oracle on a bounded sample of tokens
# ------------------------------------------------------------------------------------------------
def oracle_sample(li, cfg, n_tokens: int, seed: int, table=None):
    """Times the oracle's layer forward on n_tokens sampled tokens (experts fetched to host first)."""
    import oracle as O
    from mixture_experts_routing_gate_b200 import workloads as W
    rows = W.sample_rows(cfg.T, n_tokens, seed)
    x = li.x[rows].to(torch.float64).cpu().numpy()
    wg = li.w_gate.to(torch.float64).cpu().numpy()
    bias = None if li.bias is None else li.bias.cpu().numpy()
    off = None if li.logit_offset is None else li.logit_offset.cpu().numpy()
    hp = O.Hyper.of(cfg)
    kw = {}
    if table is not None:
        kw = dict(token_ids=li.token_ids.cpu().numpy()[rows], tid2eid=table)
    # which experts the sample needs (routing is per token), staged in host memory as bf16
    if table is not None:
        idx = table[kw["token_ids"]]
    else:
        idx = O.gate(x, wg, hp, bias, off).indices
    need = sorted(set(idx.reshape(-1).tolist()) | {cfg.n_experts})
    host = {e: (li.w1[e].cpu(), li.w3[e].cpu(), li.w2[e].cpu()) for e in need}
    fetch = lambda e: tuple(t.to(torch.float64).numpy() for t in host[e])
    t0 = time.perf_counter()
    O.moe_forward(x, hp, fetch, wg, bias, off, **kw)
    dt = time.perf_counter() - t0
    return dt, len(rows), len(need)


def routing_stats(counts, T: int, k: int) -> dict:
    """Load statistics of one step's routing: rows per expert (max, min, mean, variance), idle
    experts, and the balance metric of the tid2eid page, max_vio = E * max_e f_e - 1 with
    f_e = counts_e / (T * k) the expert's share of the routed slots."""
    c = np.asarray(counts, np.float64)
    E = c.shape[0]
    return {"rows_max": int(c.max()), "rows_min": int(c.min()), "rows_mean": float(c.mean()),
            "rows_variance": float(c.var()), "idle_experts": int((c == 0).sum()),
            "max_vio": float(E * c.max() / (T * k) - 1.0)}


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------------------------------------
# main
# ------------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="v3_prefill")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=8, help="tokens in the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the routed-expert count (a smaller layer of the same shape, for profiling)")
    ap.add_argument("--tokens", type=int, default=0, help="override the batch size T")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "mxfp4"],
                    help="expert weight format (mxfp4: E2M1 codes with UE8M0 block scales)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank, world, local = dist_setup(args.gpus)
    from mixture_experts_routing_gate_b200 import workloads as W
    cfg = W.CONFIGS[args.workload]
    if args.experts:
        cfg = cfg.replace(n_experts=args.experts, name=f"{cfg.name}-{args.experts}e")
    if args.tokens:
        cfg = cfg.replace(T=args.tokens, name=f"{cfg.name}-T{args.tokens}")
    fmt = "" if args.weights == "bf16" else ", MXFP4 expert weights"
    config = {"workload": f"{cfg.name}: T={cfg.T} d={cfg.dim} E={cfg.n_experts} G={cfg.n_groups} "
                          f"g={cfg.n_limited_groups} k={cfg.topk} I={cfg.inter_dim} +1 shared, {cfg.score_func}{fmt}",
              "T": cfg.T, "dim": cfg.dim, "n_experts": cfg.n_experts, "topk": cfg.topk,
              "inter_dim": cfg.inter_dim, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
              "l2": "no flush: expert weights stream from HBM every step (far larger than the 126 MB L2)"}

    if args.impl == "reference":
        run_reference(args, cfg, config, rank, world)
        return
    run_ours(args, cfg, config, rank, world, local)


def run_reference(args, cfg, config, rank, world):
    if rank != 0:
        return
    from mixture_experts_routing_gate_b200 import workloads as W
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    li = W.make_layer(cfg, device=dev)
    table = None
    if cfg.is_hash:
        import oracle as O
        table, _ = O.build_tid2eid(li.p, cfg.n_experts, cfg.topk)
    n_tok = 2
    for i in range(args.warmup):
        oracle_sample(li, cfg, n_tok, seed=1000 + i, table=table)
    times = []
    for i in range(args.steps):
        dt, n, _ = oracle_sample(li, cfg, n_tok, seed=2000 + i, table=table)
        times.append((dt, n))
    tot_t = sum(t for t, _ in times)
    tot_n = sum(n for _, n in times)
    v = tot_n / tot_t
    cores = cpu_threads()
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config,
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n_tok} seeded tokens of the workload per step (numpy fp64 oracle)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, cfg, config, rank, world, local):
    from mixture_experts_routing_gate_b200 import moe as M
    from mixture_experts_routing_gate_b200 import workloads as W
    dev = torch.device("cuda", torch.cuda.current_device())
    fp4 = args.weights == "mxfp4"
    li = W.make_layer(cfg, device=dev, bf16_experts=not fp4)
    w4 = W.make_mxfp4_weights(cfg, device=dev) if fp4 else None
    T, k, E, d, I = cfg.T, cfg.topk, cfg.n_experts, cfg.dim, cfg.inter_dim
    S = T * k
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, T, device=dev)
    table = None
    tid2eid = None
    if cfg.is_hash:
        table, _ = M.moe_build_tid2eid(li.p, E, k)
        tid2eid = torch.from_numpy(table).to(dev)
    # MOE_FUSED_GATHER=1 (as for moe_forward): the up-projection kernel gathers its token rows of x
    # itself (moe_expert_ffn_gather, no x_perm) instead of dispatch's gather kernel writing x_perm.
    gather = (I % 256 == 0 and os.environ.get("MOE_FUSED_GATHER") == "1"
              and os.environ.get("MOE_GEMM_SINGLE_CTA") != "1")
    # gate (planes + router, or the hash gate), dispatch (count, column scan, offsets, rank, and the
    # gather unless fused), experts (tile list, two GEMMs), combine
    launches_per_step = (1 if cfg.is_hash else 2) + (4 if gather else 5) + 3 + 1
    # stage buffers (the layer's intermediate tensors)
    weights = torch.empty((T, k), dtype=torch.float32, device=dev)
    indices = torch.empty((T, k), dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ros = torch.empty(S, dtype=torch.int32, device=dev)
    tor = torch.empty(S, dtype=torch.int32, device=dev)
    x_perm = None if gather else torch.empty((S, d), dtype=torch.bfloat16, device=dev)
    out_perm = torch.empty((S, d), dtype=torch.bfloat16, device=dev)
    out_sh = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    nstage = 4

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if cfg.is_hash:
            M.moe_hash_gate(desc, li.token_ids, tid2eid, li.x, li.w_gate, weights, indices, ws)
        else:
            M.moe_gate(desc, li.x, li.w_gate, li.bias, li.logit_offset, weights, indices, ws)
        if ev is not None:
            ev[1].record(stream)
        M.moe_dispatch(desc, indices, li.x, counts, offsets, ros, tor, None if gather else x_perm, ws)
        if ev is not None:
            ev[2].record(stream)
        if fp4 and gather:
            M.moe_expert_ffn_mxfp4_gather(desc, tor, offsets, li.x, w4, out_perm, out_sh, ws)
        elif fp4:
            M.moe_expert_ffn_mxfp4(desc, x_perm, offsets, li.x, w4, out_perm, out_sh, ws)
        elif gather:
            M.moe_expert_ffn_gather(desc, tor, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws)
        else:
            M.moe_expert_ffn(desc, x_perm, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws)
        if ev is not None:
            ev[3].record(stream)
        M.moe_combine(desc, T, out_perm, ros, weights, out_sh, y)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    M.check_device_errors(ws, "warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage + 1)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        wall0 = time.perf_counter()
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        wall_ms = (time.perf_counter() - wall0) * 1e3
        barrier(world)
    clocks = clk.summary()
    M.check_device_errors(ws, "timed steps")
    total_ms = t_start.elapsed_time(t_end)
    stage_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(nstage)] for i in range(args.steps)])
    ms_step = max_over_ranks(total_ms / args.steps, world)
    value = world * T / (ms_step * 1e-3)

    # ---------------- e2e: moe_forward through the C ABI, host buffers in and out ----------------
    # A serving loop: every step uploads its batch from pinned host memory, runs moe_forward and
    # downloads y.  The uploads and downloads run on their own streams, double-buffered, so that step
    # i+1's upload and step i-1's download overlap step i's layer; the timed region spans the first
    # upload to the last download.
    x_host = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(li.x.cpu())
    y_host = [torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    ids_host = None
    if cfg.is_hash:
        ids_host = torch.empty(T, dtype=torch.int32, pin_memory=True)
        ids_host.copy_(li.token_ids.cpu())
    x_dev = [torch.empty_like(li.x) for _ in range(2)]
    ids_dev = [torch.empty(T, dtype=torch.int32, device=dev) if cfg.is_hash else None for _ in range(2)]
    y_dev = [torch.empty_like(li.x) for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)

        def upload(i):
            b = i % 2
            up.wait_event(start)
            if i >= 2:
                up.wait_event(ev_done[b])     # step i-2 no longer reads x_dev[b]
            with torch.cuda.stream(up):
                x_dev[b].copy_(x_host, non_blocking=True)
                if ids_host is not None:
                    ids_dev[b].copy_(ids_host, non_blocking=True)
            ev_up[b].record(up)

        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            stream.wait_event(ev_up[b])
            if i >= 2:
                stream.wait_event(ev_down[b])   # y_dev[b] of step i-2 has been downloaded
            if fp4:
                M.moe_forward_mxfp4(desc, x_dev[b], li.w_gate, w4, y_dev[b], ws, bias=li.bias,
                                    logit_offset=li.logit_offset, token_ids=ids_dev[b], tid2eid=tid2eid)
            else:
                M.moe_forward(desc, x_dev[b], li.w_gate, li.w1, li.w3, li.w2, y_dev[b], ws, bias=li.bias,
                              logit_offset=li.logit_offset, token_ids=ids_dev[b], tid2eid=tid2eid)
            ev_done[b].record(stream)
            down.wait_event(ev_done[b])
            with torch.cuda.stream(down):
                y_host[b].copy_(y_dev[b], non_blocking=True)
            ev_down[b].record(down)
        for b in range(2):
            stream.wait_event(ev_down[b])
        end.record(stream)
        return start, end, (n - 1) % 2

    e2e_run(args.warmup)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1, last = e2e_run(args.steps)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    assert torch.equal(y_host[last], y.cpu()), "moe_forward and the staged entry points disagree"
    h2d = T * d * 2 + (T * 4 if cfg.is_hash else 0)
    d2h = T * d * 2

    # ---------------- roofline of the dominant unit: the grouped expert FFN ----------------
    peaks, peak_src = load_peaks()
    cnt = counts.cpu().numpy()
    active = int((cnt > 0).sum())
    bytes_per_weight = (0.5 + 1.0 / 32) if fp4 else 2.0   # MXFP4: a 4-bit code + a byte per 32 elements
    w_bytes = (active + 1) * 3 * d * I * bytes_per_weight
    ffn_bytes = w_bytes + (S + T) * d * 2 * 2          # + rows in (x_perm, x) and rows out (out_perm, out_shared)
    ffn_flops = 6.0 * d * I * (S + T)
    ffn_ms = float(stage_ms[:, 2].mean())
    kernel = "moe_expert_ffn%s (up-projection + down-projection GEMMs)" % ("_mxfp4" if fp4 else "")
    t_mem = ffn_bytes / (peaks["hbm_gbs"] * 1e9)
    t_math = ffn_flops / (peaks["bf16_tflops"] * 1e12)
    if t_math > t_mem:   # the unit's roofline: whichever of HBM and the bf16 tensor cores takes longer
        achieved = ffn_flops / (ffn_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "unit": "TFLOP/s", "achieved": achieved, "peak": peaks["bf16_tflops"],
                    "frac": achieved / peaks["bf16_tflops"], "algorithmic_flops": ffn_flops,
                    "hbm_frac": ffn_bytes / (ffn_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    else:
        achieved = ffn_bytes / (ffn_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "unit": "GB/s", "achieved": achieved, "peak": peaks["hbm_gbs"],
                    "frac": achieved / peaks["hbm_gbs"],
                    "tensor_frac": ffn_flops / (ffn_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}
    roofline.update({"kernel": kernel, "peak_source": peak_src, "algorithmic_bytes": ffn_bytes,
                     "active_experts": active, "traffic": None if fp4 else MEASURED_TRAFFIC.get(cfg.name)})
    stages = dict(zip(["gate", "dispatch", "expert_ffn", "combine"], [float(v) for v in stage_ms.mean(axis=0)]))

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based generator)",
            "config": config, "clocks": clocks,
            "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps, "stage_ms": stages,
            "wall_ms_timed_region": wall_ms, "roofline": roofline, "routing": routing_stats(cnt, T, k)}

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp4:
        dt, n, ne = oracle_sample(li, cfg, args.cpu_tokens, seed=12345, table=table)
        line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"{n} seeded tokens of the workload ({ne} experts incl. shared), "
                                          f"numpy fp64 oracle, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
