"""Benchmark of the MoE layer forward on B200: tokens/s per layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3_prefill] [--only] [--impl ours|reference]

A step is one pass of the whole layer (gate, dispatch, grouped SwiGLU experts, combine) over one
batch of the seeded synthetic workload, with inputs resident in HBM.  The four stages are issued
through their C-ABI entry points (the same launch sequence as moe_forward) with CUDA events between
them on the launching stream, so the per-stage times come from the timed region itself.  Every
layer's expert weights (4 to 23 GB, except the tiny layer's 3 MB) exceed the 126 MB L2 many times
over, so no L2 flush is needed between steps; the tiny layer is latency-bound and runs L2-resident.
`e2e` times moe_forward itself with pinned host buffers: the copy of x to the device, the layer, and
the copy of y back, every step.

The headline line is the --workload layer (the V3-shaped prefill layer by default).  Unless --only
is given, the same line also carries a `workloads` object with the other four synthetic layers
(tiny, hash-routed, decode-sized, V4-style skewed), each timed the same way with its own roofline
against the roof that binds it.

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
WORKLOADS = ("v3_prefill", "tiny", "hash", "v3_decode", "v4_skew")
# the same layers with MXFP4 expert weights (E4M3 activations on the block-scaled tensor cores)
MXFP4_WORKLOADS = ("v3_prefill", "v3_decode", "v4_skew")

# DRAM traffic of the expert-FFN GEMMs.  An ncu capture of the full workload would replay multi-GB
# launches, so the counters (dram__bytes_read.sum + dram__bytes_write.sum) come from a small case of
# the same per-expert shape (fewer experts and tokens, the same rows per expert), and the full-size
# traffic is that capture's traffic per algorithmic byte times the full launch's algorithmic bytes.
# Entries are keyed by the digest of the kernel sources they were measured on (kernel_digest): once
# the kernels change, the digest no longer matches and `traffic` is reported as null.
#   digest -> {(workload, weights): (captured DRAM bytes, the capture's algorithmic bytes, capture)}
TRAFFIC = {
    "4e5e4982d5bdd683": {   # bf16 expert GEMMs
        ("v3_prefill", "bf16"): (3072975872, 2921332736, "32 experts (32 active), T=512"),
        ("hash", "bf16"): (1825856768, 1677721600, "32 experts (32 active), T=1024"),
        ("v3_decode", "bf16"): (2561702912, 2554560512, "32 experts (28 active), T=8"),
        ("v4_skew", "bf16"): (2717005824, 2118123520, "48 experts (43 active), T=2048"),
    },
    "07ee8d7f070ad09d": {   # mxfp4 expert GEMMs
        ("v3_prefill", "mxfp4"): (873912320, 786759680, "32 experts (32 active), T=512"),
        ("v3_decode", "mxfp4"): (686870272, 678723584, "32 experts (28 active), T=8"),
        ("v4_skew", "mxfp4"): (781231616, 593428480, "48 experts (43 active), T=2048"),
    },
}
_GEMM_SOURCES = {"bf16": ("expert_gemm.cu", "expert_tiles.cuh", "common.cuh", "kernels.h"),
                 "mxfp4": ("expert_gemm_mx.cu", "expert_tiles.cuh", "common.cuh", "kernels.h")}


def kernel_digest(weights: str) -> str:
    """sha256 (first 16 hex digits) of the expert-GEMM sources of the given weight format."""
    import hashlib
    h = hashlib.sha256()
    for name in _GEMM_SOURCES[weights]:
        with open(os.path.join(ROOT, "mixture_experts_routing_gate_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def scaled_traffic(workload: str, weights: str, algorithmic_bytes: float):
    """Full-launch DRAM traffic from a matching small-case capture, or None."""
    entry = TRAFFIC.get(kernel_digest(weights), {}).get((workload, weights))
    if entry is None:
        return None
    dram, alg, _ = entry
    return dram / alg * algorithmic_bytes
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
# one synthetic layer: inputs resident on the device, stage buffers, one step through the C ABI
# ------------------------------------------------------------------------------------------------
class Layer:
    """A synthetic layer with all inputs on the device and the buffers of the four stages."""

    def __init__(self, cfg, dev, fp4: bool, gather: bool):
        from mixture_experts_routing_gate_b200 import moe as M
        from mixture_experts_routing_gate_b200 import workloads as W
        self.M, self.cfg, self.dev, self.fp4 = M, cfg, dev, fp4
        self.li = W.make_layer(cfg, device=dev, bf16_experts=not fp4)
        self.w4 = W.make_mxfp4_weights(cfg, device=dev) if fp4 else None
        T, k, E, d = cfg.T, cfg.topk, cfg.n_experts, cfg.dim
        S = T * k
        # MOE_OPT_FUSED_GATHER (as moe_forward with that option): the up-projection kernel gathers
        # its token rows of x itself (moe_expert_ffn_gather, no x_perm) instead of dispatch writing x_perm.
        # MXFP4 experts always take the gather entry point: it quantises x to E4M3 once and copies the
        # quantised rows (the work moe_forward_mxfp4's dispatch does), where the x_perm entry point
        # would quantise every bf16 copy again.
        self.gather = fp4 or (gather and cfg.inter_dim % 256 == 0)
        self.desc = M.layer_desc(cfg, options=M.MOE_OPT_FUSED_GATHER if self.gather else 0)
        self.ws = M.Workspace(self.desc, T, device=dev)
        # the router weight's bf16 planes are prepared once, with the weights, outside any timed region
        self.gate_planes = M.prepare_gate(self.desc, self.li.w_gate)
        self.table = self.tid2eid = None
        if cfg.is_hash:   # the greedy table is built once, on the host, outside any timed region
            self.table, _ = M.moe_build_tid2eid(self.li.p, E, k)
            self.tid2eid = torch.from_numpy(self.table).to(dev)
        f32, i32, bf = dict(dtype=torch.float32, device=dev), dict(dtype=torch.int32, device=dev), \
            dict(dtype=torch.bfloat16, device=dev)
        self.weights = torch.empty((T, k), **f32)
        self.indices = torch.empty((T, k), **i32)
        self.counts = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.ros = torch.empty(S, **i32)
        self.tor = torch.empty(S, **i32)
        self.x_perm = None if self.gather else torch.empty((S, d), **bf)
        self.out_perm = torch.empty((S, d), **bf)
        self.out_sh = torch.empty((T, d), **bf)
        self.y = torch.empty((T, d), **bf)

    def kernels_per_step(self) -> int:
        """Kernel launches of one step: gate (the router on the prepared weight planes, or one warp per
        token for hash layers whose expert count the cluster router does not take), dispatch
        (histogram, then rank and gather), experts (tile list, up and down projections; with MXFP4
        weights also the quantisation of x to E4M3 and the gather of its routed rows), combine."""
        return 1 + 2 + 3 + (2 if self.fp4 else 0) + 1   # MXFP4: quantisation of x, gather of its rows

    def step(self, stream, ev=None):
        M, li, desc, ws = self.M, self.li, self.desc, self.ws
        if ev is not None:
            ev[0].record(stream)
        if self.cfg.is_hash:
            M.moe_hash_gate(desc, li.token_ids, self.tid2eid, li.x, li.w_gate, self.weights, self.indices, ws)
        else:
            M.moe_gate(desc, li.x, li.w_gate, li.bias, li.logit_offset, self.weights, self.indices, ws)
        if ev is not None:
            ev[1].record(stream)
        M.moe_dispatch(desc, self.indices, li.x, self.counts, self.offsets, self.ros, self.tor, self.x_perm, ws)
        if ev is not None:
            ev[2].record(stream)
        if self.fp4 and self.gather:
            M.moe_expert_ffn_mxfp4_gather(desc, self.tor, self.offsets, li.x, self.w4, self.out_perm, self.out_sh, ws)
        elif self.fp4:
            M.moe_expert_ffn_mxfp4(desc, self.x_perm, self.offsets, li.x, self.w4, self.out_perm, self.out_sh, ws)
        elif self.gather:
            M.moe_expert_ffn_gather(desc, self.tor, self.offsets, li.x, li.w1, li.w3, li.w2, self.out_perm,
                                    self.out_sh, ws)
        else:
            M.moe_expert_ffn(desc, self.x_perm, self.offsets, li.x, li.w1, li.w3, li.w2, self.out_perm, self.out_sh,
                             ws)
        if ev is not None:
            ev[3].record(stream)
        M.moe_combine(desc, self.cfg.T, self.out_perm, self.ros, self.weights, self.out_sh, self.y)
        if ev is not None:
            ev[4].record(stream)

    def time_steps(self, steps: int, warmup: int, world: int, clocks: bool):
        """Warm-up, then exactly `steps` steps between a barrier + synchronize on both sides; returns
        (ms per step over the whole timed region, per-stage ms [steps, 4], clock summary, wall ms)."""
        stream = torch.cuda.current_stream(self.dev)
        for _ in range(warmup):
            self.step(stream)
        self.M.check_device_errors(self.ws, f"{self.cfg.name} warm-up")
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
        if sampler is not None:
            sampler.__enter__()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        wall0 = time.perf_counter()
        t_start.record(stream)
        for i in range(steps):
            self.step(stream, evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        wall_ms = (time.perf_counter() - wall0) * 1e3
        barrier(world)
        clk = None
        if sampler is not None:
            sampler.__exit__()
            clk = sampler.summary()
        self.M.check_device_errors(self.ws, f"{self.cfg.name} timed steps")
        stage_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(steps)])
        return t_start.elapsed_time(t_end) / steps, stage_ms, clk, wall_ms

    def e2e(self, steps: int, warmup: int, world: int):
        """moe_forward through the C ABI with host buffers: a serving loop in which every step uploads
        its batch from pinned host memory, runs the layer and downloads y.  Uploads and downloads run
        on their own streams, double-buffered, so that step i+1's upload and step i-1's download
        overlap step i's layer; the timed region spans the first upload to the last download.
        Returns (ms per step, h2d bytes per step, d2h bytes per step)."""
        M, li, cfg, dev = self.M, self.li, self.cfg, self.dev
        T, d = cfg.T, cfg.dim
        stream = torch.cuda.current_stream(dev)
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

        def run(n):
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
                if self.fp4:
                    M.moe_forward_mxfp4(self.desc, x_dev[b], li.w_gate, self.w4, y_dev[b], self.ws, bias=li.bias,
                                        logit_offset=li.logit_offset, token_ids=ids_dev[b], tid2eid=self.tid2eid)
                else:
                    M.moe_forward(self.desc, x_dev[b], li.w_gate, li.w1, li.w3, li.w2, y_dev[b], self.ws,
                                  bias=li.bias, logit_offset=li.logit_offset, token_ids=ids_dev[b],
                                  tid2eid=self.tid2eid)
                ev_done[b].record(stream)
                down.wait_event(ev_done[b])
                with torch.cuda.stream(down):
                    y_host[b].copy_(y_dev[b], non_blocking=True)
                ev_down[b].record(down)
            for b in range(2):
                stream.wait_event(ev_down[b])
            end.record(stream)
            return start, end, (n - 1) % 2

        run(warmup)
        barrier(world)
        torch.cuda.synchronize()
        e0, e1, last = run(steps)
        torch.cuda.synchronize()
        barrier(world)
        assert torch.equal(y_host[last], self.y.cpu()), "moe_forward and the staged entry points disagree"
        h2d = T * d * 2 + (T * 4 if cfg.is_hash else 0)
        return e0.elapsed_time(e1) / steps, h2d, T * d * 2

    def release(self):
        for name in list(vars(self)):
            if name not in ("M", "cfg", "dev", "fp4", "gather"):
                setattr(self, name, None)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def ffn_roofline(cfg, counts, ffn_ms: float, fp4: bool, peaks: dict, peak_src: str) -> dict:
    """Roofline of the dominant unit, the grouped expert FFN (moe_expert_ffn: tile list, up and down
    projections).  Algorithmic bytes: the weights of the active experts and of the shared expert, each
    read once, the T input rows of x and one output row per token (T*d*2 each way); the permuted copies
    (x_perm in, out_perm out) are reported apart as `materialised_bytes`.  Algorithmic flops:
    6*d*I per routed row and per shared row.  The unit is graded against whichever roof takes longer
    at the measured peaks: HBM bandwidth, or the dense bf16 tensor peak (burst)."""
    T, k, d, I = cfg.T, cfg.topk, cfg.dim, cfg.inter_dim
    S = T * k
    active = int((np.asarray(counts) > 0).sum())
    per_weight = (0.5 + 1.0 / 32) if fp4 else 2.0   # MXFP4: a 4-bit code + one scale byte per 32 elements
    w_bytes = (active + 1) * 3 * d * I * per_weight
    alg_bytes = w_bytes + 2 * T * d * 2
    mat_bytes = w_bytes + (S + T) * d * 2 * 2
    flops = 6.0 * d * I * (S + T)
    # MXFP4 experts run on the block-scaled FP8-class tensor cores: the measured bf16 burst peak times
    # the nominal ratio of dense FP8 (4.5 PFLOP/s) to dense bf16 (2.25 PFLOP/s)
    tflops_peak = peaks["bf16_tflops"] * (2.0 if fp4 else 1.0)
    sec = ffn_ms * 1e-3
    hbm_frac = alg_bytes / sec / 1e9 / peaks["hbm_gbs"]
    tensor_frac = flops / sec / 1e12 / tflops_peak
    t_mem = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    t_math = flops / (tflops_peak * 1e12)
    if t_math > t_mem:
        out = {"bound": "tensor", "achieved": flops / sec / 1e12, "peak": tflops_peak, "unit": "TFLOP/s",
               "frac": tensor_frac, "hbm_frac": hbm_frac}
    else:
        out = {"bound": "hbm", "achieved": alg_bytes / sec / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
               "frac": hbm_frac, "tensor_frac": tensor_frac}
    weights = "mxfp4" if fp4 else "bf16"
    out.update({"traffic": scaled_traffic(cfg.name, weights, alg_bytes), "kernel_digest": kernel_digest(weights),
                "kernel": "moe_expert_ffn%s (tile list, up- and down-projection GEMMs)" %
                ("_mxfp4" if fp4 else ""), "kernel_ms": ffn_ms,
                "peak_source": peak_src + (" (burst peaks; MXFP4 tensor peak = bf16 burst x 2)" if fp4 else
                                           " (burst peaks)"),
                "algorithmic_bytes": alg_bytes, "algorithmic_flops": flops, "materialised_bytes": mat_bytes,
                "active_experts": active, "floor_ms": 1e3 * max(t_mem, t_math)})
    if cfg.T * cfg.dim * 2 < 8 * 2 ** 20 and w_bytes < 64 * 2 ** 20:
        out["note"] = "latency-bound layer: its weights fit in L2 and launch latency dominates"
    return out


def config_of(cfg, world: int, fp4: bool) -> dict:
    fmt = "" if not fp4 else ", MXFP4 expert weights"
    return {"workload": f"{cfg.name}: T={cfg.T} d={cfg.dim} E={cfg.n_experts} G={cfg.n_groups} "
                        f"g={cfg.n_limited_groups} k={cfg.topk} I={cfg.inter_dim} +1 shared, {cfg.score_func}{fmt}",
            "T": cfg.T, "dim": cfg.dim, "n_experts": cfg.n_experts, "topk": cfg.topk, "inter_dim": cfg.inter_dim,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "no flush: expert weights stream from HBM every step (far larger than the 126 MB L2)"
                  if cfg.name != "tiny" else "no flush: the tiny layer is latency-bound and L2-resident"}


# ------------------------------------------------------------------------------------------------
# main
# ------------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="v3_prefill", help="the headline layer")
    ap.add_argument("--only", action="store_true", help="the headline layer alone (no `workloads` object)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=8, help="tokens in the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the routed-expert count (a smaller layer of the same shape, for profiling)")
    ap.add_argument("--tokens", type=int, default=0, help="override the batch size T")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "mxfp4"],
                    help="expert weight format (mxfp4: E2M1 codes with UE8M0 block scales)")
    ap.add_argument("--fused-gather", action="store_true",
                    help="the up projection gathers the rows of x itself (MOE_OPT_FUSED_GATHER, no x_perm)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank, world, local = dist_setup(args.gpus)
    from mixture_experts_routing_gate_b200 import workloads as W
    cfg = W.CONFIGS[args.workload]
    if args.experts:
        cfg = cfg.replace(n_experts=args.experts, name=f"{cfg.name}-{args.experts}e")
    if args.tokens:
        cfg = cfg.replace(T=args.tokens, name=f"{cfg.name}-T{args.tokens}")
    if args.experts or args.tokens:
        args.only = True
    config = config_of(cfg, world, args.weights == "mxfp4")
    if args.impl == "reference":
        run_reference(args, cfg, config, rank, world)
        return
    run_ours(args, cfg, config, rank, world)


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


def run_ours(args, cfg, config, rank, world):
    from mixture_experts_routing_gate_b200 import workloads as W
    dev = torch.device("cuda", torch.cuda.current_device())
    fp4 = args.weights == "mxfp4"
    peaks, peak_src = load_peaks()

    # ---------------- the headline layer ----------------
    layer = Layer(cfg, dev, fp4, args.fused_gather)
    ms_local, stage_ms, clocks, wall_ms = layer.time_steps(args.steps, args.warmup, world, clocks=True)
    ms_step = max_over_ranks(ms_local, world)
    value = world * cfg.T / (ms_step * 1e-3)
    e2e_local, h2d, d2h = layer.e2e(args.steps, args.warmup, world)
    e2e_ms = max_over_ranks(e2e_local, world)
    cnt = layer.counts.cpu().numpy()
    stages = dict(zip(["gate", "dispatch", "expert_ffn", "combine"], [float(v) for v in stage_ms.mean(axis=0)]))
    roofline = ffn_roofline(cfg, cnt, stages["expert_ffn"], fp4, peaks, peak_src)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based generator)",
            "config": config, "clocks": clocks,
            "e2e": {"value": world * cfg.T / (e2e_ms * 1e-3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": layer.kernels_per_step() * args.steps, "stage_ms": stages,
            "wall_ms_timed_region": wall_ms, "roofline": roofline, "routing": routing_stats(cnt, cfg.T, cfg.topk)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp4:
        dt, n, ne = oracle_sample(layer.li, cfg, args.cpu_tokens, seed=12345, table=layer.table)
        line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"{n} seeded tokens of the workload ({ne} experts incl. shared), "
                                          f"numpy fp64 oracle, {dt:.1f} s"}
    layer.release()

    # ---------------- the other synthetic layers, each timed the same way ----------------
    if not args.only:
        others = {}
        for name in WORKLOADS:
            if name == cfg.name:
                continue
            c = W.CONFIGS[name]
            lay = Layer(c, dev, fp4, args.fused_gather)
            ms_l, st_ms, clk, _ = lay.time_steps(args.steps, args.warmup, world, clocks=True)
            ms = max_over_ranks(ms_l, world)
            cn = lay.counts.cpu().numpy()
            st = dict(zip(["gate", "dispatch", "expert_ffn", "combine"], [float(v) for v in st_ms.mean(axis=0)]))
            others[name] = {"value": world * c.T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
                            "steps": args.steps, "warmup": args.warmup, "config": config_of(c, world, fp4),
                            "clocks": clk, "stage_ms": st, "gpu_launches": lay.kernels_per_step() * args.steps,
                            "roofline": ffn_roofline(c, cn, st["expert_ffn"], fp4, peaks, peak_src),
                            "routing": routing_stats(cn, c.T, c.topk)}
            lay.release()
        if not fp4:
            for name in MXFP4_WORKLOADS:
                c = W.CONFIGS[name]
                lay = Layer(c, dev, True, False)
                ms_l, st_ms, clk, _ = lay.time_steps(args.steps, args.warmup, world, clocks=True)
                ms = max_over_ranks(ms_l, world)
                cn = lay.counts.cpu().numpy()
                st = dict(zip(["gate", "dispatch", "expert_ffn", "combine"], [float(v) for v in st_ms.mean(axis=0)]))
                others[name + "_mxfp4"] = {
                    "value": world * c.T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps,
                    "warmup": args.warmup, "config": config_of(c, world, True), "clocks": clk, "stage_ms": st,
                    "gpu_launches": lay.kernels_per_step() * args.steps,
                    "roofline": ffn_roofline(c, cn, st["expert_ffn"], True, peaks, peak_src)}
                lay.release()
        line["workloads"] = others
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
