"""Benchmark of the NVFP4 MoE hot path on B200.

One step of an MoE workload = one MoE FFN layer over one batch of synthetic
tokens, every stage in this library's kernels: quantize(x) -> moe_permute ->
gate/up grouped GEMM + SwiGLU -> quantize(h) -> down grouped GEMM ->
moe_unpermute_combine (the sequence moe_layer_nvfp4 runs; each MoE workload
also times the down GEMM with the combine fused into its epilogue, same box,
as an A/B). One step of the dense workload = quantize(A) + one
8192^3 NVFP4 GEMM; of the tiny workload = quantize(A) + the 4 x 16-row grouped
GEMM (K = N = 256).

A default run times all five workloads in one process and prints ONE JSON line:
the headline is the 512-token decode layer (hidden 6144, intermediate 2048,
256 experts, top-8, ~16 rows per expert); the line's `configs` object holds the
same measurement for every workload (decode, Zipf decode at 1024 tokens, prefill
at 8192 tokens, dense 8192^3, tiny). Metric: grouped-GEMM TFLOP/s of the step
(the GEMMs' FLOPs over the step's device time), with the step's algorithmic HBM
GB/s alongside. The MoE workloads stream all 5.4 GB of expert weights every
step (far above the 126 MB L2); the dense and tiny workloads flush L2 between
steps (a 256 MB write outside the timed events).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

--config NAME times that workload alone (it becomes the headline). With N > 1
(torchrun, one process per GPU) every rank runs an independent replica (its
own token batch, the same weights): the layer shards over batches with no
data-path collective, so scaling is weak. Timing: barrier + device synchronise
on both sides of each timed region, CUDA events on the launching stream, the
max over ranks.

--impl reference times the CPU oracle (the plain FP64 implementation used as
the parity reference) on this host's cores, on a bounded sample of the
headline workload; it is a slow baseline, not a target.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PAGES_DECODE_TFLOPS = 0.8   # per-expert FP4 grouped GEMM at ~16 tokens/expert, RTX PRO 6000 (context)
METRIC = "NVFP4 MoE grouped-GEMM TFLOPS and HBM GB/s at 16-256 tokens/expert"
HEADLINE = "moe_decode_t512"
ORDER = ("moe_decode_t512", "moe_zipf_t1024", "moe_prefill_t8192", "dense", "tiny")
DTYPE = "nvfp4 (e2m1 x e2m1, fp32 accumulate)"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=None, choices=list(workloads.CONFIGS),
                    help="time this workload alone (default: all five, decode as the headline)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="CPU seconds per reference-arm step (default: 120 s spread over warm-up + steps, at most 30)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # size overrides, used to make small cases of a workload for profiler captures
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--experts", type=int, default=None)
    return ap.parse_args(argv)


def ref_budget(args) -> float:
    if args.ref_seconds is not None:
        return max(0.05, float(args.ref_seconds))
    return min(30.0, max(1.0, 120.0 / max(1, args.steps + args.warmup)))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


FP4_PER_BF16 = 4.0  # nominal dense ratio (9 PF FP4 / 2.25 PF BF16)

# kernel sources a committed ncu traffic figure belongs to (the summary names them; default: all GEMM sources)
GEMM_SOURCES = ("nvfp4_block_scaled_09_b200/csrc/grouped_gemm.cu", "nvfp4_block_scaled_09_b200/csrc/grouped_gemm_pair.cu",
                "nvfp4_block_scaled_09_b200/csrc/common.cuh")


def replica_seed(seed: int, rank: int) -> int:
    """Each rank is an independent replica: its own token batch and routing (weights are shared)."""
    return int(seed) + 7919 * int(rank)


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a per-rank measurement over all ranks (the bench's timing rule); identity at world 1."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gemm_source_sha256(sources=GEMM_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(config: str, key: str = "gate_up_dram_bytes_per_launch"):
    """DRAM bytes per launch of the dominant GEMM from the committed ncu summary of this workload
    (profiles/traffic_<config>.md), or None when there is none or the kernel sources it names changed
    since it was taken."""
    path = os.path.join(ROOT, "profiles", f"traffic_{config}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    sources = tuple(x.strip().strip("`") for x in fields.get("sources", "").split(",") if x.strip()) or GEMM_SOURCES
    if fields.get("source_sha256") != gemm_source_sha256(sources):
        return None
    try:   # the dominant GEMM launch: the gate/up GEMM of a layer, the GEMM of the dense and tiny workloads
        return int(fields.get(key) or fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ----------------------------------------------------------------------------- work accounting

def moe_counts(cfg, ids):
    return np.bincount(ids.ravel(), minlength=cfg["E"])


def moe_flops(cfg):
    T, k, H, I = cfg["T"], cfg["k"], cfg["H"], cfg["I"]
    R = T * k
    return 2.0 * R * (2 * I) * H, 2.0 * R * H * I


def moe_gemm_bytes(cfg, counts):
    """Algorithmic HBM bytes of each GEMM launch: active experts' weights + scales once, activations
    and their scales once, BF16 output once."""
    T, k, H, I = cfg["T"], cfg["k"], cfg["H"], cfg["I"]
    R = T * k
    active = int(np.sum(counts > 0))
    g1 = active * (2 * I) * (H // 2 + H // 16) + R * (H // 2 + H // 16) + R * I * 2
    g2 = active * H * (I // 2 + I // 16) + R * (I // 2 + I // 16) + R * H * 2
    return g1, g2


def moe_step_bytes(cfg, counts):
    T, k, H, I = cfg["T"], cfg["k"], cfg["H"], cfg["I"]
    R = T * k
    g1, g2 = moe_gemm_bytes(cfg, counts)
    qx = T * H * 2 * 2 + T * (H // 2 + H // 16)                 # amax read + quantize read, codes+scales write
    perm = R * (H // 2 + H // 16) * 2 + T * k * 4 * 3
    qh = R * I * 2 * 2 + R * (I // 2 + I // 16)
    comb = R * H * 2 + T * H * 2 + T * k * 8
    return g1 + g2 + qx + perm + qh + comb


def gemm_bytes(M, N, K, E=1):
    """Algorithmic bytes of one GEMM launch: both operands' codes + scales once, the BF16 output once."""
    return E * N * (K // 2 + K // 16) + M * (K // 2 + K // 16) + M * N * 2


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.4)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "power_w_max": max(power) if power else None}


def start_clocks(rank, local_rank):
    if rank != 0:
        return None
    c = ClockSampler(local_rank)
    c.start()
    return c


# ----------------------------------------------------------------------------- config descriptions
# One function per workload kind builds the `config` object; the reference arm prints the same one.

def resized_cfg(name, args):
    cfg = dict(workloads.CONFIGS[name])
    if args.tokens:
        cfg["T"] = args.tokens
    if args.experts:
        cfg["E"] = args.experts
    return cfg


def moe_routing(cfg, seed):
    return workloads.routing(cfg["T"], cfg["E"], cfg["k"], cfg["routing"], seed, cfg.get("zipf_s", 1.1),
                             cfg.get("zero_experts", 0))


def parallelism(world):
    return f"replicas x{world} (no data-path collective)" if world > 1 else "single GPU"


def moe_weight_bytes(cfg):
    """Packed FP4 codes and E4M3 scales of every expert's gate/up [2I, H] and down [H, I] weights."""
    H, I = cfg["H"], cfg["I"]
    return cfg["E"] * (2 * I * (H // 2 + H // 16) + H * (I // 2 + I // 16))


def moe_config_dict(name, cfg, counts, world, resized=False):
    return {"workload": name if not resized else f"{name} resized to T={cfg['T']} E={cfg['E']}",
            "tokens": cfg["T"], "hidden": cfg["H"], "intermediate": cfg["I"], "experts": cfg["E"],
            "top_k": cfg["k"], "routing": cfg["routing"],
            "rows_per_expert": {"min": int(counts.min()), "mean": float(counts.mean()), "max": int(counts.max()),
                                "empty": int(np.sum(counts == 0))},
            "l2": f"no flush: every step streams all expert weights ({moe_weight_bytes(cfg) / 1e9:.1f} GB) through HBM, "
                  "far above L2",
            "parallelism": parallelism(world)}


def dense_config_dict(cfg, world):
    return {"workload": "dense", "M": cfg["M"], "N": cfg["N"], "K": cfg["K"],
            "l2": "flushed between steps (256 MB write, outside the timed events)",
            "step": "quantize(A) + GEMM with B quantised once beforehand", "parallelism": parallelism(world)}


def tiny_config_dict(cfg, world):
    E, r = cfg["E"], cfg["rows_per_expert"]
    return {"workload": "tiny", "experts": E, "rows_per_expert": r, "N": cfg["N"], "K": cfg["K"],
            "epilogue": "none", "l2": "flushed between steps (256 MB write, outside the timed events)",
            "step": "quantize(A) + grouped GEMM with the weights quantised once beforehand",
            "parallelism": parallelism(world)}


def config_dict(name, cfg, world, seed=0, resized=False):
    if cfg["kind"] == "moe":
        ids, _ = moe_routing(cfg, seed)
        return moe_config_dict(name, cfg, moe_counts(cfg, ids), world, resized)
    if cfg["kind"] == "dense":
        return dense_config_dict(cfg, world)
    return tiny_config_dict(cfg, world)


# ----------------------------------------------------------------------------- our implementation: MoE

def build_moe_weights(nv, torch, cfg, seed, dev):
    """Random N(0, 0.02) expert weights of the layer, quantised and packed once (not timed)."""
    E, H, I = cfg["E"], cfg["H"], cfg["I"]

    def build(N, K, tag):
        packed = torch.empty((E, N * (K // 2 + K // 16)), dtype=torch.uint8, device=dev)
        g = torch.empty(E, dtype=torch.float32, device=dev)
        q = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        sf = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
        ws = torch.empty(max(nv.quantize_workspace_size(N, K), 16), dtype=torch.uint8, device=dev)
        for e in range(E):
            w = workloads.normal_bf16((N, K), 0.02, seed, tag, e, device=dev)
            nv.quantize(w, q=q, sf=sf, g=g[e:e + 1], ws=ws)
            nv.pack_weights(q, sf, out=packed[e])
        return nv.PackedWeights(packed, g, E, N, K)

    w13 = build(2 * I, H, workloads.TAG_W13)
    w2 = build(H, I, workloads.TAG_W2)
    torch.cuda.synchronize()
    return nv.MoEWeights(w13, w2)


class MoEBench:
    def __init__(self, cfg, seed, rank, device, weights):
        import torch
        import nvfp4_block_scaled_09_b200 as nv
        self.nv, self.torch = nv, torch
        self.cfg = cfg
        T, k, H, I, E = cfg["T"], cfg["k"], cfg["H"], cfg["I"], cfg["E"]
        self.dev = device
        # Each rank is a replica: its own tokens and routing, the same weights.
        ids, w = moe_routing(cfg, replica_seed(seed, rank))
        self.ids_np, self.w_np = ids, w
        self.counts = moe_counts(cfg, ids)
        self.x = workloads.normal_bf16((T, H), 1.0, replica_seed(seed, rank), workloads.TAG_X, device=device)
        self.ids = torch.from_numpy(ids).to(device)
        self.w = torch.from_numpy(w).to(device)
        self.weights = weights
        self.ws = nv.layer_workspace(T, k, E, H, I, device)
        self.lay = nv.layer_workspace_layout(T, k, E, H, I)
        self.l2_hints = nv.layer_l2_prefetch_bytes(T, k, E, H, I)
        # amax_h and the fused combine's counters: zeroed together at the start of every layer
        self.zeroed = self.ws[self.lay["amax_h"]: self.lay["fin_counters"] + nv.lib().moe_finalize_counters_size(T, H)]
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        self.qp_ws = torch.empty(max(nv.lib().moe_quantize_permute_workspace_size(T, k, E, H), 16), dtype=torch.uint8,
                                 device=device)

    def step(self, ev=None, gemm_ev=None, fused=False):
        """One layer through the C ABI, stage by stage (the same sequence moe_layer_nvfp4 runs), with
        optional CUDA events between all stages (ev) or around the gate/up GEMM only (gemm_ev). fused=True
        runs the down GEMM with the combine fused into its epilogue instead of the down GEMM and
        moe_unpermute_combine as two launches (the layer's path)."""
        import ctypes
        nv = self.nv
        L = nv.lib()
        c = self.cfg
        T, k, H, I, E = c["T"], c["k"], c["H"], c["I"], c["E"]
        R = T * k
        b = self.ws.data_ptr()
        lay = self.lay
        P = ctypes.c_void_p
        s = P(self.torch.cuda.current_stream().cuda_stream)
        W = self.weights
        scratch, sbytes = P(b + lay["scratch"]), lay["topk_ids"] - lay["scratch"]

        def rec(i):
            if ev is not None:
                ev[i].record()

        self.zeroed.zero_()    # as moe_layer_nvfp4's one memset
        rec(0)
        # x quantised into expert order (moe_layer_nvfp4 runs the same kernels on its own workspace)
        pf13, pf2 = self.l2_hints   # the L2 prefetch hints moe_layer_nvfp4 gives (decode-sized batches)
        st = L.moe_quantize_permute_prefetch(P(self.x.data_ptr()), T, H, P(self.ids.data_ptr()), k, E,
                                             P(b + lay["q_perm"]), P(b + lay["sf_perm"]), nv.SF_KSTAGE,
                                             P(b + lay["g_x"]), P(b + lay["offsets"]), P(b + lay["perm_src"]),
                                             P(b + lay["inv_perm"]), P(self.qp_ws.data_ptr()), self.qp_ws.numel(),
                                             P(W.w13.packed.data_ptr()), pf13, s)
        rec(1)
        if gemm_ev is not None:
            gemm_ev[0].record()
        st |= L.moe_grouped_gemm_nvfp4_amax(P(b + lay["q_perm"]), P(b + lay["sf_perm"]), P(b + lay["g_x"]),
                                            P(W.w13.packed.data_ptr()), P(W.w13.gscale.data_ptr()),
                                            P(b + lay["offsets"]), E, R, 2 * I, H, 1, P(b + lay["h"]),
                                            P(b + lay["amax_h"]), s)
        if gemm_ev is not None:
            gemm_ev[1].record()
        rec(2)
        st |= L.nvfp4_quantize_from_amax_prefetch(P(b + lay["h"]), R, I, P(b + lay["amax_h"]), P(b + lay["q_h"]),
                                                  P(b + lay["sf_h"]), P(b + lay["g_h"]), nv.SF_KSTAGE,
                                                  P(W.w2.packed.data_ptr()), pf2, s)
        rec(3)
        if fused:
            st |= L.moe_grouped_gemm_nvfp4_finalize(P(b + lay["q_h"]), P(b + lay["sf_h"]), P(b + lay["g_h"]),
                                                    P(W.w2.packed.data_ptr()), P(W.w2.gscale.data_ptr()),
                                                    P(b + lay["offsets"]), E, R, H, I, P(b + lay["y"]),
                                                    P(b + lay["perm_src"]), P(b + lay["inv_perm"]),
                                                    P(self.w.data_ptr()), T, k, P(b + lay["fin_counters"]),
                                                    P(self.out.data_ptr()), s)
            rec(4)
        else:
            st |= L.moe_grouped_gemm_nvfp4(P(b + lay["q_h"]), P(b + lay["sf_h"]), P(b + lay["g_h"]),
                                           P(W.w2.packed.data_ptr()), P(W.w2.gscale.data_ptr()),
                                           P(b + lay["offsets"]), E, R, H, I, 0, P(b + lay["y"]), s)
            rec(4)
            st |= L.moe_unpermute_combine(P(b + lay["y"]), P(b + lay["inv_perm"]), P(self.w.data_ptr()), T, k, H,
                                          P(self.out.data_ptr()), s)
        rec(5)
        if st != 0:
            raise RuntimeError(f"library call failed (status bits {st})")

    def layer_call(self, x, ids, w, out):
        """The public one-call API."""
        return self.nv.moe_layer(x, ids, w, self.weights, ws=self.ws, out=out)


def barrier(world):
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()


def run_moe(args, name, cfg, weights, rank, world, local_rank, dev, peaks, resized=False):
    """Time one MoE workload; returns its summary (the `configs` entry)."""
    import torch
    import nvfp4_block_scaled_09_b200 as nv
    bench = MoEBench(cfg, args.seed, rank, dev, weights)
    K, W = args.steps, args.warmup
    for _ in range(W):
        bench.step()
    torch.cuda.synchronize()
    st = nv.device_status()
    if st != 0:
        raise RuntimeError(f"{name}: device status {nv.status_string(st)} after warm-up")

    clocks = start_clocks(rank, local_rank)
    barrier(world)
    launches0 = nv.launch_count()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    # the dominant kernel (gate/up GEMM) is bracketed by events inside the timed region; events between
    # the other stages would serialise their programmatic launches, so those are timed in a later pass
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    start.record()
    for i in range(K):
        bench.step(gemm_ev=gev[i])
    stop.record()
    barrier(world)
    launches = nv.launch_count() - launches0
    clk = clocks.stop() if clocks else None
    max_ms = max_over_ranks(start.elapsed_time(stop), world, dev)
    gemm1_ms = float(np.mean([g[0].elapsed_time(g[1]) for g in gev]))
    # per-stage breakdown in a separate, untimed pass: events between stages serialise the kernels
    # that otherwise overlap their launch with the previous kernel's tail
    nev = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(K)]
    for i in range(K):
        bench.step(evs[i])
    barrier(world)
    stage_ms = np.zeros(nev - 1)
    for i in range(K):
        for j in range(nev - 1):
            stage_ms[j] += evs[i][j].elapsed_time(evs[i][j + 1])
    stage_ms /= K
    st = nv.device_status()
    if st != 0:
        raise RuntimeError(f"{name}: device status {nv.status_string(st)} after the timed region")
    # same-box A/B of the combine: the layer with the down GEMM's fused combine instead of the separate kernel
    for _ in range(W):
        bench.step(fused=True)
    barrier(world)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for i in range(K):
        bench.step(fused=True)
    a1.record()
    barrier(world)
    fused_ms = max_over_ranks(a0.elapsed_time(a1), world, dev) / K
    st = nv.device_status()
    if st != 0:
        raise RuntimeError(f"{name}: device status {nv.status_string(st)} after the separate-combine pass")

    e2e = None if args.no_e2e else run_moe_e2e(bench, cfg, K, W, world, dev)

    f1, f2 = moe_flops(cfg)
    g1b, g2b = moe_gemm_bytes(cfg, bench.counts)
    step_bytes = moe_step_bytes(cfg, bench.counts)
    step_s = max_ms / K * 1e-3
    value = world * (f1 + f2) / step_s / 1e12
    gemm1_s = gemm1_ms * 1e-3
    gemm2_s = stage_ms[3] * 1e-3
    fp4_peak = peaks["bf16_tflops_sustained"] * FP4_PER_BF16
    # the roof a kernel sits under is set by its arithmetic intensity against the ridge point
    tensor_bound = f1 / g1b >= fp4_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    rows_mean = float(bench.counts.mean())
    plan = nv.gemm_plan()
    shape = ("CTA-pair" if rows_mean >= plan["pair_min_avg_rows"] else
             "wide" if rows_mean >= plan["wide_min_avg_rows"] else "narrow")
    tflops1 = f1 / gemm1_s / 1e12
    # bytes of each GEMM's weights the kernel before it pulled into L2 (the layer's prefetch hints): the GEMM's
    # own HBM stream is the algorithmic bytes less those
    pf1, pf2 = bench.l2_hints
    roof = ({"bound": "tensor", "achieved": tflops1, "peak": fp4_peak, "unit": "TFLOP/s", "frac": tflops1 / fp4_peak,
             "algorithmic_flops": f1} if tensor_bound else
            {"bound": "hbm", "achieved": (g1b - pf1) / gemm1_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": (g1b - pf1) / gemm1_s / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes": g1b})
    roof["l2_prefetch_bytes"] = pf1
    if pf1:
        roof["bytes_note"] = ("achieved counts algorithmic_bytes less l2_prefetch_bytes: the first weight tiles "
                              "were pulled into L2 by the kernel before this one")
    roof |= {"traffic": measured_traffic(name if not resized else "", "gate_up_dram_bytes_per_launch"),
             "kernel": f"grouped GEMM gate/up + SwiGLU ({shape} tiles)",
             "peak_source": f"{peaks['source']} ({'HBM copy' if not tensor_bound else 'sustained bf16 x 4'})",
             "avg_launch_ms": gemm1_ms, "timing": "CUDA events around this kernel inside the timed region",
             "tensor_frac": tflops1 / fp4_peak, "tensor_achieved_tflops": tflops1,
             "tensor_peak_tflops": fp4_peak}
    del bench
    torch.cuda.empty_cache()
    return {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "ms_per_step": max_ms / K,
        "config": moe_config_dict(name, cfg, moe_counts(cfg, moe_routing(cfg, replica_seed(args.seed, 0))[0]),
                                  world, resized),
        "hbm_gbs": world * step_bytes / step_s / 1e9,
        "stage_ms": {"quantize_permute_x": stage_ms[0], "gemm_gate_up": stage_ms[1],
                     "quantize_h": stage_ms[2], "gemm_down": stage_ms[3], "combine": stage_ms[4]},
        "stage_ms_note": "separate pass after the timed region, events between every stage",
        "combine_ab": {"separate_ms_per_step": max_ms / K, "fused_ms_per_step": fused_ms,
                       "note": "same box, same inputs: the down GEMM followed by moe_unpermute_combine (the "
                               "layer's path) against the down GEMM with the combine fused into its epilogue"},
        "roofline": roof,
        "roofline_down": {"bound": "hbm", "achieved": (g2b - pf2) / gemm2_s / 1e9, "peak": peaks["hbm_gbs"],
                          "unit": "GB/s", "frac": (g2b - pf2) / gemm2_s / 1e9 / peaks["hbm_gbs"],
                          "algorithmic_bytes": g2b, "l2_prefetch_bytes": pf2, "kernel": "grouped GEMM down",
                          "avg_launch_ms": stage_ms[3], "tensor_frac": f2 / gemm2_s / 1e12 / fp4_peak,
                          "traffic": measured_traffic(name if not resized else "", "down_dram_bytes_per_launch")},
        "clocks": clk, "gpu_launches": int(launches), "e2e": e2e,
    }


def run_moe_e2e(bench, cfg, K, W, world, dev):
    """End to end through the public one-call API, host buffers in pinned memory: every step copies its
    inputs host -> device and its output device -> host inside the timed region. Steps are pipelined the
    way a serving loop would run them: inputs and outputs are double-buffered, the uploads run on one copy
    stream and the downloads on another while the layer runs on the compute stream."""
    import torch
    x_h = bench.x.cpu().pin_memory()
    ids_h = bench.ids.cpu().pin_memory()
    w_h = bench.w.cpu().pin_memory()
    out_h = [torch.empty(bench.out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xs = [torch.empty_like(bench.x) for _ in range(2)]
    idss = [torch.empty_like(bench.ids) for _ in range(2)]
    wts = [torch.empty_like(bench.w) for _ in range(2)]
    outs = [torch.empty_like(bench.out) for _ in range(2)]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])        # the layer of step i-2 has read these inputs
            xs[b].copy_(x_h, non_blocking=True)
            idss[b].copy_(ids_h, non_blocking=True)
            wts[b].copy_(w_h, non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])             # step i-2's output has left this buffer
        bench.layer_call(xs[b], idss[b], wts[b], outs[b])
        ev_comp[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            out_h[b].copy_(outs[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(W):
        e2e_step(i)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(K):
        e2e_step(i)
    e1.record(s_out)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    f1, f2 = moe_flops(cfg)
    return {"value": world * (f1 + f2) * K / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(x_h.numel() * 2 + ids_h.numel() * 4 + w_h.numel() * 4),
            "d2h_bytes_per_step": int(out_h[0].numel() * 2), "api": "moe_layer_nvfp4",
            "ms_per_step": e2e_ms / K,
            "pipelining": "double-buffered inputs/outputs; uploads and downloads on two copy streams"}


# ----------------------------------------------------------------------------- our implementation: GEMMs

def run_gemm_workload(args, name, cfg, rank, world, local_rank, dev, peaks):
    """The dense 8192^3 GEMM or the tiny grouped GEMM: quantize(A) + GEMM per step, L2 flushed between steps
    outside the events. Returns the `configs` entry."""
    import torch
    import nvfp4_block_scaled_09_b200 as nv
    seed = replica_seed(args.seed, rank)
    if cfg["kind"] == "dense":
        M, N, K, E = cfg["M"], cfg["N"], cfg["K"], 1
        a = workloads.normal_bf16((M, K), 1.0, seed, workloads.TAG_A, device=dev)
        b = workloads.normal_bf16((1, N, K), 0.02, args.seed, workloads.TAG_B, device=dev)
        off = torch.tensor([0, M], dtype=torch.int32, device=dev)
        desc = dense_config_dict(cfg, world)
        kernel = "grouped GEMM, E=1 (CTA-pair tiles)"
    else:
        E, rpe, N, K = cfg["E"], cfg["rows_per_expert"], cfg["N"], cfg["K"]
        M = E * rpe
        a = workloads.normal_bf16((M, K), 1.0, seed, workloads.TAG_A, device=dev)
        b = workloads.normal_bf16((E, N, K), 0.02, args.seed, workloads.TAG_B, device=dev)
        off = torch.arange(0, M + 1, rpe, dtype=torch.int32, device=dev)
        desc = tiny_config_dict(cfg, world)
        kernel = "grouped GEMM, 4 experts x 16 rows (narrow tiles)"
    pw = nv.prepare_expert_weights(b)
    del b
    a_q = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    a_sf = torch.empty((K // 256, M, 16), dtype=torch.uint8, device=dev)   # K-stage slabs (the GEMM's layout)
    a_g = torch.empty(1, dtype=torch.float32, device=dev)
    qws = torch.empty(max(nv.quantize_workspace_size(M, K), 16), dtype=torch.uint8, device=dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # larger than the 126 MB L2

    def step(e0=None, e1=None, e2=None):
        if e0 is not None:
            e0.record()
        nv.quantize(a, q=a_q, sf=a_sf, g=a_g, ws=qws, layout=nv.SF_KSTAGE)
        if e1 is not None:
            e1.record()
        nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False, out=c)
        if e2 is not None:
            e2.record()

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    st = nv.device_status()
    if st != 0:
        raise RuntimeError(f"{name}: device status {nv.status_string(st)} after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = start_clocks(rank, local_rank)
    barrier(world)
    l0 = nv.launch_count()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)                      # evict A, B and C from L2 between steps (not timed)
        step(*evs[i])
    barrier(world)
    launches = nv.launch_count() - l0
    clk = clocks.stop() if clocks else None
    step_ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    gemm_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    max_step_ms = max_over_ranks(step_ms, world, dev)
    st = nv.device_status()
    if st != 0:
        raise RuntimeError(f"{name}: device status {nv.status_string(st)} after the timed region")
    flops = 2.0 * M * N * K
    value = world * flops * args.steps / (max_step_ms * 1e-3) / 1e12
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16      # burst: a kernel timed in isolation
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    nbytes = gemm_bytes(M, N, K, E)
    del a, pw, a_q, a_sf, c, flush, qws
    torch.cuda.empty_cache()
    return {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "ms_per_step": max_step_ms / args.steps,
        "config": desc,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp4_peak, "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
                     "hbm_frac": nbytes / (gemm_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "traffic": measured_traffic(name, "dram_bytes_per_launch"), "kernel": kernel,
                     "peak_source": peaks["source"] + " bf16 x 4 (nominal FP4/BF16 ratio), burst",
                     "avg_launch_ms": gemm_ms,
                     "timing": "CUDA events around this kernel, L2 flushed between steps outside the events"},
        "clocks": clk, "gpu_launches": int(launches), "e2e": None,
    }


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(cfg, seed, budget_s=10.0):
    """Run the oracle's layer on a bounded sample: quantize + permute over the whole batch, then the two
    GEMMs (and h quantisation) for as many experts' rows as fit the time budget, then the combine.
    Returns (sampled grouped-GEMM FLOPs, seconds, description)."""
    import oracle
    T, k, H, I, E = cfg["T"], cfg["k"], cfg["H"], cfg["I"], cfg["E"]
    ids, w = moe_routing(cfg, seed)
    x = workloads.random_bf16_bits((T, H), seed=seed, tag=workloads.TAG_X)
    rng = np.random.default_rng(seed)
    # one expert's worth of random quantised weights, reused for every sampled expert (drawn untimed)
    w13_q = rng.integers(0, 256, size=(1, 2 * I, H // 2), dtype=np.uint8)
    w13_sf = rng.integers(0x20, 0x40, size=(1, 2 * I, H // 16), dtype=np.uint8)
    w2_q = rng.integers(0, 256, size=(1, H, I // 2), dtype=np.uint8)
    w2_sf = rng.integers(0x20, 0x40, size=(1, H, I // 16), dtype=np.uint8)
    one = np.ones(1, np.float32)
    y = workloads.random_bf16_bits((T * k, H), seed=seed + 1)
    t0 = time.perf_counter()
    q, sf, g = oracle.quantize(x)
    off, src, inv = oracle.permute(ids, E)
    q_perm, sf_perm = oracle.gather_rows(q, src), oracle.gather_rows(sf, src)
    flops = 0.0
    n_exp = 0
    counts = np.diff(off)
    for e in range(E):
        if counts[e] == 0:
            continue
        r0, r1 = int(off[e]), int(off[e + 1])
        M = r1 - r0
        sub = np.array([0, M], np.int32)
        hf = oracle.grouped_gemm(q_perm[r0:r1], sf_perm[r0:r1], g, w13_q, w13_sf, one, sub, 2 * I, H, True)
        hb = oracle.bf16_round(hf)
        hq, hsf, hg = oracle.quantize(hb)
        oracle.grouped_gemm(hq, hsf, hg, w2_q, w2_sf, one, sub, H, I, False)
        flops += 2.0 * M * 2 * I * H + 2.0 * M * H * I
        n_exp += 1
        if time.perf_counter() - t0 > budget_s:
            break
    oracle.combine(y, inv, w)
    dt = time.perf_counter() - t0
    desc = (f"oracle layer on {cfg['T']} tokens: quantize+permute+combine of the whole batch, both GEMMs for "
            f"the rows of {n_exp} of {int(np.sum(counts > 0))} active experts (FP64, {oracle.num_threads()} threads)")
    return flops, dt, desc, n_exp


def oracle_gemm_sample(M, N, K, E, seed, budget_s):
    """Oracle GEMM on a bounded sample of rows of a [M, K] x [E experts of N, K] problem (quantise the sampled
    activation rows + their GEMM against one expert), repeated until the budget is spent."""
    import oracle
    rng = np.random.default_rng(seed)
    w_q = rng.integers(0, 256, size=(1, N, K // 2), dtype=np.uint8)
    w_sf = rng.integers(0x20, 0x40, size=(1, N, K // 16), dtype=np.uint8)
    rows_per_call = min(8, M)
    t0 = time.perf_counter()
    rows = 0
    flops = 0.0
    while time.perf_counter() - t0 < budget_s:
        a = workloads.random_bf16_bits((rows_per_call, K), seed=seed + rows, tag=workloads.TAG_A)
        aq, asf, ag = oracle.quantize(a)
        oracle.grouped_gemm(aq, asf, ag, w_q, w_sf, np.ones(1, np.float32), np.array([0, rows_per_call], np.int32),
                            N, K, False)
        rows += rows_per_call
        flops += 2.0 * rows_per_call * N * K
    dt = time.perf_counter() - t0
    return flops, dt, f"oracle GEMM on {rows} activation rows of [{M} x {K}] x [{N} x {K}] (FP64, " \
                      f"{oracle.num_threads()} threads)"


def cpu_baseline(name, cfg, seed, budget_s, threads=None):
    """The oracle timed on this host's cores on a bounded sample of the workload (`threads`: 1 for the
    single-thread figure, None for every core the process may use)."""
    import oracle
    before = oracle.num_threads()
    if threads is not None:
        oracle.set_num_threads(threads)
    try:
        if cfg["kind"] == "moe":
            f, dt, desc, _ = oracle_sample(cfg, seed, budget_s)
        elif cfg["kind"] == "dense":
            f, dt, desc = oracle_gemm_sample(cfg["M"], cfg["N"], cfg["K"], 1, seed, budget_s)
        else:
            f, dt, desc = oracle_gemm_sample(cfg["E"] * cfg["rows_per_expert"], cfg["N"], cfg["K"], cfg["E"], seed,
                                             budget_s)
        cores = oracle.num_threads()
    finally:
        oracle.set_num_threads(before)
    return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
            "seconds": dt, "cpu_model": cpu_model()}


def cpu_baselines(names, cfgs, seed):
    """Per workload: the oracle on every core (bounded), plus a single-thread figure for tiny and decode."""
    out = {}
    for n in names:
        budget = 10.0 if n == HEADLINE else 3.0
        cb = cpu_baseline(n, cfgs[n], seed, budget)
        if n in ("tiny", HEADLINE):
            one = cpu_baseline(n, cfgs[n], seed, 4.0 if n == HEADLINE else 1.0, threads=1)
            cb["value_1thread"] = one["value"]
            cb["sample_1thread"] = one["sample"]
        out[n] = cb
    return out


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, name, cfg, world):
    """The oracle as it stands, timed on the host's cores on a bounded sample of the workload per step."""
    import oracle
    K, W = args.steps, args.warmup
    budget = ref_budget(args)
    tot_f = tot_t = 0.0
    desc = ""
    for i in range(W + K):
        if cfg["kind"] == "moe":
            f, dt, desc, _ = oracle_sample(cfg, args.seed, budget_s=budget)
        elif cfg["kind"] == "dense":
            f, dt, desc = oracle_gemm_sample(cfg["M"], cfg["N"], cfg["K"], 1, args.seed, budget)
        else:
            f, dt, desc = oracle_gemm_sample(cfg["E"] * cfg["rows_per_expert"], cfg["N"], cfg["K"], cfg["E"],
                                             args.seed, budget)
        if i >= W:
            tot_f += f
            tot_t += dt
    v = tot_f / tot_t / 1e12
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": K, "warmup": W, "ms_per_step": tot_t / K * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(name, cfg, world, args.seed, bool(args.tokens or args.experts)),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": desc, "cpu_model": cpu_model()},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main

def main(argv=None):
    args = parse(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    names = [args.config] if args.config else list(ORDER)
    headline = names[0]
    resized = bool(args.tokens or args.experts)
    cfgs = {n: (resized_cfg(n, args) if n == args.config else dict(workloads.CONFIGS[n])) for n in names}

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, headline, cfgs[headline], world)))
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        # a short bound on every collective: a rank that stops ends the others' next barrier with an error
        dist.init_process_group("nccl", device_id=torch.device("cuda", local_rank),
                                timeout=datetime.timedelta(seconds=300))
    from nvfp4_block_scaled_09_b200 import build as nvbuild
    nvbuild.build()
    import nvfp4_block_scaled_09_b200 as nv
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()

    results = {}
    moe_names = [n for n in names if cfgs[n]["kind"] == "moe"]
    if moe_names:
        # the three MoE workloads share one layer shape, hence one set of weights
        weights = build_moe_weights(nv, torch, cfgs[moe_names[0]], args.seed, dev)
        for n in moe_names:
            results[n] = run_moe(args, n, cfgs[n], weights, rank, world, local_rank, dev, peaks,
                                 resized and n == args.config)
        del weights
        torch.cuda.empty_cache()
    for n in names:
        if cfgs[n]["kind"] != "moe":
            results[n] = run_gemm_workload(args, n, cfgs[n], rank, world, local_rank, dev, peaks)

    cbs = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cbs = cpu_baselines(names, cfgs, args.seed)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    for n in names:
        results[n]["cpu_baseline"] = cbs[n] if cbs else None
    top = results[headline]
    line = {
        "metric": METRIC,
        "value": top["value"],
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": top["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": (top["value"] / PAGES_DECODE_TFLOPS if headline == HEADLINE and not resized else None),
        "dtype": DTYPE,
        "data": "synthetic",
    }
    line |= {k: v for k, v in top.items() if k not in ("metric", "value", "unit", "ms_per_step")}
    if line["vs_baseline"] is not None:
        line["vs_baseline_basis"] = ("0.8 TFLOPS: per-expert FP4 grouped GEMM at ~16 tokens/expert on RTX PRO "
                                     "6000 (SM120), quoted by the pages as context")
    if len(names) > 1:
        line["configs"] = results
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
