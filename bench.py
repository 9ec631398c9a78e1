"""Benchmark of the NVFP4 MoE hot path on B200.

One step = one MoE FFN layer over one batch of synthetic tokens, every stage in
this library's kernels: quantize(x) -> moe_permute -> gate/up grouped GEMM +
SwiGLU -> quantize(h) -> down grouped GEMM -> moe_unpermute_combine.

Default workload: the 512-token decode layer (hidden 6144, intermediate 2048,
256 experts, top-8, ~16 rows per expert). Metric: grouped-GEMM TFLOP/s of the
step (both GEMMs' FLOPs over the whole step's device time), with the step's
algorithmic HBM GB/s alongside. Inputs are larger than L2: every step streams
all 5.4 GB of expert weights, so no L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica (its own token batch, the same weights): the layer shards over batches
with no data-path collective, so scaling is weak. Timing: barrier + device
synchronise on both sides of the timed region, CUDA events on the launching
stream, the max over ranks.

--impl reference times the CPU oracle (the plain FP64 implementation used as
the parity reference) on this host's cores, on a bounded sample of the same
workload; it is a slow baseline, not a target.
"""
from __future__ import annotations

import argparse
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="moe_decode_t512", choices=[n for n in workloads.CONFIGS if n != "tiny"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="CPU seconds per reference-arm step (default: 120 s spread over warm-up + steps, at most 30)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # size overrides, used to make small cases of a workload for profiler captures
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--experts", type=int, default=None)
    return ap.parse_args()


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


def measured_traffic(config: str):
    """DRAM bytes per gate/up GEMM launch from the committed ncu summary of this workload, or None when
    there is none or the kernel sources it names changed since it was taken."""
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
    try:   # the dominant GEMM launch: the gate/up GEMM of a layer, the GEMM of the dense workload
        return int(fields.get("gate_up_dram_bytes_per_launch") or fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- work accounting

def moe_counts(cfg, ids):
    E = cfg["E"]
    counts = np.bincount(ids.ravel(), minlength=E)
    return counts


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


# ----------------------------------------------------------------------------- our implementation

class MoEBench:
    def __init__(self, cfg, seed, rank, device):
        import torch
        import nvfp4_block_scaled_09_b200 as nv
        self.nv, self.torch = nv, torch
        self.cfg = cfg
        T, k, H, I, E = cfg["T"], cfg["k"], cfg["H"], cfg["I"], cfg["E"]
        self.dev = device
        # Each rank is a replica: its own tokens and routing, the same weights.
        ids, w = workloads.routing(T, E, k, cfg["routing"], replica_seed(seed, rank), cfg.get("zipf_s", 1.1),
                                   cfg.get("zero_experts", 0))
        self.ids_np, self.w_np = ids, w
        self.counts = moe_counts(cfg, ids)
        self.x = workloads.normal_bf16((T, H), 1.0, replica_seed(seed, rank), workloads.TAG_X, device=device)
        self.ids = torch.from_numpy(ids).to(device)
        self.w = torch.from_numpy(w).to(device)
        self.weights = self._weights(seed)
        self.ws = nv.layer_workspace(T, k, E, H, I, device)
        self.lay = nv.layer_workspace_layout(T, k, E, H, I)
        self.amax_h = self.ws[self.lay["amax_h"]: self.lay["amax_h"] + 4]
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=device)

    def _weights(self, seed):
        nv, torch = self.nv, self.torch
        c = self.cfg
        E, H, I = c["E"], c["H"], c["I"]
        d = self.dev

        def build(N, K, tag):
            packed = torch.empty((E, N * (K // 2 + K // 16)), dtype=torch.uint8, device=d)
            g = torch.empty(E, dtype=torch.float32, device=d)
            q = torch.empty((N, K // 2), dtype=torch.uint8, device=d)
            sf = torch.empty((N, K // 16), dtype=torch.uint8, device=d)
            ws = torch.empty(max(nv.quantize_workspace_size(N, K), 16), dtype=torch.uint8, device=d)
            for e in range(E):
                w = workloads.normal_bf16((N, K), 0.02, seed, tag, e, device=d)
                nv.quantize(w, q=q, sf=sf, g=g[e:e + 1], ws=ws)
                nv.pack_weights(q, sf, out=packed[e])
            return nv.PackedWeights(packed, g, E, N, K)

        w13 = build(2 * I, H, workloads.TAG_W13)
        w2 = build(H, I, workloads.TAG_W2)
        torch.cuda.synchronize()
        return nv.MoEWeights(w13, w2)

    def step(self, ev=None, gemm_ev=None):
        """One layer through the C ABI, stage by stage (the same sequence moe_layer_nvfp4 runs), with
        optional CUDA events between all stages (ev) or around the gate/up GEMM only (gemm_ev)."""
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
        scratch, sbytes = P(b + lay["scratch"]), lay["total"] - lay["scratch"]

        def rec(i):
            if ev is not None:
                ev[i].record()

        self.amax_h.zero_()    # the gate/up GEMM raises it (moe_layer_nvfp4 does the same with a memset)
        rec(0)
        st = L.nvfp4_quantize(P(self.x.data_ptr()), T, H, None, P(b + lay["q_x"]), P(b + lay["sf_x"]),
                              P(b + lay["g_x"]), 0, scratch, sbytes, s)
        rec(1)
        st |= L.moe_permute(P(self.ids.data_ptr()), T, k, E, P(b + lay["q_x"]), P(b + lay["sf_x"]), H,
                            P(b + lay["q_perm"]), P(b + lay["sf_perm"]), nv.SF_KSTAGE, P(b + lay["offsets"]),
                            P(b + lay["perm_src"]), P(b + lay["inv_perm"]), scratch, sbytes, s)
        rec(2)
        if gemm_ev is not None:
            gemm_ev[0].record()
        st |= L.moe_grouped_gemm_nvfp4_amax(P(b + lay["q_perm"]), P(b + lay["sf_perm"]), P(b + lay["g_x"]),
                                            P(W.w13.packed.data_ptr()), P(W.w13.gscale.data_ptr()),
                                            P(b + lay["offsets"]), E, R, 2 * I, H, 1, P(b + lay["h"]),
                                            P(b + lay["amax_h"]), s)
        if gemm_ev is not None:
            gemm_ev[1].record()
        rec(3)
        st |= L.nvfp4_quantize_from_amax(P(b + lay["h"]), R, I, P(b + lay["amax_h"]), P(b + lay["q_h"]),
                                         P(b + lay["sf_h"]), P(b + lay["g_h"]), nv.SF_KSTAGE, s)
        rec(4)
        st |= L.moe_grouped_gemm_nvfp4(P(b + lay["q_h"]), P(b + lay["sf_h"]), P(b + lay["g_h"]),
                                       P(W.w2.packed.data_ptr()), P(W.w2.gscale.data_ptr()),
                                       P(b + lay["offsets"]), E, R, H, I, 0, P(b + lay["y"]), s)
        rec(5)
        st |= L.moe_unpermute_combine(P(b + lay["y"]), P(b + lay["inv_perm"]), P(self.w.data_ptr()), T, k, H,
                                      P(self.out.data_ptr()), s)
        rec(6)
        if st != 0:
            raise RuntimeError(f"library call failed (status bits {st})")

    def layer_call(self, x, ids, w, out):
        """The public one-call API."""
        return self.nv.moe_layer(x, ids, w, self.weights, ws=self.ws, out=out)


def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import nvfp4_block_scaled_09_b200 as nv
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    bench = MoEBench(cfg, args.seed, rank, dev)
    K, W = args.steps, args.warmup
    for _ in range(W):
        bench.step()
    torch.cuda.synchronize()
    st = nv.device_status()
    if st != 0:
        raise RuntimeError(f"device status {nv.status_string(st)} after warm-up")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    nev = 7
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(K)]
    clocks = ClockSampler(local_rank) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.4)
    barrier()
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
    barrier()
    launches = nv.launch_count() - launches0
    clk = clocks.stop() if clocks else None
    elapsed_ms = start.elapsed_time(stop)
    max_ms = max_over_ranks(elapsed_ms, world, dev)
    gemm1_timed_ms = float(np.mean([g[0].elapsed_time(g[1]) for g in gev]))
    # per-stage breakdown in a separate, untimed pass: events between stages serialise the kernels
    # that otherwise overlap their launch with the previous kernel's tail
    stage_ms = np.zeros(nev - 1)
    for i in range(K):
        bench.step(evs[i])
    barrier()
    for i in range(K):
        for j in range(nev - 1):
            stage_ms[j] += evs[i][j].elapsed_time(evs[i][j + 1])
    stage_ms /= K
    st = nv.device_status()
    if st != 0:
        raise RuntimeError(f"device status {nv.status_string(st)} after the timed region")

    # end-to-end through the public one-call API, host buffers in pinned memory: every step copies its
    # inputs host -> device and its output device -> host inside the timed region. Steps are pipelined the
    # way a serving loop would run them: inputs and outputs are double-buffered, the uploads run on one
    # copy stream and the downloads on another while the layer runs on the compute stream.
    e2e = None
    if not args.no_e2e:
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
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(K):
            e2e_step(i)
        e1.record(s_out)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        f1, f2 = moe_flops(cfg)
        e2e = {"value": world * (f1 + f2) * K / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(x_h.numel() * 2 + ids_h.numel() * 4 + w_h.numel() * 4),
               "d2h_bytes_per_step": int(out_h[0].numel() * 2), "api": "moe_layer_nvfp4",
               "ms_per_step": e2e_ms / K,
               "pipelining": "double-buffered inputs/outputs; uploads and downloads on two copy streams"}
    return bench, max_ms, stage_ms, launches, clk, e2e, gemm1_timed_ms


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(cfg, seed, budget_s=10.0):
    """Run the oracle's layer on a bounded sample: quantize + permute over the whole batch, then the two
    GEMMs (and h quantisation) for as many experts' rows as fit the time budget, then the combine.
    Returns (sampled grouped-GEMM FLOPs, seconds, description)."""
    import oracle
    T, k, H, I, E = cfg["T"], cfg["k"], cfg["H"], cfg["I"], cfg["E"]
    ids, w = workloads.routing(T, E, k, cfg["routing"], seed, cfg.get("zipf_s", 1.1), cfg.get("zero_experts", 0))
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


def cpu_baseline(cfg, seed):
    import oracle
    flops, dt, desc, _ = oracle_sample(cfg, seed, budget_s=10.0)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": desc, "seconds": dt}


# ----------------------------------------------------------------------------- dense 8192^3

def oracle_dense_sample(M, N, K, seed, budget_s):
    """Oracle GEMM on a bounded sample of rows of the dense problem (quantise A's sampled rows + GEMM)."""
    import oracle
    rng = np.random.default_rng(seed)
    w_q = rng.integers(0, 256, size=(1, N, K // 2), dtype=np.uint8)
    w_sf = rng.integers(0x20, 0x40, size=(1, N, K // 16), dtype=np.uint8)
    t0 = time.perf_counter()
    rows = 0
    flops = 0.0
    while time.perf_counter() - t0 < budget_s:
        a = workloads.random_bf16_bits((8, K), seed=seed + rows, tag=workloads.TAG_A)
        aq, asf, ag = oracle.quantize(a)
        oracle.grouped_gemm(aq, asf, ag, w_q, w_sf, np.ones(1, np.float32), np.array([0, 8], np.int32), N, K, False)
        rows += 8
        flops += 2.0 * 8 * N * K
    dt = time.perf_counter() - t0
    return flops, dt, f"oracle dense GEMM on {rows} of {M} rows (FP64, {oracle.num_threads()} threads)"


def main_dense(args, cfg, metric, world, rank, local_rank):
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    if args.impl == "reference":
        raise AssertionError("unreachable")
    import torch
    import torch.distributed as dist
    import nvfp4_block_scaled_09_b200 as nv
    from nvfp4_block_scaled_09_b200 import build as nvbuild
    nvbuild.build()
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local_rank))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    a = workloads.normal_bf16((M, K), 1.0, replica_seed(args.seed, rank), workloads.TAG_A, device=dev)
    b = workloads.normal_bf16((1, N, K), 0.02, args.seed, workloads.TAG_B, device=dev)
    pw = nv.prepare_expert_weights(b)
    del b
    a_q = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    a_sf = torch.empty((K // 256, M, 16), dtype=torch.uint8, device=dev)   # K-stage slabs (the GEMM's layout)
    a_g = torch.empty(1, dtype=torch.float32, device=dev)
    qws = torch.empty(nv.quantize_workspace_size(M, K), dtype=torch.uint8, device=dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    off = torch.tensor([0, M], dtype=torch.int32, device=dev)
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
    assert nv.device_status() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.4)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    l0 = nv.launch_count()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)                      # evict A, B and C from L2 between steps (not timed)
        step(*evs[i])
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches = nv.launch_count() - l0
    clk = clocks.stop() if clocks else None
    step_ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    gemm_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    max_step_ms = max_over_ranks(step_ms, world, dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    K_steps = args.steps
    flops = 2.0 * M * N * K
    value = world * flops * K_steps / (max_step_ms * 1e-3) / 1e12
    peaks = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    cb = None
    if world == 1 and not args.no_cpu_baseline:
        f, dt, desc = oracle_dense_sample(M, N, K, args.seed, 10.0)
        import oracle
        cb = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
              "sample": desc}
    line = {
        "metric": metric, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K_steps,
        "warmup": args.warmup, "ms_per_step": max_step_ms / K_steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": "dense", "M": M, "N": N, "K": K,
                   "l2": "flushed between steps (256 MB write, outside the timed events)",
                   "step": "quantize(A) + GEMM with B quantised once beforehand"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp4_peak, "traffic": measured_traffic("dense"),
                     "kernel": "grouped GEMM, E=1 (CTA-pair tiles)",
                     "peak_source": peaks["source"] + " bf16 x 4 (nominal FP4/BF16 ratio)",
                     "avg_launch_ms": gemm_ms},
        "clocks": clk, "gpu_launches": int(launches), "e2e": None, "cpu_baseline": cb,
    }
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- main

def main():
    args = parse()
    cfg = dict(workloads.CONFIGS[args.config])
    if args.tokens:
        cfg["T"] = args.tokens
    if args.experts:
        cfg["E"] = args.experts
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    metric = "NVFP4 MoE grouped-GEMM TFLOPS and HBM GB/s at 16-256 tokens/expert"

    if args.impl == "reference" and cfg["kind"] == "dense":
        if rank != 0:
            return 0
        import oracle
        tot_f = tot_t = 0.0
        desc = ""
        budget = ref_budget(args)
        for i in range(args.warmup + args.steps):
            f, dt, desc = oracle_dense_sample(cfg["M"], cfg["N"], cfg["K"], args.seed, budget)
            if i >= args.warmup:
                tot_f += f
                tot_t += dt
        v = tot_f / tot_t / 1e12
        print(json.dumps({"impl": "reference", "metric": metric, "value": v, "unit": "TFLOP/s",
                          "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
                          "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                          "config": {"workload": "dense", "M": cfg["M"], "N": cfg["N"], "K": cfg["K"]},
                          "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                                           "kind": "oracle", "sample": desc},
                          "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0
    if args.impl == "reference":
        if rank != 0:
            return 0
        import oracle
        K, W = args.steps, args.warmup
        budget = ref_budget(args)
        for _ in range(W):
            oracle_sample(cfg, args.seed, budget_s=budget)
        tot_f, tot_t = 0.0, 0.0
        desc = ""
        for i in range(K):
            f, dt, desc, _ = oracle_sample(cfg, args.seed, budget_s=budget)
            tot_f += f
            tot_t += dt
        v = tot_f / tot_t / 1e12
        line = {"impl": "reference", "metric": metric, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": K, "warmup": W, "ms_per_step": tot_t / K * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": args.config, **{kk: cfg[kk] for kk in ("T", "H", "I", "E", "k")}},
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    if cfg["kind"] == "dense":
        return main_dense(args, cfg, metric, world, rank, local_rank)
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local_rank))
    from nvfp4_block_scaled_09_b200 import build as nvbuild
    nvbuild.build()
    bench, max_ms, stage_ms, launches, clk, e2e, gemm1_timed_ms = run_ours(args, cfg, rank, world, local_rank)
    K = args.steps
    peaks = load_peaks()
    f1, f2 = moe_flops(cfg)
    g1b, g2b = moe_gemm_bytes(cfg, bench.counts)
    step_bytes = moe_step_bytes(cfg, bench.counts)
    step_s = max_ms / K * 1e-3
    value = world * (f1 + f2) / step_s / 1e12
    gemm1_s = gemm1_timed_ms * 1e-3   # event-bracketed inside the timed region
    gemm2_s = stage_ms[4] * 1e-3      # from the per-stage pass
    achieved = g1b / gemm1_s / 1e9
    fp4_peak = peaks["bf16_tflops_sustained"] * FP4_PER_BF16
    # the roof a kernel sits under is set by its arithmetic intensity against the ridge point
    tensor_bound = f1 / g1b >= fp4_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    rows_mean = float(bench.counts.mean())
    plan = bench.nv.gemm_plan()
    shape = ("CTA-pair" if rows_mean >= plan["pair_min_avg_rows"] else
             "wide" if rows_mean >= plan["wide_min_avg_rows"] else "narrow")
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(cfg, args.seed)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    rows = bench.counts
    line = {
        "metric": metric,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": max_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": (value / PAGES_DECODE_TFLOPS
                        if args.config == "moe_decode_t512" and not (args.tokens or args.experts) else None),
        "dtype": "nvfp4 (e2m1 x e2m1, fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": args.config if not (args.tokens or args.experts) else
                   f"{args.config} resized to T={cfg['T']} E={cfg['E']}", "tokens": cfg["T"], "hidden": cfg["H"], "intermediate": cfg["I"],
                   "experts": cfg["E"], "top_k": cfg["k"], "routing": cfg["routing"],
                   "rows_per_expert": {"min": int(rows.min()), "mean": float(rows.mean()), "max": int(rows.max()),
                                       "empty": int(np.sum(rows == 0))},
                   "l2": "no flush: every step streams all expert weights (5.4 GB) through HBM, far above L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "hbm_gbs": world * step_bytes / step_s / 1e9,
        "stage_ms": {"quantize_x": stage_ms[0], "permute": stage_ms[1], "gemm_gate_up": stage_ms[2],
                     "quantize_h": stage_ms[3], "gemm_down": stage_ms[4], "combine": stage_ms[5]},
        "stage_ms_note": "separate pass after the timed region, events between every stage",
        "roofline": ({"bound": "tensor", "achieved": f1 / gemm1_s / 1e12, "peak": fp4_peak, "unit": "TFLOP/s",
                      "frac": f1 / gemm1_s / 1e12 / fp4_peak, "traffic": measured_traffic(args.config),
                      "algorithmic_flops": f1}
                     if tensor_bound else
                     {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic(args.config),
                      "algorithmic_bytes": g1b})
        | {"kernel": f"grouped GEMM gate/up + SwiGLU ({shape} tiles)", "peak_source": peaks["source"],
           "avg_launch_ms": gemm1_timed_ms, "timing": "CUDA events around this kernel inside the timed region"},
        "roofline_down": {"bound": "hbm", "achieved": g2b / gemm2_s / 1e9, "peak": peaks["hbm_gbs"],
                          "unit": "GB/s", "frac": g2b / gemm2_s / 1e9 / peaks["hbm_gbs"]},
        "tensor_frac_gemm_gate_up": (f1 / gemm1_s / 1e12) / (peaks["bf16_tflops_sustained"] * FP4_PER_BF16),
        "clocks": clk,
        "gpu_launches": int(launches),
        "e2e": e2e,
        "cpu_baseline": cb,
    }
    if line["vs_baseline"] is not None:
        line["vs_baseline_basis"] = ("0.8 TFLOPS: per-expert FP4 grouped GEMM at ~16 tokens/expert on RTX PRO "
                                     "6000 (SM120), quoted by the pages as context")
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
