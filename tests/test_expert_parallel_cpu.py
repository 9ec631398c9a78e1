"""The expert-parallel layer's exchange on CPU ranks (gloo).

nvfp4_block_scaled_09_b200.expert_parallel runs with the oracle as each rank's backend (the same five
operations as the library: amax, quantise from an amax, permute, grouped GEMM with an amax side output,
combine) on CPU tensors. Every rank's output must equal, bit for bit, the oracle's single-process layer
over the concatenation of all ranks' tokens with all experts -- the property the design claims for the
GPU path (one global scale for x and for h over the whole batch; every other step per row).
"""
import datetime
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    """The layer's five operations through the oracle, on CPU tensors."""

    def __init__(self, oracle):
        self.o = oracle

    def amax(self, x):
        b = _bits(x)
        return torch.tensor([int((b & 0x7FFF).max()) if b.size else 0], dtype=torch.int32)

    def quantize_from_amax(self, x, amax_bits, gemm_operand=False):   # row-major scales throughout
        amax = float(self.o.bf16_bits_to_f64(np.array([int(amax_bits[0])], dtype=np.uint16))[0])
        q, sf, g = self.o.quantize_with_amax(_bits(x), amax)
        return torch.from_numpy(q), torch.from_numpy(sf), torch.tensor([g], dtype=torch.float32)

    def permute(self, ids, q, sf, num_experts, gemm_operand=False):
        off, src, inv = self.o.permute(ids.numpy(), num_experts)
        return SimpleNamespace(q_perm=torch.from_numpy(self.o.gather_rows(q.numpy(), src)),
                               sf_perm=torch.from_numpy(self.o.gather_rows(sf.numpy(), src)),
                               offsets=torch.from_numpy(off), perm_src=torch.from_numpy(src),
                               inv_perm=torch.from_numpy(inv))

    def gemm(self, a_q, a_sf, a_g, w, offsets, swiglu, amax_out=None):
        ref = self.o.grouped_gemm(a_q.numpy(), a_sf.numpy(), float(a_g[0]), w.q, w.sf, w.g, offsets.numpy(), w.N,
                                  w.K, swiglu)
        b = self.o.bf16_round(ref)
        if amax_out is not None and b.size:
            amax_out[0] = max(int(amax_out[0]), int((b & 0x7FFF).max()))
        return _bf16(b)

    def combine(self, y, inv_perm, topk_w):
        return _bf16(self.o.bf16_round(self.o.combine(_bits(y), inv_perm.numpy(), topk_w.numpy())))


def build_weights(oracle, workloads, E, N, K, tag):
    """Quantised weights of all E experts (row-major codes and scales, per-expert global scale)."""
    q = np.empty((E, N, K // 2), np.uint8)
    sf = np.empty((E, N, K // 16), np.uint8)
    g = np.empty(E, np.float32)
    for e in range(E):
        wb = workloads.random_bf16_bits((N, K), seed=100 + e, std=0.02, tag=tag)
        q[e], sf[e], g[e] = oracle.quantize(wb)
    return SimpleNamespace(q=q, sf=sf, g=g, N=N, K=K)


def local_slice(w, lo, hi):
    return SimpleNamespace(q=w.q[lo:hi], sf=w.sf[lo:hi], g=w.g[lo:hi], N=w.N, K=w.K)


def rank_inputs(workloads, r, T, H, E, k, routing):
    x = workloads.random_bf16_bits((T, H), seed=10 + r, std=1.0)
    if routing == "owner0":   # every token routed to rank 0's experts only: other ranks receive nothing
        rng = np.random.default_rng(r)
        ids = np.stack([rng.choice(E // 2, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        w = rng.random((T, k)).astype(np.float32)
        w /= w.sum(1, keepdims=True)
    else:
        ids, w = workloads.routing(T, E, k, routing, seed=20 + r)
    return x, ids, w


def reference(oracle, xs, idss, ws, w13, w2, E):
    """The oracle's single-process layer over all ranks' tokens."""
    X, IDS, W = np.concatenate(xs), np.concatenate(idss), np.concatenate(ws)
    q, sf, g = oracle.quantize(X)
    off, src, inv = oracle.permute(IDS, E)
    h = oracle.bf16_round(oracle.grouped_gemm(oracle.gather_rows(q, src), oracle.gather_rows(sf, src), g, w13.q,
                                              w13.sf, w13.g, off, w13.N, w13.K, True))
    qh, sfh, gh = oracle.quantize(h)
    y = oracle.bf16_round(oracle.grouped_gemm(qh, sfh, gh, w2.q, w2.sf, w2.g, off, w2.N, w2.K, False))
    return oracle.bf16_round(oracle.combine(y, inv, W))


def _rank_main(rank, world, port, cfg, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    import workloads
    from nvfp4_block_scaled_09_b200 import expert_parallel as ep
    oracle.set_num_threads(1)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, H, I, E, k, routing = cfg
        w13 = build_weights(oracle, workloads, E, 2 * I, H, workloads.TAG_W13)
        w2 = build_weights(oracle, workloads, E, H, I, workloads.TAG_W2)
        lo, hi = ep.expert_range(E, world, rank)
        local = SimpleNamespace(w13=local_slice(w13, lo, hi), w2=local_slice(w2, lo, hi))
        x, ids, w = rank_inputs(workloads, rank, T, H, E, k, routing)
        out = ep.ep_moe_layer(_bf16(x), torch.from_numpy(ids), torch.from_numpy(w), local, E,
                              ops=OracleOps(oracle))
        res = {"rank": rank, "out": _bits(out).copy()}
        if rank == 0:
            ins = [rank_inputs(workloads, r, T, H, E, k, routing) for r in range(world)]
            res["ref"] = reference(oracle, [a[0] for a in ins], [a[1] for a in ins], [a[2] for a in ins], w13, w2,
                                   E)
        out_q.put(res)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cfg", [
    (2, (24, 256, 256, 8, 2, "uniform")),
    (4, (16, 256, 256, 8, 3, "uniform")),
    (2, (32, 256, 256, 8, 2, "zipf")),
    (2, (12, 256, 256, 8, 2, "owner0")),    # rank 1 receives no rows
])
def test_expert_parallel_equals_single_process_layer(world, cfg):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, cfg, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda d: d["rank"])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    T = cfg[0]
    ref = res[0]["ref"]
    for d in res:
        r = d["rank"]
        assert np.array_equal(d["out"], ref[r * T:(r + 1) * T]), f"rank {r} differs from the single-process layer"
