"""Expert-parallel NVFP4 MoE layer over torch.distributed (one process per GPU, NCCL between GPUs).

G ranks each hold their own tokens and the weights of E/G consecutive experts. One layer:

  1. amax of x on every rank, combined with an all-reduce (max): x is quantised with the global scale of
     the whole batch, so every rank's FP4 rows are the rows one GPU would produce for all G*T tokens.
  2. moe_permute over all E experts. Each rank's experts are consecutive, so the expert-ordered rows are
     also grouped by the rank that owns them.
  3. all-to-all of the per-expert row counts, then of the FP4 codes and scales (dispatch; the scales of
     this permute are row-major, so that each row's bytes are contiguous).
  4. The received rows (source-major) are regrouped by local expert with a second moe_permute (k = 1),
     whose scales come out in the K-stage layout the grouped GEMM reads.
  5. The gate/up GEMM reports the amax of h; an all-reduce (max) makes it the amax over all ranks' rows;
     h is quantised from it and the down GEMM runs. A k = 1 combine with weight 1 (an exact copy) puts
     the rows back in arrival order.
  6. all-to-all of the output rows back to the ranks that own the tokens (return), then the top-k
     weighted combine.

Each rank's output is bit-identical to moe_layer_nvfp4 on one GPU over the concatenation of all ranks'
tokens with all E experts: the global scales are the same, and every other step is computed per row.
The exchange is the one step with data moving between GPUs (the expert-parallel split of the pages'
MoE layer: "Peering into the CUTLASS Kernel Cache", Knowledge Required -- each expert's weights multiply
the tokens routed to it). Routing bookkeeping (split sizes, local expert ids) is host-side; every
arithmetic step runs in the library's kernels (LibraryOps) -- tests substitute another backend with the
same five operations to exercise the exchange on CPU ranks.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

import nvfp4_block_scaled_09_b200 as nv


class LibraryOps:
    """The five operations of the layer, on device tensors, through the library's C ABI."""

    def amax(self, x):
        return nv.amax(x)

    def quantize_from_amax(self, x, amax_bits, gemm_operand=False):
        # row-major scales for x (they travel to other ranks row by row); K-stage slabs for an operand of
        # the grouped GEMM
        return nv.quantize_from_amax(x, amax_bits, layout=nv.SF_KSTAGE if gemm_operand else nv.SF_ROWMAJOR)

    def permute(self, ids, q, sf, num_experts, gemm_operand=False):
        return nv.permute(ids, q, sf, num_experts, sf_layout=nv.SF_KSTAGE if gemm_operand else nv.SF_ROWMAJOR)

    def gemm(self, a_q, a_sf, a_g, w, offsets, swiglu, amax_out=None):
        return nv.grouped_gemm(a_q, a_sf, a_g, w, offsets, swiglu, amax_out=amax_out)

    def combine(self, y, inv_perm, topk_w):
        return nv.unpermute_combine(y, inv_perm, topk_w)


def expert_range(num_experts: int, world: int, rank: int) -> tuple[int, int]:
    """Experts [lo, hi) held by `rank`."""
    if num_experts % world:
        raise ValueError(f"{num_experts} experts do not split evenly over {world} ranks")
    n = num_experts // world
    return rank * n, (rank + 1) * n


def _all_to_all_rows(t: torch.Tensor, send_rows: list[int], recv_rows: list[int], group) -> torch.Tensor:
    """all_to_all_single along dim 0 with per-rank row counts; rows travel as raw bytes."""
    raw = t.contiguous().view(torch.uint8)
    out = torch.empty((sum(recv_rows), raw.shape[1]), dtype=torch.uint8, device=raw.device)
    dist.all_to_all_single(out, raw, output_split_sizes=recv_rows, input_split_sizes=send_rows, group=group)
    return out.view(t.dtype)


def ep_moe_layer(x: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor, local_weights,
                 num_experts: int, group=None, ops=None) -> torch.Tensor:
    """One expert-parallel MoE layer. x [T, H] BF16, topk_ids [T, k] int32 (global expert ids), topk_w
    [T, k] FP32, local_weights: the MoEWeights of this rank's experts (w13 [E/G, 2I, H], w2 [E/G, H, I]).
    Returns out [T, H] BF16 for this rank's tokens. Every rank takes the same collective steps."""
    ops = ops or LibraryOps()
    G = dist.get_world_size(group)
    r = dist.get_rank(group)
    E = num_experts
    lo, hi = expert_range(E, G, r)
    El = hi - lo
    T, k = topk_ids.shape
    dev = x.device

    # 1. global scale of x
    amax_x = ops.amax(x)
    dist.all_reduce(amax_x, op=dist.ReduceOp.MAX, group=group)
    q_x, sf_x, g_x = ops.quantize_from_amax(x, amax_x)

    # 2. rows grouped by expert, hence by owning rank
    perm = ops.permute(topk_ids, q_x, sf_x, E)
    off = perm.offsets.cpu().numpy().astype(np.int64)
    send_e = np.diff(off).reshape(G, El)                      # rows for (owner rank, its local expert)

    # 3. dispatch: counts first, then codes and scales
    send_counts = torch.from_numpy(send_e.reshape(-1).astype(np.int32)).to(dev)
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    recv_e = recv_counts.cpu().numpy().astype(np.int64).reshape(G, El)   # rows from (source rank, local expert)
    send_rows = [int(v) for v in send_e.sum(1)]
    recv_rows = [int(v) for v in recv_e.sum(1)]
    R_send = int(off[-1])
    q_recv = _all_to_all_rows(perm.q_perm[:R_send], send_rows, recv_rows, group)
    sf_recv = _all_to_all_rows(perm.sf_perm[:R_send], send_rows, recv_rows, group)
    Rr = sum(recv_rows)

    # 4.-5. local experts on the received rows (global scale of h over all ranks)
    H = x.shape[1]
    amax_h = torch.zeros(1, dtype=torch.int32, device=dev)
    if Rr > 0:
        local_ids = np.repeat(np.tile(np.arange(El, dtype=np.int32), G), recv_e.reshape(-1))
        loc = ops.permute(torch.from_numpy(local_ids.reshape(-1, 1)).to(dev), q_recv, sf_recv, El,
                          gemm_operand=True)
        h = ops.gemm(loc.q_perm, loc.sf_perm, g_x, local_weights.w13, loc.offsets, True, amax_out=amax_h)
    dist.all_reduce(amax_h, op=dist.ReduceOp.MAX, group=group)
    if Rr > 0:
        q_h, sf_h, g_h = ops.quantize_from_amax(h, amax_h, gemm_operand=True)
        y_loc = ops.gemm(q_h, sf_h, g_h, local_weights.w2, loc.offsets, False)
        y_recv = ops.combine(y_loc, loc.inv_perm, torch.ones((Rr, 1), dtype=torch.float32, device=dev))
    else:
        y_recv = torch.empty((0, H), dtype=torch.bfloat16, device=dev)

    # 6. return and combine
    y_back = _all_to_all_rows(y_recv, recv_rows, send_rows, group)
    return ops.combine(y_back, perm.inv_perm, topk_w)
