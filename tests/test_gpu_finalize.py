"""moe_grouped_gemm_nvfp4_finalize (the down GEMM with the top-k combine fused into its epilogue) against
the separate path: the same GEMM followed by moe_unpermute_combine must give the same bits (y and the
combined output), on every tile shape (narrow, wide, CTA pairs), on a half column tile (N % 256 == 128), on
two calls in a row with the same counters, and at the full decode and prefill sizes. The combined output is
also checked against the oracle's combine of the GPU's y (bit-exact: FP64 accumulation, one rounding)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import gpu_bf16, host, host_bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def case(T, k, E, N, K, kind, seed, pad_rows=0):
    ids, w = workloads.routing(T, E, k, kind, seed=seed)
    R = T * k
    h_bits = workloads.random_bf16_bits((T, K), seed=seed + 1)
    q, sf, g = nv.quantize(gpu_bf16(h_bits))
    perm = nv.permute(torch.from_numpy(ids).cuda(), q, sf, E)
    if pad_rows:
        # more activation rows than routed pairs: the GEMM's max_rows picks the tile shape
        qa = torch.zeros((R + pad_rows, K // 2), dtype=torch.uint8, device="cuda")
        qa[:R] = perm.q_perm
        sfa = torch.zeros((nv.kstage_slabs(K), R + pad_rows, 16), dtype=torch.uint8, device="cuda")
        sfa[:, :R] = perm.sf_perm
        src = torch.full((R + pad_rows,), -1, dtype=torch.int32, device="cuda")
        src[:R] = perm.perm_src
    else:
        qa, sfa, src = perm.q_perm, perm.sf_perm, perm.perm_src
    wt = nv.prepare_expert_weights(workloads.normal_bf16((E, N, K), 0.02, seed, workloads.TAG_W2, device="cuda"))
    return dict(qa=qa, sfa=sfa, g=g, w=wt, off=perm.offsets, src=src, inv=perm.inv_perm,
                topk_w=torch.from_numpy(w).cuda(), T=T, k=k, R=R)


def check(c, calls=2):
    y_ref = nv.grouped_gemm(c["qa"], c["sfa"], c["g"], c["w"], c["off"], False)
    out_ref = nv.unpermute_combine(y_ref, c["inv"], c["topk_w"])
    counters = nv.finalize_counters(c["T"], c["w"].N)
    for _ in range(calls):
        out, y = nv.grouped_gemm_finalize(c["qa"], c["sfa"], c["g"], c["w"], c["off"], c["src"], c["inv"],
                                          c["topk_w"], counters)
        assert nv.device_status() == 0
        R = c["R"]
        assert torch.equal(y[:R].view(torch.int16), y_ref[:R].view(torch.int16))
        assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
        assert int(counters.abs().sum()) == 0                 # every counter left at zero
    # and against the oracle's combine of the GPU's y (bit-exact)
    ref = oracle.bf16_round(oracle.combine(host_bits(y)[: c["R"]], host(c["inv"]), host(c["topk_w"])))
    assert np.array_equal(host_bits(out), ref)


@pytest.mark.parametrize("T,k,E,N,K,kind", [(64, 8, 32, 512, 256, "uniform"),     # narrow tiles
                                             (200, 4, 8, 768, 512, "zipf"),       # wide tiles, skewed
                                             (37, 2, 5, 384, 256, "uniform"),     # half column tile
                                             (1, 1, 1, 256, 128, "uniform")])     # one row, K = 128
def test_finalize_one_sm_tiles(T, k, E, N, K, kind):
    check(case(T, k, E, N, K, kind, seed=T + N))


def test_finalize_pair_tiles():
    # experts averaging >= 192 rows: the CTA-pair kernel, each CTA combining its own 128-column block
    check(case(400, 8, 12, 512, 256, "uniform", seed=5))
    check(case(50, 4, 4, 512, 384, "uniform", seed=6, pad_rows=800))   # padded rows select the pair tiles


@pytest.mark.parametrize("name", ["moe_decode_t512", "moe_prefill_t8192"])
def test_finalize_full_size(name):
    cfg = workloads.CONFIGS[name]
    T, k, E, H, I = cfg["T"], cfg["k"], cfg["E"], cfg["H"], cfg["I"]
    ids, w = workloads.config_routing(name)
    h_bits = workloads.normal_bf16((T, I), 1.0, 0, workloads.TAG_X, device="cuda")
    q, sf, g = nv.quantize(h_bits)
    perm = nv.permute(torch.from_numpy(ids).cuda(), q, sf, E)
    wt = nv.prepare_expert_weights(workloads.normal_bf16((E, H, I), 0.02, 0, workloads.TAG_W2, device="cuda"))
    c = dict(qa=perm.q_perm, sfa=perm.sf_perm, g=g, w=wt, off=perm.offsets, src=perm.perm_src, inv=perm.inv_perm,
             topk_w=torch.from_numpy(w).cuda(), T=T, k=k, R=T * k)
    check(c, calls=2)
