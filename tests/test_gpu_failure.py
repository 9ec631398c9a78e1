"""Failure detection on the GPU without a GPU fault: the grouped GEMM's waits
are bounded. With the test flag set, the producer warp issues no loads, so the
MMA, scale and epilogue warps' waits run out after a short limit; the kernel
must latch NVFP4_ERR_DEVICE_TIMEOUT, free its tensor memory and return, and the
next normal call on the same context must produce correct results."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import compare_bf16, gpu_bf16, host, host_bits, kstage_sf_to_rowmajor, require_gpu

pytestmark = pytest.mark.gpu


def small_case():
    rows, N, K = [16, 16], 256, 256
    a_bits = workloads.random_bf16_bits((32, K), seed=21)
    a_q, a_sf, a_g = nv.quantize(gpu_bf16(a_bits), layout=nv.SF_KSTAGE)
    w = workloads.normal_bf16((2, N, K), 0.02, 21, workloads.TAG_W13, device="cuda")
    pw = nv.prepare_expert_weights(w, keep_rowmajor=True)
    off = torch.tensor([0, 16, 32], dtype=torch.int32, device="cuda")
    return a_q, a_sf, a_g, pw, off


def test_stalled_producer_times_out_then_context_recovers():
    require_gpu()
    a_q, a_sf, a_g, pw, off = small_case()
    assert nv.device_status() == 0
    old = nv.get_wait_timeout_ns()
    try:
        nv.set_wait_timeout_ns(2_000_000)          # 2 ms per wait
        nv.debug_set_flags(1)                      # producer issues nothing
        nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False)
        assert nv.device_status() == 7             # NVFP4_ERR_DEVICE_TIMEOUT, latched and cleared
    finally:
        nv.debug_set_flags(0)
        nv.set_wait_timeout_ns(old)
    assert nv.device_status() == 0
    out = nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False)
    assert nv.device_status() == 0
    args = (host(a_q), kstage_sf_to_rowmajor(host(a_sf), 32, 256), host(a_g)[0], host(pw.q), host(pw.sf),
            host(pw.gscale), np.array([0, 16, 32], np.int32), 256, 256, False)
    ref = oracle.grouped_gemm(*args)
    compare_bf16(host_bits(out), oracle.bf16_round(ref), "gemm after a timed-out launch", exact=ref,
                 band=oracle.grouped_gemm_bound(*args))
    # every counter slot of the dynamic schedule (the timed-out launch's among them) is clean when drawn
    # again: 2 x 64 more launches, each equal to the first
    first = host_bits(out)
    outs = [nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False) for _ in range(128)]
    assert nv.device_status() == 0
    for o in outs:
        assert np.array_equal(host_bits(o), first)


def pair_case(swiglu):
    """Ragged experts on the CTA-pair kernel: the activations are padded to 192 rows per expert, which
    selects the pair tiles (256 weight rows x up to 256 activation rows on two SMs)."""
    rows, N, K = [0, 200, 256, 257, 40], 512, 512
    E, R = len(rows), sum(rows)
    plan = nv.gemm_plan()
    rows_a = max(R, plan["pair_min_avg_rows"] * E)
    a_bits = workloads.random_bf16_bits((rows_a, K), seed=31)
    a_q, a_sf, a_g = nv.quantize(gpu_bf16(a_bits), layout=nv.SF_KSTAGE)
    w = workloads.normal_bf16((E, N, K), 0.02, 31, workloads.TAG_W13, device="cuda")
    pw = nv.prepare_expert_weights(w, keep_rowmajor=True)
    off_np = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    return a_q, a_sf, a_g, pw, torch.from_numpy(off_np).cuda(), off_np, rows_a, R, N, K


@pytest.mark.parametrize("swiglu", [False, True])
def test_pair_kernel_stalled_producer_times_out_then_recovers(swiglu):
    # The CTA-pair kernel's abort path: with the producer stalled, every wait of both CTAs of a pair runs
    # out (the odd CTA's waits on the work-item ring acquire at cluster scope), both CTAs drain, meet at
    # the cluster barrier and release the pair's tensor memory.
    require_gpu()
    a_q, a_sf, a_g, pw, off, off_np, rows_a, R, N, K = pair_case(swiglu)
    assert nv.device_status() == 0
    old = nv.get_wait_timeout_ns()
    try:
        nv.set_wait_timeout_ns(2_000_000)
        nv.debug_set_flags(1)
        nv.grouped_gemm(a_q, a_sf, a_g, pw, off, swiglu)
        assert nv.device_status() == 7
    finally:
        nv.debug_set_flags(0)
        nv.set_wait_timeout_ns(old)
    assert nv.device_status() == 0
    out = nv.grouped_gemm(a_q, a_sf, a_g, pw, off, swiglu)
    assert nv.device_status() == 0
    args = (host(a_q)[:R], kstage_sf_to_rowmajor(host(a_sf), rows_a, K)[:R], host(a_g)[0], host(pw.q), host(pw.sf),
            host(pw.gscale), off_np, N, K, swiglu)
    ref = oracle.grouped_gemm(*args)
    compare_bf16(host_bits(out)[:R], oracle.bf16_round(ref), f"pair gemm after a timed-out launch swiglu={swiglu}",
                 exact=ref, band=oracle.grouped_gemm_bound(*args))
    first = host_bits(out)[:R]
    outs = [nv.grouped_gemm(a_q, a_sf, a_g, pw, off, swiglu) for _ in range(72)]
    assert nv.device_status() == 0
    for o in outs:
        assert np.array_equal(host_bits(o)[:R], first)


def test_concurrent_launches_on_several_streams():
    # GEMMs in flight on four streams at once draw different counter slots of the dynamic schedule; each
    # result equals the serial one bit for bit
    require_gpu()
    a_q, a_sf, a_g, pw, off = small_case()
    ref = host_bits(nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False))
    streams = [torch.cuda.Stream() for _ in range(4)]
    outs = []
    torch.cuda.synchronize()
    for i in range(48):
        s = streams[i % 4]
        with torch.cuda.stream(s):
            outs.append(nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False, stream=s))
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    for o in outs:
        assert np.array_equal(host_bits(o), ref)
