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
    ref = oracle.grouped_gemm(host(a_q), kstage_sf_to_rowmajor(host(a_sf), 32, 256), host(a_g)[0], host(pw.q),
                              host(pw.sf), host(pw.gscale),
                              np.array([0, 16, 32], np.int32), 256, 256, False)
    compare_bf16(host_bits(out), oracle.bf16_round(ref), "gemm after a timed-out launch", exact=ref)
    # every counter slot of the dynamic schedule (the timed-out launch's among them) is clean when drawn
    # again: 2 x 64 more launches, each equal to the first
    first = host_bits(out)
    for _ in range(128):
        again = nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False)
    assert nv.device_status() == 0
    assert np.array_equal(host_bits(again), first)


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
