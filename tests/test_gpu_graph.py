"""The grouped GEMM inside a captured CUDA graph: a replay reuses the work counter its capture drew, so
replays are run one after another (the header's concurrency rule); here they alternate between two streams,
ordered by events, and every replay equals the direct launch bit for bit."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import workloads
from tests.helpers import gpu_bf16, host_bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pad", [0, 900])    # one-SM and CTA-pair tiles
def test_captured_gemm_replays_on_two_streams(pad):
    require_gpu()
    rows, N, K = [30, 0, 65, 17, 40], 512, 512
    E, R = len(rows), sum(rows)
    a_bits = workloads.random_bf16_bits((R + pad, K), seed=77)
    a_q, a_sf, a_g = nv.quantize(gpu_bf16(a_bits), layout=nv.SF_KSTAGE)
    pw = nv.prepare_expert_weights(workloads.normal_bf16((E, N, K), 0.02, 77, workloads.TAG_W13, device="cuda"))
    off = torch.from_numpy(np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)).cuda()
    ref = host_bits(nv.grouped_gemm(a_q, a_sf, a_g, pw, off, True))     # direct launch (also the warm-up)
    out = torch.zeros((R + pad, N // 2), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=cap):
        nv.grouped_gemm(a_q, a_sf, a_g, pw, off, True, out=out, stream=cap)
    s = [torch.cuda.Stream(), torch.cuda.Stream()]
    done = torch.cuda.Event()
    done.record(torch.cuda.current_stream())
    results = []
    for i in range(8):
        st = s[i % 2]
        st.wait_event(done)                 # the previous replay finished: replays never overlap
        with torch.cuda.stream(st):
            out.fill_(0)
            g.replay()
            snap = out.clone()
            done = torch.cuda.Event()
            done.record(st)
        results.append(snap)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    for r in results:
        assert np.array_equal(host_bits(r)[:R], ref[:R])
    del g
