"""moe_grouped_gemm_nvfp4_quant: the gate/up GEMM whose SwiGLU epilogue writes h as NVFP4 with a static
global scale. Its codes and K-stage scales must equal nvfp4_quantize(h, global_scale_in=g) of the BF16 h the
plain SwiGLU call writes, bit for bit, and the oracle's static-scale quantisation of that h, on every tile
shape; its amax side output equals the amax of h. Rows outside every expert stay untouched."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import gpu_bf16, host, host_bits, kstage_sf_to_rowmajor, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def run(rows, N, K, seed, pad_rows=0, g_scale=None):
    E, R = len(rows), sum(rows)
    rows_a = R + pad_rows
    a_bits = workloads.random_bf16_bits((max(rows_a, 1), K), seed=seed)
    a_q, a_sf, a_g = nv.quantize(gpu_bf16(a_bits), layout=nv.SF_KSTAGE)
    pw = nv.prepare_expert_weights(workloads.normal_bf16((E, N, K), 0.02, seed, workloads.TAG_W13, device="cuda"))
    off = torch.from_numpy(np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)).cuda()
    h = nv.grouped_gemm(a_q, a_sf, a_g, pw, off, True)                          # BF16 h, the reference input
    amax_h = int((host_bits(h)[:R] & 0x7FFF).max()) if R else 0
    g = float(np.float32(g_scale if g_scale is not None else
                         (np.frombuffer(np.uint32(amax_h << 16).tobytes(), np.float32)[0] / 2688.0 * 1.25)))
    g_t = torch.tensor([g], dtype=torch.float32, device="cuda")
    amax = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_h = torch.full((rows_a, N // 4), 0x5A, dtype=torch.uint8, device="cuda")     # canaries outside the rows
    q_h, sf_h = nv.grouped_gemm_quant(a_q, a_sf, a_g, pw, off, g_t, q_h=q_h, amax_out=amax)
    assert nv.device_status() == 0
    assert int(host(amax)[0]) == amax_h
    ref_q, ref_sf, _ = nv.quantize(h[:R], global_scale=g_t, layout=nv.SF_KSTAGE)
    assert np.array_equal(host(q_h)[:R], host(ref_q))
    got_sf = kstage_sf_to_rowmajor(host(sf_h), rows_a, N // 2)[:R]
    assert np.array_equal(got_sf, kstage_sf_to_rowmajor(host(ref_sf), R, N // 2))
    oq, osf, _ = oracle.quantize(host_bits(h)[:R], g)
    assert np.array_equal(host(q_h)[:R], oq) and np.array_equal(got_sf, osf)
    assert np.all(host(q_h)[R:] == 0x5A)


@pytest.mark.parametrize("rows,N,K,pad", [([16, 0, 5, 33, 64], 512, 256, 0),            # narrow tiles
                                          ([0, 100, 129, 300, 17], 768, 512, 0),         # wide tiles
                                          ([0, 200, 256, 257, 40], 512, 384, 800),       # CTA pairs, K % 256 = 128
                                          ([3, 40], 768, 256, 0)])                       # h width 384: padded slab
def test_quantised_h_equals_static_quantize_of_h(rows, N, K, pad):
    run(rows, N, K, seed=sum(rows) + N, pad_rows=pad)


def test_saturating_static_scale():
    # a calibrated scale below the true amax: block scales saturate at 448 and codes at 6, as nvfp4_quantize does
    run([30, 20], 512, 256, seed=3, g_scale=1e-6)
