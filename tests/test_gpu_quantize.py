"""nvfp4_quantize on the GPU against the oracle: codes, block scales and the
global scale must match bit for bit (both sides take every rounding decision
in FP32 round-to-nearest-even)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import gpu_bf16, host, kstage_sf_to_rowmajor, require_gpu, untile_sf

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def gpu_quantize(xbits, gscale=None, layout=nv.SF_ROWMAJOR):
    x = gpu_bf16(xbits)
    g_in = None if gscale is None else torch.tensor([gscale], dtype=torch.float32, device="cuda")
    q, sf, g = nv.quantize(x, global_scale=g_in, layout=layout)
    torch.cuda.synchronize()
    return host(q), host(sf), np.float32(host(g)[0])


def check(xbits, gscale=None):
    q, sf, g = gpu_quantize(xbits, gscale)
    oq, osf, og = oracle.quantize(xbits, gscale)
    assert g == og, (g, og)
    assert np.array_equal(sf.reshape(osf.shape), osf), np.argwhere(sf.reshape(osf.shape) != osf)[:5]
    mism = np.argwhere(q != oq)
    assert mism.size == 0, (mism[:5], q[tuple(mism[0])], oq[tuple(mism[0])])


@pytest.mark.parametrize("rows,K,std,seed", [
    (1, 16, 1.0, 0), (3, 48, 1.0, 1), (64, 256, 1.0, 2), (100, 6144, 1.0, 3), (33, 2048, 0.02, 4),
    (7, 512, 100.0, 5), (128, 1024, 1e-3, 6),
])
def test_random_bit_exact(rows, K, std, seed):
    check(workloads.random_bf16_bits((rows, K), seed=seed, std=std))


def bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_ties_saturation_and_signed_zero():
    # global scale 1 and block amax 6 make f = 1, so x lands on the E2M1 grid's tie points directly
    ties = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.1, -0.0, 0.0, -5.0, -2.5, 0.1, -6.0]
    check(bf16_bits([ties, [v * 0.5 for v in ties]]), gscale=1.0)
    # static scale small enough to saturate both the block scale and the codes
    check(bf16_bits([[12.0, -30.0] + [1.0] * 14]), gscale=1.0 / 448.0)


def test_zero_tensor_and_zero_block():
    check(np.zeros((4, 64), dtype=np.uint16))
    x = workloads.random_bf16_bits((4, 64), seed=9)
    x[1, 16:32] = 0
    x[2, :16] = 0x8000  # negative zeros
    check(x)


def test_tiled_layout_is_a_permutation_of_rowmajor():
    x = workloads.random_bf16_bits((256, 512), seed=11, std=0.02)
    q, sf_t, g = gpu_quantize(x, layout=nv.SF_MMA_TILED)
    oq, osf, og = oracle.quantize(x)
    assert g == og and np.array_equal(q, oq)
    assert np.array_equal(untile_sf(sf_t, 256, 512), osf)


@pytest.mark.parametrize("rows,K", [(1, 256), (37, 768), (300, 6144), (5, 128), (33, 384)])
def test_kstage_layout_is_a_permutation_of_rowmajor(rows, K):
    # the grouped GEMM's activation-scale layout: one [rows x 16 B] slab per 256-element K step (K % 256 == 128:
    # the last slab zero-padded, which the converter checks)
    x = workloads.random_bf16_bits((rows, K), seed=rows, std=1.0)
    q, sf_k, g = gpu_quantize(x, layout=nv.SF_KSTAGE)
    oq, osf, og = oracle.quantize(x)
    assert sf_k.shape == ((K + 255) // 256, rows, 16)
    assert g == og and np.array_equal(q, oq)
    assert np.array_equal(kstage_sf_to_rowmajor(sf_k, rows, K), osf)


def test_decode_activation_size():
    # x of the 512-token decode layer, and an h-sized tensor
    check(workloads.random_bf16_bits((512, 6144), seed=12))
    check(workloads.random_bf16_bits((4096, 2048), seed=13, std=0.3))


def test_rejects_bad_arguments():
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.quantize(x)
    assert e.value.status == 3
    x = torch.zeros((100, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.quantize(x, layout=nv.SF_MMA_TILED)
    assert e.value.status == 3
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")    # K-stage slabs need K % 128 == 0
    with pytest.raises(nv.NVFP4Error) as e:
        nv.quantize(x, layout=nv.SF_KSTAGE)
    assert e.value.status == 3
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")   # one padded slab: 4 rows x 16 bytes
    with pytest.raises(ValueError):
        nv.quantize(x, layout=nv.SF_KSTAGE, sf=torch.empty((4, 8), dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("rows,K,std,seed", [(1, 16, 1.0, 10), (96, 2048, 0.5, 11), (300, 512, 3.0, 12)])
def test_from_amax_equals_dynamic(rows, K, std, seed):
    # quantize_from_amax with the tensor's own amax (BF16 bits, as the GEMM side output carries it) is the
    # dynamic-scale quantiser: compared with the oracle bit for bit, and with an all-zero tensor
    xbits = workloads.random_bf16_bits((rows, K), seed=seed, std=std)
    for bits in (xbits, np.zeros_like(xbits)):
        amax = torch.tensor([int((bits & 0x7FFF).max())], dtype=torch.int32, device="cuda")
        q, sf, g = nv.quantize_from_amax(gpu_bf16(bits), amax)
        oq, osf, og = oracle.quantize(bits)
        assert np.float32(host(g)[0]) == og
        assert np.array_equal(host(sf).reshape(osf.shape), osf)
        assert np.array_equal(host(q), oq)
        if K % 256 == 0:   # the same in the K-stage layout (what the layer feeds the down GEMM)
            qk, sfk, gk = nv.quantize_from_amax(gpu_bf16(bits), amax, layout=nv.SF_KSTAGE)
            assert np.float32(host(gk)[0]) == og and np.array_equal(host(qk), oq)
            assert np.array_equal(kstage_sf_to_rowmajor(host(sfk), rows, K), osf)
