"""moe_quantize_permute (x quantised straight into expert order) against nvfp4_quantize followed by
moe_permute -- the same bytes -- and against the oracle."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import gpu_bf16, host, kstage_sf_to_rowmajor, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def both(T, E, k, H, kind, seed, layout=nv.SF_KSTAGE):
    ids, _ = workloads.routing(T, E, k, kind, seed=seed)
    x = gpu_bf16(workloads.random_bf16_bits((T, H), seed=seed + 1))
    idsd = torch.from_numpy(ids).cuda()
    got, g = nv.quantize_permute(x, idsd, E, sf_layout=layout)
    q, sf, g_ref = nv.quantize(x)
    ref = nv.permute(idsd, q, sf, E, sf_layout=layout)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    for name in ("q_perm", "sf_perm", "offsets", "perm_src", "inv_perm"):
        assert torch.equal(getattr(got, name), getattr(ref, name)), name
    assert torch.equal(g, g_ref)
    return ids, x, got, g


@pytest.mark.parametrize("T,E,k,H,kind", [(512, 256, 8, 6144, "uniform"),     # the decode layer (fused path)
                                          (1024, 256, 8, 6144, "zipf"),       # Zipf layer (fused path)
                                          (37, 5, 2, 256, "uniform"),         # ragged, few experts
                                          (1, 1, 1, 128, "uniform"),          # one row, K = 128
                                          (64, 16, 4, 384, "uniform"),        # K % 256 == 128 (half slab)
                                          (64, 1024, 32, 256, "uniform"),     # E = 1024, k = 32 (every lane a slot)
                                          (5000, 64, 8, 256, "uniform")])     # 40,000 pairs: quantise, then permute
def test_same_bytes_as_quantize_then_permute(T, E, k, H, kind):
    both(T, E, k, H, kind, seed=T + H)


def test_rowmajor_scales():
    both(200, 16, 4, 512, "uniform", seed=3, layout=nv.SF_ROWMAJOR)


def test_against_the_oracle():
    T, E, k, H = 48, 8, 2, 512
    ids, x, got, g = both(T, E, k, H, "uniform", seed=21)
    x_bits = host(x.view(torch.int16)).view(np.uint16)
    oq, osf, og = oracle.quantize(x_bits)
    off, src, inv = oracle.permute(ids, E)
    assert host(g)[0] == og
    assert np.array_equal(host(got.offsets), off) and np.array_equal(host(got.perm_src), src)
    assert np.array_equal(host(got.inv_perm), inv)
    assert np.array_equal(host(got.q_perm), oracle.gather_rows(oq, src))
    sf_rm = kstage_sf_to_rowmajor(host(got.sf_perm), T * k, H)
    assert np.array_equal(sf_rm, oracle.gather_rows(osf, src))


def test_bad_expert_id_latches_status():
    T, E, k, H = 32, 8, 2, 256
    ids, _ = workloads.routing(T, E, k, "uniform", seed=4)
    ids = ids.copy()
    ids[3, 1] = E + 2
    x = gpu_bf16(workloads.random_bf16_bits((T, H), seed=5))
    nv.quantize_permute(x, torch.from_numpy(ids).cuda(), E)
    assert nv.device_status() == 8   # NVFP4_ERR_DEVICE_INPUT


def test_l2_prefetch_hint_changes_no_byte():
    # moe_quantize_permute_prefetch and nvfp4_quantize_from_amax_prefetch with a 96 MB hint (the decode layer's)
    # give the bytes of the calls without one; a hint longer than its tensor is clipped to the tensor by the binding
    T, E, k, H = 512, 256, 8, 6144
    ids, _ = workloads.routing(T, E, k, "uniform", seed=5)
    x = gpu_bf16(workloads.random_bf16_bits((T, H), seed=6))
    idsd = torch.from_numpy(ids).cuda()
    weights = torch.empty(128 << 20, dtype=torch.uint8, device="cuda")
    plain, g0 = nv.quantize_permute(x, idsd, E)
    hinted, g1 = nv.quantize_permute(x, idsd, E, l2_next=weights, l2_next_bytes=96 << 20)
    h = gpu_bf16(workloads.random_bf16_bits((T * k, 2048), seed=7))
    amax = nv.amax(h)
    q0, sf0, gh0 = nv.quantize_from_amax(h, amax, layout=nv.SF_KSTAGE)
    q1, sf1, gh1 = nv.quantize_from_amax(h, amax, layout=nv.SF_KSTAGE, l2_next=weights, l2_next_bytes=1 << 40)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    for name in ("q_perm", "sf_perm", "offsets", "perm_src", "inv_perm"):
        assert torch.equal(getattr(plain, name), getattr(hinted, name)), name
    assert torch.equal(g0, g1)
    assert torch.equal(q0, q1) and torch.equal(sf0, sf1) and torch.equal(gh0, gh1)
