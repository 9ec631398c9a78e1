"""moe_permute on the GPU against the oracle: offsets, indices and gathered
bytes bit-exact, for every routing pattern of the workloads, with the scales
written in either layout (K-stage slabs, as the grouped GEMM reads them, and
row-major)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import host, kstage_sf_to_rowmajor, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def run(ids, E, K, seed=0, sf_layout=nv.SF_KSTAGE):
    T, k = ids.shape
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, size=(T, K // 2), dtype=np.uint8)
    sf = rng.integers(0, 256, size=(T, K // 16), dtype=np.uint8)
    out = nv.permute(torch.from_numpy(ids).cuda(), torch.from_numpy(q).cuda(), torch.from_numpy(sf).cuda(), E,
                     sf_layout=sf_layout)
    assert nv.device_status() == 0
    off, src, inv = oracle.permute(ids, E)
    assert np.array_equal(host(out.offsets), off)
    assert np.array_equal(host(out.perm_src), src)
    assert np.array_equal(host(out.inv_perm), inv)
    assert np.array_equal(host(out.q_perm), oracle.gather_rows(q, src))
    sf_perm = host(out.sf_perm)
    if sf_layout == nv.SF_KSTAGE:
        assert sf_perm.shape == ((K + 255) // 256, T * k, 16)
        sf_perm = kstage_sf_to_rowmajor(sf_perm, T * k, K)
    assert np.array_equal(sf_perm, oracle.gather_rows(sf, src))


@pytest.mark.parametrize("name", ["moe_decode_t512", "moe_zipf_t1024", "moe_prefill_t8192"])
def test_workload_routing(name):
    ids, _ = workloads.config_routing(name)
    run(ids, 256, 6144 if name != "moe_prefill_t8192" else 256)


@pytest.mark.parametrize("T,E,k,kind", [(1, 4, 1, "uniform"), (37, 5, 3, "uniform"), (300, 1024, 8, "zipf"),
                                        (257, 64, 16, "uniform"), (513, 3, 2, "zipf"),
                                        (5000, 1024, 8, "zipf")])   # > 32768 pairs: the multi-kernel path
def test_ragged_shapes(T, E, k, kind):
    # up to 32768 pairs (and 160 KB of rank tables) one CTA ranks every pair; beyond, four kernels do
    ids, _ = workloads.routing(T, E, k, kind, seed=T)
    run(ids, E, 256, seed=T)


@pytest.mark.parametrize("T,E,k,K", [(37, 5, 3, 768), (300, 64, 8, 2048), (37, 5, 3, 128), (129, 16, 4, 384)])
def test_scale_layouts(T, E, k, K):
    # several K steps, so the K-stage slabs and the row-major rows differ; both layouts from one routing
    ids, _ = workloads.routing(T, E, k, "uniform", seed=T)
    run(ids, E, K, seed=T, sf_layout=nv.SF_KSTAGE)
    run(ids, E, K, seed=T, sf_layout=nv.SF_ROWMAJOR)


def test_invalid_and_duplicate_ids_latch_status():
    ids = np.array([[0, 1], [2, 7]], dtype=np.int32)       # 7 >= E
    q = torch.zeros((2, 128), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((2, 16), dtype=torch.uint8, device="cuda")
    nv.permute(torch.from_numpy(ids).cuda(), q, sf, 4)
    assert nv.device_status() == 8
    ids = np.array([[1, 1], [2, 3]], dtype=np.int32)       # expert listed twice by token 0
    nv.permute(torch.from_numpy(ids).cuda(), q, sf, 4)
    assert nv.device_status() == 8
    assert nv.device_status() == 0                          # reading clears the word
