"""moe_unpermute_combine on the GPU against the oracle (FP64 sum, BF16-rounded)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import combine_band, compare_bf16, gpu_bf16, host, host_bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("T,E,k,H", [(1, 4, 1, 8), (37, 8, 4, 256), (512, 256, 8, 6144), (1024, 256, 8, 6144),
                                     (70000, 16, 2, 16)])   # more tokens than one grid dimension holds
def test_combine_parity(T, E, k, H):
    ids, w = workloads.routing(T, E, k, "uniform", seed=T)
    _, _, inv = oracle.permute(ids, E)
    y = workloads.random_bf16_bits((T * k, H), seed=T + 1)
    out = nv.unpermute_combine(gpu_bf16(y), torch.from_numpy(inv).cuda(), torch.from_numpy(w).cuda())
    exact = oracle.combine(y, inv, w)
    ref = oracle.bf16_round(exact)
    compare_bf16(host_bits(out), ref, "combine", exact=exact, band=combine_band(y, inv, w))
    # FP64 accumulation of exact products in the oracle's order: bit-identical
    assert np.array_equal(host_bits(out), ref)


def test_one_hot_weights_select_rows_exactly():
    T, E, k, H = 16, 8, 4, 64
    ids, _ = workloads.routing(T, E, k, "uniform", seed=3)
    _, _, inv = oracle.permute(ids, E)
    y = workloads.random_bf16_bits((T * k, H), seed=4)
    w = np.zeros((T, k), dtype=np.float32)
    w[:, 1] = 1.0
    out = nv.unpermute_combine(gpu_bf16(y), torch.from_numpy(inv).cuda(), torch.from_numpy(w).cuda())
    assert np.array_equal(host_bits(out), y[inv.reshape(T, k)[:, 1]])


def test_combine_chunked_rows_and_skipped_slots():
    # k = 32 rows of 4000 columns do not fit one shared-memory stage: 1536-column chunks with a ragged last
    # chunk (928 columns); slots marked -1 are skipped
    T, E, k, H = 40, 64, 32, 4000
    ids, w = workloads.routing(T, E, k, "uniform", seed=9)
    _, _, inv = oracle.permute(ids, E)
    inv = inv.copy()
    inv[::7] = -1
    y = workloads.random_bf16_bits((T * k, H), seed=10)
    out = nv.unpermute_combine(gpu_bf16(y), torch.from_numpy(inv).cuda(), torch.from_numpy(w).cuda())
    assert nv.device_status() == 0
    assert np.array_equal(host_bits(out), oracle.bf16_round(oracle.combine(y, inv, w)))


def test_combine_row_index_past_y_is_skipped_and_latched():
    T, E, k, H = 16, 8, 4, 256
    ids, w = workloads.routing(T, E, k, "uniform", seed=11)
    _, _, inv = oracle.permute(ids, E)
    y = workloads.random_bf16_bits((T * k, H), seed=12)
    bad = inv.copy()
    bad[5] = T * k + 3                                     # past the last row of y
    out = nv.unpermute_combine(gpu_bf16(y), torch.from_numpy(bad).cuda(), torch.from_numpy(w).cuda())
    assert nv.device_status() == 8                         # NVFP4_ERR_DEVICE_INPUT
    skipped = inv.copy()
    skipped[5] = -1
    assert np.array_equal(host_bits(out), oracle.bf16_round(oracle.combine(y, skipped, w)))
