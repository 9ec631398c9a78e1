"""moe_permute_noalloc: the permute entry point for callers that cannot hand
the library device memory (code inside a CUDA stream capture, where cudaMalloc
is not allowed, real-time paths that forbid allocation, frameworks that own all
device memory through a pool they do not expose). It keeps its count table in
the library's fixed device array instead of a caller workspace.

Called here through the C ABI and compared with moe_permute (the workspace
entry point) on the same inputs: the results are integer indices and byte
copies, so they must agree exactly, on two calls in a row (the second call
reuses the array the first one left behind). This file is collected last so a
stop-at-first-failure run has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import workloads
from tests.helpers import host, require_gpu

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def call_noalloc(ids, q, sf, E, K):
    T, k = ids.shape
    R = T * k
    out = {
        "q_perm": torch.empty((R, K // 2), dtype=torch.uint8, device="cuda"),
        "sf_perm": torch.empty((K // 256, R, 16), dtype=torch.uint8, device="cuda"),   # K-stage slabs
        "offsets": torch.empty(E + 1, dtype=torch.int32, device="cuda"),
        "perm_src": torch.empty(R, dtype=torch.int32, device="cuda"),
        "inv_perm": torch.empty(R, dtype=torch.int32, device="cuda"),
    }
    st = nv.lib().moe_permute_noalloc(
        P(ids.data_ptr()), T, k, E, P(q.data_ptr()), P(sf.data_ptr()), K, P(out["q_perm"].data_ptr()),
        P(out["sf_perm"].data_ptr()), nv.SF_KSTAGE, P(out["offsets"].data_ptr()), P(out["perm_src"].data_ptr()),
        P(out["inv_perm"].data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    assert st == 0, nv.status_string(st)
    return out


@pytest.mark.parametrize("name,K", [("moe_decode_t512", 6144), ("moe_zipf_t1024", 256),
                                    ("moe_prefill_t8192", 256)])
def test_noalloc_matches_workspace_entry_point_twice(name, K):
    require_gpu()
    cfg = workloads.CONFIGS[name]
    E = cfg["E"]
    ids_np, _ = workloads.config_routing(name)
    T = ids_np.shape[0]
    rng = np.random.default_rng(7)
    ids = torch.from_numpy(ids_np).cuda()
    q = torch.from_numpy(rng.integers(0, 256, size=(T, K // 2), dtype=np.uint8)).cuda()
    sf = torch.from_numpy(rng.integers(0, 256, size=(T, K // 16), dtype=np.uint8)).cuda()
    ref = nv.permute(ids, q, sf, E)
    for _ in range(2):
        got = call_noalloc(ids, q, sf, E, K)
        assert nv.device_status() == 0
        for field in ("offsets", "perm_src", "inv_perm", "q_perm", "sf_perm"):
            assert np.array_equal(host(got[field]), host(getattr(ref, field))), field


def test_noalloc_rejects_shapes_beyond_its_array():
    require_gpu()
    # ceil(T / 256) * E must fit the fixed array; 65535 tokens x 1024 experts does not
    T, k, E, K = 65535, 1, 1024, 256
    d = P(256)
    st = nv.lib().moe_permute_noalloc(d, T, k, E, d, d, K, d, d, nv.SF_KSTAGE, d, d, d, None)
    assert st == 3, nv.status_string(st)
