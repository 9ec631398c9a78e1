"""moe_route_topk (the router kernel) against the oracle's router.

Integer results (the chosen experts and their order) must match exactly; the
weights are computed in FP64 on both sides and rounded once to FP32, so they
agree to the last bit unless the two FP64 exponentials differ by an ulp right at
an FP32 rounding boundary: the bound is one FP32 ulp. The layer entry point that
takes logits must equal the layer fed with the router's output, bit for bit.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import host, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def check(z, k):
    ids, w = nv.route_topk(torch.from_numpy(z).cuda(), k)
    assert nv.device_status() == 0
    ref_ids, ref_w = oracle.route_topk(z, k)
    got_ids, got_w = host(ids), host(w)
    assert np.array_equal(got_ids, ref_ids)
    diff = np.abs(got_w.astype(np.float64) - ref_w.astype(np.float64))
    ulp = np.spacing(np.abs(ref_w)).astype(np.float64)
    assert np.all(diff <= ulp), float((diff / np.maximum(ulp, 1e-45)).max())
    print(f"[route] T={z.shape[0]} E={z.shape[1]} k={k}: ids exact, weights bit-exact "
          f"{float(np.mean(diff == 0)):.6f}, max {float((diff / np.maximum(ulp, 1e-45)).max()):.1f} ulp")


@pytest.mark.parametrize("name", ["moe_decode_t512", "moe_zipf_t1024", "moe_prefill_t8192"])
def test_router_workloads(name):
    c = workloads.CONFIGS[name]
    z = workloads.router_logits(c["T"], c["E"], c["routing"], 0, c.get("zipf_s", 1.1), c.get("zero_experts", 0))
    check(z.astype(np.float32), c["k"])     # Zipf logits hold -inf for the experts nobody routes to


@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (37, 1024, 32), (19, 8, 8), (64, 33, 1), (300, 1000, 5),
                                   (8, 1, 1)])
def test_router_shapes(T, E, k):
    z = np.random.default_rng(T + E + k).standard_normal((T, E)).astype(np.float32)
    check(z, k)


def test_router_ties_and_infinities():
    rng = np.random.default_rng(4)
    z = rng.integers(-2, 3, size=(500, 256)).astype(np.float32)    # many equal logits
    z[::7, :] = 0.0
    z[::7, 1::2] = -0.0                                              # signed zeros are equal
    z[3, :] = -np.inf                                                # a row of -inf only
    z[5, 10:] = -np.inf                                              # fewer finite logits than k
    check(z, 8)


def test_router_rejects_bad_shapes():
    z = torch.zeros((4, 16), dtype=torch.float32, device="cuda")
    ids = torch.empty((4, 32), dtype=torch.int32, device="cuda")
    w = torch.empty((4, 32), dtype=torch.float32, device="cuda")
    L = nv.lib()
    P = nv.ctypes.c_void_p
    s = P(torch.cuda.current_stream().cuda_stream)
    assert L.moe_route_topk(P(z.data_ptr()), 4, 16, 17, P(ids.data_ptr()), P(w.data_ptr()), s) == 3   # k > E
    assert L.moe_route_topk(P(z.data_ptr()), 4, 1025, 8, P(ids.data_ptr()), P(w.data_ptr()), s) == 3  # E > 1024
    assert L.moe_route_topk(P(z.data_ptr()), 4, 16, 0, P(ids.data_ptr()), P(w.data_ptr()), s) == 1
    assert L.moe_route_topk(P(z.data_ptr() + 2), 4, 16, 4, P(ids.data_ptr()), P(w.data_ptr()), s) == 2


def test_layer_from_logits_equals_layer_on_router_output():
    T, k, E, H, I = 200, 4, 8, 512, 512
    dev = torch.device("cuda", 0)
    z = torch.from_numpy(workloads.router_logits(T, E, "uniform", 3).astype(np.float32)).to(dev)
    x = workloads.normal_bf16((T, H), 1.0, 3, workloads.TAG_X, device=dev)
    w13 = nv.prepare_expert_weights(workloads.normal_bf16((E, 2 * I, H), 0.02, 3, workloads.TAG_W13, device=dev))
    w2 = nv.prepare_expert_weights(workloads.normal_bf16((E, H, I), 0.02, 3, workloads.TAG_W2, device=dev))
    weights = nv.MoEWeights(w13, w2)
    ids, w = nv.route_topk(z, k)
    ref = nv.moe_layer(x, ids, w, weights)
    ws = nv.layer_workspace(T, k, E, H, I, dev)
    got = nv.moe_layer_from_logits(x, z, k, weights, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    lay = nv.layer_workspace_layout(T, k, E, H, I)
    ids_ws = ws[lay["topk_ids"]: lay["topk_ids"] + T * k * 4].view(torch.int32).view(T, k)
    assert torch.equal(ids_ws, ids)
