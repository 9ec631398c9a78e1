"""moe_layer_nvfp4 (one call) against the same layer run call by call, at the full decode and prefill
sizes (the launch configurations the bench times: its throughput runs the calls one by one, its end-to-end
figure runs the one-call API). Both must agree bit for bit; each call is checked against the oracle by
the per-call tests, and the whole layer against the oracle stage by stage by smoke()."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import workloads
from tests.helpers import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def layer_weights(E, H, I, dev):
    def build(N, K, tag):
        packed = torch.empty((E, N * (K // 2 + K // 16)), dtype=torch.uint8, device=dev)
        g = torch.empty(E, dtype=torch.float32, device=dev)
        q = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        sf = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
        for e in range(E):
            nv.quantize(workloads.normal_bf16((N, K), 0.02, 0, tag, e, device=dev), q=q, sf=sf, g=g[e:e + 1])
            nv.pack_weights(q, sf, out=packed[e])
        return nv.PackedWeights(packed, g, E, N, K)
    return nv.MoEWeights(build(2 * I, H, workloads.TAG_W13), build(H, I, workloads.TAG_W2))


def staged_layer(x, ids, w, weights, E):
    q, sf, g = nv.quantize(x)
    perm = nv.permute(ids, q, sf, E)
    amax = torch.zeros(1, dtype=torch.int32, device=x.device)
    h = nv.grouped_gemm(perm.q_perm, perm.sf_perm, g, weights.w13, perm.offsets, True, amax_out=amax)
    qh, sfh, gh = nv.quantize_from_amax(h, amax, layout=nv.SF_KSTAGE)
    # the amax side output equals the amax pass of the dynamic quantiser on h
    assert torch.equal(gh, nv.quantize(h)[2])
    y = nv.grouped_gemm(qh, sfh, gh, weights.w2, perm.offsets, False)
    return nv.unpermute_combine(y, perm.inv_perm, w)


@pytest.mark.parametrize("name", ["moe_decode_t512", "moe_prefill_t8192"])
def test_one_call_layer_equals_call_by_call(name):
    cfg = workloads.CONFIGS[name]
    T, H, I, E, k = cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"]
    dev = torch.device("cuda", 0)
    weights = layer_weights(E, H, I, dev)
    ids, w = workloads.config_routing(name)
    x = workloads.normal_bf16((T, H), 1.0, 0, workloads.TAG_X, device=dev)
    ids_d, w_d = torch.from_numpy(ids).to(dev), torch.from_numpy(w).to(dev)
    ws = nv.layer_workspace(T, k, E, H, I, dev)
    out_one = nv.moe_layer(x, ids_d, w_d, weights, ws=ws)
    out_two = nv.moe_layer(x, ids_d, w_d, weights, ws=ws)   # same workspace: its amax word is re-zeroed per call
    out_staged = staged_layer(x, ids_d, w_d, weights, E)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    assert torch.equal(out_one.view(torch.int16), out_staged.view(torch.int16))
    assert torch.equal(out_two.view(torch.int16), out_one.view(torch.int16))
    assert torch.isfinite(out_one.float()).all() and out_one.float().abs().max() > 0


def test_smoke_entry_point_passes():
    # __graft_entry__.smoke(): one small layer against the oracle, stage by stage
    import __graft_entry__
    __graft_entry__.smoke()
