"""The expert-parallel layer on the GPU with one rank (NCCL, world size 1): every kernel of its path runs
(amax, quantise from the amax, both permutes, both GEMMs with the amax side output, the k = 1 regrouping
combine and the top-k combine) and the result must equal moe_layer_nvfp4 bit for bit. Ranks on several
GPUs are covered by the CPU tests of the exchange (tests/test_expert_parallel_cpu.py); one GPU cannot host
several ranks whose collectives wait on one another."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import nvfp4_block_scaled_09_b200 as nv
import workloads
from nvfp4_block_scaled_09_b200 import expert_parallel as ep
from tests.helpers import require_gpu

pytestmark = pytest.mark.gpu


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture(scope="module")
def group():
    require_gpu()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=datetime.timedelta(seconds=60))
    yield dist.group.WORLD
    dist.destroy_process_group()


@pytest.mark.parametrize("T,E,k,routing", [(64, 8, 2, "uniform"), (200, 16, 4, "zipf")])
def test_world1_equals_single_gpu_layer(group, T, E, k, routing):
    H, I = 256, 256
    dev = torch.device("cuda", 0)
    w13 = nv.prepare_expert_weights(workloads.normal_bf16((E, 2 * I, H), 0.02, 0, workloads.TAG_W13, device=dev))
    w2 = nv.prepare_expert_weights(workloads.normal_bf16((E, H, I), 0.02, 0, workloads.TAG_W2, device=dev))
    weights = nv.MoEWeights(w13, w2)
    x = workloads.normal_bf16((T, H), 1.0, 3, workloads.TAG_X, device=dev)
    ids, w = workloads.routing(T, E, k, routing, seed=4)
    ids_d, w_d = torch.from_numpy(ids).to(dev), torch.from_numpy(w).to(dev)
    out_ep = ep.ep_moe_layer(x, ids_d, w_d, weights, E, group=group)
    out_ref = nv.moe_layer(x, ids_d, w_d, weights)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    assert torch.equal(out_ep.view(torch.int16), out_ref.view(torch.int16))
