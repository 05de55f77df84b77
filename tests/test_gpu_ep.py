"""The expert-parallel forward (mixture_experts_layer_53_b200.ep) with the
library's kernels, on one GPU as one NCCL rank: the exchanges are NCCL
all-to-alls with the rank itself and the regroup is the identity, so the
output must equal moe_forward's bit for bit (the same route, dispatch,
expert GEMM tile rule and combine).  Ranks on several GPUs need more than
one GPU; their exchange logic runs on gloo ranks in tests/test_ep.py.
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import mixture_experts_layer_53_b200 as M
import workloads as W
from mixture_experts_layer_53_b200 import ep as EP
from parity import config_of, gpu_forward, np64

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral_single_cta": W.WORKLOADS["mixtral"].scaled(N=300, d_model=256, d_ff=384),
    "mixtral_pairs": W.WORKLOADS["mixtral"].scaled(N=1100, d_model=320, d_ff=384),
    "gpt2_gelu_biases": W.WORKLOADS["gpt2_moe"].scaled(N=130, d_model=128, d_ff=256),
    "deepseek_sigmoid_bias": W.WORKLOADS["deepseek_v3"].scaled(N=128, d_model=192, d_ff=64, E=64),
}


@pytest.fixture(scope="module")
def one_rank():
    from mixture_experts_layer_53_b200 import build
    build.build()
    M.library()
    torch.cuda.set_device(0)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(CASES))
def test_single_rank_matches_forward(one_rank, name):
    wl = CASES[name]
    inp = W.make_inputs(wl, "cuda")
    ref = gpu_forward(wl, inp, z_loss=False)
    layer = EP.ExpertParallelMoE(config_of(wl))
    y, aux = layer.forward(inp["x"], inp["W_g"], inp["W1"], inp["W2"], W3=inp["W3"], b1=inp["b1"], b2=inp["b2"],
                           b_e=inp["b_e"])
    torch.cuda.synchronize()
    assert np.array_equal(np64(y), ref["y"]), "expert-parallel output differs from moe_forward"
    assert abs(float(aux[0]) - float(ref["aux"][0])) <= 1e-6 * max(1.0, abs(float(ref["aux"][0])))


def test_configuration_checks(one_rank):
    wl = W.WORKLOADS["mixtral"].scaled(N=8, d_model=64, d_ff=64)
    layer = EP.ExpertParallelMoE(config_of(wl))
    assert layer.E_r == wl.E  # one rank holds every expert
    with pytest.raises(ValueError):  # the shared expert is not exchanged
        EP.ExpertParallelMoE(config_of(W.WORKLOADS["mixtral"].scaled(N=8, d_model=64, d_ff=64, d_ff_shared=64)))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_permute_rows(dtype):
    g = torch.Generator().manual_seed(11)
    rows, d = 301, 136
    src = torch.randn((rows, d), generator=g).to(dtype).cuda()
    dst_row = torch.randperm(rows, generator=g).to(torch.int32)
    dst_row[5] = rows + 3  # out of range: source row 5 is not copied
    out = torch.full((rows, d), 7.0, dtype=dtype, device="cuda")
    M.moe_permute_rows(src, dst_row.cuda(), out=out)
    torch.cuda.synchronize()
    want = torch.full((rows, d), 7.0, dtype=dtype)
    keep = torch.arange(rows) != 5
    want[dst_row[keep].long()] = src.cpu()[keep]
    assert torch.equal(out.cpu(), want)
