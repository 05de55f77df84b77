"""The expert-parallel forward (mixture_experts_layer_53_b200.ep) with the
library's kernels on one GPU.

* Several ranks emulated in one process: each rank routes and dispatches
  its own tokens, the all-to-alls are done by concatenating the row blocks
  the ranks would send each other, and each rank's experts run on the rows
  it would receive (the regroup is then not the identity).  Every expert
  output row and every rank's y and Switch loss are compared with the fp64
  oracle (course module "Going further": experts on different devices,
  tokens moved by all-to-all; the sec. 2.2 forward is unchanged by where
  the experts live).
* One NCCL rank: the exchanges are all-to-alls with the rank itself, and
  the output must equal moe_forward's bit for bit.
Ranks on several GPUs need more than one GPU; their exchange logic runs on
gloo ranks in tests/test_ep.py.
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import mixture_experts_layer_53_b200 as M
import oracle as O
import workloads as W
from mixture_experts_layer_53_b200 import ep as EP
from parity import MARGIN, TOL_AUX, TOL_Y, config_of, gpu_forward, np64

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


@pytest.mark.parametrize("name,world", [("mixtral_pairs", 2), ("gpt2_gelu_biases", 3), ("deepseek_sigmoid_bias", 4),
                                        ("mixtral_single_cta", 4)])
def test_emulated_ranks_match_oracle(name, world):
    from mixture_experts_layer_53_b200 import build
    build.build()
    wl = CASES[name]
    E_r = wl.E // world
    inp = W.make_inputs(wl, "cuda")
    cfg = config_of(wl)
    xs = [W.make_x(wl.scaled(seed=wl.seed + 17 * r)).cuda() for r in range(world)]
    layers = [EP.ExpertParallelMoE(cfg, world=world, rank=r) for r in range(world)]
    st = [layers[r].dispatch_phase(xs[r], inp["W_g"], inp["b_e"]) for r in range(world)]
    counts = [s_.counts.cpu().numpy() for s_ in st]
    # the counts exchange: rank q receives, from every rank s, s's rows per local expert of q
    plans = [EP.plan(counts[q], np.stack([counts[s_][q * E_r:(q + 1) * E_r] for s_ in range(world)]), world)
             for q in range(world)]
    send_start = [np.concatenate([[0], np.cumsum(plans[s_].send_rows)]) for s_ in range(world)]
    recv_start = [np.concatenate([[0], np.cumsum(plans[q].recv_rows)]) for q in range(world)]
    assert any(not np.array_equal(p.regroup, np.arange(len(p.regroup))) for p in plans), "regroup is the identity"

    def local(t, q):
        return None if t is None else t[q * E_r:(q + 1) * E_r].contiguous()

    y_recv = []
    worst_row = 0.0
    for q in range(world):
        # the rows rank q receives: from each source in rank order, its block for q's experts
        x_recv = torch.cat([st[s_].x_sorted[send_start[s_][q]:send_start[s_][q + 1]] for s_ in range(world)])
        yr = layers[q].expert_phase(x_recv, plans[q], local(inp["W1"], q), local(inp["W2"], q),
                                    W3=local(inp["W3"], q), b1=local(inp["b1"], q), b2=local(inp["b2"], q))
        torch.cuda.synchronize()
        # every received row through its expert, against the oracle
        xr, yr64 = np64(x_recv), np64(yr)
        row = 0
        for s_ in range(world):
            for j in range(E_r):
                e = q * E_r + j
                ew = [None if inp[k_] is None else np64(inp[k_][e]) for k_ in ("W1", "W2", "W3", "b1", "b2")]
                for _ in range(int(counts[s_][e])):
                    ref = O.expert_ffn(xr[row], ew[0], ew[1], wl.act, ew[3], ew[2], ew[4])
                    worst_row = max(worst_row, float(np.max(np.abs(yr64[row] - ref)) / max(np.max(np.abs(ref)), 1e-30)))
                    row += 1
        assert row == x_recv.shape[0]
        y_recv.append(yr)
    assert worst_row <= TOL_Y[wl.dtype], worst_row

    b = None if inp["b_e"] is None else np64(inp["b_e"])
    for s_ in range(world):
        # the reverse exchange: rank s gets back its block from every rank, in rank order
        y_sorted = torch.cat([y_recv[q][recv_start[q][s_]:recv_start[q][s_ + 1]] for q in range(world)])
        y, aux = layers[s_].combine_phase(st[s_], y_sorted)
        torch.cuda.synchronize()
        x64 = np64(xs[s_])
        ids = st[s_].ids.cpu().numpy()
        r = O.route(x64, np64(inp["W_g"]), wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=b)
        near = r["margin"] < MARGIN
        assert np.array_equal(ids[~near], r["ids"][~near])
        rf = O.route(x64, np64(inp["W_g"]), wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=b,
                     forced_ids=ids, forced=near.astype(np.uint8))
        y_o = O.dense_forward(x64, ids, rf["w"], np64(inp["W1"]), np64(inp["W2"]), wl.act, np64(inp["W3"]),
                              np64(inp["b1"]), np64(inp["b2"]))
        denom = np.max(np.abs(y_o), axis=1)
        err = float(np.max(np.max(np.abs(np64(y) - y_o), axis=1) / np.where(denom > 0, denom, 1.0)))
        assert err <= TOL_Y[wl.dtype], (s_, err)
        L_o, _ = O.aux_loss(rf["probs"], ids)
        assert abs(float(aux[0]) - L_o) <= TOL_AUX
