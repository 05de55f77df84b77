"""The data-parallel Switch loss through the C ABI (marked gpu).

Course module sec. 2.3 (f_e and P_e are averages over the whole batch) and
sec. 2.5 (the sign rule on the whole batch's load).  A batch is split into
parts that run as separate moe_forward_partials calls, as the ranks of a
data-parallel group would; their counts and probability sums are added
(the all-reduce's sum, done here with torch on one device) and
moe_aux_from_partials must give the oracle's whole-batch loss (1e-5) and
sign-rule step (1e-7).  DataParallelMoE on one NCCL rank must equal
moe_forward.
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import mixture_experts_layer_53_b200 as M
import oracle as O
import workloads as W
from mixture_experts_layer_53_b200 import dp as DP
from parity import MARGIN, TOL_AUX, config_of, gpu_forward, np64

pytestmark = pytest.mark.gpu

CASES = {
    # E <= 32: one-CTA scan; E > 32: per-expert scan columns
    "mixtral_small": (W.WORKLOADS["mixtral"].scaled(N=333, d_model=256, d_ff=256), (100, 200, 33)),
    "deepseek_small": (W.WORKLOADS["deepseek_v3"].scaled(N=256, d_model=384, d_ff=128, E=64), (128, 128)),
    "qwen3_small": (W.WORKLOADS["qwen3_skew"].scaled(N=512, d_model=256, d_ff=128), (31, 481)),
    "gpt2_one_part": (W.WORKLOADS["gpt2_moe"].scaled(N=130, d_model=128, d_ff=256), (130,)),
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_layer_53_b200 import build
    build.build()
    M.library()


def _part(inp, lo, hi):
    part = dict(inp)
    part["x"] = inp["x"][lo:hi].contiguous()
    return part


@pytest.mark.parametrize("name", sorted(CASES))
def test_loss_from_partials_matches_whole_batch(name):
    wl, parts = CASES[name]
    assert sum(parts) == wl.N
    inp = W.make_inputs(wl, "cuda")
    b0 = None if inp["b_e"] is None else inp["b_e"].clone()
    counts = torch.zeros(wl.E, dtype=torch.int32, device="cuda")
    psum = torch.zeros(wl.E, dtype=torch.float64, device="cuda")
    ids, lo = [], 0
    for n in parts:
        cfg = config_of(wl.scaled(N=n))
        p = _part(inp, lo, lo + n)
        out = M.moe_forward_partials(cfg, p["x"], p["W_g"], p["W1"], p["W2"], W3=p["W3"], b1=p["b1"], b2=p["b2"],
                                     b_e=inp["b_e"])
        # the same rows as a stand-alone forward of the part, bit for bit
        ref = M.moe_forward(cfg, p["x"], p["W_g"], p["W1"], p["W2"], W3=p["W3"], b1=p["b1"], b2=p["b2"],
                            b_e=None if inp["b_e"] is None else inp["b_e"].clone())
        torch.cuda.synchronize()
        assert int(out["status"][0]) == 0
        assert torch.equal(out["y"], ref["y"]) and torch.equal(out["topk_ids"], ref["topk_ids"])
        assert torch.equal(out["counts"], ref["counts"])
        counts += out["counts"]
        psum += out["psum"]
        ids.append(out["topk_ids"].cpu().numpy())
        lo += n
    if b0 is not None:
        assert torch.equal(inp["b_e"], b0), "moe_forward_partials moved the selection bias"
    b = None if inp["b_e"] is None else inp["b_e"].clone()
    aux = M.moe_aux_from_partials(wl.E, wl.k, counts, psum, gamma=wl.gamma, b_e=b)
    torch.cuda.synchronize()

    # the oracle on the whole batch, with the CUDA ids where the choice was a near-tie
    ids = np.concatenate(ids)
    bsel = None if b0 is None else np64(b0)
    r = O.route(np64(inp["x"]), np64(inp["W_g"]), wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=bsel)
    near = r["margin"] < MARGIN
    assert np.array_equal(ids[~near], r["ids"][~near])
    rf = O.route(np64(inp["x"]), np64(inp["W_g"]), wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=bsel,
                 forced_ids=ids, forced=near.astype(np.uint8))
    L_o, counts_o = O.aux_loss(rf["probs"], ids)
    assert np.array_equal(counts.cpu().numpy(), counts_o)
    assert abs(float(aux[0]) - L_o) <= TOL_AUX, (float(aux[0]), L_o)
    # the probability sums themselves, against the oracle's fp64 sums (fp32 p per token)
    assert np.max(np.abs(psum.cpu().numpy() - rf["probs"].sum(axis=0))) <= 1e-6 * wl.N
    if b is not None and wl.gamma > 0:
        want = O.bias_update(np64(b0), counts_o, wl.N, wl.k, wl.gamma)
        assert np.max(np.abs(b.cpu().numpy() - want)) <= 1e-7


def test_finalizer_checks_arguments():
    c = torch.zeros(8, dtype=torch.int32, device="cuda")
    p = torch.zeros(8, dtype=torch.float64, device="cuda")
    lib = M.library()
    P = M._ptr
    a = torch.empty(1, dtype=torch.float32, device="cuda")
    assert lib.moe_aux_from_partials(8, 9, P(c), P(p), P(a), 0.0, None, None) == 1   # k > E
    assert lib.moe_aux_from_partials(300, 2, P(c), P(p), P(a), 0.0, None, None) == 2  # E > 256
    assert lib.moe_aux_from_partials(8, 2, P(c), P(p), None, 0.0, None, None) == 1   # no output
    assert lib.moe_aux_from_partials(8, 2, P(c), P(p), P(a), -1.0, None, None) == 1  # gamma < 0
    assert lib.moe_aux_from_partials(8, 2, P(c), P(p), P(a), 0.0, None, None) == 0
    torch.cuda.synchronize()
    assert float(a[0]) == 0.0  # no assignments: empty sums


@pytest.fixture(scope="module")
def one_rank():
    torch.cuda.set_device(0)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("name", ["deepseek_small", "mixtral_small"])
def test_data_parallel_layer_on_one_rank(one_rank, name):
    wl, _ = CASES[name]
    inp = W.make_inputs(wl, "cuda")
    ref = gpu_forward(wl, inp, z_loss=False)  # moe_forward, b_e moved by its own step
    b = None if inp["b_e"] is None else inp["b_e"].clone()
    layer = DP.DataParallelMoE(config_of(wl), gamma=wl.gamma)
    y, aux, counts = layer.forward(inp["x"], inp["W_g"], inp["W1"], inp["W2"], W3=inp["W3"], b1=inp["b1"],
                                   b2=inp["b2"], b_e=b)
    torch.cuda.synchronize()
    assert np.array_equal(np64(y), ref["y"])
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert abs(float(aux[0]) - float(ref["aux"][0])) <= 1e-6 * max(1.0, abs(float(ref["aux"][0])))
    if b is not None:
        assert np.array_equal(b.cpu().numpy(), ref["b_e_after"])
