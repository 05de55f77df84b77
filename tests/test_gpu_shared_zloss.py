"""Shared expert and router z-loss on the GPU against the fp64 oracle.

Course module sec. 2.1 (y_n = routed sum + Shared(x_n)); "nano-moe",
"Router z-loss" (mean over tokens of the squared log-sum-exp of the logits).
The shared-expert checks run through moe_forward_ex and through the staged
entry points (moe_shared_ffn, moe_combine_shared), which must agree bit for
bit: they launch the same kernels on the same data.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_53_b200 as M
import oracle as O
import workloads as W
from parity import TOL_Z, check_forward, config_of, gpu_forward, np64, oracle_routing, sample_tokens

pytestmark = pytest.mark.gpu

DEV = "cuda"

SHARED = {
    # fp32 SIMT path, GELU with biases, ragged
    "fp32_gelu_bias": W.WORKLOADS["tiny_fp32"].scaled(N=150, d_model=72, d_ff=136, E=5, k=3, d_ff_shared=88),
    # bf16, <= 192 tokens: 128-row tiles for the shared slice
    "bf16_swiglu_single": W.WORKLOADS["mixtral"].scaled(N=160, d_model=256, d_ff=384, d_ff_shared=512),
    # bf16, > 192 tokens: CTA-pair tiles for the shared slice; routed slices single
    "bf16_swiglu_pair": W.WORKLOADS["deepseek_v3_shared"].scaled(N=700, d_model=384, d_ff=256, E=64,
                                                                  d_ff_shared=256),
    # bf16 GELU with biases, ragged widths, pair tiles on both
    "bf16_gelu_ragged": W.WORKLOADS["gpt2_moe"].scaled(N=777, d_model=200, d_ff=328, E=3, d_ff_shared=136),
    "one_token": W.WORKLOADS["mixtral"].scaled(N=1, d_model=128, d_ff=256, d_ff_shared=128),
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_layer_53_b200 import build
    build.build()
    M.library()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("name", sorted(SHARED))
def test_forward_with_shared_expert(name):
    wl = SHARED[name]
    inp = W.make_inputs(wl, DEV)
    assert inp["shared"] is not None
    gpu = gpu_forward(wl, inp)
    rep = check_forward(wl, inp, gpu)
    print(name, rep.as_dict())


def test_shared_expert_full_size_deepseek():
    wl = W.WORKLOADS["deepseek_v3_shared"]
    inp = W.make_inputs(wl, DEV)
    gpu = gpu_forward(wl, inp)
    rep = check_forward(wl, inp, gpu, y_tokens=sample_tokens(wl.N, 4, seed=5))
    print(wl.name, rep.as_dict())


def test_shared_expert_changes_the_output():
    """The shared part is really added: zeroing its W2 gives the routed-only layer."""
    wl = SHARED["bf16_swiglu_pair"]
    inp = W.make_inputs(wl, DEV)
    with_shared = gpu_forward(wl, inp)["y"]
    zero = dict(inp["shared"])
    zero["W2"] = torch.zeros_like(zero["W2"])
    routed_only = gpu_forward(wl, dict(inp, shared=zero))["y"]
    plain = gpu_forward(wl.scaled(d_ff_shared=0), dict(inp, shared=None), z_loss=False)["y"]
    assert np.array_equal(routed_only, plain)
    assert np.max(np.abs(with_shared - plain)) > 1e-3


@pytest.mark.parametrize("name", ["fp32_gelu_bias", "bf16_swiglu_pair", "bf16_gelu_ragged"])
def test_staged_shared_path_matches_forward(name):
    wl = SHARED[name]
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    ws = M.workspace(cfg, DEV)
    b_e = inp["b_e"]
    ids, w, _ = M.moe_route(cfg, inp["x"], inp["W_g"], b_e, ws=ws)
    dp = M.moe_dispatch(cfg, ids, inp["x"], ws=ws)
    ys = M.moe_expert_ffn(cfg, dp["x_sorted"], dp["offsets"], inp["W1"], inp["W2"], b1=inp["b1"], W3=inp["W3"],
                          b2=inp["b2"], ws=ws)
    ysh = M.moe_shared_ffn(cfg, inp["x"], inp["shared"], ws=ws)
    y = M.moe_combine_shared(cfg, ys, w, dp["inv_perm"], ysh)
    y_plain = M.moe_combine(cfg, ys, w, dp["inv_perm"])
    out = M.moe_forward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], W3=inp["W3"], b1=inp["b1"],
                        b2=inp["b2"], b_e=None if b_e is None else b_e.clone(), gamma=0.0, shared=inp["shared"])
    torch.cuda.synchronize()
    assert torch.equal(y, out["y"])
    # the shared output itself against the oracle (every token)
    sh = inp["shared"]
    want = O.shared_add(np.zeros((wl.N, wl.d_model)), np64(inp["x"]), np64(sh["W1"]), np64(sh["W2"]), wl.act,
                        np64(sh["W3"]), np64(sh["b1"]), np64(sh["b2"]))
    got = np64(ysh)
    denom = np.maximum(np.max(np.abs(want), axis=1), 1e-30)
    err = float(np.max(np.max(np.abs(got - want), axis=1) / denom))
    assert err <= (1e-5 if wl.dtype == "f32" else 2e-2), err
    # y_shared NULL is the plain combine
    assert torch.equal(M.moe_combine_shared(cfg, ys, w, dp["inv_perm"], None), y_plain)


Z_CASES = {
    "fp32": W.WORKLOADS["tiny_fp32"].scaled(N=333, d_model=72, d_ff=136, E=5, k=3),
    "bf16_mixtral_small": W.WORKLOADS["mixtral"].scaled(N=200, d_model=512, d_ff=768),
    "bf16_deepseek_small": W.WORKLOADS["deepseek_v3"].scaled(N=256, d_model=384, d_ff=256, E=64),
    "bf16_qwen3_small": W.WORKLOADS["qwen3_skew"].scaled(N=512, d_model=256, d_ff=128),
    # logits of size ~100: exp overflows fp32 without the max shift
    "fp32_large_logits": W.WORKLOADS["tiny_fp32"].scaled(N=100, x_std=1.0, w_std=15.0),
    "bf16_large_logits": W.WORKLOADS["gpt2_moe"].scaled(N=300, d_model=256, d_ff=256, x_std=1.0, w_std=6.0,
                                                        x_dist="normal"),
}


@pytest.mark.parametrize("name", sorted(Z_CASES))
def test_router_z_loss(name):
    wl = Z_CASES[name]
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    z_alone = M.moe_router_z_loss(cfg, inp["x"], inp["W_g"])
    gpu = gpu_forward(wl, inp)
    z_o = O.z_loss(oracle_routing(wl, inp)["logits"])
    assert abs(float(gpu["z"][0]) - z_o) <= TOL_Z * max(1.0, abs(z_o)), (gpu["z"][0], z_o)
    # same kernels, same order: the standalone entry point gives the same bits
    assert float(z_alone.cpu()[0]) == float(gpu["z"][0])
    if "large" in name:
        assert z_o > 1e3  # the case really exercises big logits


@pytest.mark.parametrize("name", ["mixtral", "qwen3_skew"])
def test_router_z_loss_full_size(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, DEV)
    z = float(M.moe_router_z_loss(config_of(wl), inp["x"], inp["W_g"]).cpu()[0])
    z_o = O.z_loss(oracle_routing(wl, inp)["logits"])
    assert abs(z - z_o) <= TOL_Z * max(1.0, abs(z_o)), (z, z_o)


@pytest.mark.parametrize("N", [0, 1, 31, 33])
def test_router_z_loss_edges(N):
    wl = W.WORKLOADS["mixtral"].scaled(N=N, d_model=128, d_ff=256)
    inp = W.make_inputs(wl, DEV)
    z = float(M.moe_router_z_loss(config_of(wl), inp["x"] if N else inp["x"].new_empty((0, 128)),
                                  inp["W_g"]).cpu()[0])
    z_o = O.z_loss(oracle_routing(wl, inp)["logits"]) if N else 0.0
    assert abs(z - z_o) <= TOL_Z * max(1.0, abs(z_o)), (z, z_o)
