"""moe_backward on the GPU against the fp64 oracle's backward.

The scalar is <dy, y> + aux_coef L_aux + z_coef L_z (course module sec. 2.1,
2.3 and 2.4; "nano-moe" router z-loss).  The GPU recomputes the routing with
the forward's kernels (bf16: expert products on the tensor cores, fp32: on
the CUDA cores); tokens whose top-k margin is under 1e-4 are replayed
in the oracle with the GPU's choice, as in the forward parity.  Every
gradient is compared normwise: max |g - r| / max |r| per tensor.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_53_b200 as M
import oracle as O
import workloads as W
from parity import MARGIN, config_of, np64

pytestmark = pytest.mark.gpu

DEV = "cuda"
# fp32: every product accumulates in fp32 from inputs the oracle sees exactly (errors are fp32
# rounding).  bf16: the expert products run on the tensor cores, whose operands da, du and w h are
# rounded to bf16 (2^-9 = 1.95e-3 relative per element) before the fp32 accumulation.  Per gradient,
# normwise against max |r|:
#   dW2 = dy_s^T (w h):        one bf16 operand rounding (w h)           -> about 2^-9 of a typical term
#   dW1, dW3 = [da | du]^T x_s: da / du rounded once, and they carry h's recomputation from the
#                              bf16 pre-activations                      -> 2-3 x 2^-9
#   dx = sum_j [da | du] W:    the same da / du roundings                 -> 2-3 x 2^-9
#   dW_g, db: fp32 operands (CUDA-core products)                        -> fp32 rounding
# Measured worst cases are 1.5e-3 .. 2.6e-3; 1e-2 (about 5 x 2^-9) bounds a sum of a few such
# roundings with no cancellation, and is half the forward's bf16 output tolerance of 2e-2.
TOL_G = {"f32": 1e-5, "bf16": 1e-2}

CASES = {
    "fp32_gelu_bias": (W.WORKLOADS["tiny_fp32"].scaled(N=97, d_model=40, d_ff=48, E=5, k=2, x_std=1.0), 0.3, 0.2),
    "fp32_swiglu_shared": (W.WORKLOADS["tiny_fp32"].scaled(N=70, d_model=32, d_ff=40, E=4, k=2, act="swiglu",
                                                           biases=False, x_std=1.0, d_ff_shared=24), 0.5, 0.1),
    "bf16_gpt2_small": (W.WORKLOADS["gpt2_moe"].scaled(N=160, d_model=128, d_ff=256), 0.01, 0.001),
    "bf16_mixtral_small": (W.WORKLOADS["mixtral"].scaled(N=200, d_model=256, d_ff=384), 0.5, 0.1),
    "bf16_topk_softmax": (W.WORKLOADS["gpt2_moe"].scaled(N=130, d_model=128, d_ff=128, E=7, k=3,
                                                         router="topk_softmax"), 0.2, 0.0),
    "bf16_softmax_no_norm": (W.WORKLOADS["qwen3_skew"].scaled(N=96, d_model=128, d_ff=64, E=40, k=4, zipf=False,
                                                              norm_topk=False), 1.0, 0.05),
    "bf16_deepseek_shared": (W.WORKLOADS["deepseek_v3_shared"].scaled(N=128, d_model=192, d_ff=64, E=64,
                                                                      d_ff_shared=64), 0.1, 0.01),
    "bf16_gpt2_shared_bias": (W.WORKLOADS["gpt2_moe"].scaled(N=150, d_model=128, d_ff=128, d_ff_shared=96),
                              0.05, 0.01),
    # more than 192 rows per group: the ragged-M products run on CTA pairs
    # (d_model 320 and d_ff 384 leave partial 256-column tiles)
    "bf16_mixtral_pairs": (W.WORKLOADS["mixtral"].scaled(N=1100, d_model=320, d_ff=384), 0.5, 0.1),
    "bf16_gpt2_shared_pairs": (W.WORKLOADS["gpt2_moe"].scaled(N=420, d_model=128, d_ff=128, d_ff_shared=96),
                               0.05, 0.01),
    "one_token": (W.WORKLOADS["mixtral"].scaled(N=1, d_model=64, d_ff=64), 0.5, 0.5),
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_layer_53_b200 import build
    build.build()
    M.library()
    assert torch.cuda.is_available()


def make_dy(wl):
    g = torch.Generator().manual_seed(wl.seed * 7 + 9)
    return torch.randn((wl.N, wl.d_model), generator=g).to(wl.torch_dtype).to(DEV)


def run_case(wl, aux_coef, z_coef):
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    dy = make_dy(wl)
    out = M.moe_backward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], dy, W3=inp["W3"], b1=inp["b1"],
                         b2=inp["b2"], b_e=inp["b_e"], shared=inp["shared"], aux_coef=aux_coef, z_coef=z_coef)
    ids_g, _, _ = M.moe_route(cfg, inp["x"], inp["W_g"], inp["b_e"])
    torch.cuda.synchronize()
    assert int(out["status"][0]) == 0
    ids_g = ids_g.cpu().numpy()
    b_sel = None if inp["b_e"] is None else np64(inp["b_e"])
    r = O.route(np64(inp["x"]), np64(inp["W_g"]), wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=b_sel)
    near = r["margin"] < MARGIN
    assert np.array_equal(ids_g[~near], r["ids"][~near]), "routing differs away from near-ties"
    sh = inp["shared"]
    ref = O.backward(np64(inp["x"]), np64(inp["W_g"]), wl.k, np64(inp["W1"]), np64(inp["W2"]), np64(dy),
                     wl.router, wl.norm_topk, wl.routed_scaling, wl.act, np64(inp["W3"]), np64(inp["b1"]),
                     np64(inp["b2"]), b_sel, None if sh is None else {kk: np64(v) for kk, v in sh.items()},
                     aux_coef, z_coef, forced_ids=ids_g, forced=near.astype(np.uint8))
    errs = {}
    for key, want in ref.items():
        if want is None:
            continue
        got = out["dW_g" if key == "dWg" else key].cpu().numpy().astype(np.float64)
        scale = max(float(np.max(np.abs(want))), 1e-30)
        errs[key] = float(np.max(np.abs(got - want))) / scale
    return errs, int(near.sum())


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_oracle(name):
    wl, aux_coef, z_coef = CASES[name]
    errs, near = run_case(wl, aux_coef, z_coef)
    print(name, "near-ties", near, {k: f"{v:.2e}" for k, v in errs.items()})
    tol = TOL_G[wl.dtype]
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"gradients off: {bad}"


def test_backward_is_deterministic():
    wl, aux_coef, z_coef = CASES["bf16_mixtral_small"]
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    dy = make_dy(wl)
    a = M.moe_backward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], dy, W3=inp["W3"], aux_coef=aux_coef,
                       z_coef=z_coef)
    b = M.moe_backward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], dy, W3=inp["W3"], aux_coef=aux_coef,
                       z_coef=z_coef)
    torch.cuda.synchronize()
    for key in ("dx", "dW_g", "dW1", "dW3", "dW2"):
        assert torch.equal(a[key], b[key]), key


def test_backward_without_tokens():
    wl = W.WORKLOADS["gpt2_moe"].scaled(N=0, d_model=64, d_ff=64)
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    dy = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    out = M.moe_backward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], dy, b1=inp["b1"], b2=inp["b2"],
                         aux_coef=1.0, z_coef=1.0)
    torch.cuda.synchronize()
    for key in ("dW_g", "dW1", "dW2", "db1", "db2"):
        assert float(out[key].abs().max()) == 0.0, key
