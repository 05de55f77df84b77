"""Seeded workload recipe checks (CPU)."""
import numpy as np
import torch

import oracle as O
import workloads as W


def test_shapes_and_determinism():
    wl = W.WORKLOADS["tiny_fp32"]
    a = W.make_inputs(wl)
    b = W.make_inputs(wl)
    assert a["x"].shape == (64, 64) and a["x"].dtype == torch.float32
    assert a["W_g"].shape == (4, 64)
    assert a["W1"].shape == (4, 128, 64) and a["W2"].shape == (4, 64, 128)
    assert a["b1"].shape == (4, 128) and a["b2"].shape == (4, 64)
    assert a["W3"] is None and a["b_e"] is None
    for key in a:
        if a[key] is not None:
            assert torch.equal(a[key], b[key]), key


def test_bf16_values_are_rounded_once():
    wl = W.WORKLOADS["gpt2_moe"].scaled(N=32, d_model=64, d_ff=128)
    x = W.make_x(wl)
    assert x.dtype == torch.bfloat16
    xf = x.float()
    # LayerNorm'd rows: mean ~0, variance ~1 before rounding
    assert torch.all(xf.mean(dim=1).abs() < 0.05)
    assert torch.all((xf.var(dim=1, unbiased=False) - 1).abs() < 0.05)


def test_deepseek_bias_range():
    wl = W.WORKLOADS["deepseek_v3"]
    b = W.make_router(wl)["b_e"]
    assert b.shape == (256,) and b.dtype == torch.float32
    assert float(b.min()) >= -0.1 and float(b.max()) <= 0.1


def test_qwen3_skew_recipe():
    """Top expert picked by ~40% of tokens; >= 20 experts with 0-4 tokens."""
    wl = W.WORKLOADS["qwen3_skew"]
    x = W.make_x(wl).float().numpy()
    Wg = W.make_router(wl)["W_g"].float().numpy()
    r = O.route(x, Wg, wl.k)
    ids = r["ids"]
    token_frac = np.array([(ids == e).any(axis=1).mean() for e in range(wl.E)])
    counts = np.bincount(ids.reshape(-1), minlength=wl.E)
    assert abs(token_frac.max() - 0.40) <= 0.01, token_frac.max()
    assert int((counts <= 4).sum()) >= 20, counts
