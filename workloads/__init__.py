"""Seeded synthetic workloads for the MoE layer forward.

This module is shared by the tests, the benchmark and the smoke check.  It
only draws random inputs (and knows the five workload shapes); it holds none
of the layer's arithmetic -- no routing, no top-k, no expert FFN, no loss.

Workloads (shapes of the pages' models, synthetic values; no dataset and no
trained weights are used):

  tiny_fp32    N=64    d=64   E=4   k=2 GELU   F=128   fp32, biases
  gpt2_moe     N=8192  d=768  E=6   k=2 GELU   F=3072  bf16, biases, LayerNorm'd x
  mixtral      N=4096  d=4096 E=8   k=2 SwiGLU F=14336 bf16
  deepseek_v3  N=4096  d=7168 E=256 k=8 SwiGLU F=2048  bf16, sigmoid + b_e, gamma=1e-3
  qwen3_skew   N=16384 d=2048 E=128 k=8 SwiGLU F=768   bf16, Zipf(1.2) router offsets

Value recipe: weights ~ N(0, 0.02) (router, experts, biases), x ~ N(0, 1)
except tiny_fp32 (x ~ N(0, 0.02)) and gpt2_moe (N(0,1) then a row-wise
LayerNorm without affine, eps 1e-5).  bf16 workloads round every value once,
round-to-nearest-even, and both the CUDA path and the oracle read those same
values.  deepseek_v3 draws b_e ~ U(-0.1, 0.1) in fp32.

qwen3_skew adds a per-expert offset o_e to the router logits.  It is carried
by the inputs themselves: feature 0 of every token is the constant 1 and
column 0 of W_g holds o_e, so z_{n,e} = o_e + (the usual product).  With
experts ranked r = 1..E by a seeded permutation,
    o_e = ALPHA * ln(r_e^-1.2 / sum_r r^-1.2),   and -3 more for the 24
lowest-ranked experts; ALPHA is the fixed constant below, chosen so that the
top expert is picked by about 40% of tokens and at least 20 experts get 0-4
tokens (a CPU test checks both on the generated inputs).

Large expert weights are drawn directly on the target device, one expert at a
time from a per-(tensor, expert) seed, so a 22.5 GB weight set never passes
through host memory.  Everything else is drawn on the CPU (device-independent
values) and copied.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

ZIPF_S = 1.2
ZIPF_ALPHA = 0.256         # logit scale of the Zipf offsets (see module doc)
ZIPF_COLD = 24             # lowest-ranked experts that get an extra offset
ZIPF_COLD_OFFSET = -3.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    d_model: int
    d_ff: int
    E: int
    k: int
    act: str                 # "gelu" | "swiglu"
    router: str              # "softmax_topk" | "topk_softmax" | "sigmoid"
    dtype: str               # "f32" | "bf16"
    norm_topk: bool = True
    routed_scaling: float = 1.0
    biases: bool = False     # b1 and b2 (GELU experts)
    sel_bias: bool = False   # aux-free selection bias b_e
    gamma: float = 0.0       # sign-rule step applied after the forward
    x_dist: str = "normal"   # "normal" | "layernorm"
    x_std: float = 1.0
    w_std: float = 0.02
    zipf: bool = False
    seed: int = 1000
    d_ff_shared: int = 0     # width of the shared expert (0 = none)

    @property
    def mats(self) -> int:
        return 3 if self.act == "swiglu" else 2

    @property
    def expert_flops(self) -> int:
        """Algorithmic FLOPs of the expert FFNs: 2 * mats * d * F per assignment,
        plus 2 * mats * d * Fs per token for the shared expert."""
        return 2 * self.mats * self.d_model * (self.d_ff * self.N * self.k + self.d_ff_shared * self.N)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", N=64, d_model=64, d_ff=128, E=4, k=2, act="gelu",
                          router="softmax_topk", dtype="f32", biases=True, x_std=0.02, seed=1000),
    "gpt2_moe": Workload("gpt2_moe", N=8192, d_model=768, d_ff=3072, E=6, k=2, act="gelu",
                         router="softmax_topk", dtype="bf16", biases=True, x_dist="layernorm",
                         seed=1001),
    "mixtral": Workload("mixtral", N=4096, d_model=4096, d_ff=14336, E=8, k=2, act="swiglu",
                        router="softmax_topk", dtype="bf16", seed=1002),
    "deepseek_v3": Workload("deepseek_v3", N=4096, d_model=7168, d_ff=2048, E=256, k=8,
                            act="swiglu", router="sigmoid", dtype="bf16", sel_bias=True,
                            gamma=1e-3, seed=1003),
    "qwen3_skew": Workload("qwen3_skew", N=16384, d_model=2048, d_ff=768, E=128, k=8,
                           act="swiglu", router="softmax_topk", dtype="bf16", zipf=True, seed=1004),
    # DeepSeek-V3 as the course module's router table describes it: one
    # shared expert of the routed width beside the 256 routed ones, and
    # routed_scaling 2.5 (beyond the five configurations above)
    "deepseek_v3_shared": Workload("deepseek_v3_shared", N=4096, d_model=7168, d_ff=2048, E=256, k=8,
                                   act="swiglu", router="sigmoid", dtype="bf16", sel_bias=True,
                                   gamma=1e-3, routed_scaling=2.5, d_ff_shared=2048, seed=1005),
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_offsets(wl: Workload) -> torch.Tensor:
    """Per-expert logit offsets o_e (fp32, [E]) of the skewed workload."""
    g = _gen(wl.seed * 7 + 5)
    ranks = torch.randperm(wl.E, generator=g) + 1            # rank of expert e
    r = torch.arange(1, wl.E + 1, dtype=torch.float64)
    z = torch.sum(r ** (-ZIPF_S))
    o = ZIPF_ALPHA * torch.log(ranks.double() ** (-ZIPF_S) / z)
    o = torch.where(ranks > wl.E - ZIPF_COLD, o + ZIPF_COLD_OFFSET, o)
    return o.float()


def make_x(wl: Workload) -> torch.Tensor:
    """Token activations [N, d] in the workload's dtype (on the CPU)."""
    g = _gen(wl.seed * 7 + 1)
    x = torch.randn((wl.N, wl.d_model), generator=g, dtype=torch.float32) * wl.x_std
    if wl.x_dist == "layernorm" and wl.N > 0:  # an empty batch has no rows to normalise
        mu = x.mean(dim=1, keepdim=True)
        var = x.var(dim=1, unbiased=False, keepdim=True)
        x = (x - mu) / torch.sqrt(var + 1e-5)
    if wl.zipf:
        x[:, 0] = 1.0
    return x.to(wl.torch_dtype)


def make_router(wl: Workload) -> Dict[str, Optional[torch.Tensor]]:
    """W_g [E, d] (workload dtype) and the selection bias b_e [E] fp32 or None."""
    g = _gen(wl.seed * 7 + 2)
    Wg = torch.randn((wl.E, wl.d_model), generator=g, dtype=torch.float32) * wl.w_std
    if wl.zipf:
        Wg[:, 0] = zipf_offsets(wl)
    b_e = None
    if wl.sel_bias:
        gb = _gen(wl.seed * 7 + 3)
        b_e = (torch.rand((wl.E,), generator=gb, dtype=torch.float32) * 0.2 - 0.1)
    return {"W_g": Wg.to(wl.torch_dtype), "b_e": b_e}


def _expert_seed(wl: Workload, tensor: int, e: int) -> int:
    return (wl.seed * 1_000_003 + tensor * 65_537 + e) & 0x7FFF_FFFF_FFFF


def make_expert(wl: Workload, e: int, device="cpu") -> Dict[str, Optional[torch.Tensor]]:
    """Weights of expert e: W1 [F,d], W3 [F,d] or None, W2 [d,F], b1 [F], b2 [d]."""
    dev = torch.device(device)
    F, d = wl.d_ff, wl.d_model

    def draw(tensor: int, shape):
        g = _gen(_expert_seed(wl, tensor, e), dev)
        t = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        return (t * wl.w_std).to(wl.torch_dtype)

    out = {"W1": draw(1, (F, d)), "W2": draw(2, (d, F)), "W3": None, "b1": None, "b2": None}
    if wl.act == "swiglu":
        out["W3"] = draw(3, (F, d))
    if wl.biases:
        out["b1"] = draw(4, (F,))
        out["b2"] = draw(5, (d,))
    return out


def make_shared(wl: Workload, device="cpu") -> Optional[Dict[str, Optional[torch.Tensor]]]:
    """The shared expert: W1 [Fs,d], W3 [Fs,d] or None, W2 [d,Fs], b1 [Fs], b2 [d]; None if Fs = 0."""
    if wl.d_ff_shared == 0:
        return None
    dev = torch.device(device)
    Fs, d = wl.d_ff_shared, wl.d_model

    def draw(tensor: int, shape):
        g = _gen(_expert_seed(wl, tensor, 0x5A5A), dev)
        t = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        return (t * wl.w_std).to(wl.torch_dtype)

    out = {"W1": draw(11, (Fs, d)), "W2": draw(12, (d, Fs)), "W3": None, "b1": None, "b2": None}
    if wl.act == "swiglu":
        out["W3"] = draw(13, (Fs, d))
    if wl.biases:
        out["b1"] = draw(14, (Fs,))
        out["b2"] = draw(15, (d,))
    return out


def make_experts(wl: Workload, device="cpu") -> Dict[str, Optional[torch.Tensor]]:
    """All expert weights stacked: W1 [E,F,d], W3 [E,F,d]|None, W2 [E,d,F], b1 [E,F]|None, b2 [E,d]|None."""
    dev = torch.device(device)
    F, d, E = wl.d_ff, wl.d_model, wl.E
    dt = wl.torch_dtype
    W1 = torch.empty((E, F, d), dtype=dt, device=dev)
    W2 = torch.empty((E, d, F), dtype=dt, device=dev)
    W3 = torch.empty((E, F, d), dtype=dt, device=dev) if wl.act == "swiglu" else None
    b1 = torch.empty((E, F), dtype=dt, device=dev) if wl.biases else None
    b2 = torch.empty((E, d), dtype=dt, device=dev) if wl.biases else None
    for e in range(E):
        ex = make_expert(wl, e, dev)
        W1[e].copy_(ex["W1"])
        W2[e].copy_(ex["W2"])
        if W3 is not None:
            W3[e].copy_(ex["W3"])
        if b1 is not None:
            b1[e].copy_(ex["b1"])
            b2[e].copy_(ex["b2"])
    return {"W1": W1, "W3": W3, "W2": W2, "b1": b1, "b2": b2}


def make_inputs(wl: Workload, device="cpu") -> Dict[str, Optional[torch.Tensor]]:
    """Every input of one forward, on ``device``: x, W_g, b_e, W1, W3, W2, b1, b2, shared."""
    dev = torch.device(device)
    out = {"x": make_x(wl).to(dev)}
    r = make_router(wl)
    out["W_g"] = r["W_g"].to(dev)
    out["b_e"] = None if r["b_e"] is None else r["b_e"].to(dev)
    out.update(make_experts(wl, dev))
    out["shared"] = make_shared(wl, dev)
    return out


def flush_bytes_for_l2() -> int:
    """Bytes to write to evict a 126 MB L2 twice over."""
    return 2 * 128 * 1024 * 1024


def describe(wl: Workload) -> Dict[str, object]:
    return {"workload": wl.name, "N": wl.N, "d_model": wl.d_model, "d_ff": wl.d_ff, "E": wl.E,
            "k": wl.k, "act": wl.act, "router": wl.router, "dtype": wl.dtype,
            **({"d_ff_shared": wl.d_ff_shared, "routed_scaling": wl.routed_scaling} if wl.d_ff_shared else {})}


__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_x", "make_router", "make_expert",
           "make_experts", "make_shared", "zipf_offsets", "describe"]
