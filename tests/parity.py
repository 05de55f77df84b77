"""Comparison of the CUDA layer with the fp64 oracle (test infrastructure).

Rules (the tolerance is the one the task fixes for this layer):
  * routing: expert ids must equal the oracle's bit for bit, except for tokens
    whose top-k margin (oracle, fp64, selection-score space) is below 1e-4 --
    those are excluded from the id comparison and counted;
  * dispatch (counts, offsets, perm, inv_perm) must equal the oracle's
    dispatch of the CUDA path's ids exactly; it must equal the oracle's own
    when no token was excluded;
  * y and the Switch loss are compared with the oracle evaluated on the CUDA
    path's ids for the excluded tokens (their weights recomputed in fp64),
    because a single flipped near-tie moves L by ~E/N * dP;
  * y: max over tokens of ||y_n - r_n||_inf / ||r_n||_inf <= 1e-5 (fp32) or
    2e-2 (bf16, fp32 accumulation); L within 1e-5 absolute; gate weights
    within 2e-5 absolute;
  * router z-loss within 1e-5 relative (max(1, z) scale): each token's
    log-sum-exp comes from fp32 logits of the same accuracy as the gates;
  * the shared expert is part of y (same tolerance).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence

import numpy as np
import torch

import mixture_experts_layer_53_b200 as M
import oracle as O
import workloads as W

MARGIN = 1e-4
TOL_Y = {"f32": 1e-5, "bf16": 2e-2}
TOL_AUX = 1e-5
TOL_W = 2e-5
TOL_Z = 1e-5


def np64(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    if t is None:
        return None
    return t.detach().float().cpu().numpy().astype(np.float64)


def config_of(wl: W.Workload) -> M.MoeConfig:
    return M.make_config(wl.N, wl.d_model, wl.d_ff, wl.E, wl.k, wl.router, wl.norm_topk, wl.routed_scaling,
                         wl.act, wl.dtype, wl.d_ff_shared)


def gpu_forward(wl: W.Workload, inp: Dict[str, torch.Tensor], z_loss: bool = True) -> Dict[str, np.ndarray]:
    """One forward on the device (moe_forward_ex with the z-loss and any shared
    expert; moe_forward when z_loss is False and there is no shared expert);
    returns host copies of every output."""
    cfg = config_of(wl)
    b_e = inp["b_e"].clone() if inp["b_e"] is not None else None
    out = M.moe_forward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], W3=inp["W3"], b1=inp["b1"],
                        b2=inp["b2"], b_e=b_e, gamma=wl.gamma, shared=inp.get("shared"), z_loss=z_loss)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items() if k != "y" and (k != "z" or z_loss)}
    res["y"] = np64(out["y"])
    res["b_e_after"] = None if b_e is None else b_e.cpu().numpy()
    return res


@dataclasses.dataclass
class Report:
    near: int = 0
    id_mismatch: int = 0
    y_err: float = 0.0
    aux_err: float = 0.0
    z_err: float = 0.0
    w_err: float = 0.0
    tokens_checked_y: int = 0

    def as_dict(self):
        return dataclasses.asdict(self)


def oracle_routing(wl: W.Workload, inp) -> Dict[str, np.ndarray]:
    b = None if inp["b_e"] is None else np64(inp["b_e"])
    return O.route(np64(inp["x"]), np64(inp["W_g"]), wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=b)


def expert_getter(inp):
    def get(e: int):
        return {"W1": np64(inp["W1"][e]), "W2": np64(inp["W2"][e]),
                "W3": None if inp["W3"] is None else np64(inp["W3"][e]),
                "b1": None if inp["b1"] is None else np64(inp["b1"][e]),
                "b2": None if inp["b2"] is None else np64(inp["b2"][e])}
    return get


def ffn_tile_m(wl: W.Workload) -> int:
    """Rows per m-tile of the library's expert GEMMs for this workload: 256
    (CTA pairs) for bf16 when the experts average more than 192 rows, else
    128 (the rule the library states for its grouped GEMM)."""
    return 256 if wl.dtype == "bf16" and wl.N * wl.k / wl.E > 192 else 128


def tile_rows(offsets: np.ndarray, tile_m: int) -> np.ndarray:
    """Sorted rows that start every (expert, m-tile) of the grouped GEMM's
    tile schedule -- tile t of expert e starts at offsets[e] + t * tile_m --
    plus each non-empty expert's last row."""
    rows = []
    for e in range(len(offsets) - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            rows.extend(range(lo, hi, tile_m))
            rows.append(hi - 1)
    return np.unique(np.asarray(rows, dtype=np.int64))


def covering_tokens(ids: np.ndarray, E: int, tile_m: int, budget: int) -> np.ndarray:
    """Tokens whose routed rows touch as many (expert, m-tile) pairs of the
    tile schedule as possible, at most `budget` of them (greedy set cover;
    ties to the lowest token).  Each token's k rows sit at their sorted
    positions; a tile counts as touched by any of its rows."""
    dp = O.dispatch(ids, E)
    N, k = ids.shape
    inv = dp["inv_perm"].reshape(N, k)
    off = dp["offsets"]
    expert_of = np.searchsorted(off, inv, side="right") - 1
    tile_of = expert_of.astype(np.int64) * (1 << 32) + (inv - off[expert_of]) // tile_m
    need = set(np.unique(tile_of).tolist())
    chosen = []
    covers = [set(tile_of[n].tolist()) for n in range(N)]
    while need and len(chosen) < budget:
        best = max(range(N), key=lambda n: (len(covers[n] & need), -n))
        gain = covers[best] & need
        if not gain:
            break
        chosen.append(best)
        need -= gain
    return np.unique(np.asarray(chosen, dtype=np.int64))


def sample_tokens(N: int, count: int, seed: int = 0) -> np.ndarray:
    if count >= N:
        return np.arange(N)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, N - 1), size=count - 2, replace=False)
    return np.unique(np.concatenate([[0, N - 1], mid]))


def check_forward(wl: W.Workload, inp, gpu: Dict[str, np.ndarray], y_tokens: Optional[Sequence[int]] = None,
                  routing: Optional[Dict[str, np.ndarray]] = None) -> Report:
    """Assert the CUDA forward matches the oracle; y on all tokens or on y_tokens."""
    rep = Report()
    r = routing if routing is not None else oracle_routing(wl, inp)
    near = r["margin"] < MARGIN
    rep.near = int(near.sum())
    ids_g = gpu["topk_ids"]
    mism = np.any(ids_g != r["ids"], axis=1) & ~near
    rep.id_mismatch = int(mism.sum())
    assert rep.id_mismatch == 0, f"{rep.id_mismatch} tokens chose other experts (first {np.nonzero(mism)[0][:5]})"
    assert gpu["status"][0] == 0, f"device status {gpu['status'][0]}"

    # oracle on the CUDA ids where the choice was a near-tie
    b = None if inp["b_e"] is None else np64(inp["b_e"])
    rf = O.route(np64(inp["x"]), np64(inp["W_g"]), wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=b,
                 forced_ids=ids_g, forced=near.astype(np.uint8))
    assert np.array_equal(rf["ids"], ids_g)
    rep.w_err = float(np.max(np.abs(gpu["topk_w"] - rf["w"]))) if wl.N else 0.0
    assert rep.w_err <= TOL_W, f"gate weights off by {rep.w_err}"

    dp = O.dispatch(ids_g, wl.E)
    assert np.array_equal(gpu["counts"], dp["counts"]), "counts differ from the dispatch of the CUDA ids"
    if rep.near == 0:
        assert np.array_equal(gpu["counts"], O.dispatch(r["ids"], wl.E)["counts"])

    if wl.N:
        aux_o, _ = O.aux_loss(rf["probs"], ids_g)
        rep.aux_err = abs(float(gpu["aux"][0]) - aux_o)
        assert rep.aux_err <= TOL_AUX, f"aux loss {gpu['aux'][0]} vs {aux_o}"
    if "z" in gpu:
        z_o = O.z_loss(r["logits"]) if wl.N else 0.0
        rep.z_err = abs(float(gpu["z"][0]) - z_o) / max(1.0, abs(z_o))
        assert rep.z_err <= TOL_Z, f"router z-loss {gpu['z'][0]} vs {z_o}"

    if inp["b_e"] is not None and wl.gamma > 0:
        want = O.bias_update(np64(inp["b_e"]), dp["counts"], wl.N, wl.k, wl.gamma)
        assert np.max(np.abs(gpu["b_e_after"] - want)) <= 1e-7, "sign-rule bias step"

    tokens = np.arange(wl.N) if y_tokens is None else np.asarray(y_tokens)
    rep.tokens_checked_y = len(tokens)
    if len(tokens):
        x = np64(inp["x"])
        if y_tokens is None:
            y_o = O.dense_forward(x, ids_g, rf["w"], np64(inp["W1"]), np64(inp["W2"]), wl.act,
                                  np64(inp["W3"]), np64(inp["b1"]), np64(inp["b2"]))
        else:
            y_o = O.forward_tokens(x[tokens], ids_g[tokens], rf["w"][tokens], expert_getter(inp), wl.act)
        sh = inp.get("shared")
        if sh is not None:
            y_o = O.shared_add(y_o, x[tokens], np64(sh["W1"]), np64(sh["W2"]), wl.act, np64(sh["W3"]),
                               np64(sh["b1"]), np64(sh["b2"]))
        y_g = gpu["y"][tokens]
        denom = np.max(np.abs(y_o), axis=1)
        denom = np.where(denom > 0, denom, 1.0)
        rep.y_err = float(np.max(np.max(np.abs(y_g - y_o), axis=1) / denom))
        assert rep.y_err <= TOL_Y[wl.dtype], f"max normwise relative error {rep.y_err:.3e}"
    return rep
