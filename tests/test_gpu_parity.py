"""CUDA layer vs the fp64 oracle, through the C ABI, on a B200 (marked gpu).

Small cases (all tokens compared) span several 128-row GEMM tiles with
ragged expert slices, reduction dims that are not multiples of the 64-wide
k-block and hidden widths that are not multiples of the N tile.  The five
full-size workloads run in the launch configuration the benchmark times;
there the routing, dispatch and loss are compared on every token and y on
sampled tokens.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_53_b200 as M
import oracle as O
import workloads as W
from parity import (MARGIN, TOL_Y, check_forward, config_of, covering_tokens, ffn_tile_m, gpu_forward, np64,
                    oracle_routing, tile_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"

SMALL = {
    "tiny_fp32": W.WORKLOADS["tiny_fp32"],
    "tiny_fp32_ragged": W.WORKLOADS["tiny_fp32"].scaled(N=333, d_model=72, d_ff=136, E=5, k=3),
    "gpt2_small": W.WORKLOADS["gpt2_moe"].scaled(N=300, d_model=256, d_ff=512),
    "gpt2_odd": W.WORKLOADS["gpt2_moe"].scaled(N=257, d_model=200, d_ff=328, E=5),
    "mixtral_small": W.WORKLOADS["mixtral"].scaled(N=200, d_model=512, d_ff=768),
    "mixtral_odd": W.WORKLOADS["mixtral"].scaled(N=161, d_model=136, d_ff=200, E=3),
    "deepseek_small": W.WORKLOADS["deepseek_v3"].scaled(N=256, d_model=384, d_ff=256, E=64),
    "qwen3_small": W.WORKLOADS["qwen3_skew"].scaled(N=512, d_model=256, d_ff=128),
    "topk_softmax_small": W.WORKLOADS["gpt2_moe"].scaled(N=130, d_model=128, d_ff=256, E=7, k=3,
                                                         router="topk_softmax"),
    "sigmoid_no_norm_scaled": W.WORKLOADS["deepseek_v3"].scaled(N=96, d_model=128, d_ff=128, E=16, k=4,
                                                               norm_topk=False, routed_scaling=2.5),
    # > 192 rows per expert: the CTA-pair GEMM (256-row tiles), ragged shapes
    "pair_swiglu_odd": W.WORKLOADS["mixtral"].scaled(N=600, d_model=136, d_ff=200, E=3),
    "pair_gelu_odd": W.WORKLOADS["gpt2_moe"].scaled(N=700, d_model=200, d_ff=328, E=3),
    "pair_swiglu_tiles": W.WORKLOADS["mixtral"].scaled(N=1100, d_model=320, d_ff=640, E=4),
    # the fused tcgen05 router with 17..32 experts (32-wide registers), and a
    # sigmoid router there
    "fused_e24": W.WORKLOADS["mixtral"].scaled(N=333, d_model=256, d_ff=256, E=24, k=3),
    "fused_e32_sigmoid": W.WORKLOADS["deepseek_v3"].scaled(N=130, d_model=192, d_ff=128, E=32, k=8),
    # the E > 32 selection: k > 8 (two choices per lane of a token's group),
    # E not a multiple of 4 (padded logit rows), a 200-expert sigmoid router
    "select_e50_k10": W.WORKLOADS["qwen3_skew"].scaled(N=161, d_model=136, d_ff=64, E=50, k=10, zipf=False),
    "select_e200_k16_sigmoid": W.WORKLOADS["deepseek_v3"].scaled(N=97, d_model=128, d_ff=64, E=200, k=16),
}

# Token budgets for y at full size: tokens are chosen so that their routed
# rows touch as many (expert, m-tile) pairs of the GEMM tile schedule as the
# budget allows (None: every token).
FULL_BUDGET = {"tiny_fp32": None, "gpt2_moe": 48, "mixtral": 40, "deepseek_v3": 48, "qwen3_skew": 96}


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_layer_53_b200 import build
    build.build()
    M.library()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("name", sorted(SMALL))
def test_forward_small(name):
    wl = SMALL[name]
    inp = W.make_inputs(wl, DEV)
    gpu = gpu_forward(wl, inp)
    rep = check_forward(wl, inp, gpu)
    print(name, rep.as_dict())


@pytest.mark.parametrize("name", ["tiny_fp32", "gpt2_moe", "mixtral", "deepseek_v3", "qwen3_skew"])
def test_forward_full_size(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, DEV)
    gpu = gpu_forward(wl, inp)
    n = FULL_BUDGET[name]
    tokens = None
    if n is not None:
        tokens = covering_tokens(gpu["topk_ids"], wl.E, ffn_tile_m(wl), n)
        tokens = np.union1d(tokens, [0, wl.N - 1])
    rep = check_forward(wl, inp, gpu, y_tokens=tokens)
    print(name, rep.as_dict())
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["gpt2_moe", "mixtral", "deepseek_v3", "qwen3_skew"])
def test_expert_ffn_full_size_rows(name):
    """moe_expert_ffn at full size on the forward's own x_sorted and offsets
    (moe_route + moe_dispatch), in the tile configuration the benchmark runs:
    the first row of every (expert, m-tile) and each expert's last row are
    compared with the oracle's expert FFN, row by row."""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    ws = M.workspace(cfg, DEV)
    ids, _, _ = M.moe_route(cfg, inp["x"], inp["W_g"], b_e=inp["b_e"], ws=ws)
    d = M.moe_dispatch(cfg, ids, x=inp["x"], ws=ws)
    ys = M.moe_expert_ffn(cfg, d["x_sorted"], d["offsets"], inp["W1"], inp["W2"], b1=inp["b1"], W3=inp["W3"],
                          b2=inp["b2"], ws=ws)
    torch.cuda.synchronize()
    offsets = d["offsets"].cpu().numpy()
    rows = tile_rows(offsets, ffn_tile_m(wl))
    expert_of = np.searchsorted(offsets, rows, side="right") - 1
    worst, checked = 0.0, 0
    for e in np.unique(expert_of):
        sel = rows[expert_of == e]
        ew = {"W1": np64(inp["W1"][e]), "W2": np64(inp["W2"][e]),
              "W3": None if inp["W3"] is None else np64(inp["W3"][e]),
              "b1": None if inp["b1"] is None else np64(inp["b1"][e]),
              "b2": None if inp["b2"] is None else np64(inp["b2"][e])}
        xr = np64(d["x_sorted"][torch.from_numpy(sel).to(DEV)])
        yr = np64(ys[torch.from_numpy(sel).to(DEV)])
        for i in range(len(sel)):
            ref = O.expert_ffn(xr[i], ew["W1"], ew["W2"], wl.act, ew["b1"], ew["W3"], ew["b2"])
            worst = max(worst, float(np.max(np.abs(yr[i] - ref)) / max(np.max(np.abs(ref)), 1e-30)))
            checked += 1
    print(name, {"rows_checked": checked, "tile_m": ffn_tile_m(wl), "max_rel_err": worst})
    assert checked == len(rows)
    assert worst <= TOL_Y[wl.dtype], worst
    del inp, ws, ys, d
    torch.cuda.empty_cache()


def test_forward_is_deterministic():
    wl = SMALL["qwen3_small"]
    inp = W.make_inputs(wl, DEV)
    a = gpu_forward(wl, inp)
    b = gpu_forward(wl, inp)
    for key in ("y", "topk_ids", "topk_w", "counts", "aux"):
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("name", ["gpt2_small", "deepseek_small", "tiny_fp32"])
def test_route_entry_point(name):
    wl = SMALL[name]
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    ids, w, probs = M.moe_route(cfg, inp["x"], inp["W_g"], b_e=inp["b_e"], want_probs=True)
    torch.cuda.synchronize()
    r = oracle_routing(wl, inp)
    near = r["margin"] < MARGIN
    ids = ids.cpu().numpy()
    assert np.all(ids[~near] == r["ids"][~near])
    assert np.max(np.abs(probs.cpu().numpy() - r["probs"])) <= 1e-6
    ok = ~near
    assert np.max(np.abs(w.cpu().numpy()[ok] - r["w"][ok])) <= 2e-5


@pytest.mark.parametrize("E,k,N", [(4, 2, 64), (128, 8, 777), (6, 2, 1), (1, 1, 40), (8, 8, 50), (256, 16, 99)])
def test_dispatch_entry_point(E, k, N):
    rng = np.random.default_rng(E * 1000 + k)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    cfg = M.make_config(N, 64, 64, E, k, dtype="bf16")
    x = torch.randn((N, 64), device=DEV).to(torch.bfloat16)
    out = M.moe_dispatch(cfg, torch.from_numpy(ids).to(DEV), x=x)
    torch.cuda.synchronize()
    want = O.dispatch(ids, E)
    for key in ("perm", "inv_perm", "offsets", "counts"):
        assert np.array_equal(out[key].cpu().numpy(), want[key]), key
    assert torch.equal(out["x_sorted"], x[torch.from_numpy(want["perm"] // k).long().to(DEV)])
    assert int(out["status"][0]) == 0


@pytest.mark.parametrize("E,k,N", [(4, 2, 64), (128, 8, 777), (6, 2, 1)])
def test_dispatch_entry_point_without_rows(E, k, N):
    """x = NULL: positions only (the scatter kernel instead of the fused row pass)."""
    rng = np.random.default_rng(E * 1000 + k + 7)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    cfg = M.make_config(N, 64, 64, E, k, dtype="bf16")
    out = M.moe_dispatch(cfg, torch.from_numpy(ids).to(DEV))
    torch.cuda.synchronize()
    want = O.dispatch(ids, E)
    for key in ("perm", "inv_perm", "offsets", "counts"):
        assert np.array_equal(out[key].cpu().numpy(), want[key]), key


def test_dispatch_reports_bad_expert_id():
    N, E, k = 50, 8, 2
    ids = np.tile(np.array([[0, 1]], np.int32), (N, 1))
    ids[7, 1] = 8
    ids[20, 0] = -1
    cfg = M.make_config(N, 64, 64, E, k, dtype="bf16")
    x = torch.randn((N, 64), device=DEV).to(torch.bfloat16)
    out = M.moe_dispatch(cfg, torch.from_numpy(ids).to(DEV), x=x)
    torch.cuda.synchronize()
    assert int(out["status"][0]) == 6
    # the valid assignments keep their stable positions; the two invalid ones
    # get inv_perm = -1 and no row
    inv = out["inv_perm"].cpu().numpy().reshape(N, k)
    assert inv[7, 1] == -1 and inv[20, 0] == -1
    valid = (ids >= 0) & (ids < E)
    got_rows = x.float().cpu().numpy()[np.arange(N).repeat(k).reshape(N, k)[valid]]
    xs = out["x_sorted"].float().cpu().numpy()
    assert np.array_equal(xs[inv[valid]], got_rows)
    assert len(set(inv[valid].tolist())) == int(valid.sum())


@pytest.mark.parametrize("dtype,act,big", [("bf16", "swiglu", False), ("bf16", "gelu", False),
                                           ("f32", "gelu", False), ("f32", "swiglu", False),
                                           ("bf16", "swiglu", True), ("bf16", "gelu", True)])
def test_expert_ffn_entry_point(dtype, act, big):
    """Random ragged slices with idle experts; every row checked.  `big`
    slices (> 192 rows per expert on average) take the CTA-pair kernel."""
    rng = np.random.default_rng(3)
    E, d, F = 9, 200, 264
    counts = np.array([0, 130, 1, 0, 257, 5, 128, 0, 40], np.int32)
    if big:
        counts = np.array([0, 700, 1, 0, 257, 5, 513, 0, 300], np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(offsets[-1])
    wl = W.Workload("ffn", N=rows, d_model=d, d_ff=F, E=E, k=1, act=act, router="softmax_topk",
                    dtype=dtype, biases=(act == "gelu"), seed=77)
    ex = W.make_experts(wl, DEV)
    xs = torch.randn((rows, d), device=DEV).to(wl.torch_dtype)
    cfg = M.make_config(rows, d, F, E, 1, act=act, dtype=dtype)
    ys = M.moe_expert_ffn(cfg, xs, torch.from_numpy(offsets).to(DEV), ex["W1"], ex["W2"], b1=ex["b1"],
                          W3=ex["W3"], b2=ex["b2"])
    torch.cuda.synchronize()
    ys = np64(ys)
    x64 = np64(xs)
    worst = 0.0
    for e in range(E):
        for i in range(offsets[e], offsets[e + 1]):
            ref = O.expert_ffn(x64[i], np64(ex["W1"][e]), np64(ex["W2"][e]), act,
                               None if ex["b1"] is None else np64(ex["b1"][e]),
                               None if ex["W3"] is None else np64(ex["W3"][e]),
                               None if ex["b2"] is None else np64(ex["b2"][e]))
            worst = max(worst, float(np.max(np.abs(ys[i] - ref)) / max(np.max(np.abs(ref)), 1e-30)))
    assert worst <= TOL_Y[dtype], worst


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_combine_entry_point(dtype):
    rng = np.random.default_rng(5)
    N, k, d = 300, 3, 136
    inv = rng.permutation(N * k).astype(np.int32)
    w = rng.uniform(0, 1, (N, k)).astype(np.float32)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    ys = torch.randn((N * k, d), device=DEV).to(td)
    cfg = M.make_config(N, d, 64, 8, k, dtype=dtype)
    y = M.moe_combine(cfg, ys, torch.from_numpy(w).to(DEV), torch.from_numpy(inv).to(DEV))
    torch.cuda.synchronize()
    ref = O.combine(np64(ys), w, inv)
    err = np.max(np.max(np.abs(np64(y) - ref), axis=1) / np.max(np.abs(ref), axis=1))
    assert err <= TOL_Y[dtype], err


def test_aux_loss_entry_point_and_bias_rule():
    rng = np.random.default_rng(8)
    N, E, k = 500, 16, 4
    z = rng.standard_normal((N, E))
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ids = np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)
    cfg = M.make_config(N, 64, 64, E, k, router="sigmoid", dtype="bf16")
    b = torch.from_numpy(rng.uniform(-0.1, 0.1, E).astype(np.float32)).to(DEV)
    b0 = b.cpu().numpy().copy()
    aux, counts, status = M.moe_aux_loss(cfg, torch.from_numpy(p.astype(np.float32)).to(DEV),
                                         torch.from_numpy(ids).to(DEV), gamma=1e-3, b_e=b)
    torch.cuda.synchronize()
    want, want_counts = O.aux_loss(p.astype(np.float32), ids)
    assert abs(float(aux[0]) - want) <= 1e-5
    assert np.array_equal(counts.cpu().numpy(), want_counts)
    assert np.max(np.abs(b.cpu().numpy() - O.bias_update(b0, want_counts, N, k, 1e-3))) <= 1e-7
    assert int(status[0]) == 0


@pytest.mark.parametrize("E,k,router,group", [(128, 8, "softmax_topk", 1), (128, 8, "softmax_topk", 2),
                                                (128, 8, "topk_softmax", 16), (256, 8, "sigmoid", 2),
                                                (256, 8, "sigmoid", 32), (64, 4, "softmax_topk", 2),
                                                (64, 8, "softmax_topk", 1)])
def test_route_exact_ties_large_E(E, k, router, group):
    """Exact ties through the E > 32 selection, both of its paths.

    Experts come in groups of `group` with identical W_g rows, a constant c_g
    per group (distinct, exact in bf16), and x is positive: tied experts get
    bitwise-equal logits, groups are far apart, and the course module's rule
    (ties to the lowest id, sec. 2.1) fixes the choice: groups by c_g
    descending, ids ascending inside a group, the same for every token.
    Groups of 1-2 leave about ten candidates per token (the short path);
    groups of 16-32 leave more than a lane group holds (the k-round path).
    """
    N, d = 96, 64
    wl = W.Workload("ties", N=N, d_model=d, d_ff=64, E=E, k=k, act="swiglu", router=router, dtype="bf16",
                    seed=31 + E + group)
    inp = W.make_inputs(wl, DEV)
    g = torch.Generator().manual_seed(7 + group)
    ngroups = E // group
    c = (torch.randperm(ngroups, generator=g).to(torch.float32) + 1.0) / (2.0 * ngroups)  # 1/2n .. 1/2, exact
    inp["W_g"] = c.repeat_interleave(group)[:, None].expand(E, d).contiguous().to(DEV, torch.bfloat16)
    inp["x"] = (inp["x"].float().abs() * 0.05 + 0.01).to(torch.bfloat16)  # z = c_g * sum(x) in (0, 3)
    if inp["b_e"] is not None:
        inp["b_e"] = torch.zeros_like(inp["b_e"])
    cg = c.repeat_interleave(group).numpy()
    want = np.array(sorted(range(E), key=lambda e: (-cg[e], e))[:k], dtype=np.int32)
    cfg = config_of(wl)
    ids, w, _ = M.moe_route(cfg, inp["x"], inp["W_g"], b_e=inp["b_e"], want_probs=True)
    torch.cuda.synchronize()
    ids = ids.cpu().numpy()
    assert np.array_equal(ids, np.tile(want, (N, 1)))
    r = oracle_routing(wl, inp)
    assert np.array_equal(r["ids"], ids)
    assert np.max(np.abs(w.cpu().numpy() - r["w"])) <= 2e-5


def test_balanced_router_gives_loss_k():
    """Circulant router: every expert in exactly k top-k sets, so L = k."""
    E, k = 8, 2
    v = np.array([1.5, -0.5, 0.75, 0.0, -1.25, 0.5, 1.0, -0.25], np.float32)
    Wg = np.array([[v[(e - n) % E] for n in range(E)] for e in range(E)], np.float32)
    wl = W.Workload("bal", N=E, d_model=E, d_ff=64, E=E, k=k, act="gelu", router="softmax_topk", dtype="f32",
                    biases=True, seed=5)
    inp = W.make_inputs(wl.scaled(d_model=8), DEV)
    inp["x"] = torch.eye(E, device=DEV)
    inp["W_g"] = torch.from_numpy(Wg).to(DEV)
    gpu = gpu_forward(wl, inp)
    assert np.array_equal(gpu["counts"], np.full(E, k))
    assert abs(float(gpu["aux"][0]) - k) <= 1e-5


@pytest.mark.parametrize("N,E,k", [(1, 8, 2), (0, 8, 2), (37, 1, 1), (45, 4, 4), (129, 16, 1)])
def test_edge_shapes(N, E, k):
    wl = W.Workload("edge", N=N, d_model=64, d_ff=128, E=E, k=k, act="swiglu", router="softmax_topk",
                    dtype="bf16", seed=11 + N)
    inp = W.make_inputs(wl, DEV)
    gpu = gpu_forward(wl, inp)
    if N == 0:
        assert gpu["counts"].sum() == 0 and float(gpu["aux"][0]) == 0.0
        return
    check_forward(wl, inp, gpu)


def test_collapsed_routing_single_expert_gets_everything():
    wl = W.Workload("collapse", N=300, d_model=64, d_ff=128, E=8, k=2, act="swiglu", router="softmax_topk",
                    dtype="bf16", seed=21)
    inp = W.make_inputs(wl, DEV)
    Wg = torch.zeros((8, 64), device=DEV)
    Wg[3, :] = 1.0
    Wg[6, :] = 0.5
    inp["x"] = inp["x"].abs()
    inp["W_g"] = Wg.to(torch.bfloat16)
    gpu = gpu_forward(wl, inp)
    assert gpu["counts"][3] == 300 and gpu["counts"][6] == 300
    check_forward(wl, inp, gpu)


@pytest.mark.parametrize("graphs", [True, False])
def test_host_pipeline_matches_forward(graphs):
    """Batches in pinned host memory through the overlapped copy pipeline
    (graph-pipelined or eager) give the same y and loss as moe_forward on
    device tensors, batch by batch."""
    wl = SMALL["mixtral_small"]
    inp = W.make_inputs(wl, DEV)
    cfg = config_of(wl)
    weights = {k: inp[k] for k in ("W_g", "W1", "W2", "W3", "b1", "b2", "b_e")}
    xs = [W.make_x(wl.scaled(seed=wl.seed + i)).pin_memory() for i in range(4)]
    ys = [torch.empty((wl.N, wl.d_model), dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    auxs = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(4)]
    pipe = M.HostPipeline(cfg, weights, device=DEV, graphs=graphs)
    n = 6  # fresh buffers on every call: the pipeline's work is enqueued directly
    xs = xs + [W.make_x(wl.scaled(seed=wl.seed + i)).pin_memory() for i in range(4, n)]
    ys = ys + [torch.empty((wl.N, wl.d_model), dtype=torch.bfloat16).pin_memory() for _ in range(4, n)]
    auxs = auxs + [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(4, n)]
    for i in range(n):
        pipe.step(xs[i], ys[i], auxs[i])
    pipe.finish()
    for i in range(3):  # a second pipeline on the same object, fewer batches than its depth
        pipe.step(xs[i], ys[i], auxs[i])
    pipe.finish()
    for i in range(n):
        ref = M.moe_forward(cfg, xs[i].to(DEV), inp["W_g"], inp["W1"], inp["W2"], W3=inp["W3"])
        torch.cuda.synchronize()
        assert torch.equal(ys[i], ref["y"].cpu()), i
        assert torch.equal(auxs[i], ref["aux"].cpu()), i
    # two buffer sets used in turn: each parity's work is enqueued directly on
    # its first use, captured on its second and replayed after that
    for j in (4, 5):  # no copy is in flight after finish()
        ys[j].zero_()
        auxs[j].zero_()
    for i in range(8):
        j = 4 + (i & 1)
        pipe.step(xs[j], ys[j], auxs[j])
    pipe.finish()
    if graphs:
        assert len(pipe.policy.graphs) >= 2
    for j in (4, 5):
        ref = M.moe_forward(cfg, xs[j].to(DEV), inp["W_g"], inp["W1"], inp["W2"], W3=inp["W3"])
        torch.cuda.synchronize()
        assert torch.equal(ys[j], ref["y"].cpu()), j
        assert torch.equal(auxs[j], ref["aux"].cpu()), j
