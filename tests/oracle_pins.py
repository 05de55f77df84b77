"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``pin_*`` function takes a loaded oracle library (``oracle.load()``) and
raises AssertionError (or oracle.OracleError) when the oracle disagrees with
an externally fixed value.  ``tests/test_oracle_pins.py`` runs them on the
real oracle; ``tests/test_oracle_mutants.py`` runs them on copies of the
oracle with one plausible mistake planted each, and requires that every
mistake makes at least one pin fail.

What pins what:
  course worked example (sec. 3)         routing with a tie, weights, dispatch
                                         arrays, combine, P, L = 161/72, margin
  hand 8-expert top-2 case               top/boundary ties, renormalised gates,
                                         dispatch arrays, P, L, combine
  GPT-2 blog six-expert printout         softmax values, masked top-2 softmax
  circulant router                       L = k exactly at perfect balance
  bounds / collapse                      0 <= L <= E, L -> E when collapsed
  sigmoid hand case (sec. 2.5)           bias selects, never weighs; sign rule
  60 sign-rule steps (sec. 4 tests)      imbalance falls
  dense loop vs sorted dispatch          bitwise equal, three routers
  numpy float64 reference FFN            expert arithmetic (GELU erf, SwiGLU,
                                         biases, layouts); k=E dense mixture;
                                         E=k=1 plain FFN
  brute force over all subsets           selection on tiny random cases
  invariants                             sum w, counts, bijection, stability
  C per-token loop and numpy             forward_tokens (sampled-token y at
                                         full size), bit for bit / to 1e-12
  batch split into parts                 L from summed counts and P sums
                                         equals the whole batch's; = k at
                                         balance
"""
from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
from scipy.special import erf as sp_erf

import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _fr(s) -> float:
    return float(Fraction(str(s)))


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}\n{a}\n{b}"


def _eq(a, b, what):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape and np.array_equal(a, b), f"{what}: {a.tolist()} != {b.tolist()}"


def _logit_router(z):
    """x = identity, W_g[e, n] = z_n[e], so W_g x_n = z_n exactly."""
    z = np.asarray(z, dtype=np.float64)
    N, E = z.shape
    return np.eye(N), np.ascontiguousarray(z.T)


# ------------------------------------------------------------ numpy reference

def np_gelu(v):
    return 0.5 * v * (1.0 + sp_erf(v / math.sqrt(2.0)))


def np_silu(v):
    return v / (1.0 + np.exp(-v))


def np_expert(x, W1, W2, act, W3=None, b1=None, b2=None):
    """Expert FFN with numpy float64 matrix products (x is [S, d])."""
    g = x @ W1.T
    if act == "swiglu":
        h = np_silu(g) * (x @ W3.T)
    else:
        h = np_gelu(g + (0.0 if b1 is None else b1))
    o = h @ W2.T
    return o + (0.0 if b2 is None else b2)


def _rand_problem(rng, N, d, F, E, act, biases):
    x = rng.standard_normal((N, d))
    Wg = rng.standard_normal((E, d)) * 0.7
    W1 = rng.standard_normal((E, F, d)) / math.sqrt(d)
    W2 = rng.standard_normal((E, d, F)) / math.sqrt(F)
    W3 = rng.standard_normal((E, F, d)) / math.sqrt(d) if act == "swiglu" else None
    b1 = rng.standard_normal((E, F)) * 0.1 if biases else None
    b2 = rng.standard_normal((E, d)) * 0.1 if biases else None
    return x, Wg, W1, W2, W3, b1, b2


# ------------------------------------------------------------------- pins

def pin_course_worked_example(L):
    g = _golden("course_worked_example.json")
    z = np.log(np.array([[float(v) for v in row] for row in g["logits_ln"]]))
    x, Wg = _logit_router(z)
    r = O.route(x, Wg, g["k"], "softmax_topk", L=L)
    _close(r["probs"], [[_fr(v) for v in row] for row in g["probs"]], 1e-15, "probs")
    _eq(r["ids"], g["ids"], "ids")
    _close(r["w"], [[_fr(v) for v in row] for row in g["weights"]], 1e-15, "weights")
    # margins in p-space: token 0 gaps (1/4, 1/8); token 1 tie at the top -> 0
    _close(r["margin"], [1 / 8, 0.0], 1e-15, "margin")
    dp = O.dispatch(r["ids"], g["E"], L=L)
    _eq(dp["perm"], g["perm"], "perm")
    _eq(dp["perm"] // g["k"], g["tokens_of_perm"], "perm // k")
    _eq(dp["counts"], g["counts"], "counts")
    _eq(dp["offsets"], g["offsets"], "offsets")
    _eq(dp["inv_perm"], g["inv_perm"], "inv_perm")
    ys = np.array(g["y_sorted"], dtype=np.float64)[:, None]
    y = O.combine(ys, r["w"], dp["inv_perm"], L=L)
    _close(y[:, 0], [_fr(v) for v in g["y"]], 1e-13, "combine")
    _close(r["probs"].mean(axis=0), [_fr(v) for v in g["P"]], 1e-15, "P")
    loss, counts = O.aux_loss(r["probs"], r["ids"], L=L)
    _eq(counts, g["counts"], "aux counts")
    _close(loss, _fr(g["aux_loss"]), 1e-14, "aux loss")


def pin_hand_8expert(L):
    g = _golden("hand_8expert_top2.json")
    z = np.log(np.array(g["q"], dtype=np.float64))
    x, Wg = _logit_router(z)
    r = O.route(x, Wg, g["k"], "softmax_topk", L=L)
    _eq(r["ids"], g["ids"], "ids")
    _close(r["w"], [[_fr(v) for v in row] for row in g["weights"]], 1e-15, "weights")
    _close(r["w"].sum(axis=1), np.ones(4), 1e-15, "weights sum to 1")
    dp = O.dispatch(r["ids"], g["E"], L=L)
    for key in ("perm", "counts", "offsets", "inv_perm"):
        _eq(dp[key], g[key], key)
    _eq(dp["perm"] // g["k"], g["tokens_of_perm"], "perm // k")
    _close(r["probs"].mean(axis=0) * 20160, g["P_times_20160"], 1e-9, "P")
    loss, _ = O.aux_loss(r["probs"], r["ids"], L=L)
    _close(loss, _fr(g["aux_loss"]), 1e-14, "aux loss")
    ys = np.array(g["y_sorted"], dtype=np.float64)[:, None]
    y = O.combine(ys, r["w"], dp["inv_perm"], L=L)
    _close(y[:, 0], [_fr(v) for v in g["y"]], 1e-12, "combine")


def pin_gpt2_blog_six_expert(L):
    g = _golden("gpt2_blog_six_expert.json")
    z = np.array([g["logits"]])
    x, Wg = _logit_router(z)
    r = O.route(x, Wg, g["k"], "topk_softmax", L=L)
    _close(r["probs"][0], g["softmax"], 5e-5, "softmax printout")
    dense = np.zeros(6)
    dense[r["ids"][0]] = r["w"][0]
    _close(dense, g["topk_softmax_dense"], 5e-5, "masked top-2 softmax printout")
    _eq(r["ids"][0], [4, 2], "top-2 largest first")
    r2 = O.route(x, Wg, g["k"], "softmax_topk", norm_topk=True, L=L)
    _close(r2["w"], r["w"], 1e-15, "renormalised softmax == softmax over chosen logits")


def pin_balance_equals_k(L):
    rng = np.random.default_rng(7)
    for E, k in ((4, 1), (4, 2), (8, 2), (6, 3), (16, 4), (5, 5)):
        v = rng.standard_normal(E) * 2.0
        # W_g[e, n] = v[(e - n) mod E]: every token sees the same logits rotated
        Wg = np.array([[v[(e - n) % E] for n in range(E)] for e in range(E)])
        x = np.eye(E)
        r = O.route(x, Wg, k, "softmax_topk", L=L)
        loss, counts = O.aux_loss(r["probs"], r["ids"], L=L)
        _eq(counts, np.full(E, k), f"balanced counts E={E} k={k}")
        _close(loss, float(k), 1e-12, f"L == k at balance (E={E}, k={k})")


def pin_loss_bounds_and_collapse(L):
    rng = np.random.default_rng(11)
    for _ in range(20):
        N, d, E = 17, 5, 6
        k = int(rng.integers(1, E + 1))
        r = O.route(rng.standard_normal((N, d)), rng.standard_normal((E, d)) * 2, k, L=L)
        loss, _ = O.aux_loss(r["probs"], r["ids"], L=L)
        assert -1e-12 <= loss <= E + 1e-12, f"L={loss} outside [0, E]"
    # collapse: same k experts win every token with overwhelming logits
    N, E, k = 32, 8, 2
    z = rng.standard_normal((N, E)) * 0.1
    z[:, 3] += 40.0
    z[:, 5] += 40.0
    x, Wg = _logit_router(z)
    r = O.route(x, Wg, k, L=L)
    loss, counts = O.aux_loss(r["probs"], r["ids"], L=L)
    _eq(counts, [0, 0, 0, N, 0, N, 0, 0], "collapsed counts")
    _close(loss, float(E), 1e-6, "collapsed L -> E")
    # concentration raises the loss above its balanced value k
    assert loss > k


def pin_bias_selects_not_weighs(L):
    s = np.array([0.5, 0.6, 0.7, 0.8])
    z = np.log(s / (1.0 - s))[None, :]
    x, Wg = _logit_router(z)
    r = O.route(x, Wg, 2, "sigmoid", L=L)
    _eq(r["ids"][0], [3, 2], "sigmoid top-2 without bias")
    _close(r["w"][0], [8 / 15, 7 / 15], 1e-15, "sigmoid weights")
    b = np.array([0.4, 0.0, 0.0, 0.0])
    r = O.route(x, Wg, 2, "sigmoid", b_sel=b, L=L)
    _eq(r["ids"][0], [0, 3], "bias changes the selection (0.9 > 0.8)")
    _close(r["w"][0], [5 / 13, 8 / 13], 1e-15, "weights from unbiased scores")
    _close(r["margin"][0], 0.1, 1e-15, "sigmoid margin on biased scores")
    r = O.route(x, Wg, 2, "sigmoid", b_sel=b, routed_scaling=2.5, L=L)
    _close(r["w"][0], [2.5 * 5 / 13, 2.5 * 8 / 13], 1e-14, "routed_scaling")
    r = O.route(x, Wg, 2, "sigmoid", b_sel=b, norm_topk=False, L=L)
    _close(r["w"][0], [0.5, 0.8], 1e-15, "sigmoid without renormalisation")


def pin_softmax_norm_topk_false(L):
    g = _golden("course_worked_example.json")
    z = np.log(np.array([[float(v) for v in row] for row in g["logits_ln"]]))
    x, Wg = _logit_router(z)
    r = O.route(x, Wg, 2, "softmax_topk", norm_topk=False, L=L)
    _close(r["w"], [[1 / 2, 1 / 4], [1 / 3, 1 / 3]], 1e-15, "raw p without renormalisation")


def pin_sign_rule_by_hand(L):
    counts = np.array([3, 1, 0, 4])
    b0 = np.array([0.25, -0.5, 0.0, 1.0])
    b1 = O.bias_update(b0, counts, N=4, k=2, gamma=1e-3, L=L)
    _close(b1 - b0, 1e-3 * np.array([-1.0, 1.0, 1.0, -1.0]), 1e-18, "sign rule by hand")
    b2 = O.bias_update(b0, np.array([2, 2, 2, 2]), N=4, k=2, gamma=1e-3, L=L)
    _close(b2, b0, 0.0, "sign(0) = 0 at exact balance")


def pin_sign_rule_balances(L):
    """64 tokens, skewed sigmoid router, E=8, k=2, gamma=0.01, 60 steps."""
    rng = np.random.default_rng(3)
    N, d, E, k = 64, 16, 8, 2
    x = rng.standard_normal((N, d))
    Wg = rng.standard_normal((E, d)) * 0.3
    # skew: two experts get a large constant advantage through feature 0
    x[:, 0] = 1.0
    Wg[:, 0] = 0.0
    Wg[2, 0] = 1.5
    Wg[5, 0] = 1.2
    b = np.zeros(E)
    r = O.route(x, Wg, k, "sigmoid", b_sel=b, L=L)
    _, c0 = O.aux_loss(r["probs"], r["ids"], L=L)
    for _ in range(60):
        r = O.route(x, Wg, k, "sigmoid", b_sel=b, L=L)
        _, c = O.aux_loss(r["probs"], r["ids"], L=L)
        b = O.bias_update(b, c, N, k, 0.01, L=L)
    r = O.route(x, Wg, k, "sigmoid", b_sel=b, L=L)
    _, c1 = O.aux_loss(r["probs"], r["ids"], L=L)
    assert c0.max() >= 2 * N * k // E, f"start should be skewed (max >= 2x mean): {c0}"
    assert c1.max() < c0.max(), f"max load did not fall: {c0} -> {c1}"
    assert np.var(c1) < np.var(c0), f"load variance did not fall: {c0} -> {c1}"


def pin_sorted_equals_dense(L):
    rng = np.random.default_rng(5)
    for router, act, biases in (("softmax_topk", "gelu", True), ("topk_softmax", "swiglu", False),
                                ("sigmoid", "swiglu", True)):
        N, d, F, E, k = 23, 12, 20, 5, 3
        x, Wg, W1, W2, W3, b1, b2 = _rand_problem(rng, N, d, F, E, act, biases)
        bsel = rng.uniform(-0.1, 0.1, E) if router == "sigmoid" else None
        r = O.route(x, Wg, k, router, b_sel=bsel, L=L)
        yd = O.dense_forward(x, r["ids"], r["w"], W1, W2, act, W3, b1, b2, L=L)
        s = O.sorted_forward(x, r["ids"], r["w"], W1, W2, act, W3, b1, b2, L=L)
        assert np.array_equal(yd, s["y"]), f"sorted != dense bitwise ({router})"
        dp = O.dispatch(r["ids"], E, L=L)
        _eq(s["x_sorted"], x[dp["perm"] // k], "x_sorted = x[perm // k]")


def pin_ffn_matches_numpy(L):
    rng = np.random.default_rng(9)
    for act, biases in (("gelu", True), ("gelu", False), ("swiglu", False), ("swiglu", True)):
        d, F = 7, 11
        x = rng.standard_normal((3, d))
        W1 = rng.standard_normal((F, d))
        W2 = rng.standard_normal((d, F))
        W3 = rng.standard_normal((F, d)) if act == "swiglu" else None
        b1 = rng.standard_normal(F) if (biases and act == "gelu") else None
        b2 = rng.standard_normal(d) if biases else None
        ref = np_expert(x, W1, W2, act, W3, b1, b2)
        got = np.stack([O.expert_ffn(x[i], W1, W2, act, b1, W3, b2, L=L) for i in range(3)])
        scale = np.max(np.abs(ref))
        _close(got / scale, ref / scale, 1e-13, f"expert FFN vs numpy ({act}, biases={biases})")
    # exact GELU: erf, not the tanh form
    for v in (-3.0, -0.7, 0.0, 0.3, 1.9):
        W1 = np.array([[v]])
        W2 = np.array([[1.0]])
        got = O.expert_ffn(np.array([1.0]), W1, W2, "gelu", L=L)[0]
        assert abs(got - 0.5 * v * (1 + math.erf(v / math.sqrt(2)))) < 1e-15, "GELU erf form"


def pin_dense_mixture_k_equals_E(L):
    rng = np.random.default_rng(13)
    N, d, F, E = 9, 6, 10, 4
    x, Wg, W1, W2, W3, b1, b2 = _rand_problem(rng, N, d, F, E, "gelu", True)
    r = O.route(x, Wg, E, "softmax_topk", L=L)
    y = O.dense_forward(x, r["ids"], r["w"], W1, W2, "gelu", None, b1, b2, L=L)
    z = x @ Wg.T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ref = sum(p[:, e:e + 1] * np_expert(x, W1[e], W2[e], "gelu", None, b1[e], b2[e])
              for e in range(E))
    _close(y, ref, 1e-12, "k=E is the dense softmax mixture")
    _close(r["w"], np.take_along_axis(p, r["ids"], axis=1), 1e-14, "k=E weights are p")


def pin_plain_ffn_single_expert(L):
    rng = np.random.default_rng(17)
    N, d, F = 5, 8, 6
    x, Wg, W1, W2, W3, b1, b2 = _rand_problem(rng, N, d, F, 1, "swiglu", False)
    r = O.route(x, Wg, 1, "softmax_topk", L=L)
    _eq(r["ids"], np.zeros((N, 1)), "E=k=1 ids")
    _close(r["w"], np.ones((N, 1)), 1e-15, "E=k=1 weight")
    y = O.dense_forward(x, r["ids"], r["w"], W1, W2, "swiglu", W3, L=L)
    _close(y, np_expert(x, W1[0], W2[0], "swiglu", W3[0]), 1e-12, "E=k=1 is a plain FFN")


def pin_brute_force_selection(L):
    rng = np.random.default_rng(19)
    for trial in range(40):
        N = int(rng.integers(1, 7))
        E = int(rng.integers(1, 7))
        k = int(rng.integers(1, E + 1))
        router = ("softmax_topk", "topk_softmax", "sigmoid")[trial % 3]
        # few distinct values so that ties are frequent
        z = rng.integers(-2, 3, size=(N, E)).astype(np.float64) * 0.5
        b = rng.integers(-1, 2, size=E) * 0.25 if router == "sigmoid" else None
        x, Wg = _logit_router(z)
        r = O.route(x, Wg, k, router, b_sel=b, L=L)
        for n in range(N):
            score = 1 / (1 + np.exp(-z[n])) + b if router == "sigmoid" else z[n]
            valid = []
            for S in itertools.combinations(range(E), k):
                rest = [e for e in range(E) if e not in S]
                if all(score[e] > score[o] or (score[e] == score[o] and e < o)
                       for e in S for o in rest):
                    valid.append(S)
            assert len(valid) == 1, "exactly one subset obeys the tie rule"
            S = valid[0]
            assert set(r["ids"][n].tolist()) == set(S), f"chosen set {r['ids'][n]} vs {S}"
            want = sorted(S, key=lambda e: (-score[e], e))
            _eq(r["ids"][n], want, "slots in (score desc, id asc) order")
            # weights recomputed from the chosen set
            if router == "sigmoid":
                s = 1 / (1 + np.exp(-z[n, want]))
            else:
                s = np.exp(z[n, want] - z[n].max())
            _close(r["w"][n], s / s.sum(), 1e-14, "weights of the brute-force set")


def pin_ties_lowest_id(L):
    z = np.zeros((1, 6))
    x, Wg = _logit_router(z)
    for k in range(1, 7):
        r = O.route(x, Wg, k, L=L)
        _eq(r["ids"][0], list(range(k)), f"all-equal logits take ids 0..{k - 1}")


def pin_invariants(L):
    rng = np.random.default_rng(23)
    for router in ("softmax_topk", "topk_softmax", "sigmoid"):
        N, d, E, k = 41, 9, 7, 3
        x = rng.standard_normal((N, d))
        Wg = rng.standard_normal((E, d))
        b = rng.uniform(-0.1, 0.1, E) if router == "sigmoid" else None
        r = O.route(x, Wg, k, router, b_sel=b, L=L)
        _close(r["w"].sum(axis=1), np.ones(N), 1e-14, "sum_j w = 1")
        assert all(len(set(row)) == k for row in r["ids"].tolist()), "k distinct experts"
        _close(r["probs"].sum(axis=1), np.ones(N), 1e-14, "sum_e p = 1")
        dp = O.dispatch(r["ids"], E, L=L)
        assert dp["counts"].sum() == N * k
        _eq(np.sort(dp["perm"]), np.arange(N * k), "perm is a bijection")
        _eq(dp["inv_perm"][dp["perm"]], np.arange(N * k), "inv_perm[perm[i]] = i")
        _eq(np.diff(dp["offsets"]), dp["counts"], "offsets[e+1]-offsets[e] = counts[e]")
        assert dp["offsets"][0] == 0 and dp["offsets"][-1] == N * k
        flat = r["ids"].reshape(-1)
        for e in range(E):
            sl = dp["perm"][dp["offsets"][e]:dp["offsets"][e + 1]]
            assert np.all(flat[sl] == e), "slice holds only its expert"
            assert np.all(np.diff(sl) > 0), "assignments ascend inside a slice (stable)"


def pin_forced_ids(L):
    rng = np.random.default_rng(29)
    N, d, E, k = 6, 5, 5, 2
    x = rng.standard_normal((N, d))
    Wg = rng.standard_normal((E, d))
    r = O.route(x, Wg, k, L=L)
    forced_ids = r["ids"][:, ::-1].copy()
    forced = np.zeros(N, np.uint8)
    forced[[1, 4]] = 1
    r2 = O.route(x, Wg, k, forced_ids=forced_ids, forced=forced, L=L)
    _eq(r2["ids"][[1, 4]], forced_ids[[1, 4]], "forced tokens take the given ids")
    _eq(r2["ids"][[0, 2, 3, 5]], r["ids"][[0, 2, 3, 5]], "other tokens unchanged")
    _close(r2["w"][[1, 4]], r["w"][[1, 4]][:, ::-1], 1e-15, "weights follow the forced slots")


def pin_rejects_bad_ids(L):
    try:
        O.dispatch(np.array([[0, 4]]), 4, L=L)
    except O.OracleError:
        pass
    else:
        raise AssertionError("dispatch accepted an expert id >= E")




def pin_z_loss_closed_forms(L):
    """Router z-loss = mean_n (logsumexp z_n)^2 ("nano-moe", router z-loss)."""
    for E in (1, 4, 8):
        _close(O.z_loss(np.zeros((5, E)), L=L), math.log(E) ** 2, 1e-14, f"zero logits, E={E}")
    g = _golden("course_worked_example.json")
    z = np.log(np.array([[float(v) for v in row] for row in g["logits_ln"]]))
    # token 0: sum q = 8, token 1: sum q = 9
    _close(O.z_loss(z, L=L), (math.log(8) ** 2 + math.log(9) ** 2) / 2, 1e-14, "worked-example logits")
    zz = np.array([[1.5], [-2.0], [0.25]])
    _close(O.z_loss(zz, L=L), float(np.mean(zz[:, 0] ** 2)), 1e-14, "one expert: lse = z")
    rng = np.random.default_rng(31)
    z = rng.standard_normal((6, 5)) * 3
    lse = np.log(np.sum(np.exp(z), axis=1))
    _close(O.z_loss(z + 7.0, L=L), float(np.mean((lse + 7.0) ** 2)), 1e-12, "shift by c moves lse by c")


def pin_shared_expert_numpy(L):
    """y_n = sum_j w_j Expert_j(x_n) + Shared(x_n) (course module sec. 2.1)."""
    rng = np.random.default_rng(37)
    for act, biases in (("swiglu", False), ("gelu", True)):
        N, d, F, Fs, E, k = 7, 6, 9, 12, 4, 2
        x, Wg, W1, W2, W3, b1, b2 = _rand_problem(rng, N, d, F, E, act, biases)
        Ws1 = rng.standard_normal((Fs, d)) / math.sqrt(d)
        Ws2 = rng.standard_normal((d, Fs)) / math.sqrt(Fs)
        Ws3 = rng.standard_normal((Fs, d)) / math.sqrt(d) if act == "swiglu" else None
        bs1 = rng.standard_normal(Fs) * 0.1 if biases else None
        bs2 = rng.standard_normal(d) * 0.1 if biases else None
        r = O.route(x, Wg, k, routed_scaling=2.5, L=L)
        y = O.dense_forward(x, r["ids"], r["w"], W1, W2, act, W3, b1, b2, L=L)
        y = O.shared_add(y, x, Ws1, Ws2, act, Ws3, bs1, bs2, L=L)
        ref = sum(r["w"][:, j:j + 1] * np.stack([np_expert(x[n:n + 1], W1[r["ids"][n, j]], W2[r["ids"][n, j]],
                                                           act, None if W3 is None else W3[r["ids"][n, j]],
                                                           None if b1 is None else b1[r["ids"][n, j]],
                                                           None if b2 is None else b2[r["ids"][n, j]])[0]
                                                 for n in range(N)]) for j in range(k))
        ref = ref + np_expert(x, Ws1, Ws2, act, Ws3, bs1, bs2)  # shared part carries no weight
        _close(y, ref, 1e-12, f"routed sum + shared expert ({act})")
    z = O.shared_add(np.ones((3, 4)), rng.standard_normal((3, 4)), np.zeros((5, 4)), np.zeros((4, 5)), "gelu", L=L)
    _close(z, np.ones((3, 4)), 0.0, "zero shared expert adds nothing")



def _fd_case(L, rng, N, d, F, E, k, act, router, norm_topk, scaling, biases, shared_F, sel_bias, aux_coef, z_coef):
    """Central finite differences of the oracle's own forward loss
    <dy, y> + aux_coef L_aux + z_coef L_z against oracle_backward, for every
    entry of every input and parameter (ids held at the unperturbed routing)."""
    x, Wg, W1, W2, W3, b1, b2 = _rand_problem(rng, N, d, F, E, act, biases)
    b_sel = rng.uniform(-0.1, 0.1, E) if sel_bias else None
    sh = None
    if shared_F:
        sh = {"W1": rng.standard_normal((shared_F, d)) / math.sqrt(d),
              "W2": rng.standard_normal((d, shared_F)) / math.sqrt(shared_F),
              "W3": rng.standard_normal((shared_F, d)) / math.sqrt(d) if act == "swiglu" else None,
              "b1": rng.standard_normal(shared_F) * 0.1 if (biases and act == "gelu") else None,
              "b2": rng.standard_normal(d) * 0.1 if biases else None}
    dy = rng.standard_normal((N, d))
    r0 = O.route(x, Wg, k, router, norm_topk, scaling, b_sel=b_sel, L=L)
    assert np.min(r0["margin"]) > 1e-4, "pick a seed with clear routing"
    ids0 = r0["ids"]
    forced = np.ones(N, np.uint8)
    P = {"x": x, "Wg": Wg, "W1": W1, "W2": W2, "W3": W3, "b1": b1, "b2": b2}
    if sh:
        P.update({"Ws1": sh["W1"], "Ws2": sh["W2"], "Ws3": sh["W3"], "bs1": sh["b1"], "bs2": sh["b2"]})

    def loss():
        r = O.route(P["x"], P["Wg"], k, router, norm_topk, scaling, b_sel=b_sel, forced_ids=ids0, forced=forced, L=L)
        y = O.dense_forward(P["x"], ids0, r["w"], P["W1"], P["W2"], act, P["W3"], P["b1"], P["b2"], L=L)
        if sh:
            y = O.shared_add(y, P["x"], P["Ws1"], P["Ws2"], act, P["Ws3"], P["bs1"], P["bs2"], L=L)
        aux, _ = O.aux_loss(r["probs"], ids0, L=L)
        return float(np.sum(dy * y)) + aux_coef * aux + z_coef * O.z_loss(r["logits"], L=L)

    shared = None if not sh else {"W1": P["Ws1"], "W2": P["Ws2"], "W3": P["Ws3"], "b1": P["bs1"], "b2": P["bs2"]}
    g = O.backward(x, Wg, k, W1, W2, dy, router, norm_topk, scaling, act, W3, b1, b2, b_sel, shared,
                   aux_coef, z_coef, L=L)
    names = {"x": "dx", "Wg": "dWg", "W1": "dW1", "W2": "dW2", "W3": "dW3", "b1": "db1", "b2": "db2",
             "Ws1": "dWs1", "Ws2": "dWs2", "Ws3": "dWs3", "bs1": "dbs1", "bs2": "dbs2"}
    h = 1e-5
    for pname, arr in P.items():
        if arr is None:
            continue
        fd = np.zeros_like(arr)
        flat = arr.reshape(-1)
        for i in range(flat.size):
            v = flat[i]
            flat[i] = v + h
            lp = loss()
            flat[i] = v - h
            lm = loss()
            flat[i] = v
            fd.reshape(-1)[i] = (lp - lm) / (2 * h)
        an = g[names[pname]]
        assert an is not None and an.shape == arr.shape, pname
        err = float(np.max(np.abs(fd - an) / np.maximum(1.0, np.abs(an))))
        assert err <= 1e-6, f"{router}/{act}: d{pname} off by {err:.2e} (finite differences)"


def pin_backward_finite_differences(L):
    """Every gradient of oracle_backward equals the central difference of the
    forward loss (routing held fixed: the choice and f_e are piecewise
    constant), for each router, both activations, biases, a shared expert,
    routed_scaling, the aux-free bias, the Switch loss and the router z-loss."""
    rng = np.random.default_rng(91)
    _fd_case(L, rng, 4, 4, 5, 4, 2, "gelu", "softmax_topk", True, 1.0, True, 3, False, 0.3, 0.2)
    _fd_case(L, rng, 4, 4, 3, 5, 2, "swiglu", "sigmoid", True, 2.5, False, 3, True, 0.5, 0.1)
    _fd_case(L, rng, 3, 4, 3, 4, 3, "swiglu", "topk_softmax", True, 1.0, False, 0, False, 1.0, 0.0)
    _fd_case(L, rng, 4, 3, 4, 4, 2, "gelu", "softmax_topk", False, 1.0, False, 0, False, 0.7, 0.3)
    _fd_case(L, rng, 3, 3, 3, 3, 3, "gelu", "sigmoid", False, 1.0, True, 0, True, 0.4, 0.0)


def pin_aux_gradient_is_E_f_over_N(L):
    """[course] sec. 2.3: dL_aux / dp_{n,e} = E f_e / N.  With dy = 0 and only
    the Switch loss, dW_g = sum_n (J_softmax(z_n) c) x_n^T, c_e = E f_e / N."""
    rng = np.random.default_rng(93)
    N, d, E, k = 7, 5, 6, 2
    x = rng.standard_normal((N, d))
    Wg = rng.standard_normal((E, d))
    W1 = rng.standard_normal((E, 3, d))
    W2 = rng.standard_normal((E, d, 3))
    r = O.route(x, Wg, k, L=L)
    f = np.bincount(r["ids"].reshape(-1), minlength=E) / N
    c = E * f / N
    p = r["probs"]
    dz = p * (c[None, :] - (p @ c)[:, None])
    g = O.backward(x, Wg, k, W1, W2, np.zeros((N, d)), aux_coef=1.0, L=L)
    _close(g["dWg"], dz.T @ x, 1e-12, "dW_g of the Switch loss")
    _close(g["dW1"], np.zeros_like(W1), 0.0, "no expert gradient without dy")

def pin_forward_tokens(L, forward_tokens=None):
    """The per-token loop for sampled tokens (``oracle.forward_tokens``, the
    oracle of y at full size) equals the C per-token loop
    ``oracle_dense_forward`` bit for bit, and numpy's float64 restatement
    y_n = sum_j w_nj Expert_{e_nj}(x_n) (course module sec. 2.1) to 1e-12.
    Problems: k = 8 with experts shared across tokens and one idle expert, a
    GELU layer with biases, a single token with k = 1, and slot weights that
    differ per slot (so a slot swap shows)."""
    fwd = forward_tokens or O.forward_tokens
    rng = np.random.default_rng(29)
    cases = (("swiglu", False, 9, 10, 8), ("gelu", True, 6, 7, 3), ("swiglu", True, 1, 4, 1))
    for act, biases, S, E, k in cases:
        d, F = 12, 10
        x, _, W1, W2, W3, b1, b2 = _rand_problem(rng, S, d, F, E, act, biases)
        if act == "swiglu":
            b1 = None  # SwiGLU experts carry no hidden bias
        idle = E // 2
        pool = [e for e in range(E) if e != idle]
        ids = np.stack([rng.permutation(pool)[:k] for _ in range(S)]).astype(np.int32)
        w = rng.uniform(0.05, 1.0, (S, k))
        fetched = []

        def getter(e):
            fetched.append(e)
            return {"W1": W1[e], "W2": W2[e], "W3": None if W3 is None else W3[e],
                    "b1": None if b1 is None else b1[e], "b2": None if b2 is None else b2[e]}

        got = fwd(x, ids, w, getter, act, L=L)
        assert idle not in fetched, "an expert no token chose was evaluated"
        want = O.dense_forward(x, ids, w, W1, W2, act, W3, b1, b2, L=L)
        assert np.array_equal(got, want), f"forward_tokens != dense_forward bitwise ({act}, k={k})"
        ref = np.zeros((S, d))
        for s_ in range(S):
            for j in range(k):
                e = int(ids[s_, j])
                ref[s_] += w[s_, j] * np_expert(x[s_:s_ + 1], W1[e], W2[e], act, None if W3 is None else W3[e],
                                                None if b1 is None else b1[e], None if b2 is None else b2[e])[0]
        scale = np.max(np.abs(ref))
        _close(got / scale, ref / scale, 1e-12, f"forward_tokens vs numpy ({act}, k={k})")


def pin_loss_from_partials(L):
    """A batch split into parts (course module sec. 2.3: f and P are averages
    over the whole batch): summing each part's counts and probability sums
    and applying the loss gives the whole batch's L to rounding; at the
    circulant router's perfect balance it is k; with one part it is the
    part's own L; an empty batch gives 0."""
    rng = np.random.default_rng(31)
    for router, E, k, parts in (("softmax_topk", 8, 2, (13, 1, 30)), ("sigmoid", 16, 4, (20, 20)),
                                ("topk_softmax", 5, 5, (7,))):
        N = sum(parts)
        x, Wg, *_ = _rand_problem(rng, N, 9, 4, E, "gelu", False)
        bsel = rng.uniform(-0.1, 0.1, E) if router == "sigmoid" else None
        r = O.route(x, Wg, k, router, b_sel=bsel, L=L)
        whole, whole_counts = O.aux_loss(r["probs"], r["ids"], L=L)
        counts = np.zeros(E, np.int64)
        psum = np.zeros(E)
        lo = 0
        for n in parts:
            part_counts = np.bincount(r["ids"][lo:lo + n].reshape(-1), minlength=E)
            counts += part_counts
            psum += r["probs"][lo:lo + n].sum(axis=0)
            if len(parts) == 1:
                own, _ = O.aux_loss(r["probs"][lo:lo + n], r["ids"][lo:lo + n], L=L)
                _close(O.aux_from_partials(part_counts, r["probs"][lo:lo + n].sum(axis=0), k, L=L), own, 1e-14,
                       "one part: its own L")
            lo += n
        _eq(counts, whole_counts, "summed counts are the whole batch's")
        _close(O.aux_from_partials(counts, psum, k, L=L), whole, 1e-13, f"L from partials ({router})")
    E, k = 8, 3
    v = np.array([1.5, -0.5, 0.75, 0.0, -1.25, 0.5, 1.0, -0.25])
    x = np.eye(E)
    Wg = np.array([[v[(e - n) % E] for n in range(E)] for e in range(E)])
    r = O.route(x, Wg, k, L=L)
    halves = [slice(0, 3), slice(3, E)]
    counts = sum(np.bincount(r["ids"][h].reshape(-1), minlength=E) for h in halves)
    psum = sum(r["probs"][h].sum(axis=0) for h in halves)
    _close(O.aux_from_partials(counts, psum, k, L=L), k, 1e-12, "balanced split batch: L = k")
    assert O.aux_from_partials(np.zeros(E, np.int32), np.zeros(E), k, L=L) == 0.0, "empty batch"


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
