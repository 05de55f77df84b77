"""Plant one mistake at a time in a copy of the oracle; the pins must catch each.

The mistakes follow the course module's pitfall table (sec. 5: renormalising
when told not to, weighing by the biased score, scattering with perm instead
of inv_perm, reading tokens in token order, counting f from probabilities, a
flipped bias sign, ties to the highest id, routed_scaling ignored, offsets
holding ends, topk_softmax weighing by the full softmax) plus slips of the
kind that break any numeric code (a dropped bias, a transposed index, the
tanh GELU, the wrong SwiGLU operand, an unstable sort, a wrong P).
The planted copies are compiled to a temporary directory on the CPU; the
oracle under ``oracle/`` is never modified.
"""
import inspect
import os
import subprocess
import textwrap

import pytest

import oracle as O
from oracle_pins import ALL_PINS, pin_forward_tokens

SRC = os.path.join(os.path.dirname(O.__file__), "moe_oracle.c")

MUTANTS = {
    "s01_renormalise_always": ("if (norm_topk) for (int j = 0; j < k; ++j) wn[j] /= s;\n        } else if (router == ORC_TOPK_SOFTMAX)",
                               "for (int j = 0; j < k; ++j) wn[j] /= s;\n        } else if (router == ORC_TOPK_SOFTMAX)"),
    "s02_weigh_by_biased_score": ("wn[j] = sigmoid(z[idn[j]]); s += wn[j];", "wn[j] = sel[idn[j]]; s += wn[j];"),
    "s03_scatter_with_perm": ("oracle_combine(N, d, k, ys, w, inv, y);", "oracle_combine(N, d, k, ys, w, perm, y);"),
    "s04_token_order": ("memcpy(xs + i * d, x + (int64_t)(perm[i] / k) * d", "memcpy(xs + i * d, x + (int64_t)(i / k) * d"),
    "s05_f_from_probs": ("double f = (double)cnt[e] / (double)N;", "double f = P[e] / (double)N;"),
    "s06_sign_flipped": ("b[e] += gamma * (double)s;", "b[e] -= gamma * (double)s;"),
    "s07_ties_highest_id": ("    return a < b;\n}", "    return a > b;\n}"),
    "s09_routed_scaling_ignored": ("for (int j = 0; j < k; ++j) wn[j] *= routed_scaling;", ""),
    "s11_offsets_hold_ends": ("offsets[e + 1] = offsets[e] + cnt[e];", "offsets[e + 1] = offsets[e] + cnt[e] + (e + 1 < E ? cnt[e + 1] : 0) - cnt[e];"),
    "s12_topk_softmax_full_softmax": ("wn[j] = exp(z[idn[j]] - cmax); s += wn[j]; }\n            for (int j = 0; j < k; ++j) wn[j] /= s;",
                                      "wn[j] = p[idn[j]]; s += wn[j]; }"),
    "dropped_b2": ("if (b2) o += b2[c];", ""),
    "dropped_b1": ("if (b1) g += b1[f];", ""),
    "transposed_W2": ("o += W2[(int64_t)c * F + f] * h[f];", "o += W2[(int64_t)f * d + c] * h[f];"),
    "transposed_router": ("acc += Wg[(int64_t)e * d + i] * xn[i];", "acc += Wg[(int64_t)i * E + e] * xn[i];"),
    "gelu_tanh_form": ("return 0.5 * v * (1.0 + erf(v / sqrt(2.0)));",
                       "return 0.5 * v * (1.0 + tanh(0.7978845608028654 * (v + 0.044715 * v * v * v)));"),
    "swiglu_operands_swapped": ("h[f] = silu(g) * u;", "h[f] = silu(u) * g;"),
    "unstable_within_expert": ("return (u->a > v->a) - (u->a < v->a);", "return (u->a < v->a) - (u->a > v->a);"),
    "P_sums_skip_last_token": ("for (int64_t n = 0; n < N; ++n)\n        for (int e = 0; e < E; ++e) P[e] += probs[n * E + e];",
                               "for (int64_t n = 0; n + 1 < N; ++n)\n        for (int e = 0; e < E; ++e) P[e] += probs[n * E + e];"),
    "loss_missing_E": ("L *= (double)E;", ""),
    "sigmoid_bias_ignored": ("sel[e] = sigmoid(z[e]) + (b_sel ? b_sel[e] : 0.0);", "sel[e] = sigmoid(z[e]);"),
    "margin_from_wrong_neighbour": ("double g = gap_score[order[r]] - gap_score[order[r + 1]];",
                                    "double g = gap_score[order[0]] - gap_score[order[r + 1]];"),
    "softmax_no_normalise": ("for (int e = 0; e < E; ++e) p[e] /= denom;", ""),
    "wrong_expert_block": ("oracle_expert_ffn(d, F, act, xrow, W1 + (int64_t)e * F * d,",
                           "oracle_expert_ffn(d, F, act, xrow, W1 + (int64_t)(e ^ 1) * F * d,"),
    "z_loss_not_squared": ("total += lse * lse;", "total += lse;"),
    "z_loss_no_max_shift": ("const double lse = zmax + log(s);", "const double lse = log(s);"),
    "shared_not_added": ("for (int c = 0; c < d; ++c) y[n * d + c] += o[c];", "for (int c = 0; c < d; ++c) y[n * d + c] = o[c];"),
    "bwd_softmax_jacobian_no_mean": ("for (int e = 0; e < E; ++e) dz[e] += p[e] * (dp[e] - pdp);",
                                     "for (int e = 0; e < E; ++e) dz[e] += p[e] * dp[e];"),
    "bwd_silu_derivative_short": ("da = dh[f] * u[f] * sg * (1.0 + a[f] * (1.0 - sg));", "da = dh[f] * u[f] * sg;"),
    "bwd_gelu_derivative_short": ("da = dh[f] * (Phi + a[f] * phi);", "da = dh[f] * Phi;"),
    "bwd_aux_missing_E": ("dp[e] += aux_coef * (double)E * (cnt[e] / (double)N) / (double)N;",
                          "dp[e] += aux_coef * (cnt[e] / (double)N) / (double)N;"),
    "bwd_z_loss_not_doubled": ("dz[e] += z_coef * 2.0 * lse_n * p[e] / (double)N;",
                               "dz[e] += z_coef * lse_n * p[e] / (double)N;"),
    "bwd_gate_scaling_dropped": ("dg[e] += routed_scaling * dwj;", "dg[e] += dwj;"),
    "bwd_norm_term_dropped": ("for (int j = 0; j < k; ++j) dp[idn[j]] += dg[idn[j]] / S - gp / (S * S);",
                              "for (int j = 0; j < k; ++j) dp[idn[j]] += dg[idn[j]] / S;"),
    "bwd_W2_grad_transposed": ("for (int f = 0; f < F; ++f) dW2[(int64_t)c * F + f] += go[c] * h[f];",
                               "for (int f = 0; f < F; ++f) dW2[(int64_t)c * F + f] += go[f % d] * h[c % F];"),
    "partials_N_not_over_k": ("const double N = (double)total / (double)k;", "const double N = (double)total;"),
    "partials_P_unnormalised": ("double Pe = psum[e] / N;\n        L += f * Pe;\n    }\n    return L * (double)E;",
                                "double Pe = psum[e];\n        L += f * Pe;\n    }\n    return L * (double)E;"),
    "combine_drops_last_slot": ("for (int j = 0; j < k; ++j) {\n            const double *src",
                                "for (int j = 0; j + 1 < k; ++j) {\n            const double *src"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def test_unmutated_oracle_passes_every_pin():
    L = O.load()
    for pin in ALL_PINS:
        pin(L)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *O.GCC_FLAGS, str(src), "-lm", "-o", str(so)])
    L = O.load(str(so))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(L)
        except (AssertionError, O.OracleError, FloatingPointError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


# Mistakes planted in a copy of oracle.forward_tokens (plain Python): the
# per-token loop the full-size parity tests use for y on sampled tokens.
FORWARD_TOKENS_MUTANTS = {
    "slot_weights_swapped": ("y[s] += w[s, j] * outs[(s, j)]", "y[s] += w[s, k - 1 - j] * outs[(s, j)]"),
    "other_slot_output": ("y[s] += w[s, j] * outs[(s, j)]", "y[s] += w[s, j] * outs[(s, (j + 1) % k)]"),
    "wrong_expert_fetched": ("ew = expert_weights(e)", "ew = expert_weights(sorted(by_expert)[0])"),
    "wrong_token_row": ("outs[(s, j)] = expert_ffn(x_rows[s],", "outs[(s, j)] = expert_ffn(x_rows[(s + 1) % S],"),
    "key_transposed": ("by_expert.setdefault(int(ids[s, j]), []).append((s, j))",
                       "by_expert.setdefault(int(ids[s, j]), []).append((j % S, s % k))"),
}


@pytest.mark.parametrize("name", sorted(FORWARD_TOKENS_MUTANTS))
def test_forward_tokens_mutant_is_caught(name):
    old, new = FORWARD_TOKENS_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(O.forward_tokens))
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    scope = dict(vars(O))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), scope)
    L = O.load()
    pin_forward_tokens(L)  # the real function passes
    with pytest.raises((AssertionError, KeyError, IndexError, ValueError)):
        pin_forward_tokens(L, forward_tokens=scope["forward_tokens"])
