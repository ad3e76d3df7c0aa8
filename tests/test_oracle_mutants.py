"""Plant one mistake at a time in a copy of the oracle source and require the
pin suite to catch every one of them.  The mutants are compiled on the CPU
and never touch a GPU."""
import os

import pytest

from oracle.oracle import Oracle, compile_oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "moe_oracle.c")

# (name, exact source text, replacement): each a plausible slip.
MUTANTS = [
    ("drop_bias", "logit[e] += (double)bias[e];", "logit[e] += 0.0 * (double)bias[e];"),
    ("no_routing_weight", "const double yc = wj * o[c];", "const double yc = o[c];"),
    ("silu_sign", "h[n] = g[n] / (1.0 + exp(-g[n])) * u[n];", "h[n] = g[n] / (1.0 + exp(g[n])) * u[n];"),
    ("renormalise", "weights[t * k + j] = ranked[j].p;",
     "weights[t * k + j] = ranked[j].p / (ranked[0].p + ranked[k - 1].p);"),
    ("transposed_down", "o[c] += hn * bf16_to_double(drow[c]);", "o[c] += hn * bf16_to_double(wd[c * f + n]);"),
    ("tie_highest_index", "return (ra->e > rb->e) - (ra->e < rb->e);", "return (ra->e < rb->e) - (ra->e > rb->e);"),
    ("reverse_group_order", "for (int64_t a = 0; a < n; ++a) {\n        int32_t pos",
     "for (int64_t a = n - 1; a >= 0; --a) {\n        int32_t pos"),
    ("up_uses_gate", "u[n] += xi * bf16_to_double(urow[n]);", "u[n] += xi * bf16_to_double(grow[n]);"),
    ("dropped_last_hidden_term", "for (int64_t i = 0; i < d; ++i) {\n            double xi",
     "for (int64_t i = 0; i < d - 1; ++i) {\n            double xi"),
    ("softmax_no_norm", "for (int64_t e = 0; e < E; ++e) prob[e] /= s;", "for (int64_t e = 0; e < E; ++e) prob[e] /= 1.0;"),
    ("weights_from_wrong_slot", "weights[t * k + j] = ranked[j].p;", "weights[t * k + j] = ranked[0].p;"),
    ("sum_only_first_slot", "orow[c] += yc;", "orow[c] += (j == 0) ? yc : 0.0;"),
    ("renorm_no_divide", "weights[t * k + j] /= s;", "weights[t * k + j] /= 1.0;"),
    ("round_drops_largest", "qsort(in, (size_t)n_in, sizeof(cand_t), drop_order);",
     "qsort(in, (size_t)n_in, sizeof(cand_t), add_order);"),
    ("round_adds_smallest", "qsort(out, (size_t)n_out, sizeof(cand_t), add_order);",
     "qsort(out, (size_t)n_out, sizeof(cand_t), drop_order);"),
    ("round_drop_tie_smaller_index", "return (x->t < y->t) - (x->t > y->t);",
     "return (x->t > y->t) - (x->t < y->t);"),
    ("round_one_short", "const int64_t add = R - r;", "const int64_t add = R - r - 1;"),
    ("masked_weight_one", "const double we = probs[t * E + e];", "const double we = 1.0;"),
    ("shared_first_only", "for (int64_t sidx = 0; sidx < n_s; ++sidx) {",
     "for (int64_t sidx = 0; sidx < 1; ++sidx) {"),
    ("shared_half_weight", "for (int64_t c = 0; c < d; ++c) out[r * d + c] += o[c];",
     "for (int64_t c = 0; c < d; ++c) out[r * d + c] += 0.5 * o[c];"),
    ("renorm_partial_sum", "for (int64_t j = 0; j < k; ++j) s += weights[t * k + j];",
     "for (int64_t j = 0; j + 1 < k; ++j) s += weights[t * k + j];"),
    ("bwd_silu_derivative_short", "dg[n] = dh[n] * u[n] * sg * (1.0 + g[n] * (1.0 - sg));",
     "dg[n] = dh[n] * u[n] * sg;"),
    ("bwd_no_routing_weight", "for (int64_t c = 0; c < d; ++c) dz[c] = wj * drow_out[c];",
     "for (int64_t c = 0; c < d; ++c) dz[c] = drow_out[c];"),
    ("bwd_softmax_no_centering", "for (int64_t e = 0; e < E; ++e) dl[e] = p[e] * (dp[e] - pdp);",
     "for (int64_t e = 0; e < E; ++e) dl[e] = p[e] * dp[e];"),
    ("bwd_dx_without_router", "acc += dl[e] * bf16_to_double(wrow[e]);", "acc += 0.0 * dl[e] * bf16_to_double(wrow[e]);"),
    ("bwd_up_grad_uses_gate", "du[n] = dh[n] * (g[n] * sg);", "du[n] = dh[n] * g[n];"),
    ("bwd_renorm_no_dot", "dp[ids[t * k + j]] = (dwj[j] - dot) / ssum;", "dp[ids[t * k + j]] = dwj[j] / ssum;"),
    ("bwd_down_transposed", "acc += dz[c] * bf16_to_double(wd[n * d + c]);",
     "acc += dz[c] * bf16_to_double(wd[c * f + n]);"),
    ("bwd_rows_without_router", "            for (int64_t e = 0; e < E; ++e) acc += dl[e] * bf16_to_double(wrow[e]);\n            dxr[i] += acc;",
     "            for (int64_t e = 0; e < E; ++e) acc += 0.0 * dl[e] * bf16_to_double(wrow[e]);\n            dxr[i] += acc;"),
    ("bwd_rows_no_routing_weight", "for (int64_t c = 0; c < d; ++c) dz[c] = w[j] * drow_out[c];",
     "for (int64_t c = 0; c < d; ++c) dz[c] = drow_out[c];"),
    ("bwd_expert_no_routing_weight", "for (int64_t c = 0; c < d; ++c) dz[c] = w[t * k + j] * drow_out[c];",
     "for (int64_t c = 0; c < d; ++c) dz[c] = drow_out[c];"),
    ("bwd_expert_up_uses_gate", "                    dw_up_e[i * f + n] += xrow[i] * du[n];",
     "                    dw_up_e[i * f + n] += xrow[i] * dg[n];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    # the per-token and per-expert restrictions of the backward repeat some of
    # its lines; a slip in such a line is planted in every copy of it
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mut_src = tmp_path / f"mut_{name}.c"
    mut_src.write_text(src.replace(old, new))
    lib = compile_oracle(str(mut_src), str(tmp_path / f"lib_{name}.so"), force=True)
    o = Oracle(lib)
    failed = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(o)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {name}"
