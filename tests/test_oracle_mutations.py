"""Planted mistakes in the oracle are caught by its pins (CPU only).

Each case copies oracle/oracle.c, plants one plausible mistake in the copy (a
flipped sign, a dropped term, a wrong index, a transposed operand, a wrong
rounding rule), compiles it, and runs the pin tests of test_oracle_pins.py
against that build.  The case passes only if the pin named beside the mistake
fails; a mistake that no pin notices would mean that part of the oracle is
unpinned.  The control case runs the pins on an unmodified copy built the same
way and needs them all to pass.

The copies live in a temporary directory; the committed oracle is never
touched.  The mistakes cover the expert arithmetic, the routing and its top-k
margins, the backward, the number formats and the placement of the bf16
rounding mirrors in the forward and the backward (a mirror dropped, moved or
added where the layer keeps fp32).
"""
import concurrent.futures
import os
import re
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_C = os.path.join(ROOT, "oracle", "oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (id, text in oracle.c (occurs exactly once), replacement, pin that must fail)
MUTATIONS = [
    # expert arithmetic
    ("silu_sign",
     "return g / (1.0 + exp(-g)); }", "return g / (1.0 + exp(g)); }",
     "test_single_expert_equals_dense_swiglu"),
    ("swiglu_operands_swapped",
     "h[i] = silu(g[i]) * u[i];\n    if (c->mx)", "h[i] = silu(u[i]) * g[i];\n    if (c->mx)",
     "test_single_expert_equals_dense_swiglu"),
    ("up_rows_read_from_gate_half",
     "b += xd[h] * ld(s->Wgu, s->gu_off + (int64_t)(s->I + i) * H + h, c->w_kind);",
     "b += xd[h] * ld(s->Wgu, s->gu_off + (int64_t)i * H + h, c->w_kind);",
     "test_single_expert_equals_dense_swiglu"),
    ("down_weight_transposed",
     "a += h[i] * ld(s->Wdn, s->dn_off + (int64_t)n * s->I + i, c->w_kind);",
     "a += h[i] * ld(s->Wdn, s->dn_off + (int64_t)i * c->H + n, c->w_kind);",
     "test_single_expert_equals_dense_swiglu"),
    ("shared_expert_dropped",
     "double wj = shared ? 1.0 : w[(int64_t)t * k + j];\n            gate_up(c, &s, xd, g, u);\n            swiglu_h",
     "double wj = shared ? 0.0 : w[(int64_t)t * k + j];\n            gate_up(c, &s, xd, g, u);\n            swiglu_h",
     "test_single_expert_equals_dense_swiglu"),
    ("routing_weight_not_applied",
     "acc[n2] += wj * o[n2];", "acc[n2] += o[n2];",
     "test_mirrors_sit_at_stored_tensors"),
    ("y_not_rounded_to_bf16",
     "y[(int64_t)ti * H + n2] = mirror(c, acc[n2]);", "y[(int64_t)ti * H + n2] = acc[n2];",
     "test_mirrors_sit_at_stored_tensors"),
    ("h_not_rounded_to_bf16",
     "for (int i = 0; i < I; i++) h[i] = mirror(c, h[i]);", "for (int i = 0; i < I; i++) h[i] = h[i];",
     "test_mirrors_sit_at_stored_tensors"),
    # routing
    ("weights_not_renormalised",
     "w[j] = c->routed_scale * prob[ord[j]] / tot;", "w[j] = c->routed_scale * prob[ord[j]];",
     "test_softmax_topk_bruteforce"),
    ("routed_scale_dropped",
     "w[j] = c->routed_scale * prob[ord[j]] / tot;", "w[j] = prob[ord[j]] / tot;",
     "test_sigmoid_group_limited_bruteforce"),
    ("selection_bias_in_weights",
     "w[j] = c->routed_scale * prob[ord[j]] / tot;", "w[j] = c->routed_scale * sc[ord[j]] / tot;",
     "test_sigmoid_group_limited_bruteforce"),
    ("ties_to_higher_index",
     "(key[idx[j]] == key[v] && idx[j] > v)", "(key[idx[j]] == key[v] && idx[j] < v)",
     "test_ties_go_to_lower_index"),
    ("group_score_best_only",
     "gsc[g] = sc[g * gs + wo[0]] + (gs > 1 ? sc[g * gs + wo[1]] : 0.0);", "gsc[g] = sc[g * gs + wo[0]];",
     "test_sigmoid_group_limited_bruteforce"),
    ("dispatch_tokens_descending",
     "for (int t = 0; t < T; t++)\n        for (int j = 0; j < k; j++) {\n            int64_t s",
     "for (int t = T - 1; t >= 0; t--)\n        for (int j = 0; j < k; j++) {\n            int64_t s",
     "test_dispatch_invariants"),
    # backward
    ("softmax_dlogit_sign",
     "dl[j] = w[j] * (G[j] - gbar);", "dl[j] = w[j] * (gbar - G[j]);",
     "test_gradients_match_finite_differences"),
    ("sigmoid_derivative_term_dropped",
     "dl[j] = rho / S * (G[j] - gbar) * s * (1.0 - s);", "dl[j] = rho / S * (G[j] - gbar) * s;",
     "test_gradients_match_finite_differences"),
    ("silu_derivative_term_dropped",
     "double dg = dh[i] * ub * sg * (1.0 + gb * (1.0 - sg)), du = dh[i] * gb * sg;",
     "double dg = dh[i] * ub * sg, du = dh[i] * gb * sg;",
     "test_gradients_match_finite_differences"),
    ("du_uses_g_not_silu",
     "double dg = dh[i] * ub * sg * (1.0 + gb * (1.0 - sg)), du = dh[i] * gb * sg;",
     "double dg = dh[i] * ub * sg * (1.0 + gb * (1.0 - sg)), du = dh[i] * gb;",
     "test_gradients_match_finite_differences"),
    ("dx_misses_router_path",
     "dx[(int64_t)ti * H + q] = mirror(c, acc[q] + r);", "dx[(int64_t)ti * H + q] = mirror(c, acc[q]);",
     "test_gradients_match_finite_differences"),
    ("drouter_wrong_slot",
     "a += dl[(int64_t)r * k + slot[r]] * ld(", "a += dl[(int64_t)r * k] * ld(",
     "test_gradients_match_finite_differences"),
    ("down_dgrad_transposed",
     "dh[i] += d * ld(s->Wdn, s->dn_off + (int64_t)n * s->I + i, c->w_kind);",
     "dh[i] += d * ld(s->Wdn, s->dn_off + (int64_t)i * c->H + n, c->w_kind);",
     "test_gradients_match_finite_differences"),
    ("dw_down_unweighted_h",
     "HW[(int64_t)r * I + i] = mirror(c, wr[r] * h[i]);", "HW[(int64_t)r * I + i] = mirror(c, h[i]);",
     "test_gradients_match_finite_differences"),
    # top-k margins (the gap margin rejection reads) and non-finite scores
    ("gap_on_unbiased_scores",
     "double d = tmp[ord[j]] - tmp[ord[j + 1]];", "double d = prob[ord[j]] - prob[ord[j + 1]];",
     "test_margin_gap_sigmoid_groups_bruteforce"),
    ("group_gap_dropped",
     "double d = gsc[gord[i]] - gsc[gord[i + 1]];\n            if (d < gap) gap = d;",
     "double d = gsc[gord[i]] - gsc[gord[i + 1]];\n            (void)d;",
     "test_margin_gap_sigmoid_groups_bruteforce"),
    ("gap_misses_kth_neighbour",
     "for (int j = 0; j < k && j + 1 < ncand; j++) {", "for (int j = 0; j + 1 < k && j + 1 < ncand; j++) {",
     "test_margin_gap_softmax_bruteforce"),
    ("nan_score_not_ranked_last",
     "for (int e = 0; e < E; e++) if (isnan(sc[e])) sc[e] = -INFINITY;", "",
     "test_nan_scores_rank_last"),
    # where the backward rounds to bf16 (the stored tensors)
    ("saved_gu_not_rounded",
     "double gb = mirror(c, g[i]), ub = mirror(c, u[i]);", "double gb = g[i], ub = u[i];",
     "test_backward_mirrors_sit_at_stored_tensors"),
    ("dh_rounded_instead_of_dgu",
     "double dg = dh[i] * ub * sg * (1.0 + gb * (1.0 - sg)), du = dh[i] * gb * sg;\n        dgu[i] = mirror(c, dg);\n"
     "        dgu[I + i] = mirror(c, du);",
     "double dg = mirror(c, dh[i]) * ub * sg * (1.0 + gb * (1.0 - sg)), du = mirror(c, dh[i]) * gb * sg;\n"
     "        dgu[i] = dg;\n        dgu[I + i] = du;",
     "test_backward_mirrors_sit_at_stored_tensors"),
    ("wh_not_rounded",
     "HW[(int64_t)r * I + i] = mirror(c, wr[r] * h[i]);", "HW[(int64_t)r * I + i] = wr[r] * h[i];",
     "test_backward_mirrors_sit_at_stored_tensors"),
    ("dx_not_rounded",
     "dx[(int64_t)ti * H + q] = mirror(c, acc[q] + r);", "dx[(int64_t)ti * H + q] = acc[q] + r;",
     "test_backward_mirrors_sit_at_stored_tensors"),
    ("dw_gate_up_not_rounded",
     "dWgu[(int64_t)n * H + q] = mirror(c, a);", "dWgu[(int64_t)n * H + q] = a;",
     "test_backward_mirrors_sit_at_stored_tensors"),
    ("slot_dx_rows_rounded",
     "acc[q] += dxs[q];     /* per-slot dx rows are stored in fp32 */",
     "acc[q] += mirror(c, dxs[q]);",
     "test_backward_mirrors_sit_at_stored_tensors"),
    # number formats
    ("bf16_truncates",
     "double r = ldexp(nearbyint(ldexp(a, -q)), q);\n    if (r > 3.3895313892515355e38)",
     "double r = ldexp(trunc(ldexp(a, -q)), q);\n    if (r > 3.3895313892515355e38)",
     "test_bf16_rounding_matches_torch"),
    ("e4m3_ties_away_from_zero",
     "double r = ldexp(nearbyint(ldexp(a, -q)), q);\n    if (r > 448.0)",
     "double r = ldexp(round(ldexp(a, -q)), q);\n    if (r > 448.0)",
     "test_e4m3_rounding_matches_torch"),
    ("e4m3_no_saturation",
     "if (r > 448.0) r = 448.0;", "if (r > 1e300) r = 448.0;",
     "test_e4m3_rounding_matches_torch"),
    ("mx_scale_boundary",
     "while (amax > ldexp(448.0, e)) e++;", "while (amax >= ldexp(448.0, e)) e++;",
     "test_mx_scale_golden"),
    ("mx_x_not_quantised",
     "if (c->mx)\n        for (int b = 0; b < c->H; b += 32) mx_block(xd + b",
     "if (0)\n        for (int b = 0; b < c->H; b += 32) mx_block(xd + b",
     "test_mxfp8_single_expert_matches_fakequant_mlp"),
    ("mx_h_not_quantised",
     "for (int b = 0; b < I; b += 32) mx_block(h + b, 32, NULL, NULL);",
     "for (int b = 0; b < 0; b += 32) mx_block(h + b, 32, NULL, NULL);",
     "test_mxfp8_single_expert_matches_fakequant_mlp"),
    # MXFP8 backward (the data-gradient products on MXFP8 operands)
    ("mx_dy_not_quantised",
     "if (c->mx)\n        for (int b = 0; b < c->H; b += 32) mx_block(dyq + b",
     "if (0)\n        for (int b = 0; b < c->H; b += 32) mx_block(dyq + b",
     "test_mxfp8_backward_restated"),
    ("mx_down_dgrad_reads_forward_copy",
     "a[i] += d * ld(s->Wdn_b,", "a[i] += d * ld(s->Wdn,",
     "test_mxfp8_backward_restated"),
    ("mx_gate_up_dgrad_reads_forward_copy",
     "const void *Wg = c->mx ? s->Wgu_b : s->Wgu;", "const void *Wg = s->Wgu;",
     "test_mxfp8_backward_restated"),
    ("mx_slot_grad_after_routing_weight",
     "        down_dgrad_mx(c, s, dyq, dh);\n        if (G) {",
     "        down_dgrad_mx(c, s, dyq, dh);\n        for (int i = 0; i < I; i++) dh[i] *= wj;\n        if (G) {",
     "test_mxfp8_backward_restated"),
    ("mx_dgu_not_quantised",
     "for (int b = 0; b < 2 * I; b += 32) mx_block(raw + b, 32, NULL, NULL);",
     "for (int b = 0; b < 0; b += 32) mx_block(raw + b, 32, NULL, NULL);",
     "test_mxfp8_backward_restated"),
    ("mx_dw_down_unquantised_h",
     "swiglu_h(c, g, u, I, h);                  /* stored h: bf16, or MX blocks */",
     "for (int i = 0; i < I; i++) h[i] = mirror(c, silu(g[i]) * u[i]);",
     "test_mxfp8_backward_restated"),
    ("mx_column_blocks_skipped",
     "for (int64_t r0 = 0; r0 < R; r0 += 32) {", "for (int64_t r0 = 0; r0 < R; r0 += 64) {",
     "test_mx_fakequant_cols_is_rows_of_transpose"),
]
CONTROL = ("control", None, None, None)


def _build_and_run(tmp, case):
    name, old, new, _ = case
    src = open(ORACLE_C).read()
    if old is not None:
        if src.count(old) != 1:
            return name, ("bad-site", src.count(old))
        src = src.replace(old, new)
    d = os.path.join(tmp, name)
    os.makedirs(d, exist_ok=True)
    c_path, so_path = os.path.join(d, "oracle.c"), os.path.join(d, "liboracle.so")
    open(c_path, "w").write(src)
    cc = subprocess.run(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", c_path, "-o", so_path, "-lm"],
                        capture_output=True, text=True)
    if cc.returncode != 0:
        return name, ("compile", cc.stderr[-2000:])
    env = dict(os.environ, **{oracle.LIB_ENV: so_path, "OMP_NUM_THREADS": "2"})
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-rf", PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    failed = sorted(set(re.findall(r"FAILED \S+::(test_\w+)", r.stdout)))
    return name, (r.returncode, failed, r.stdout[-3000:])


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    tmp = str(tmp_path_factory.mktemp("planted"))
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        return dict(ex.map(lambda c: _build_and_run(tmp, c), MUTATIONS + [CONTROL]))


def test_control_copy_passes_every_pin(outcomes):
    rc, failed, out = outcomes["control"]
    assert rc == 0 and not failed, out


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(outcomes, name, old, new, pin):
    res = outcomes[name]
    assert res[0] not in ("bad-site", "compile"), res
    rc, failed, out = res
    assert rc == 1, out          # 1: tests ran and some failed (not a collection or usage error)
    assert pin in failed, (failed, out)
