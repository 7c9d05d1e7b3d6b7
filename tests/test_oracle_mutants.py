"""Mutation check of the oracle's pins.

Each case below plants one plausible mistake in a copy of the oracle's source (on
the CPU, in a temporary directory) and runs the pin tests against that copy: the C
token loop against ``test_oracle_pins``, the gates and gated output of
``oracle/gates.py`` against ``test_oracle_gates``.  The pins must reject every
mutant; a mutant that survives means a mistake of that kind would go unnoticed.
"""
import importlib.util
import os
import subprocess

import numpy as np
import pytest

import oracle
import tests.test_oracle_gates as gate_pins
import tests.test_oracle_pins as pins
import tests.test_oracle_segments as seg_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

# (name, original text, replacement) -- every replacement keeps memory accesses in bounds.
MUTANTS = [
    ("no_decay", "for (int i = 0; i < DK * DV; ++i) S[i] *= a;", "(void)a;"),
    ("error_sign", "e[j] = v[j] - p;", "e[j] = v[j] + p;"),
    ("no_beta", "S[i * DV + j] += b * kh[i] * e[j];", "S[i * DV + j] += kh[i] * e[j];"),
    ("error_from_undecayed_state",
     "    for (int i = 0; i < DK * DV; ++i) S[i] *= a;\n    /* (2) e = v - St^T kh */\n"
     "    for (int j = 0; j < DV; ++j) {\n        double p = 0.0;\n"
     "        for (int i = 0; i < DK; ++i) p += S[i * DV + j] * kh[i];\n"
     "        e[j] = v[j] - p;\n    }\n",
     "    for (int j = 0; j < DV; ++j) {\n        double p = 0.0;\n"
     "        for (int i = 0; i < DK; ++i) p += S[i * DV + j] * kh[i];\n"
     "        e[j] = v[j] - p;\n    }\n    for (int i = 0; i < DK * DV; ++i) S[i] *= a;\n"),
    ("output_reads_query_unnormalised", "l2norm_vec(J->q + th * DK, DK, J->eps, J->l2norm, qh);\n"
     "        gdn_step(S, kh, qh, J->v + th * DV, J->alpha[th], J->beta[th], J->scale,\n"
     "                 J->y ? J->y + th * DV : NULL, e, DK, DV);",
     "l2norm_vec(J->q + th * DK, DK, J->eps, 0, qh);\n"
     "        gdn_step(S, kh, qh, J->v + th * DV, J->alpha[th], J->beta[th], J->scale,\n"
     "                 J->y ? J->y + th * DV : NULL, e, DK, DV);"),
    ("norm_without_sqrt", "double r = 1.0 / sqrt(ss + eps);", "double r = 1.0 / (ss + eps);"),
    ("y_scale_dropped", "y[j] = scale * acc;", "y[j] = acc;"),
    ("bwd_dalpha_uses_dS", "for (size_t i = 0; i < ssz; ++i) da += dSt[i] * Sprev[i];",
     "for (size_t i = 0; i < ssz; ++i) da += dS[i] * Sprev[i];"),
    ("bwd_dk_sign", "dkh[i] -= acc;", "dkh[i] += acc;"),
    ("bwd_state_grad_not_decayed", "for (size_t i = 0; i < ssz; ++i) dS[i] = a * dSt[i];",
     "for (size_t i = 0; i < ssz; ++i) dS[i] = dSt[i];"),
    ("bwd_norm_projection_dropped", "for (int i = 0; i < n; ++i) dx[i] = (dxh[i] - xh[i] * dot) * r;",
     "for (int i = 0; i < n; ++i) dx[i] = dxh[i] * r;"),
    ("bwd_dbeta_missing_error", "db += kh[i] * acc;", "db += kh[i];"),
    ("bwd_output_grad_unscaled", "dS[i * DV + j] += J->scale * qh[i] * dyv[j];",
     "dS[i * DV + j] += qh[i] * dyv[j];"),
]

# Pin tests that only use the C oracle (the chunked form is a separate implementation).
PIN_TESTS = [
    lambda: pins.test_hand_worked_examples("scalar_three_tokens.txt"),
    lambda: pins.test_hand_worked_examples("two_by_three.txt"),
    lambda: pins.test_hand_worked_examples("l2norm_one_token.txt"),
    pins.test_hand_worked_backward,
    pins.test_alpha1_beta0_is_identity,
    pins.test_one_token_outer_product,
    pins.test_beta1_unit_key_writes_exactly,
    pins.test_beta0_closed_form,
    pins.test_scale_multiplies_y_only,
    lambda: pins.test_chunked_form_matches_token_loop(16, True),
    lambda: pins.test_chunked_form_matches_token_loop(16, False),
    lambda: pins.test_backward_matches_central_differences(True),
    lambda: pins.test_backward_matches_central_differences(False),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mut = tmp_path / f"{name}.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o",
                           str(lib), str(mut), "-lm"])
    caught = []
    with oracle.use_library(str(lib)):
        for t in PIN_TESTS:
            try:
                t()
            except AssertionError:
                caught.append(t)
    assert caught, f"no pin rejects the planted mistake {name!r}"


GATES_SRC = os.path.join(os.path.dirname(oracle.__file__), "gates.py")

GATE_MUTANTS = [
    ("decay_rate_not_exponentiated", "g = -np.exp(A_log) * softplus(a + b_alpha)",
     "g = -A_log * softplus(a + b_alpha)"),
    ("decay_bias_outside_softplus", "g = -np.exp(A_log) * softplus(a + b_alpha)",
     "g = -np.exp(A_log) * (softplus(a) + b_alpha)"),
    ("softplus_as_log1p", "return np.logaddexp(0.0, _f64(x))", "return np.log1p(_f64(x))"),
    ("sigmoid_sign", "return 1.0 / (1.0 + np.exp(-x))", "return 1.0 / (1.0 + np.exp(x))"),
    ("norm_not_zero_centred", "return (1.0 + w) * y * r", "return w * y * r"),
    ("norm_sum_not_mean",
     "r = 1.0 / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)\n    return",
     "r = 1.0 / np.sqrt(np.sum(y * y, axis=-1, keepdims=True) + eps)\n    return"),
    ("bwd_alpha_chain_dropped", "dg_tot += _f64(dalpha) * alpha", "dg_tot += _f64(dalpha)"),
    ("bwd_dA_missing_g", "dA_log = np.sum(dg_tot * g, axis=(0, 1))",
     "dA_log = np.sum(dg_tot, axis=(0, 1))"),
    ("bwd_db_alpha_sign", "db_alpha = np.sum(da, axis=(0, 1))",
     "db_alpha = -np.sum(da, axis=(0, 1))"),
    ("bwd_beta_derivative", "* beta * (1.0 - beta)", "* beta"),
    ("bwd_gate_derivative", "dz = do * (1.0 + w) * n * s * (1.0 - s)",
     "dz = do * (1.0 + w) * n * s"),
    ("bwd_norm_projection_dropped",
     "dy = r * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))", "dy = r * dn"),
    ("layer_gate_swapped", "return gated_output(y, z, w, eps), y, sf",
     "return gated_output(z, y, w, eps), y, sf"),
]


def _python_mutant_caught(tmp_path, src_path, checks, name, old, new):
    src = open(src_path).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = tmp_path / f"mutant_{name}.py"
    path.write_text(src.replace(old, new))
    # a submodule of the oracle package, so that its relative imports resolve
    spec = importlib.util.spec_from_file_location(f"oracle._mutant_{name}", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    caught = []
    for check in checks:
        try:
            with np.errstate(all="ignore"):
                check(mod)
        except AssertionError:
            caught.append(check)
    return caught


@pytest.mark.parametrize("name,old,new", GATE_MUTANTS, ids=[m[0] for m in GATE_MUTANTS])
def test_gate_pins_reject_mutant(tmp_path, name, old, new):
    caught = _python_mutant_caught(tmp_path, GATES_SRC, gate_pins.CHECKS, name, old, new)
    assert caught, f"no pin rejects the planted mistake {name!r}"


SEGMENTS_SRC = os.path.join(os.path.dirname(oracle.__file__), "segments.py")

SEGMENT_MUTANTS = [
    ("token_map_without_decay", "M = alpha_t * (np.eye(kh.shape[0]) - beta_t * np.outer(kh, kh))",
     "M = np.eye(kh.shape[0]) - beta_t * np.outer(kh, kh)"),
    ("token_map_sign", "M = alpha_t * (np.eye(kh.shape[0]) - beta_t * np.outer(kh, kh))",
     "M = alpha_t * (np.eye(kh.shape[0]) + beta_t * np.outer(kh, kh))"),
    ("token_write_without_beta", "N = beta_t * np.outer(kh, v_t)", "N = np.outer(kh, v_t)"),
    ("compose_order", "return M2 @ M1, M2 @ N1 + N2", "return M1 @ M2, M2 @ N1 + N2"),
    ("compose_offset_not_carried", "return M2 @ M1, M2 @ N1 + N2", "return M2 @ M1, N1 + N2"),
    ("scan_inclusive", "        starts.append(S)\n        S = apply(m, S)",
     "        S = apply(m, S)\n        starts.append(S)"),
    ("chunk_map_decay_dropped", "mc = (gam[-1] * np.eye(dk) - Kd.T @ W, Kd.T @ Ut)",
     "mc = (np.eye(dk) - Kd.T @ W, Kd.T @ Ut)"),
    ("chunk_map_unscaled_keys", "Kd = Gam[-1][:, None] * K", "Kd = K"),
    ("segments_restart_from_s0", "                                beta[b:b + 1, t0:t1, h:h + 1], Ss[None, None], scale=scale,",
     "                                beta[b:b + 1, t0:t1, h:h + 1], S0[None, None], scale=scale,"),
]


@pytest.mark.parametrize("name,old,new", SEGMENT_MUTANTS, ids=[m[0] for m in SEGMENT_MUTANTS])
def test_segment_pins_reject_mutant(tmp_path, name, old, new):
    caught = _python_mutant_caught(tmp_path, SEGMENTS_SRC, seg_pins.CHECKS, name, old, new)
    assert caught, f"no pin rejects the planted mistake {name!r}"


CHUNKED_SRC = os.path.join(os.path.dirname(oracle.__file__), "chunked.py")

CHUNKED_CHECKS = [
    lambda m: pins.test_chunked_form_matches_token_loop(16, True, m),
    lambda m: pins.test_chunked_form_matches_token_loop(64, False, m),
    lambda m: pins.test_chunked_form_small_alpha_no_overflow(m),
    lambda m: pins.test_chunked_backward_matches_reverse_recurrence(16, True, m),
    lambda m: pins.test_chunked_backward_matches_reverse_recurrence(64, False, m),
    lambda m: pins.test_coupled_chunk_form_matches_token_loop(False, m),
    lambda m: pins.test_coupled_chunk_form_matches_token_loop(True, m),
    lambda m: pins.test_lag2_coupled_chunk_form_matches_token_loop(m),
    lambda m: pins.test_blocked_inverse_matches_dense_inverse(64, m),
    lambda m: pins.test_blocked_inverse_matches_dense_inverse(50, m),
]

CHUNKED_MUTANTS = [
    ("A_sign", "A = np.tril(be[:, None] * (K @ K.T) * Gam, k=-1)",
     "A = -np.tril(be[:, None] * (K @ K.T) * Gam, k=-1)"),
    ("output_without_decay_mask", "((Q @ K.T) * Gam) @ U", "(Q @ K.T) @ U"),
    ("state_not_decayed", "S = gam[-1] * S + (Gam[-1][:, None] * K).T @ U", "S = S + (Gam[-1][:, None] * K).T @ U"),
    ("W_without_gamma", "W = solve_triangular(IA, (be * gam)[:, None] * K, lower=True, unit_diagonal=True)\n"
     "                Ut = solve_triangular(IA, be[:, None] * V,",
     "W = solve_triangular(IA, be[:, None] * K, lower=True, unit_diagonal=True)\n"
     "                Ut = solve_triangular(IA, be[:, None] * V,"),
    ("bwd_dV_without_beta", "dV = be[:, None] * Z1", "dV = Z1"),
    ("bwd_dA_sign", "dA = np.tril(-(Tm.T @ dT @ Tm.T), k=-1)", "dA = np.tril(Tm.T @ dT @ Tm.T, k=-1)"),
    ("bwd_forward_cumsum", "dlna = np.cumsum(dG[::-1])[::-1]", "dlna = np.cumsum(dG)"),
    ("bwd_E_transpose_dropped", "dKh += E @ Kh + E.T @ Kh + F.T @ Qh", "dKh += E @ Kh + F.T @ Qh"),
    ("coupled_X_sign", 'ch[c]["X"] = -ch[c]["W"] @ ch[c - 1]["K"].T',
     'ch[c]["X"] = ch[c]["W"] @ ch[c - 1]["K"].T'),
    ("coupled_state_one_back_undecayed",
     'U.append(d["Ut"] + m["g"] * (-d["W"] @ S[c - 1]) + d["X"] @ (m["D"] * U[c - 1]))',
     'U.append(d["Ut"] + (-d["W"] @ S[c - 1]) + d["X"] @ (m["D"] * U[c - 1]))'),
    ("lag2_X2_term_dropped",
     '                             + m["g"] * (X2 @ (mm["D"] * U[c - 2])) + d["X"] @ (m["D"] * U[c - 1]))',
     '                             + d["X"] @ (m["D"] * U[c - 1]))'),
    ("lag2_state_decay_single", 'U.append(d["Ut"] + m["g"] * mm["g"] * (-d["W"] @ S[c - 2])',
     'U.append(d["Ut"] + m["g"] * (-d["W"] @ S[c - 2])'),
    ("unrolled_A2_second_term_dropped",
     'A2 = d["X"] @ (m["D"] * m["X"]) - m["g"] * d["W"] @ mm["K"].T', 'A2 = d["X"] @ (m["D"] * m["X"])'),
    ("inverse_offdiag_sign", "T[blk(bi), blk(bj)] = -T[blk(bi), blk(bi)] @ acc",
     "T[blk(bi), blk(bj)] = T[blk(bi), blk(bi)] @ acc"),
    ("inverse_offdiag_missing_far_terms",
     "acc = sum(A[blk(bi), blk(mb)] @ T[blk(mb), blk(bj)] for mb in range(bj, bi))",
     "acc = A[blk(bi), blk(bj)] @ T[blk(bj), blk(bj)]"),
    ("bwd_dU_without_decay", 'c["dU"] = c["dec"][:, None] * (c["Kh"] @ dS) + scale * c["QK"].T @ c["dY"]',
     'c["dU"] = (c["Kh"] @ dS) + scale * c["QK"].T @ c["dY"]'),
]


@pytest.mark.parametrize("name,old,new", CHUNKED_MUTANTS, ids=[m[0] for m in CHUNKED_MUTANTS])
def test_chunked_pins_reject_mutant(tmp_path, name, old, new):
    caught = _python_mutant_caught(tmp_path, CHUNKED_SRC, CHUNKED_CHECKS, name, old, new)
    assert caught, f"no pin rejects the planted mistake {name!r}"


CONV_SRC = os.path.join(os.path.dirname(oracle.__file__), "short_conv.py")

CONV_MUTANTS = [
    ("taps_reversed", "acc += w[:, i] * ext[t + i]", "acc += w[:, W - 1 - i] * ext[t + i]"),
    ("window_off_by_one", "acc += w[:, i] * ext[t + i]",
     "acc += w[:, i] * ext[min(t + i + 1, ext.shape[0] - 1)]"),
    ("state_ignored", "ext = np.concatenate([st[n], x[a:b]], axis=0)",
     "ext = np.concatenate([0.0 * st[n], x[a:b]], axis=0)"),
    ("final_state_from_first_rows", "final[n] = ext[ext.shape[0] - (W - 1):] if W > 1 else final[n]",
     "final[n] = ext[:W - 1] if W > 1 else final[n]"),
    ("silu_as_sigmoid", "return x / (1.0 + np.exp(-x))", "return 1.0 / (1.0 + np.exp(-x))"),
    ("documents_not_reset", "ext = np.concatenate([st[n], x[a:b]], axis=0)",
     "ext = np.concatenate([x[max(a - (W - 1), 0):a] if a >= W - 1 else st[n], x[a:b]], axis=0)"),
]


@pytest.mark.parametrize("name,old,new", CONV_MUTANTS, ids=[m[0] for m in CONV_MUTANTS])
def test_short_conv_pins_reject_mutant(tmp_path, name, old, new):
    import tests.test_oracle_short_conv as conv_pins
    caught = _python_mutant_caught(tmp_path, CONV_SRC, conv_pins.CHECKS, name, old, new)
    assert caught, f"no pin rejects the planted mistake {name!r}"


QSA_SRC = os.path.join(os.path.dirname(oracle.__file__), "qsa_indexer.py")

QSA_MUTANTS = [
    ("relu_dropped", "out.append(np.maximum(sim, 0.0).sum(axis=0))", "out.append(sim.sum(axis=0))"),
    ("max_over_heads", "out.append(np.maximum(sim, 0.0).sum(axis=0))",
     "out.append(np.maximum(sim, 0.0).max(axis=0))"),
    ("mask_misses_completed_block", "nvis = (i + 1) // r", "nvis = i // r"),
    ("mask_admits_partial_block", "nvis = (i + 1) // r", "nvis = (i + r) // r"),
    ("ties_to_higher_index", "key=lambda b: (-s[b], b)", "key=lambda b: (-s[b], -b)"),
    ("norm_without_gain", "return _f64(g) * x / np.sqrt(", "return x / np.sqrt("),
    ("partial_block_pooled", "nb = (b - a) // r", "nb = -(-(b - a) // r)"),
    ("selection_in_score_order", "sel = sorted(order)", "sel = list(order)"),
    ("blocks_from_stream_start", "rows.append(np.mean(k[a + r * j:a + r * (j + 1)], axis=0))",
     "rows.append(np.mean(k[r * j:r * (j + 1)], axis=0))"),
]


@pytest.mark.parametrize("name,old,new", QSA_MUTANTS, ids=[m[0] for m in QSA_MUTANTS])
def test_qsa_pins_reject_mutant(tmp_path, name, old, new):
    import tests.test_oracle_qsa as qsa_pins
    caught = _python_mutant_caught(tmp_path, QSA_SRC, qsa_pins.CHECKS, name, old, new)
    assert caught, f"no pin rejects the planted mistake {name!r}"
