"""Planted mistakes in the oracle, each of which one of its pins must catch.

The oracle is trusted because the tests in ``test_oracle_*.py`` pin it to what
the pages and the mathematics fix (printed figures, closed forms, brute force
over walks, finite differences, an independent route to log Z).  This file
checks that those pins are sharp: for every entry below it copies the oracle,
its pin tests and the seeded input generators into a scratch directory, plants
one plausible mistake there (a dropped term, a wrong sign, constant or index,
a transposed operand, a non-strict tie rule), rebuilds the copy and runs the
named pin, which must fail on an assertion.  A control run checks that the
unmodified copy passes every named pin, so a failure comes from the planted
mistake.  Nothing here touches the oracle in the repository, and nothing here
runs on a GPU.

Each entry: (name, file, text, replacement, occurrence, pin).  ``occurrence``
picks the match when the text is not unique (0 = first), else it must be.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
C = "oracle/tcq_oracle.c"
PY = "oracle/__init__.py"

MUTANTS = [
    # 1MAD codebook (QTIP blog, "The codebook is computed")
    ('lcg_mult', C,
     '34038481u * x',
     '34038483u * x',
     None, 'test_oracle_codebook.py::test_908_distinct_values_at_L16'),
    ('lcg_add', C,
     '+ 76625530u',
     '+ 76625531u',
     None, 'test_oracle_codebook.py::test_special_states_follow_the_printed_constants'),
    ('bytesum_drop_byte', C,
     '(int)((y >> 16) & 255u) + (int)((y >> 24) & 255u)',
     '(int)((y >> 16) & 255u)',
     None, 'test_oracle_codebook.py::test_908_distinct_values_at_L16'),
    ('bytesum_shift', C,
     '(int)((y >> 8) & 255u)',
     '(int)((y >> 9) & 255u)',
     None, 'test_oracle_codebook.py::test_908_distinct_values_at_L16'),
    ('center_510', C,
     '- 510.0) / 147.8',
     '- 512.0) / 147.8',
     None, 'test_oracle_codebook.py::test_special_states_follow_the_printed_constants'),
    ('scale_1478', C,
     '- 510.0) / 147.8',
     '- 510.0) / 148.7',
     None, 'test_oracle_codebook.py::test_special_states_follow_the_printed_constants'),
    # Viterbi, predecessor set and argmin rule (QTIP blog, "The trellis: a stateful codebook")
    ('vit32_pred_index', C,
     'int p = (j >> k) | (a << (L - k));\n                if (bestp < 0 || cost[p] < best)',
     'int p = (j >> k) | (a << (L - k - 1));\n                if (bestp < 0 || cost[p] < best)',
     0, 'test_oracle_viterbi.py::test_fp32_viterbi_walk_cost_is_sequential_sum[4]'),
    ('vit32_tie_le', C,
     'if (bestp < 0 || cost[p] < best) { best = cost[p]; bestp = p; }',
     'if (bestp < 0 || cost[p] <= best) { best = cost[p]; bestp = p; }',
     0, 'test_oracle_viterbi.py::test_all_ties_give_the_lowest_index_walk_by_hand'),
    ('vit32_final_tie_le', C,
     'if (cost[j] < cost[st]) st = j;',
     'if (cost[j] <= cost[st]) st = j;',
     None, 'test_oracle_viterbi.py::test_all_ties_give_the_lowest_index_walk_by_hand'),
    ('vit64_tie_le', C,
     'if (bestp < 0 || prev[p] < best)',
     'if (bestp < 0 || prev[p] <= best)',
     None, 'test_oracle_viterbi.py::test_all_ties_give_the_lowest_index_walk_by_hand'),
    ('vit64_final_tie_le', C,
     'if (last[j] < last[st]) st = j;',
     'if (last[j] <= last[st]) st = j;',
     None, 'test_oracle_viterbi.py::test_all_ties_give_the_lowest_index_walk_by_hand'),
    ('py_mse_denominator', PY,
     'mse[i] = np.float32(cost) / np.float32(T)',
     'mse[i] = np.float32(cost) / np.float32(T - 1)',
     None, 'test_oracle_viterbi.py::test_fp32_viterbi_walk_cost_is_sequential_sum[4]'),
    # Curvature-weighted step cost (XOR-Trellis explainer, "Cliff edges")
    ('vit32_D_index', C,
     'if (D) e = e * D[t];\n            next[j] = best + e;\n            back[(size_t)t * N + j] = bestp;\n        }\n        float *tmp = cost; cost = next; next = tmp;\n    }\n    int st = 0;',
     'if (D) e = e * D[t - 1];\n            next[j] = best + e;\n            back[(size_t)t * N + j] = bestp;\n        }\n        float *tmp = cost; cost = next; next = tmp;\n    }\n    int st = 0;',
     None, 'test_oracle_weighted.py::test_weighted_fp32_walk_cost_is_sequential_sum'),
    ('vit32_D_first_dropped', C,
     'cost[j] = D ? e * D[0] : e;\n    }\n    for (int t = 1; t < T; ++t) {\n        if (min_margin)',
     'cost[j] = e;\n    }\n    for (int t = 1; t < T; ++t) {\n        if (min_margin)',
     None, 'test_oracle_weighted.py::test_weighted_fp32_walk_cost_is_sequential_sum'),
    ('vit64_D_dropped', C,
     'cur[j] = best + (D ? D[t] : 1.0) * d * d;',
     'cur[j] = best + d * d;',
     None, 'test_oracle_weighted.py::test_weighted_viterbi_and_bcjr_match_brute_force[8-4]'),
    ('emis_D_dropped', C,
     'return (D ? D[t] : 1.0) * d * d;',
     'return d * d;',
     None, 'test_oracle_weighted.py::test_weighted_viterbi_and_bcjr_match_brute_force[8-4]'),
    ('vjp_D_dropped', C,
     'grad[u] = (2.0 * (D ? D[u] : 1.0) / temp)',
     'grad[u] = (2.0 / temp)',
     None, 'test_oracle_weighted.py::test_weighted_vjp_matches_central_differences'),
    # Decision margins along the returned walk
    ('margin32_absolute', C,
     '    return gap / den;',
     '    return gap;',
     None, 'test_oracle_viterbi.py::test_decision_margin_matches_enumeration[True]'),
    ('margin64_sign', C,
     'return (second - best) / den;',
     'return (best - second) / den;',
     None, 'test_oracle_viterbi.py::test_decision_margin_matches_enumeration[False]'),
    ('margin32_final_missing', C,
     'if (second < INFINITY) margin = fminf(margin, rel_gap_f32(total, second));',
     '',
     None, 'test_oracle_viterbi.py::test_decision_margin_matches_enumeration[True]'),
    # BCJR forward-backward and soft codeword (BCJR-QAT abstract)
    ('bcjr_alpha0_temp', C,
     'alpha[j] = -emis(code, s, D, 0, j) / temp;',
     'alpha[j] = -emis(code, s, D, 0, j);',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[0.1-4-2-6]'),
    ('bcjr_beta_emis_index', C,
     'tmp[b] = beta[(size_t)(t + 1) * N + nx] - emis(code, s, D, t + 1, nx) / temp;\n            }\n            beta[',
     'tmp[b] = beta[(size_t)(t + 1) * N + nx] - emis(code, s, D, t, nx) / temp;\n            }\n            beta[',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[1.0-4-2-6]'),
    ('bcjr_beta_succ', C,
     'int nx = ((i << k) | b) & (N - 1);\n                tmp[b] = beta[(size_t)(t + 1) * N + nx] - emis(code, s, D, t + 1, nx) / temp;\n            }\n            beta[',
     'int nx = ((i << k) | (b >> 1)) & (N - 1);\n                tmp[b] = beta[(size_t)(t + 1) * N + nx] - emis(code, s, D, t + 1, nx) / temp;\n            }\n            beta[',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[1.0-4-2-6]'),
    ('bcjr_beta_init_emission', C,
     'for (int i = 0; i < N; ++i) beta[(size_t)(T - 1) * N + i] = 0.0;',
     'for (int i = 0; i < N; ++i) beta[(size_t)(T - 1) * N + i] = -emis(code, s, D, T - 1, i) / temp;',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[1.0-4-2-6]'),
    ('lse_no_shift_back', C,
     'return m + log(acc);',
     'return log(acc);',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[1.0-4-2-6]'),
    ('soft_logz_row', C,
     'double lz = lse_array(alpha + (size_t)(T - 1) * N, N);\n    for (int t = 0; t < T; ++t) {\n        double acc = 0.0;',
     'double lz = lse_array(alpha + (size_t)(T - 2) * N, N);\n    for (int t = 0; t < T; ++t) {\n        double acc = 0.0;',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[1.0-4-2-6]'),
    ('bcjr_soft_abs_code', C,
     'acc += exp(alpha[(size_t)t * N + j] + beta[(size_t)t * N + j] - lz) * code[j];\n        soft[t] = acc;\n    }\n    if (log_z)',
     'acc += exp(alpha[(size_t)t * N + j] + beta[(size_t)t * N + j] - lz) * fabs(code[j]);\n        soft[t] = acc;\n    }\n    if (log_z)',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[1.0-4-2-6]'),
    # Vector-Jacobian product of the soft codeword (BCJR-QAT abstract)
    ('vjp_factor2', C,
     'grad[u] = (2.0 * (D ? D[u] : 1.0) / temp)',
     'grad[u] = ((D ? D[u] : 1.0) / temp)',
     None, 'test_oracle_bcjr.py::test_vjp_matches_central_differences[1.0]'),
    ('vjp_mean_term_dropped', C,
     '* (acc - ef * soft[u]);',
     '* acc;',
     None, 'test_oracle_bcjr.py::test_vjp_matches_central_differences[1.0]'),
    ('vjp_phi_v_index', C,
     'phi[(size_t)t * N + j] = acc + v[t] * code[j];',
     'phi[(size_t)t * N + j] = acc + v[t - 1] * code[j];',
     None, 'test_oracle_bcjr.py::test_vjp_matches_central_differences[1.0]'),
    ('vjp_psi_v_index', C,
     'acc += exp(tmp[b] - m) * (v[t + 1] * code[nx]',
     'acc += exp(tmp[b] - m) * (v[t] * code[nx]',
     None, 'test_oracle_bcjr.py::test_vjp_matches_central_differences[1.0]'),
    ('vjp_phi0_dropped', C,
     'for (int j = 0; j < N; ++j) phi[j] = v[0] * code[j];',
     'for (int j = 0; j < N; ++j) phi[j] = 0.0;',
     None, 'test_oracle_bcjr.py::test_vjp_matches_central_differences[1.0]'),
    # Brute force over walks
    ('brute_temp_dropped', C,
     'double p = exp(-(E - emin) / temp);',
     'double p = exp(-(E - emin));',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[0.1-4-2-6]'),
    ('brute_logz_emin', C,
     '*log_z = log(z) - emin / temp;',
     '*log_z = log(z);',
     None, 'test_oracle_bcjr.py::test_soft_matches_brute_force[1.0-4-2-6]'),
    ('brute_tb_wrap', C,
     'if ((x & low) == (x0 >> k) && E < emin) emin = E;',
     'if ((x & low) == (x0 & low) && E < emin) emin = E;',
     None, 'test_oracle_tailbiting.py::test_exact_equals_brute_force_over_tail_biting_walks[4-7]'),
    # Tail-biting search (QTIP blog, "Tail-biting is worth its complexity")
    ('pinned32_start_lowbits', C,
     'if ((j >> k) != o) { cost[j] = INFINITY; continue; }',
     'if ((j & low) != o) { cost[j] = INFINITY; continue; }',
     None, 'test_oracle_viterbi.py::test_all_ties_give_the_lowest_index_walk_by_hand'),
    ('pinned64_end_topbits', C,
     'if ((j & low) == o && (st < 0 || cost[j] < cost[st])) st = j;\n    double total',
     'if ((j >> k) == o && (st < 0 || cost[j] < cost[st])) st = j;\n    double total',
     None, 'test_oracle_tailbiting.py::test_exact_equals_brute_force_over_tail_biting_walks[4-7]'),
    ('pinned32_end_free', C,
     'if ((j & low) == o && (st < 0 || cost[j] < cost[st])) st = j;\n    float total',
     'if ((st < 0 || cost[j] < cost[st])) st = j;\n    float total',
     None, 'test_oracle_viterbi.py::test_all_ties_give_the_lowest_index_walk_by_hand'),
    ('py_alg4_seam_lowbits', PY,
     'overlap = st_rot[:, (T - h) % T].astype(np.int64) >> k',
     'overlap = st_rot[:, (T - h) % T].astype(np.int64) & ((1 << (L - k)) - 1)',
     None, 'test_oracle_tailbiting.py::test_algorithm4_matches_exact_at_L8'),
    ('py_exact_tb_first_overlap', PY,
     'for o in range(1 << (L - k)):',
     'for o in range(1 << (L - k - 1)):',
     None, 'test_oracle_tailbiting.py::test_exact_equals_brute_force_over_tail_biting_walks[4-7]'),
    # Bitstream decode and pack (QTIP blog, "The trellis" decode window; tail-biting stream)
    ('py_window_bit_order', PY,
     'out[:, t] |= bits[:, p].astype(np.int64) << (L - 1 - i)',
     'out[:, t] |= bits[:, p].astype(np.int64) << i',
     None, 'test_oracle_decode.py::test_free_start_windows_match_page_formula[8-13]'),
    ('py_window_no_wrap', PY,
     '            if layout == TAILBITING:\n                p %= nb\n',
     '            if layout == TAILBITING:\n                p = min(p, nb - 1)\n',
     None, 'test_oracle_decode.py::test_stream_lengths_count_the_walks[4-2-3]'),
    ('py_pack_tail_offset', PY,
     'bits[:, k * (T - 1) + i] = (states[:, T - 1] >> (L - 1 - i)) & 1',
     'bits[:, k * T + i - 1] = (states[:, T - 1] >> (L - 1 - i)) & 1',
     None, 'test_oracle_decode.py::test_stream_lengths_count_the_walks[4-2-3]'),
    ('py_pack_digit_bits', PY,
     'bits[:, k * t + i] = (states[:, t] >> (L - 1 - i)) & 1',
     'bits[:, k * t + i] = (states[:, t] >> (L - k + i)) & 1',
     None, 'test_oracle_decode.py::test_stream_lengths_count_the_walks[4-2-3]'),
    ('py_free_start_nbits', PY,
     'return k * T if layout == TAILBITING else k * T + L - k',
     'return k * T if layout == TAILBITING else k * T + L',
     None, 'test_oracle_decode.py::test_stream_lengths_count_the_walks[4-2-3]'),
    ('py_tile_order', PY,
     '.transpose(0, 2, 1, 3).reshape(rows, cols)',
     '.reshape(rows, cols)',
     None, 'test_oracle_decode.py::test_tile_layout'),
    # Random-sign Hadamard rotation (QTIP blog, "The trellis: a stateful codebook")
    ('py_hadamard_kernel', PY,
     'np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), h)',
     'np.kron(np.array([[1.0, 1.0], [-1.0, 1.0]]), h)',
     None, 'test_oracle_rht.py::test_hadamard_small_and_orthogonal'),
    ('py_rht_norm', PY,
     '@ hc) / np.sqrt(R * C)',
     '@ hc) / np.sqrt(R + C)',
     None, 'test_oracle_rht.py::test_rht_properties[16-32]'),
    ('py_rht_signs_swapped', PY,
     '(hr @ (np.asarray(sign_rows, np.float64)[:, None] * W * np.asarray(sign_cols, np.float64)[None, :])',
     '(hr @ (np.asarray(sign_cols, np.float64)[:, None] * W * np.asarray(sign_rows, np.float64)[None, :])',
     None, 'test_oracle_rht.py::test_rht_properties[16-32]'),
    ('py_hadamard_entry_parity', PY,
     'return 1.0 - 2.0 * (pc & 1)',
     'return 1.0 - 2.0 * ((pc >> 1) & 1)',
     None, 'test_oracle_rht.py::test_closed_form_entries_match_the_kronecker_construction'),
    ('py_rht_entries_transpose', PY,
     'out[a, b] = np.dot(hadamard_entry(i, rr) * s1, u)',
     'out[a, b] = np.dot(hadamard_entry(rr, i) * s1[::-1], u)',
     None, 'test_oracle_rht.py::test_closed_form_entries_match_the_kronecker_construction'),
    # Row blocks over host threads
    ('py_map_rows_edges', PY,
     'edges = np.linspace(0, n, threads + 1).astype(int)',
     'edges = np.linspace(0, n - 1, threads + 1).astype(int)',
     None, 'test_oracle_map_rows.py::test_viterbi_rows_match_direct_call[1]'),
]


def _plant(text, old, new, nth):
    count = text.count(old)
    if nth is None:
        assert count == 1, f"planted text matches {count} times"
        nth = 0
    assert count > nth, f"planted text matches {count} times"
    at = -1
    for _ in range(nth + 1):
        at = text.index(old, at + 1)
    return text[:at] + new + text[at + len(old):]


def _copy(dst):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "*.tmp*", "__pycache__"))
    shutil.copy(os.path.join(ROOT, "tcq_workloads.py"), dst)
    shutil.copy(os.path.join(ROOT, "pytest.ini"), dst)
    os.makedirs(os.path.join(dst, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for name in os.listdir(os.path.join(ROOT, "tests")):
        if name == "conftest.py" or (name.startswith("test_oracle_") and name.endswith(".py")
                                     and name != os.path.basename(__file__)):
            shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(dst, "tests", name))


def _run_pins(cwd, pins):
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        *[f"tests/{p}" for p in pins]],
                       cwd=cwd, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-1500:] + r.stderr[-500:]


def test_every_planted_mistake_is_caught(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is needed to rebuild the planted copies")
    names = [m[0] for m in MUTANTS]
    assert len(set(names)) == len(names)

    control = tmp_path / "control"
    _copy(str(control))
    rc, out = _run_pins(str(control), sorted({m[5] for m in MUTANTS}))
    assert rc == 0, "the unmodified copy fails a named pin:\n" + out

    def one(m):
        name, path, old, new, nth, pin = m
        dst = tmp_path / name
        _copy(str(dst))
        src = os.path.join(str(dst), path)
        with open(src) as f:
            text = f.read()
        with open(src, "w") as f:
            f.write(_plant(text, old, new, nth))
        rc, out = _run_pins(str(dst), [pin])
        shutil.rmtree(dst, ignore_errors=True)
        # exit code 1: tests ran and failed (2 would be a collection or build
        # error, a negative code a crash, 0 a surviving mistake)
        return None if rc == 1 else f"{name}: pin {pin} exited {rc}\n{out}"

    with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        missed = [r for r in ex.map(one, MUTANTS) if r]
    assert not missed, "planted mistakes not caught:\n" + "\n".join(missed)
