"""Plants plausible mistakes in a copy of the CPU oracle's source and checks
that the pins in test_oracle_pins.py catch every one of them.  The planted
copies are compiled into a temporary directory; the real oracle is not
touched.  CPU only."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import tests.test_oracle_pins as pins
from oracle import ref

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "externd_ref.cpp")

# (name, original text, planted text)
MUTATIONS = [
    ("deflate_sign", "if (s > 0) row[j] = row[j] - d;", "if (s > 0) row[j] = row[j] + d;"),
    ("threshold_not_strict", "out[j] = (a > thr)", "out[j] = (a >= thr)"),
    ("threshold_mean_square", "tau * std::sqrt(s / (double)len)", "tau * (s / (double)len)"),
    ("u_step_drops_weight", "s += (double)row[j] * ((double)v[j] * wt(w, j));",
     "s += (double)row[j] * ((double)v[j]);"),
    ("scale_den_unweighted", "double den = (double)nu * vw;", "double den = (double)nu * (double)nv;"),
    ("gain_not_squared", "out[5] = den > 0.0 ? p * p / den : 0.0;", "out[5] = den > 0.0 ? p / den : 0.0;"),
    ("safeguard_flipped", "if (sc[5] < M) {", "if (sc[5] > M) {"),
    ("init_row_argmin", "if (s > rho[best]) best = i;", "if (s < rho[best]) best = i;"),
    ("energy_unweighted", "s += wt(w, j) * (double)R[i * n + j] * (double)R[i * n + j];",
     "s += (double)R[i * n + j] * (double)R[i * n + j];"),
    ("v_step_transposed_sign", "z[j] += (double)u[i] * (double)row[j];",
     "z[j] -= (double)u[i] * (double)row[j];"),
    ("block_ridge_large", "return tr > 0.0 ? 1e-6 * tr / (double)b : 1.0;",
     "return tr > 0.0 ? 1e-1 * tr / (double)b : 1.0;"),
    ("block_closed_form_sign", "e -= 2.0 * (double)dl[a] * r[a];", "e += 2.0 * (double)dl[a] * r[a];"),
    ("safeguard_keeps_u", "std::fill(u.begin(), u.end(), 0);", ";"),
    ("block_gram_unweighted", "s += wt(w, j) * V[l * n + j] * V[l2 * n + j];",
     "s += V[l * n + j] * V[l2 * n + j];"),
    ("block_u_target_unweighted", "s += (double)R[i * n + j] * wt(w, j) * V[l * n + j];",
     "s += (double)R[i * n + j] * V[l * n + j];"),
    ("safeguard_score_drops_weight", "float s = sq * w[j];", "float s = sq;"),
    ("mean_abs_statistic_ignored", "s += stat == 1 ? std::fabs(x[j]) : x[j] * x[j];",
     "s += x[j] * x[j];"),
    ("naive_vstep_drops_weight", "wz[j] = (double)w[j] * z[j];", "wz[j] = z[j];"),
    ("block_naive_drops_weight", "for (int64_t j = 0; j < n; ++j) Q[l * n + j] *= (double)w[j];",
     "for (int64_t j = 0; j < n; ++j) Q[l * n + j] *= 1.0;"),
    ("sweep_addback_sign", "orc_deflate(R, m, n, Ul, Vl, -D[l]);  // add back",
     "orc_deflate(R, m, n, Ul, Vl, D[l]);  // add back"),
    ("sweep_choice_flipped", "} else if (sc[5] > g_old) {", "} else if (sc[5] < g_old) {"),
    ("sweep_old_scale_not_resolved", "d = den_old > 0.0 ? (float)(p_old / den_old) : 0.0f;",
     "d = D[l];"),
    ("sweep_single_entry_ignores_old", "const double g_best = sc[5] > g_old ? sc[5] : g_old;",
     "const double g_best = sc[5];"),
    ("apply_drops_scale", "const double sc = (double)D[c] * t[c];", "const double sc = t[c];"),
    ("apply_sign_dropped", "if (V[c * n + j]) s += (double)V[c * n + j] * (double)x[j];",
     "if (V[c * n + j]) s += (double)x[j];"),
]

PIN_TESTS = [
    pins.test_ternarize_hand_computed,
    lambda o: pins.test_prop1_scale_minimises_and_gain_is_exact(o, False),
    lambda o: pins.test_prop1_scale_minimises_and_gain_is_exact(o, True),
    pins.test_deflation_is_one_fp32_subtract,
    pins.test_half_steps_against_numpy,
    lambda o: pins.test_bruteforce_every_ternary_pair(o, 2),
    lambda o: pins.test_bruteforce_every_ternary_pair(o, 3),
    pins.test_safeguard_zeroes_best_entry,
    pins.test_weighted_safeguard_takes_largest_weighted_square,
    lambda o: pins.test_prop2_geometric_bound(o, 0.5),
    pins.test_monotone_residual_and_replay,
    pins.test_reconstruct_matches_matmul_and_energy,
    pins.test_weighted_energy_is_weighted_norm,
    pins.test_block_scales_solve_normal_equations,
    lambda o: pins.test_block_targets_solve_their_normal_equations(o, False),
    lambda o: pins.test_block_targets_solve_their_normal_equations(o, True),
    pins.test_block_energy_matches_replay,
    pins.test_exact_recovery_of_ternary_rank1,
    pins.test_exact_recovery_of_two_disjoint_components,
    pins.test_ternarize_mean_abs_hand_computed,
    pins.test_naive_vstep_against_numpy,
    lambda o: pins.test_block_variant_targets(o, True),
    lambda o: pins.test_sweep_steps_match_a_replay_by_hand(o, False),
    lambda o: pins.test_sweep_steps_match_a_replay_by_hand(o, True),
    pins.test_sweeps_never_raise_the_residual,
    pins.test_ternary_apply_against_numpy_and_the_reconstruction,
    pins.test_ternary_apply_exact_on_integers,
]


def _build_planted(tmp, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, name
    src = os.path.join(tmp, f"{name}.cpp")
    open(src, "w").write(text.replace(old, new))
    lib = os.path.join(tmp, f"lib{name}.so")
    subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", src,
                    "-o", lib], check=True)
    return lib


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new):
    real = ref.lib()
    with tempfile.TemporaryDirectory() as tmp:
        path = _build_planted(tmp, name, old, new)
        ref._lib = None
        saved = ref._build.build
        ref._build.build = lambda force=False: path
        caught = []
        try:
            ref.lib()
            for t in PIN_TESTS:
                try:
                    t(ref)
                except AssertionError:
                    # only a failed check counts as a catch; a planted copy
                    # that crashes or cannot load is an error of the harness
                    caught.append(getattr(t, "__name__", "lambda"))
                    break
        finally:
            ref._build.build = saved
            ref._lib = real
    assert caught, f"planted mistake {name} went undetected by every pin"
