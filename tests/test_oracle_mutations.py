"""The oracle's pins detect planted mistakes.

Each case copies the oracle's C source, plants one plausible slip (a dropped
term, a wrong sign, a conjugation or pairing swap), compiles the copy into a
temporary library and checks that at least one pin of test_oracle_pins.py
fails on it.  Everything runs on the CPU; the real oracle is untouched.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_bwd_pins as bwd_pins
from tests import test_oracle_mimo_proj_pins as proj_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "mamba3_oracle.c")

MUTATIONS = {
    "drop_lag_term": ("(1.0 - lam) * dt * a[k] * u_prev[k * P + p]", "0.0 * u_prev[k * P + p]"),
    "lag_without_pole": ("(1.0 - lam) * dt * a[k] * u_prev[k * P + p]", "(1.0 - lam) * dt * u_prev[k * P + p]"),
    "lag_weight_lam": ("(1.0 - lam) * dt * a[k] * u_prev[k * P + p]", "lam * dt * a[k] * u_prev[k * P + p]"),
    "rotation_sign": ("cexp(dt * (At + I * th[k]))", "cexp(dt * (At - I * th[k]))"),
    "readout_no_conj": ("creal(conj(c) * Hs[k * P + p])", "creal(c * Hs[k * P + p])"),
    "pair_swap": ("(Bt[r * N + 2 * k] + I * Bt[r * N + 2 * k + 1])", "(Bt[r * N + 2 * k + 1] + I * Bt[r * N + 2 * k])"),
    "rope_sign": ("*o1 = -sin(phi) * v0 + cos(phi) * v1;", "*o1 = sin(phi) * v0 + cos(phi) * v1;"),
    "quadratic_weight_next": ("(1.0 - io->lam[in]) * io->dt[in]", "(1.0 - io->lam[is]) * io->dt[is]"),
    "mimo_rank_drop": ("for (int r = 0; r < R; ++r)\n          s += (Bt", "for (int r = 0; r < 1; ++r)\n          s += (Bt"),
    "decay_ignores_A_t": ("return io->A_t ? io->A_t[it] : io->A[h];", "return io->A[h];"),
    "bcnorm_sum_not_mean": ("    ms /= N;\n", "\n"),
    "bcnorm_eps_outside_sqrt": ("1.0 / sqrt(ms + eps)", "1.0 / (sqrt(ms) + eps)"),
    "bc_group_interleaved": ("h / (d->nheads / d->ngroups)", "h % d->ngroups"),
    "bwd_angle_sign_of_C": ("+ dc[0] * ct[1] - dc[1] * ct[0];", "- dc[0] * ct[1] + dc[1] * ct[0];"),
    "bwd_rotate_back_wrong_way": ("oB[0] = c * db[0] - sn * db[1];", "oB[0] = c * db[0] + sn * db[1];"),
    "bwd_no_lagged_adjoint": ("gup[i] = beta * gh[i];", "gup[i] = 0.0;"),
    "bwd_beta_not_through_alpha": ("const double d_alpha_all = d_alpha + d_beta * (1.0 - lam) * dt;",
                                   "const double d_alpha_all = d_alpha;"),
    "bwd_theta_without_dt": ("g->dtheta[it * K + k] = dt * S[k];", "g->dtheta[it * K + k] = S[k];"),
    "bwd_adjoint_not_decayed": ("for (size_t i = 0; i < NP; ++i) gh[i] *= alpha;", ""),
    "gate_before_norm": ("out[row * gsize + c] = yr[c] * inv * wt * (zv / (1.0 + exp(-zv)));",
                         "out[row * gsize + c] = yr[c] * wt * (zv / (1.0 + exp(-zv)));"),
    "gate_sigmoid_only": ("(zv / (1.0 + exp(-zv)))", "(1.0 / (1.0 + exp(-zv)))"),
    "gated_norm_sum_not_mean": ("ms /= (double)gsize;", "ms /= 1.0;"),
    "gated_norm_interleaved_groups": ("const size_t h = g * hpg + c / ((size_t)R * P)",
                                      "const size_t h = g + groups * (c / ((size_t)R * P))"),
    "mimo_up_weight_transposed": ("acc += W[(size_t)rp * P + q] * ut[q];", "acc += W[(size_t)q * P + rp % P] * ut[q];"),
    "mimo_down_rank_stride": ("acc += W[(size_t)p * R * P + rq] * yt[rq];", "acc += W[(size_t)p * R * P + rq % P] * yt[rq];"),
    "bcnorm_bias_index_swapped": ("const size_t p = ((size_t)h * R + r) * N + n;", "const size_t p = ((size_t)r * H + h) * N + n;"),
}

PIN_FUNCS = [
    lambda: [pins.test_time_invariant_equals_lfilter(l) for l in (0.0, 0.3, 0.5, 1.0)],
    lambda: [pins.test_impulse_closed_form(f) for f in ("scan_complex", "scan_rope", "scan_quadratic")],
    pins.test_lambda_one_is_exponential_euler,
    pins.test_lambda_zero_is_pure_lag,
    pins.test_theta_zero_is_real_ssm,
    pins.test_parity_toy,
    lambda: [pins.test_complex_equals_rope(r) for r in (1, 3)],
    lambda: [pins.test_quadratic_equals_recurrence(r) for r in (1, 2)],
    pins.test_mimo_is_superposition_of_siso,
    lambda: [pins.test_time_varying_decay_impulse_closed_form(f) for f in ("scan_complex", "scan_rope",
                                                                           "scan_quadratic")],
    pins.test_bc_norm_constant_row_closed_form,
    pins.test_bc_norm_unit_rms_per_row,
    pins.test_bc_norm_scale_invariant_and_odd,
    pins.test_bc_norm_weight_and_bias_per_head_and_rank,
    lambda: [pins.test_grouped_bc_equals_per_head_broadcast("scan_complex", G, R) for G, R in ((2, 2), (3, 1))],
    lambda: bwd_pins.test_backward_matches_finite_differences_of_the_definition({}),
    lambda: bwd_pins.test_backward_matches_finite_differences_of_the_definition(dict(R=1, L=11, H=3, N=6, P=2)),
    bwd_pins.test_backward_linear_in_x_and_state,
    pins.test_gate_is_silu_at_exact_points,
    pins.test_gate_odd_part_is_the_identity,
    lambda: [pins.test_normalised_group_has_unit_rms(g) for g in (1, 2, 6)],
    pins.test_gated_norm_scale_invariant_and_group_local,
    pins.test_gated_norm_weight_per_head_rank_channel_and_eps,
    bwd_pins.test_backward_linear_in_C_and_D,
    lambda: [proj_pins.test_up_and_down_equal_library_matrix_products(r) for r in (1, 4)],
    proj_pins.test_rank_one_weights_closed_form,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {name}"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "mut.c"
    so = tmp_path / "libmut.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(c), "-lm", "-lpthread"])
    saved = oracle._lib
    oracle._lib = oracle._bind(ctypes.CDLL(str(so)))
    try:
        failed = 0
        for f in PIN_FUNCS:
            try:
                f()
            except AssertionError:
                failed += 1
        assert failed >= 1, f"no pin caught mutation {name}"
    finally:
        oracle._lib = saved
