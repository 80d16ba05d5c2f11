"""Plant plausible mistakes in a copy of the oracle's C source and check that
the pins catch each one (CPU only; the planted mistakes never reach a GPU)."""
import os

import pytest

import oracle
import oracle_pins

# (name, text in ln_oracle.c, replacement): each is a mistake someone could
# plausibly make when writing LayerNorm and its hand-derived gradient.
MUTANTS = [
    ("unbiased_variance", "double var = sq / (double)C;",
     "double var = sq / (double)(C - 1);"),
    ("mean_divisor", "double m = sum / (double)C;",
     "double m = sum / (double)(C + 1);"),
    ("eps_outside_root", "1.0 / sqrt(var + eps)", "1.0 / (sqrt(var) + eps)"),
    ("eps_dropped", "1.0 / sqrt(var + eps)", "1.0 / sqrt(var + 1e-300)"),
    ("affine_swapped", "o[c] = xhat * weight[c] + bias[c];",
     "o[c] = xhat * bias[c] + weight[c];"),
    ("dinp_mean_term_dropped", "(g - mean_g - xhat * mean_gxhat)",
     "(g - xhat * mean_gxhat)"),
    ("dinp_xhat_term_dropped", "(g - mean_g - xhat * mean_gxhat)", "(g - mean_g)"),
    ("dinp_sign_flipped", "(g - mean_g - xhat * mean_gxhat)",
     "(g - mean_g + xhat * mean_gxhat)"),
    ("dinp_rstd_dropped", "dx[c] = s * (", "dx[c] = ("),
    ("g_without_weight", "double g = dy[c] * weight[c];", "double g = dy[c];"),
    ("dweight_without_xhat", "dweight[c] += dy[c] * xhat;", "dweight[c] += dy[c];"),
    ("xhat_divides_by_rstd", "double xhat = (x[c] - m) * s;",
     "double xhat = (x[c] - m) / s;"),
    ("dbias_times_weight", "dbias[c] += dy[c];", "dbias[c] += dy[c] * weight[c];"),
    ("dweight_uses_g", "dweight[c] += dy[c] * xhat;", "dweight[c] += g * xhat;"),
    # rounding to a format
    ("round_ties_away", "nearbyint(ldexp(v, -q))", "round(ldexp(v, -q))"),
    ("round_truncates", "nearbyint(ldexp(v, -q))", "trunc(ldexp(v, -q))"),
    ("round_one_bit_short", "int q = e - p;", "int q = e - p + 1;"),
    ("round_no_gradual_underflow", "if (q < emin - p + 1) q = emin - p + 1;", ""),
    ("round_no_overflow", "fabs(r) > max_finite ? copysign(INFINITY, v) : r", "r"),
    # residual forward
    ("residual_drops_branch", "x[i] = resid[i] + branch[i];", "x[i] = resid[i];"),
    ("residual_not_rounded", "int rc = oracle_round_format(x, x, N * C, p, emin, max_finite);",
     "int rc = ORACLE_OK;"),
    # backward variants
    ("accumulate_dinp_ignored", "dinp[i] = accumulate_dinp ? dinp[i] + g_in[i] : g_in[i];",
     "dinp[i] = g_in[i];"),
    ("accumulate_dinp_subtracts", "dinp[i] = accumulate_dinp ? dinp[i] + g_in[i] : g_in[i];",
     "dinp[i] = accumulate_dinp ? dinp[i] - g_in[i] : g_in[i];"),
    ("accumulate_params_ignored",
     "dweight[j] = accumulate_params ? dweight[j] + g_w[j] : g_w[j];", "dweight[j] = g_w[j];"),
    ("accumulate_dbias_ignored",
     "dbias[j] = accumulate_params ? dbias[j] + g_b[j] : g_b[j];", "dbias[j] = g_b[j];"),
    ("recompute_ignored", "            m = st_m;\n            s = st_s;\n", ""),
    ("recompute_without_eps",
     "rc = oracle_ln_forward(scratch, st_m, st_s, inp, weight, zeros, N, C, eps);",
     "rc = oracle_ln_forward(scratch, st_m, st_s, inp, weight, zeros, N, C, 1e-300);"),
]


# the mutants are built inside the repository, in a folder git ignores
MUTANT_DIR = os.path.join(os.path.dirname(oracle.SOURCE), "_build", "mutants")


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, old, new):
    src = open(oracle.SOURCE).read()
    assert old in src, f"mutation site for {name} no longer in the oracle source"
    os.makedirs(MUTANT_DIR, exist_ok=True)
    mutant_src = os.path.join(MUTANT_DIR, f"{name}.c")
    with open(mutant_src, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.compile_oracle(mutant_src, os.path.join(MUTANT_DIR, f"{name}.so"))
    mutant = oracle.Oracle(library=lib, source=mutant_src)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant {name}"
