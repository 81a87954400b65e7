"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each one.

The mutants are built from the committed oracle source with one textual change
each, compiled into a temporary directory; the committed oracle is untouched.
"""
import os

import pytest

import oracle
from oracle import build as obuild
import pins

# (name, exact text in wkv_oracle.c, replacement)
MUTANTS = [
    ("wkv6_drop_bonus", "u[i] * kt[i] * vt[j]", "0.0 * kt[i] * vt[j]"),
    ("wkv6_transposed_state", "(S[i * N + j] + u[i]", "(S[j * N + i] + u[i]"),
    ("wkv6_decay_wrong_axis", "wt[i] * S[i * N + j] + kt[i] * vt[j]",
     "wt[j] * S[i * N + j] + kt[i] * vt[j]"),
    ("wkv6_decay_before_output", "o += rt[i] * (S[i * N + j]", "o += rt[i] * (wt[i] * S[i * N + j]"),
    ("wkv6_ignore_s0", "S[e] = s0 ? s0[n * N * N + e] : 0.0;", "S[e] = 0.0;"),
    ("wkv6_wrong_head_u", "u + h * N, S, y + base", "u, S, y + base"),
    ("wkv6_kv_swapped_in_update", "+ kt[i] * vt[j];", "+ kt[j] * vt[i];"),
    ("wkv4_decay_sign", "double q2 = p - w > kt ? p - w : kt;\n        double e_decay = exp(p - w - q2);",
     "double q2 = p + w > kt ? p + w : kt;\n        double e_decay = exp(p + w - q2);"),
    ("wkv4_drop_bonus", "double e_now = exp(u + kt - q);", "double e_now = exp(kt - q);"),
    ("wkv4_bonus_in_state", "double e_key = exp(kt - q2);", "double e_key = exp(u + kt - q2);"),
    ("wkv4_output_after_decay", "double e_past = exp(p - q);", "double e_past = exp(p - w - q);"),
    ("wkv4_ignore_s0_max", "p = s0[(bi * 3 + 2) * C + c];", "p = 0.0;"),
    ("wkv4_denominator_uses_v", "(e_past * b + e_now)", "(e_past * b + e_now * vt)"),
    ("norm_unbiased_variance", "var /= (double)N;", "var /= (double)(N - 1);"),
    ("norm_drops_eps", "rstd = 1.0 / sqrt(var + eps);", "rstd = 1.0 / sqrt(var);"),
    ("gate_sigmoid_not_silu", "gn / (1.0 + exp(-gn))", "1.0 / (1.0 + exp(-gn))"),
    ("norm_shared_head_params", "ln_w[h * N + n] * (x[n] - mean)", "ln_w[n] * (x[n] - mean)"),
    ("norm_no_centering", "(x[n] - mean) * rstd", "x[n] * rstd"),
    ("gate_skips_shift", "gate * (ln_w[h * N + n] * (x[n] - mean) * rstd + ln_b[h * N + n])",
     "gate * ln_w[h * N + n] * (x[n] - mean) * rstd + ln_b[h * N + n]"),
    ("logit_single_exponential", "w[i] = exp(-exp(omega[i]));", "w[i] = exp(-omega[i]);"),
    ("logit_outer_sign", "w[i] = exp(-exp(omega[i]));", "w[i] = exp(exp(omega[i]));"),
    ("logit_inner_sign", "w[i] = exp(-exp(omega[i]));", "w[i] = exp(-exp(-omega[i]));"),
    ("logit_base_two", "w[i] = exp(-exp(omega[i]));", "w[i] = exp2(-exp(omega[i]));"),
    ("logit_skips_last", "for (int64_t i = 0; i < n; ++i) w[i]", "for (int64_t i = 0; i < n - 1; ++i) w[i]"),
    ("bwd_dk_drops_bonus", "b += L[i * N + j] * vt[j] + gt[j] * rt[i] * uh[i] * vt[j];", "b += L[i * N + j] * vt[j];"),
    ("bwd_dw_uses_next_state", "c += L[i * N + j] * S[i * N + j];",
     "c += L[i * N + j] * Sall[(t + 1) * NN + i * N + j];"),
    ("bwd_adjoint_transposed", "L[i * N + j] = wt[i] * L[i * N + j] + rt[i] * gt[j];",
     "L[i * N + j] = wt[i] * L[i * N + j] + rt[j] * gt[i];"),
    ("bwd_adjoint_decay_wrong_axis", "L[i * N + j] = wt[i] * L[i * N + j] + rt[i] * gt[j];",
     "L[i * N + j] = wt[j] * L[i * N + j] + rt[i] * gt[j];"),
    ("bwd_du_not_summed_over_batch", "du[h * N + i] += d;", "du[h * N + i] = d;"),
    ("bwd_ds0_not_propagated", "ds0[n * NN + e] = L[e];", "ds0[n * NN + e] = dsT ? dsT[n * NN + e] : 0.0;"),
    ("bwd_dv_bonus_without_u", "+ gt[j] * rt[i] * uh[i] * kt[i];", "+ gt[j] * rt[i] * kt[i];"),
    ("bwd_dr_decayed_state", "a += gt[j] * (S[i * N + j] + uh[i] * kt[i] * vt[j]);",
     "a += gt[j] * (wt[i] * S[i * N + j] + uh[i] * kt[i] * vt[j]);"),
    ("bwd_logit_grad_sign", "domega[i] = dw[i] * (-e * exp(-e));", "domega[i] = dw[i] * (e * exp(-e));"),
]


@pytest.fixture(scope="module")
def source():
    with open(obuild.SRC) as f:
        return f.read()


def test_committed_oracle_passes_all_pins():
    assert pins.failing_pins(oracle.get()) == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, source, name, old, new):
    assert source.count(old) == 1, f"mutation anchor for {name} not unique/present"
    src = tmp_path / f"{name}.c"
    src.write_text(source.replace(old, new))
    lib = obuild.build(str(src), str(tmp_path / f"lib_{name}.so"))
    bad = pins.failing_pins(oracle.Oracle(lib))
    assert bad, f"no pin caught the planted mistake {name}"
