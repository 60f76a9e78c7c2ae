"""Planted mistakes in the oracle (CPU only).

Each case edits a copy of the oracle's C source in a temporary directory,
compiles it, and checks that at least one pin of ``oracle_pins`` rejects the
edited oracle. This shows the pins would catch a plausible slip anywhere in
the oracle: a dropped term, a wrong sign or index, swapped operands, a
misplaced nonlinearity. The committed oracle source is never modified.
"""
import pytest

import oracle
import oracle_pins

MUTANTS = [
    ("drop_skip_term", "double out = acc + dskip * xv;", "double out = acc;"),
    ("output_before_update",
     "h[n] = a_bar * h[n] + b_bar * xv;\n        acc += Ct[n] * h[n];",
     "acc += Ct[n] * h[n];\n        h[n] = a_bar * h[n] + b_bar * xv;"),
    ("exp_sign", "double a_bar = exp(dt * Arow[n]);",
     "double a_bar = exp(-dt * Arow[n]);"),
    ("B_and_C_swapped", "bbar_coeff(dt, Arow[n], bbar_mode) * Bt[n];",
     "bbar_coeff(dt, Arow[n], bbar_mode) * Ct[n];"),
    ("softplus_skipped", "return softplus_flag ? softplus(v) : v;", "return v;"),
    ("bias_outside_softplus",
     "double v = delta + (delta_bias ? delta_bias[d] : 0.0);\n"
     "    return softplus_flag ? softplus(v) : v;",
     "double v = delta;\n    return (softplus_flag ? softplus(v) : v)"
     " + (delta_bias ? delta_bias[d] : 0.0);"),
    ("gate_applied_twice", "out *= silu(*zv);", "out *= silu(silu(*zv));"),
    ("silu_sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    ("softplus_positive_branch", "v + log1p(exp(-v))", "v + log1p(exp(v))"),
    ("B_token_off_by_one", "int64_t j = (b * L + t) * N;\n                double dt",
     "int64_t j = (b * L + (t > 0 ? t - 1 : 0)) * N;\n                double dt"),
    ("zoh_divides_wrong", "expm1(dt * a) / a", "expm1(dt * a) * a"),
    ("compose_order", "*b_out = a_later * b_earlier + b_later;",
     "*b_out = a_earlier * b_later + b_earlier;"),
    ("decode_B_batch_ignored", "A + d * N, B + b * N,", "A + d * N, B,"),
    ("decode_dt_times_x_dropped",
     "h[n] = a_bar * h[n] + b_bar * xv;", "h[n] = a_bar * h[n] + b_bar;"),
    ("state_init_not_zero", "h[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;",
     "h[n] = h0 ? h0[(b * D + d) * N + n] : 1e-3;"),
    ("skip_uses_wrong_channel", "double dskip = Dv ? Dv[d] : 0.0;\n            for (int64_t t = 0; t < L; ++t)",
     "double dskip = Dv ? Dv[0] : 0.0;\n            for (int64_t t = 0; t < L; ++t)"),
    ("chunk_carry_dropped", "oracle_compose(P[c * N + n], H[c * N + n], 1.0,\n                                   hin[c * N + n],",
     "oracle_compose(P[c * N + n], H[c * N + n], 1.0,\n                                   0.0,"),
    # backward pass
    ("bwd_lambda_not_decayed", "lam[n] *= a_bar; /*", "lam[n] *= 1.0; /*"),
    ("bwd_dA_without_dt", "dA[d * N + n] += lam[n] * hprev * a_bar * dt;",
     "dA[d * N + n] += lam[n] * hprev * a_bar;"),
    ("bwd_softplus_grad_dropped", "double dv = softplus_flag ? ddt * sigmoid(v) : ddt;",
     "double dv = ddt;"),
    ("bwd_h_instead_of_hprev", "ddt += lam[n] * hprev * a_bar * Arow[n];",
     "ddt += lam[n] * h * a_bar * Arow[n];"),
    ("bwd_dx_skip_dropped", "dx[i] = du * dt + ds * dskip;", "dx[i] = du * dt;"),
    ("bwd_silu_grad_sign", "return sg * (1.0 + z * (1.0 - sg));",
     "return sg * (1.0 - z * (1.0 - sg));"),
    ("bwd_dB_without_x", "pB[t * N + n] += lam[n] * dt * x[i];",
     "pB[t * N + n] += lam[n] * dt;"),
    ("bwd_du_x_term_dropped", "    ddt += du * x[i];\n", "\n"),
    ("bwd_dfinal_ignored", "lam[n] = dfinal ? dfinal[(b * D + d) * N + n] : 0.0;",
     "lam[n] = 0.0;"),
    ("conv_tap_off_by_one", "int64_t s = t - (K - 1) + k;", "int64_t s = t - K + k;"),
    ("conv_silu_skipped", "x_out[(b * L + t) * D + d] = silu_flag ? silu(acc) : acc;",
     "x_out[(b * L + t) * D + d] = acc;"),
    ("conv_bias_dropped", "double acc = cb ? cb[d] : 0.0;", "double acc = 0.0;"),
    ("conv_filter_not_reversed", "acc += w[d * K + k] * x_in", "acc += w[d * K + (K - 1 - k)] * x_in"),
    ("conv_bwd_taps_not_transposed",
     "int64_t t = s + (K - 1) - k; /* the output token x_in[s] feeds via w[k] */",
     "int64_t t = s + k; /* the output token x_in[s] feeds via w[k] */"),
    ("conv_bwd_silu_grad_dropped", "dpre[i] = silu_flag ? dxc[i] * silu_grad(pre) : dxc[i];",
     "dpre[i] = dxc[i];"),
    ("bwd_gate_on_ds_dropped", "double ds = z ? dy[i] * silu(z[i]) : dy[i];",
     "double ds = dy[i];"),
    ("zoh_grad_dA_term_dropped",
     "dA[d * N + n] += lam[n] * hprev * a_bar * dt +\n"
     "                                             lam[n] * c_a * B[j + n] * x[i];",
     "dA[d * N + n] += lam[n] * hprev * a_bar * dt;"),
    ("zoh_grad_ddelta_uses_c", "lam[n] * c_dt * B[j + n] * x[i];",
     "lam[n] * c * B[j + n] * x[i];"),
    ("zoh_grad_limit_wrong", "*c_a = dt * dt * (0.5 + z / 3.0 + z * z / 8.0);",
     "*c_a = dt * dt * (1.0 + z / 3.0 + z * z / 8.0);"),
    ("bwd_dh0_missing_first_decay", "lam[n] *= a_bar; /* Abar_t",
     "if (t > 0) lam[n] *= a_bar; /* Abar_t"),
    ("bwd_dC_uses_previous_state", "pC[t * N + n] += ds * h;", "pC[t * N + n] += ds * hprev;"),
    ("bwd_bias_grad_without_softplus", "ddelta_bias[d] += dv;", "ddelta_bias[d] += ddt;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert old in src, f"mutation site for {name} not found"
    path = tmp_path / f"mutant_{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.build(str(path), str(tmp_path / f"libmutant_{name}.so"))
    mutant = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the planted mistake {name}"
