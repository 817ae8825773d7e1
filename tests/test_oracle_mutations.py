"""Plant plausible mistakes in a temporary copy of the oracle and show that the
pins catch each one. The committed oracle is never modified: every mutant is a
text substitution on a copy, compiled to a temporary library. CPU only."""

import os
import subprocess
import tempfile

import pytest

import oracle
from oracle_checks import ALL_CHECKS

SRC = os.path.join(os.path.dirname(oracle.__file__), "hstu_oracle.c")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("drop_pos_term",
     "if (pos) s += pos[(int64_t)h * num_pos + hstu_oracle_pos_index(i, j, num_pos)];", ""),
    ("drop_time_term", "if (ts && tbias)\n", "if (0)\n"),
    ("causal_excludes_diagonal", "for (int64_t j = 0; j <= i; ++j) {\n            const double* kj",
     "for (int64_t j = 0; j < i; ++j) {\n            const double* kj"),
    ("time_diff_sign", "hstu_oracle_time_bucket(ts[o + i] - ts[o + j], num_buckets)];",
     "hstu_oracle_time_bucket(ts[o + j] - ts[o + i], num_buckets)];"),
    ("pos_index_off_by_one", "int64_t r = i - j;", "int64_t r = i - j + 1;"),
    ("pos_no_clip", "if (r > num_pos - 1) r = num_pos - 1;", "if (r > num_pos - 1) r = r % num_pos;"),
    ("q_k_transposed", "const double* qi = q + t * q_tok + (int64_t)h * dqk;",
     "const double* qi = k + t * k_tok + (int64_t)h * dqk;"),
    ("no_1_over_N", "a[c] /= (double)max_seqlen;", "a[c] /= 1.0;"),
    ("sigmoid_not_silu", "return x / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(-x));"),
    ("bit_length_not_floor_log2", "while (x > 1) {", "while (x > 0) {"),
    ("no_max_1", "int64_t x = dt < 1 ? 1 : dt;", "int64_t x = dt < 0 ? -dt : (dt < 1 ? 1 : dt);"),
    ("bucket_clamp_low", "if (bkt > num_buckets - 1) bkt = num_buckets - 1;",
     "if (bkt > num_buckets - 1) bkt = num_buckets - 2;"),
    ("unbiased_variance", "var /= (double)F;", "var /= (double)(F - 1);"),
    ("eps_outside_sqrt", "double rstd = 1.0 / sqrt(var + eps);", "double rstd = 1.0 / (sqrt(var) + eps);"),
    ("gate_dropped", "*= u[m * u_ld + c];", "*= 1.0;"),
    ("split_q_k_swapped", "uvqk + 2 * F, W, uvqk + 3 * F, W,", "uvqk + 3 * F, W, uvqk + 2 * F, W,"),
    ("split_u_v_swapped", "memcpy(urow + r * F, uvqk + t * W,", "memcpy(urow + r * F, uvqk + t * W + F,"),
    ("residual_dropped", "hstu_oracle_linear(n, (int32_t)F, D, ygate, W2, b2, 0, xrow, out);",
     "hstu_oracle_linear(n, (int32_t)F, D, ygate, W2, b2, 0, NULL, out);"),
    ("linear_bias_dropped",
     "for (int32_t c = 0; c < K; ++c) acc += x[m * K + c] * W[(int64_t)n * K + c];\n"
     "            if (bias) acc += bias[n];",
     "for (int32_t c = 0; c < K; ++c) acc += x[m * K + c] * W[(int64_t)n * K + c];\n"),
    ("silu_after_bias_missing",
     "if (bias) acc += bias[n];\n            if (act_silu) acc = hstu_oracle_silu(acc);\n"
     "            if (residual) acc += residual[m * N + n];\n            y[m * N + n] = acc;\n"
     "        }\n    }\n}\n\n/* ------",
     "if (bias) acc += bias[n];\n"
     "            if (residual) acc += residual[m * N + n];\n            y[m * N + n] = acc;\n"
     "        }\n    }\n}\n\n/* ------"),
    ("input_norm_not_applied", "        xin = xn;\n", "        xin = x;\n"),
    ("input_norm_residual_normalized", "memcpy(xrow + r * D, x + t * D,", "memcpy(xrow + r * D, xin + t * D,"),
    ("layernorm_no_affine", "yr[c] = (ar[c] - mean) * rstd * (gamma ? gamma[c] : 1.0) + (beta ? beta[c] : 0.0);",
     "yr[c] = (ar[c] - mean) * rstd;"),
    ("e4m3_ties_away", "return fmod(f, 2.0) == 0.0 ? f : f + 1.0;", "return f + 1.0;"),
    ("e4m3_exponent_bias_8", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3_no_subnormals", "if (e == 0) v = ldexp((double)m / 8.0, -6);",
     "if (e == 0) v = 0.0;"),
    ("e4m3_overflow_to_nan", "if (a >= 448.0) return sign | 0x7E;",
     "if (a > 448.0) return sign | 0x7F;"),
    ("quant_scale_not_amax", "if (v > amax) amax = v;", "if (v > amax) amax = v * 0.5f;"),
    ("quant_inv_overflow_unchecked", "const int finite = amax > 0.0f && q <= FLT_MAX;",
     "const int finite = amax > 0.0f;"),
    ("fp8_scale_inverted", "acc *= (double)sx[m] * (double)sw[n];",
     "acc *= (double)sx[m] / (double)sw[n];"),
    ("bwd_silu_grad_is_sigmoid", "return sg * (1.0 + s * (1.0 - sg));", "return sg;"),
    ("bwd_dk_uses_k", "dk[((o + j) * H + h) * dqk + c] += ds * qi[c];",
     "dk[((o + j) * H + h) * dqk + c] += ds * kj[c];"),
    ("bwd_ds_missing_1_over_N", "const double ds = dp * hstu_oracle_silu_grad(s) * inv_n;",
     "const double ds = dp * hstu_oracle_silu_grad(s);"),
    ("bwd_dtime_dropped", "if (dtime && bkt >= 0) dtime[(int64_t)h * num_buckets + bkt] += ds;",
     ""),
]


@pytest.fixture(scope="module")
def tmpdir_mod():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmpdir_mod, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor for %s not unique in the oracle" % name
    path_c = os.path.join(tmpdir_mod, name + ".c")
    path_so = os.path.join(tmpdir_mod, name + ".so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o",
                           path_so, path_c, "-lm"])
    lib = oracle.load(path_so)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(lib)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, "no pin catches mutant %s" % name
