"""Plant plausible mistakes in copies of the oracle source and check that the
pins in test_oracle.py catch every one (a pin set that passes a broken oracle
pins nothing).  Runs on the CPU only; the real oracle is never modified."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sq_oracle.c")

MUTANTS = {
    "alpha_swapped": ("pow(x, a) / pow(w, 1.0 - a)", "pow(x, 1.0 - a) / pow(w, a)"),
    "truncate_not_round": ("float r = rintf(p);", "float r = truncf(p);"),
    "ties_away_from_zero": ("float r = rintf(p);", "float r = roundf(p);"),
    "scale_128": ("return amax / 127.0f;", "return amax / 128.0f;"),
    "clamp_128": ("if (r < -127.0f) r = -127.0f;", "if (r < -128.0f) r = -128.0f;"),
    "weight_index_reversed": ("sum += (int32_t)xq[t * K + k] * (int32_t)wq[n * K + k];\n      acc[t * N + n] = sum;",
                              "sum += (int32_t)xq[t * K + k] * (int32_t)wq[n * K + (K - 1 - k)];\n      acc[t * N + n] = sum;"),
    "dequant_drops_sw": ("      v = v * sw[n];\n      if (bias) v = v + h2f(bias[n]);\n      y[t * N + n] = f2h(v);\n    }\n}\n\n/* The whole",
                         "      v = v * 1.0f;\n      if (bias) v = v + h2f(bias[n]);\n      y[t * N + n] = f2h(v);\n    }\n}\n\n/* The whole"),
    "ln_sign": ("float d = h2f(h[k]) - mu;", "float d = h2f(h[k]) + mu;"),
    "ln_variance_sign": ("double var = ex2 - mean * mean;", "double var = ex2 + mean * mean;"),
    "ln_drops_beta": ("out[k] = beta ? u + beta[k] : u;", "out[k] = u;"),
    "fold_divides": ("f2h(h2f(w[n * K + j]) * s[j])", "f2h(h2f(w[n * K + j]) / s[j])"),
    "fold_ln_dropped": ("if (gamma) gamma_out[j] = gamma[j] * inv_s[j];", "if (gamma) gamma_out[j] = gamma[j];"),
    "calib_no_abs": ("float a = fabsf(scratch_row[j]);", "float a = scratch_row[j];"),
    "smooth_not_applied": ("for (int64_t k = 0; k < K; ++k) out[k] = out[k] * inv_s[k];",
                           "for (int64_t k = 0; k < K; ++k) out[k] = out[k];"),
    "zero_row_inf": ("return scale > 0.0f ? 1.0f / scale : 0.0f;", "return 1.0f / scale;"),
    "o2_range_of_last_token": ("  for (int64_t t = 0; t < M; ++t) {\n    act_row(h + t * ld, K, gamma, beta, inv_s, eps, scratch_row);\n    for (int64_t k = 0; k < K; ++k) {",
                               "  for (int64_t t = 0; t < M; ++t) {\n    act_row(h + t * ld, K, gamma, beta, inv_s, eps, scratch_row);\n    range = 0.0f;\n    for (int64_t k = 0; k < K; ++k) {"),
    "tensor_range_ignores_inv_s": ("float a = inv_s ? amax[j] * inv_s[j] : amax[j];", "float a = amax[j];"),
    "producer_relu_dropped": ("if (relu && !(a > 0.0f)) a = 0.0f;", "if (relu && 0) a = 0.0f;"),
    "producer_no_fp16_round": ("float a = h2f(f2h(v));", "float a = v;"),
    "producer_inv_s_not_applied": ("float x = inv_s_next ? a * inv_s_next[n] : a;", "float x = a;"),
    "bmm_scales_of_item_0": ("float v = (float)sum * a_scale[i * M + m];", "float v = (float)sum * a_scale[m];"),
    "bmm_b_of_item_0": ("const int8_t* bi = b + i * N * K;", "const int8_t* bi = b;"),
    "weight_tensor_scale_per_row": ("  for (int64_t n = 0; n < N; ++n) sw[n] = sc;", "  for (int64_t n = 0; n < N; ++n) sw[n] = n ? sc : 1.0f;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique in the oracle source"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                    str(mut), "-o", str(so), "-lm"], check=True)
    env = dict(os.environ, SQ_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
