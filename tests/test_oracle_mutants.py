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


# Mistakes planted in the oracle's numpy quality references (naive per-tensor W8A8 and
# per-token / per-channel W8A8 without smoothing); the copy of the package runs with the
# real C library, so only the planted line differs.
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")
PY_MUTANTS = {
    "naive_scale_per_row": ("    sx = np.abs(x).max() / 127.0\n", "    sx = np.abs(x).max(axis=1, keepdims=True) / 127.0\n"),
    "naive_weight_truncates": ("qw = np.clip(np.rint(w / sw if sw > 0 else 0 * w), -127, 127)",
                               "qw = np.clip(np.trunc(w / sw if sw > 0 else 0 * w), -127, 127)"),
    "naive_scale_128": ("    sw = np.abs(w).max() / 127.0\n", "    sw = np.abs(w).max() / 128.0\n"),
    "ptpc_ties_away": ("qx = np.clip(np.rint(np.where(sx > 0, x / sx, 0.0)), -127, 127)",
                       "qx = np.clip(np.sign(x) * np.floor(np.abs(np.where(sx > 0, x / sx, 0.0)) + 0.5), -127, 127)"),
    "ptpc_drops_sw": ("    y = (qx @ qw.T) * sx * sw.T\n", "    y = (qx @ qw.T) * sx\n"),
    "ptpc_tensor_scale_for_w": ("    sw = np.abs(w).max(axis=1, keepdims=True) / 127.0\n",
                                "    sw = np.abs(w).max() / 127.0 + 0.0 * np.abs(w).max(axis=1, keepdims=True)\n"),
    # the per-token producer-side quantization (a composition of pinned steps)
    "dyn_relu_dropped": ("        y = np.where(y > 0, y, np.float16(0)).astype(np.float16)\n",
                         "        y = y.astype(np.float16)\n"),
    "dyn_inv_s_dropped": ("    return ln_quant_act(y, None, None, inv_s_next)\n", "    return ln_quant_act(y, None, None, None)\n"),
    "dyn_relu_abs": ("        y = np.where(y > 0, y, np.float16(0)).astype(np.float16)\n",
                     "        y = np.abs(y).astype(np.float16)\n"),
}


def _run_pins_on_copy(tmp_path, src_text):
    """Run test_oracle.py against a copy of the oracle package whose __init__.py is src_text."""
    import shutil

    from oracle import build as oracle_build

    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    (tmp_path / "oracle" / "__init__.py").write_text(src_text)
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests", ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copy(os.path.join(ROOT, "sq_inputs.py"), tmp_path / "sq_inputs.py")
    env = dict(os.environ, SQ_ORACLE_LIB=oracle_build.build())
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           str(tmp_path / "tests" / "test_oracle.py")],
                          env=env, cwd=str(tmp_path), capture_output=True, text=True)


def test_python_mutant_harness_passes_the_real_oracle(tmp_path):
    # the copy itself must pass, so a failing mutant run means the planted line was caught
    r = _run_pins_on_copy(tmp_path, open(PY_SRC).read())
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_catch_python_mutant(name, tmp_path):
    old, new = PY_MUTANTS[name]
    src = open(PY_SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique in the oracle package"
    r = _run_pins_on_copy(tmp_path, src.replace(old, new))
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "1 failed" in r.stdout, r.stdout[-2000:]
