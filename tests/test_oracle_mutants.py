"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle/pe_oracle.c (on the CPU),
builds it, and runs the pin suite against it in a child process; the suite has
to fail.  The real oracle is never modified.  The children run concurrently
(one OpenMP thread each), once per module; each case then reads its result.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pe_oracle.c")

MUTANTS = {
    "window_inner_order_swapped": ("(g_h % m) * m + (g_w % m)", "(g_w % m) * m + (g_h % m)"),
    "window_outer_order_w_major": ("(g_t * (h / m) + g_h / m) * (w / m) + g_w / m",
                                   "(g_t * (w / m) + g_w / m) * (h / m) + g_h / m"),
    "bias_dropped": ("out[r * E + e] = acc + (bias ? (double)bias[e] : 0.0);",
                     "out[r * E + e] = acc;"),
    "bias_dropped_patches": ("out[n * E + e] = acc + (bias ? (double)bias[e] : 0.0);",
                             "out[n * E + e] = acc;"),
    "norm_sign": ("volatile float d = x - mean;", "volatile float d = x + mean;"),
    "norm_reciprocal_multiply": ("volatile float q = d / std;",
                                 "volatile float q = d * (1.0f / std);"),
    "pad_repeats_first_frame": ("const int src = tau < T ? tau : T - 1;",
                                "const int src = tau < T ? tau : 0;"),
    "conv_i_j_transposed": ("const int64_t y = g_h * p + i, xx = g_w * p + j;",
                            "const int64_t y = g_h * p + j, xx = g_w * p + i;"),
    "patch_x_k_order_t_major": ("oracle_bf16_round(x[n * K + k])",
                                "oracle_bf16_round(x[n * K + (((int64_t)t * C + c) * p + i) * p + j])"),
    "weight_not_rounded": ("oracle_bf16_round_array(w, wb, (int64_t)E * K);\n    const int64_t ncell",
                           "memcpy(wb, w, sizeof(float) * (size_t)(E * K));\n    const int64_t ncell"),
    "bf16_truncates": ("u = (u + 0x7fffu + ((u >> 16) & 1u)) & 0xffff0000u;",
                       "u = u & 0xffff0000u;"),
    "bf16_ties_away": ("u = (u + 0x7fffu + ((u >> 16) & 1u)) & 0xffff0000u;",
                       "u = (u + 0x8000u) & 0xffff0000u;"),
    "input_not_rounded": ("const double xv = (double)oracle_bf16_round(x[n * K + k]);",
                          "const double xv = (double)x[n * K + k];"),
    "fp32_form_rounds_input": ("const double xv = (double)x[n * K + k];",
                               "const double xv = (double)oracle_bf16_round(x[n * K + k]);"),
    "fp32_form_neighbour_column": ("const double xv = (double)x[n * K + k];",
                                   "const double xv = (double)x[n * K + (k ^ 1)];"),
    "merger_window_columns_transposed": ("hln[(int64_t)q * E + e] = (double)oracle_bf16_round((float)y);",
                                         "hln[(int64_t)e * m2 + q] = (double)oracle_bf16_round((float)y);"),
    "merger_unbiased_variance": ("            var /= E;\n", "            var /= (E - 1);\n"),
    "merger_gelu_without_half": ("const double gl = 0.5 * y * (1.0 + erf(y / sqrt(2.0)));",
                                 "const double gl = y * (1.0 + erf(y / sqrt(2.0)));"),
    "merger_ln_drops_beta": ("* (double)gamma[e] + (double)beta[e];", "* (double)gamma[e];"),
    "patchify_drops_time_offset": ("const int64_t tau = g_t * tp + t;\n                        rows",
                                   "const int64_t tau = g_t * tp;\n                        rows"),
    "norm_uses_first_channel_constants": ("oracle_normalize_pixel(s[q], mean[c], std[c])",
                                          "oracle_normalize_pixel(s[q], mean[0], std[0])"),
    "frames_temporal_slices_reversed": ("const int64_t tau = g_t * tp + t;\n                            const int64_t y",
                                        "const int64_t tau = g_t * tp + (tp - 1 - t);\n"
                                        "                            const int64_t y"),
    "patches_weight_transposed": ("const double wv = (double)wb[(int64_t)e * K + k];",
                                  "const double wv = (double)wb[k * E + e];"),
    "accumulates_in_fp32": ("double acc = 0.0, mag = 0.0;", "float acc = 0.0f; double mag = 0.0;"),
    "raster_order_w_major": ("return (g_t * h + g_h) * w + g_w;", "return (g_t * w + g_w) * h + g_h;"),
    "merger_gelu_tanh_form": ("const double gl = 0.5 * y * (1.0 + erf(y / sqrt(2.0)));",
                              "const double gl = 0.5 * y * (1.0 + tanh(0.7978845608028654 * (y + 0.044715 * y * y * y)));"),
    "merger_eps_outside_sqrt": ("const double inv = 1.0 / sqrt(var + eps);",
                                "const double inv = 1.0 / (sqrt(var) + eps);"),
    "merger_second_moment_as_variance": ("var += ((double)row[e] - mean) * ((double)row[e] - mean);",
                                         "var += (double)row[e] * (double)row[e];"),
    "merger_fc2_takes_fc1_bias": ("out[v * H + h] = acc + (b2 ? (double)b2[h] : 0.0);",
                                  "out[v * H + h] = acc + (b2 ? (double)b1[h] : 0.0);"),
}


CONTROL = "unmodified"   # the real source through the same build and run: must pass


def _run_mutant(name, src, workdir):
    if name == CONTROL:
        text = src
    else:
        old, new = MUTANTS[name]
        if src.count(old) < 1:
            return None, f"pattern for {name} not found in the oracle source"
        text = src.replace(old, new)
    mut = os.path.join(workdir, f"{name}.c")
    with open(mut, "w") as f:
        f.write(text)
    lib = oracle.compile_source(mut, os.path.join(workdir, f"lib{name}.so"))
    env = dict(os.environ, PE_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    src = open(SRC).read()
    workdir = str(tmp_path_factory.mktemp("mutants"))
    names = [CONTROL] + sorted(MUTANTS)
    with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda n: _run_mutant(n, src, workdir), names))
    return dict(zip(names, results))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_results):
    rc, out = mutant_results[name]
    assert rc is not None, out
    assert rc != 0, f"mutant {name} survived the pins:\n{out}"


def test_unmodified_oracle_passes_the_same_run(mutant_results):
    """The control: a failure above means a pin failed, not the harness."""
    rc, out = mutant_results[CONTROL]
    assert rc == 0, out
