"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the
pins of test_oracle_pins.py catch every one of them.

Each mutant is a one-line edit of oracle.c compiled into a temporary library; the
pin functions then run against it in a child process (a mutant that writes out of
bounds may crash, which also counts as caught).  A mutant that passes every pin
would show a hole in the pins.
"""
import os
import subprocess
import sys
import textwrap

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")
TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)

MUTANTS = {
    "gate_up_swapped": ("a[j] = silu(g[j]) * g[F + j];", "a[j] = silu(g[F + j]) * g[j];"),
    "silu_sign": ("v / (1.0 + exp(-v))", "v / (1.0 + exp(v))"),
    "weight_dropped_in_combine": ("o[c] += wk * y[c];\n        }\n    }\n}",
                                  "o[c] += y[c];\n        }\n    }\n}"),
    "unstable_scatter": ("for (int64_t i = 0; i < R; i++) {\n        int32_t s = cursor",
                         "for (int64_t i = R - 1; i >= 0; i--) {\n        int32_t s = cursor"),
    "offsets_off_by_one": ("offsets[e + 1] = offsets[e] + counts[e];",
                           "offsets[e + 1] = offsets[e] + counts[e] + (e == 0);"),
    "dispatch_wrong_token": ("int64_t t = perm[s] / topk;", "int64_t t = perm[s] % topk;"),
    "gemm_transposed_b": ("c[n] += a * bf16_widen(b[n]);",
                          "c[n] += a * bf16_widen(Be[(n % K) * N + (k % N)]);"),
    "w2_row_index": ("const uint16_t *wrow = W2e + j * H;",
                     "const uint16_t *wrow = W2e + (F - 1 - j) * H;"),
    "route_tie_to_higher_index": ("if (best < 0 || l[e] > l[best])", "if (best < 0 || l[e] >= l[best])"),
    "route_softmax_misses_shift": ("w[t * topk + k] = exp((double)l[out[k]] - mx) / sum;",
                                   "w[t * topk + k] = exp((double)l[out[k]]) / sum;"),
    "tile_short_edge": ("tile_row1[n] = (r + BM < offsets[e + 1]) ? r + BM : offsets[e + 1];",
                        "tile_row1[n] = r + BM;"),
    "e4m3_ties_round_up": ("if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))\n        n = fl + 1.0;\n    double r",
                           "if (rem >= 0.5)\n        n = fl + 1.0;\n    double r"),
    "fp8_row_scale_240": ("float sc = amax > 0.0f ? amax / 448.0f : 1.0f;\n        scale[r] = sc;",
                          "float sc = amax > 0.0f ? amax / 240.0f : 1.0f;\n        scale[r] = sc;"),
    "fp8_cols_not_transposed": ("qrow[k] = oracle_e4m3_encode((float)bf16_widen(Be[k * N + n]) / sc);",
                                "qrow[k] = oracle_e4m3_encode((float)bf16_widen(Be[n * K + k]) / sc);"),
    "gemm_add_alpha_beta_swapped": ("y[i] = alpha * acc[i] + beta * bf16_widen(add[i]);",
                                    "y[i] = beta * acc[i] + alpha * bf16_widen(add[i]);"),
    "gemm_add_drops_add": ("y[i] = alpha * acc[i] + beta * bf16_widen(add[i]);",
                           "y[i] = alpha * acc[i];"),
    "mx_exponent_never_rounds_up": ("    if (amax > ldexp(448.0, e))\n        e += 1;", "    if (amax > ldexp(448.0, e + 1))\n        e += 1;"),
    "mx_gemm_drops_b_scale": ("(int)b_sf[((int64_t)e * N + n) * nb + b] - 127);", "0);"),
    "mx_rows_scale_not_applied": ("q[r * K + b * 32 + k] = e4m3_encode_d(ldexp(v[k], -e));",
                                  "q[r * K + b * 32 + k] = e4m3_encode_d(v[k]);"),
    "fp8_gemm_drops_b_scale": ("C[s * N + n] = (double)a_scale[s] * (double)b_scale[(int64_t)e * N + n] * acc;",
                               "C[s * N + n] = (double)a_scale[s] * acc;"),
}

CHILD = textwrap.dedent("""
    import ctypes, sys
    sys.path[:0] = [{root!r}, {tests!r}]
    import oracle
    oracle._lib = oracle.configure(ctypes.CDLL({lib!r}))
    import test_oracle_pins as pins
    import test_oracle_fp8_pins as fp8
    import test_oracle_mx_pins as mx
    calls = [
        mx.test_exponent_is_the_smallest_that_fits,
        mx.test_row_quantiser_matches_torch_e4m3,
        mx.test_column_quantiser_matches_torch_and_round_trip,
        mx.test_mx_gemm_matches_numpy_block_sums,
        lambda: mx.test_mx_layer_within_e4m3_bound_of_the_exact_layer(40, 64, 96, 4, 2),
        mx.test_mx_layer_dense_special_case,
        fp8.test_decode_every_code_matches_torch,
        fp8.test_encode_matches_torch_and_brute_force,
        fp8.test_encode_saturates,
        fp8.test_quantize_rows_matches_torch_and_bounds,
        fp8.test_quantize_cols_matches_torch,
        fp8.test_grouped_gemm_e4m3_matches_numpy,
        fp8.test_fp8_layer_dense_special_case,
        lambda: fp8.test_fp8_layer_within_e4m3_bound_of_exact_layer(64, 4, 2),
        lambda: pins.test_plan_matches_stable_sort(33, 8, 2, True),
        lambda: pins.test_plan_matches_stable_sort(50, 5, 3, False),
        pins.test_tiling_worked_example,
        pins.test_tile_table_brute_force,
        pins.test_dispatch_and_unpermute_identity,
        pins.test_grouped_gemm_matches_numpy_matmul,
        pins.test_swiglu_closed_form,
        pins.test_dense_special_case_e1_topk1,
        pins.test_scalar_closed_form_h1_f1,
        pins.test_identical_experts_sum_of_weights,
        pins.test_layer_matches_torch_per_token_mixture,
        pins.test_route_matches_lexsort_and_softmax,
        pins.test_route_closed_form_and_permutation_equivariance,
        pins.test_gemm_add_special_cases,
        pins.test_gemm_add_linear_in_alpha_and_beta,
    ]
    caught = 0
    for c in calls:
        try:
            c()
        except Exception:
            caught += 1
    sys.exit(0 if caught == 0 else 3)
""")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site of {name} not unique"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                           "-std=c11", "-w", "-o", str(lib), str(mpath), "-lm"])
    child = CHILD.format(root=ROOT, tests=TESTS, lib=str(lib))
    r = subprocess.run([sys.executable, "-c", child], capture_output=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} passed every pin"
