"""The oracle pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (a wrong
scale, index, transpose, coefficient, association, mask or conv offset),
builds it in a temporary folder and runs the pin tests against it: every
planted mistake must make at least one pin fail. Runs on the CPU only.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "scale_full_sqrt_d": ("return 1.0 / sqrt(sqrt((double)d));", "return 1.0 / sqrt((double)d);"),
    "landmark_strided": ("x[(size_t)(j * L + t) * d + c]", "x[(size_t)(t * m + j) * d + c]"),
    "softmax_shifted_entry": ("row[c] = exp(row[c] - mx);", "row[c] = exp(row[c] - mx + 0.1*(c==0));"),
    "z0_not_transposed": ("Z[(size_t)r * m + k] = c * A[(size_t)k * m + r];",
                          "Z[(size_t)r * m + k] = c * A[(size_t)r * m + k];"),
    "coefficient_7": ("sub_from_scaled_identity(T, m, 7.0);", "sub_from_scaled_identity(T, m, 6.0);"),
    "quarter": ("Z[e] = 0.25 * U[e];", "Z[e] = 0.26 * U[e];"),
    "update_order_TZ": ("matmul(Z, T, m, m, m, U);", "matmul(T, Z, m, m, m, U);"),
    "kernel2_transposed": ("matmul_bt(ql, kl, m, d, m, k2);", "matmul_bt(kl, ql, m, d, m, k2);"),
    "kernel3_unscaled_k": ("scaled_copy(k, n, d, s, ks);", "scaled_copy(k, n, d, 1.0, ks);"),
    "kernel1_unscaled_q": ("qs[(size_t)r * d + c] = s * (double)q[(size_t)i * d + c];",
                           "qs[(size_t)r * d + c] = (double)q[(size_t)i * d + c];"),
    "conv_flipped": ("int src = i + t - half;", "int src = i - t + half;"),
    "conv_off_by_one": ("int src = i + t - half;", "int src = i + t - half - 1;"),
    "mask_finite": ("if (!keep[c]) row[c] = -INFINITY;", "if (!keep[c]) row[c] = -1.0;"),
    "init_row_sum_twice": ("return 1.0 / (max_col * max_row);", "return 1.0 / (max_row * max_row);"),
    "extra_iteration": ("for (int it = 0; it < n_iter; ++it) {", "for (int it = 0; it <= n_iter; ++it) {"),
    "z_transposed_in_product": ("matmul(k1, z, nr, m, m, probs);", "matmul_bt(k1, z, nr, m, m, probs);"),
    "init_exact_row_sums": ("        for (int r = 0; r < m; ++r) s += A[(size_t)r * m + c];\n        max_col = s > max_col ? s : max_col;\n    }\n    return 1.0 / max_col;",
                            "        for (int r = 0; r < m; ++r) s += A[(size_t)c * m + r];\n        max_col = s > max_col ? s : max_col;\n    }\n    return 1.0 / max_col;"),
    "init_option_ignored": ("const double c = init_option ? nys_oracle_init_coeff_exact(A, m) : nys_oracle_init_coeff(A, m);",
                            "const double c = nys_oracle_init_coeff(A, m);"),
    "exact_mask_ignored": ("nys_oracle_softmax_rows(p, nr, n, keep);", "nys_oracle_softmax_rows(p, nr, n, NULL);"),
    "exact_no_conv": ("    if (w) conv_rows_add(v, w, n, d, rows, nr, out);\n    if (probs_out) memcpy(probs_out, p,",
                      "    if (probs_out) memcpy(probs_out, p,"),
    "exact_unscaled_k": ("    scaled_copy(k, n, d, s, ks);\n    scaled_copy(v, n, d, 1.0, vd);\n    for (int r = 0; r < nr; ++r) {",
                         "    scaled_copy(k, n, d, 1.0, ks);\n    scaled_copy(v, n, d, 1.0, vd);\n    for (int r = 0; r < nr; ++r) {"),
    "probs_are_kernel1": ("if (probs_out) memcpy(probs_out, probs, ", "if (probs_out) memcpy(probs_out, k1, "),
}


def _run_mutant(name, tmp_root):
    a, b = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "nys_oracle.c")).read()
    assert a in src, f"mutation site for {name} is gone"
    d = os.path.join(tmp_root, name)
    ign = shutil.ignore_patterns("*.so", "__pycache__", "*.tmp*")
    for sub in ("oracle", "tests", "workloads"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub), ignore=ign)
    with open(os.path.join(d, "oracle", "nys_oracle.c"), "w") as f:
        f.write(src.replace(a, b))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), d)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=d, capture_output=True, text=True)
    return name, r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda n: _run_mutant(n, str(tmp_path)), MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mistakes not caught by any pin: {survivors}"
