"""Planted slips in copies of the oracle's C source must break at least one pin.

This checks the pins themselves: a dropped term, a wrong sign or index, or a
transposed operand anywhere in the oracle is caught.  Mutants are compiled
from the source text into a temporary directory; the oracle in the tree is
untouched.
"""
import os
import subprocess

import pytest

import oracle
from tests.pins import PINS

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "selinv_oracle.c")).read()

MUTANTS = {
    "schur_sign": ("for (size_t k = 0; k < bb; ++k) S[k] -= T2[k];",
                   "for (size_t k = 0; k < bb; ++k) S[k] += T2[k];"),
    "schur_transposed_B": ("matmul(b, T1, 0, Bi, 1, T2);", "matmul(b, T1, 0, Bi, 0, T2);"),
    "g_lower_sign": ("Gl[k] = -T2[k];", "Gl[k] = T2[k];"),
    "g_lower_transposed_B": ("matmul(b, Gn, 0, Bi, 0, T1);", "matmul(b, Gn, 0, Bi, 1, T1);"),
    "g_diag_transposed_B": ("matmul(b, Sinv + bb * i, 0, Bi, 1, T1);",
                            "matmul(b, Sinv + bb * i, 0, Bi, 0, T1);"),
    "g_diag_sign": ("Gii[k] = Sinv[bb * i + k] - T2[k];", "Gii[k] = Sinv[bb * i + k] + T2[k];"),
    "logdet_half": ("ld += 2.0 * log(R[k * b + k]);", "ld += log(R[k * b + k]);"),
    "cholesky_index": ("s -= R[i * b + k] * R[j * b + k];", "s -= R[i * b + k] * R[k * b + j];"),
    "tri_inverse_pivot": ("Rinv[i * b + j] = -s / R[i * b + i];", "Rinv[i * b + j] = -s / R[j * b + j];"),
    "sinv_order": ("matmul(b, Rinv, 1, Rinv, 0, Sinv);", "matmul(b, Rinv, 0, Rinv, 1, Sinv);"),
    "solve_forward_transposed": ("matvec(b, lower + bb * i, 0, v1, v2);",
                                 "matvec(b, lower + bb * i, 1, v1, v2);"),
    "solve_backward_transposed": ("matvec(b, lower + bb * i, 1, x + b * (i + 1), v1);",
                                  "matvec(b, lower + bb * i, 0, x + b * (i + 1), v1);"),
    "solve_rhs_index": ("y[b * (i + 1) + k] = rhs[b * (i + 1) + k] - v2[k];",
                        "y[b * (i + 1) + k] = rhs[b * i + k] - v2[k];"),
    "tree_child_transposed": ("matmul(b, T1, 0, edge + bb * c, 1, T2);",
                              "matmul(b, T1, 0, edge + bb * c, 0, T2);"),
    "tree_child_skipped": ("for (int64_t k = count[v]; k < count[v + 1]; ++k) {",
                           "for (int64_t k = count[v] + 1; k < count[v + 1]; ++k) {"),
    "tree_edge_transposed": ("matmul(b, G_diag + bb * p, 0, edge + bb * v, 0, T1);",
                             "matmul(b, G_diag + bb * p, 0, edge + bb * v, 1, T1);"),
    "sample_last_untransposed": ("matvec(b, Rinv + bb * (L - 1), 1, z + (size_t)b * (L - 1), eta + (size_t)b * (L - 1));",
                                 "matvec(b, Rinv + bb * (L - 1), 0, z + (size_t)b * (L - 1), eta + (size_t)b * (L - 1));"),
    "sample_coupling_transposed": ("matvec(b, lower + bb * i, 1, eta + (size_t)b * (i + 1), v1);",
                                   "matvec(b, lower + bb * i, 0, eta + (size_t)b * (i + 1), v1);"),
    "sample_sign": ("for (int k = 0; k < b; ++k) v1[k] = z[(size_t)b * i + k] - v2[k];",
                    "for (int k = 0; k < b; ++k) v1[k] = z[(size_t)b * i + k] + v2[k];"),
    "sample_schur_sign": ("for (size_t k = 0; k < bb; ++k) S[k] = S[k] - BSB[k];",
                          "for (size_t k = 0; k < bb; ++k) S[k] = S[k] + BSB[k];"),
    "tree_sample_root_untransposed": ("matvec(b, Rinv + bb * root, 1, z + (size_t)b * root, w + (size_t)b * root);",
                                      "matvec(b, Rinv + bb * root, 0, z + (size_t)b * root, w + (size_t)b * root);"),
    "tree_sample_edge_transposed": ("matvec(b, edge + bb * u, 1, w + (size_t)b * pu, t1);",
                                    "matvec(b, edge + bb * u, 0, w + (size_t)b * pu, t1);"),
    "tree_sample_sign": ("for (int k = 0; k < b; ++k) t1[k] = z[(size_t)b * u + k] - t2[k];",
                         "for (int k = 0; k < b; ++k) t1[k] = z[(size_t)b * u + k] + t2[k];"),
    "backward_sign": ("for (size_t k = 0; k < NN; ++k) Ab[k] = -Ab[k];",
                      "for (size_t k = 0; k < NN; ++k) Ab[k] = Ab[k];"),
    "backward_bbar_untransposed": ("Bb[bb * i + r * b + c] = Ab[lrow * N + col] + Ab[col * N + lrow];",
                                   "Bb[bb * i + r * b + c] = Ab[lrow * N + col] + Ab[lrow * N + col];"),
    "backward_dbar_mirror_dropped": ("if (c < r) v = Ab[row * N + col] + Ab[col * N + row];",
                                     "if (c < r) v = Ab[row * N + col];"),
    "backward_gbar_lower_above_untransposed": ("Gbar[lrow * N + col] = Gb_lower[bb * i + r * b + c];",
                                               "Gbar[row * N + col + b] = Gb_lower[bb * i + r * b + c];"),
    "backward_gbar_diag_dropped": ("Gbar[row * N + col] = Gb_diag[bb * i + r * b + c];",
                                   "Gbar[row * N + col] = 0.0 * Gb_diag[bb * i + r * b + c];"),
    "tree_backward_eb_untransposed": ("Eb[bb * v + r * b + c] = Ab[pr * N + vc] + Ab[vc * N + pr];",
                                      "Eb[bb * v + r * b + c] = Ab[pr * N + vc] + Ab[pr * N + vc];"),
    "tree_backward_gbar_edge_untransposed_above": ("Gbar[pr * N + vc] = Gb_edge[bb * v + r * b + c];",
                                                   "Gbar[vr * N + (size_t)(p * b + c)] = Gb_edge[bb * v + r * b + c];"),
    "tree_backward_db_mirror_dropped": ("Db[bb * v + r * b + c] = c < r ? lo + up : (c == r ? lo : 0.0);",
                                        "Db[bb * v + r * b + c] = c < r ? lo : (c == r ? lo : 0.0);"),
    "bidiag_pivot_smallest": ("if (fabs(aug[r * W + k]) > fabs(aug[piv * W + k])) piv = r;",
                              "if (fabs(aug[r * W + k]) < fabs(aug[piv * W + k])) piv = r;"),
    "bidiag_no_row_exchange": ("if (piv != k)\n", "if (piv != k && 0)\n"),
    "bidiag_lower_transposed": ("if (i + 1 < L) M[(row + b) * N + col] = lower[bb * i + r * b + c];",
                                "if (i + 1 < L) M[(row + b) * N + col] = lower[bb * i + c * b + r];"),
    "bidiag_lower_above": ("if (i + 1 < L) G_lower[bb * i + r * b + c] = Mi[(row + b) * N + col];",
                           "if (i + 1 < L) G_lower[bb * i + r * b + c] = Mi[row * N + col + b];"),
    "bidiag_backward_untransposed": ("matmul(N, Mi, 1, Gbar, 0, T);", "matmul(N, Mi, 0, Gbar, 0, T);"),
    "bidiag_backward_lower_above": ("if (i + 1 < L) Mb_lower[bb * i + r * b + c] = -Mb[(row + b) * N + col];",
                                    "if (i + 1 < L) Mb_lower[bb * i + r * b + c] = -Mb[row * N + col + b];"),
    "tree_g_diag_transposed": ("matmul(b, Sinv + bb * v, 0, edge + bb * v, 1, T1);",
                               "matmul(b, Sinv + bb * v, 0, edge + bb * v, 0, T1);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation site for {name} is not unique"
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(so), str(src), "-lm"])
    lib = oracle._bind(str(so))
    failed = []
    for pin, (fn, tol) in PINS.items():
        try:
            err = fn(lib=lib)
        except Exception:                      # a crash in the pin also counts as caught
            err = float("inf")
        if not err <= tol:
            failed.append(pin)
    assert failed, f"mutant {name} passed every pin"
