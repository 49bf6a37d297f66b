"""The element-wise training-step check (tests/parity.py: check_train with train_bounds) rejects
localised mistakes that a comparison of whole gradients by their relative L2 error lets through.

Mistakes are planted in copies of the oracle's C source (a wrong index in one outer product, one
row of one sequence dropped, the last entry of the last sequence dropped from the gradients,
one sequence missing from one weight gradient); each broken copy stands in for a GPU result and must
fail the check against the intact oracle.  CPU only.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from parity import check_train, exact_train_case, train_bounds

MISTAKES = {
    # outer product g_Wiuq = sum_b dq_b c_b^T read with the column index shifted by one
    "g_Wiuq_column_shifted": ("g_Wiuq[((size_t)l * nq + o) * r + j] += dq[lb * nq + o] * c[j];",
                              "g_Wiuq[((size_t)l * nq + o) * r + j] += dq[lb * nq + o] * c[(j + 1) % r];"),
    # one row of W^IUQ's gradient (256 of its 2 M elements) misses one sequence's contribution
    "g_Wiuq_one_row_one_sequence": ("g_Wiuq[((size_t)l * nq + o) * r + j] += dq[lb * nq + o] * c[j];",
                                    "g_Wiuq[((size_t)l * nq + o) * r + j] += (o == 100 && b == 2 ? 0.0 : dq[lb * nq + o]) * c[j];"),
    # one row of W^DQ's gradient misses one sequence's contribution
    "g_Wdq_one_row_one_sequence": ("g_Wdq[((size_t)l * r + j) * d + i] += dc[j] * elem(h, dt, hb + i);",
                                   "g_Wdq[((size_t)l * r + j) * d + i] += (j == 7 && b == 2 ? 0.0 : dc[j]) * elem(h, dt, hb + i);"),
    # the gradients skip the last entry of the last sequence (a lost partial sum at a sequence end)
    "last_entry_dropped": ("                    if (a[hh] > 0.0) {\n                        dw[",
                           "                    if (a[hh] > 0.0 && !(b == B - 1 && s + 1 == S)) {\n                        dw["),
    # W^w's gradient misses the first sequence of layer 1
    "g_Ww_sequence_missing": ("g_Ww[((size_t)l * n_h + hh) * d + i] += dw[lb * n_h + hh] * elem(h, dt, hb + i);",
                              "g_Ww[((size_t)l * n_h + hh) * d + i] += (l == 1 && b == 0 ? 0.0 : dw[lb * n_h + hh]) * elem(h, dt, hb + i);"),
}


def rel_l2(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _grads(ref):
    return [ref["g_Wdq"], ref["g_Wiuq"], ref["g_Ww"]]


@pytest.mark.slow
def test_elementwise_check_rejects_planted_mistakes(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    case = exact_train_case(torch.bfloat16, torch.bfloat16)
    h, W, K, ks, labels, offs, n_h, d_I = case
    args = (h, *W, K, ks, labels.numpy(), offs.numpy(), n_h, d_I)
    ref = oracle.train_step(*args)
    bounds = train_bounds(case)
    check_train(ref["loss"], _grads(ref), ref, bounds, what="oracle against itself")
    with open(os.path.join(os.path.dirname(oracle.__file__), "lsa_oracle.c")) as f:
        src0 = f.read()
    passes_norm = []
    for name, (old, new) in MISTAKES.items():
        assert old in src0, f"{name}: pattern not found in the oracle source"
        c = tmp_path / f"{name}.c"
        so = tmp_path / f"{name}.so"
        c.write_text(src0.replace(old, new, 1))
        subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                        str(c), "-o", str(so), "-lm"], check=True)
        with oracle.using(str(so)):
            bad = oracle.train_step(*args)
        with pytest.raises(AssertionError):
            check_train(bad["loss"], _grads(bad), ref, bounds, what=name)
        if all(rel_l2(bad[k], ref[k]) < 2e-2 for k in ("g_Wdq", "g_Wiuq", "g_Ww")):
            passes_norm.append(name)
    # a mistake in a few hundred elements is invisible to a whole-gradient norm at a 2e-2 tolerance
    assert "g_Wiuq_one_row_one_sequence" in passes_norm, passes_norm
