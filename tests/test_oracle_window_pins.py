"""Pins of the oracle's sliding-window / used-key extension.

The extension reads the window_size_left / window_size_right / seqused_k
arguments of PyTorch pull request #176015's varlen forward schema with the
page's sequence-local indices (boostr 0.2.0,
src/ops/cpu/attention/varlen_attention.rs): key ki is visible to query qi
iff ki < min(seqused_k[b], Lk_b), qi - left <= ki (left >= 0),
ki <= qi + right (right >= 0), and not (causal and qi < ki).  Rows without
a visible key give O = 0, LSE = -inf.
"""
import math
import os
import shutil
import tempfile

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
import workloads


def f64(t):
    return t.to(torch.float64).numpy()


WINDOWS = [(3, -1), (-1, 2), (5, 0), (0, 4), (7, 7), (0, 0), (1, -1)]


@pytest.mark.parametrize("left,right", WINDOWS)
@pytest.mark.parametrize("causal", [False, True])
def test_window_matches_brute_force(left, right, causal):
    case = workloads.make_case([9, 1, 17, 6], [12, 3, 17, 2], 4, 2, 8, "bf16", causal,
                               seed=200 + left + 3 * right)
    out, lse = oracle.run_case(case, window_left=left, window_right=right)
    ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v), case.cu_q.numpy(),
                                 case.cu_k.numpy(), causal, case.scale, left, right)
    assert np.max(np.abs(out - ob)) <= 1e-12
    fin = np.isfinite(lb)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.max(np.abs(lse[fin] - lb[fin]), initial=0.0) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_seqused_matches_brute_force(causal):
    lq, lk = [7, 12, 5, 9], [10, 12, 4, 9]
    used = [3, 12, 0, 20]          # 20 > Lk: clipped to Lk
    case = workloads.make_case(lq, lk, 6, 3, 8, "fp16", causal, seed=210)
    out, lse = oracle.run_case(case, seqused_k=used)
    ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v), case.cu_q.numpy(),
                                 case.cu_k.numpy(), causal, case.scale, seqused_k=used)
    assert np.max(np.abs(out - ob)) <= 1e-12
    fin = np.isfinite(lb)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.max(np.abs(lse[fin] - lb[fin])) <= 1e-12
    cu = case.cu_q.tolist()
    # a sequence with no used key: O = 0, LSE = -inf
    assert np.all(out[cu[2]:cu[3]] == 0.0) and np.all(np.isneginf(lse[cu[2]:cu[3]]))


def test_self_window_gives_own_value():
    """left = 0 with the causal rule: each query sees only its own position."""
    case = workloads.make_case([11, 4], None, 2, 1, 16, "bf16", True, seed=211)
    out, lse = oracle.run_case(case, window_left=0)
    q, k, v = f64(case.q), f64(case.k), f64(case.v)
    for tok in range(case.Tq):
        for h in range(2):
            assert np.array_equal(out[tok, h], v[tok, 0])
            s = math.fsum(q[tok, h] * k[tok, 0]) * case.scale
            assert abs(lse[tok, h] - s) <= 1e-13


def test_one_hot_window_rule():
    """V = one-hot of the key index: O[qi, d] > 0 exactly on the window."""
    L, D, left, right = 14, 16, 3, 2
    case = workloads.make_case([L], None, 1, 1, D, "bf16", False, seed=212)
    v = torch.zeros_like(case.v)
    for ki in range(L):
        v[ki, 0, ki] = 1.0
    case.v = v
    out, _ = oracle.run_case(case, window_left=left, window_right=right)
    for qi in range(L):
        lo, hi = max(0, qi - left), min(L - 1, qi + right)
        row = out[qi, 0]
        assert np.all(row[lo:hi + 1] > 0)
        assert np.all(row[:lo] == 0) and np.all(row[hi + 1:] == 0)
        assert abs(row.sum() - 1.0) <= 1e-14


def test_wide_window_and_full_seqused_equal_plain():
    case = workloads.make_case([9, 20], [15, 20], 4, 4, 8, "bf16", True, seed=213)
    ref = oracle.run_case(case)
    for mask in (dict(window_left=100, window_right=100), dict(seqused_k=[15, 20]),
                 dict(window_left=19, window_right=-1, seqused_k=[99, 99])):
        got = oracle.run_case(case, **mask)
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_rows_without_visible_key():
    # left = 0, non-causal, Lk < Lq: queries qi >= Lk see no key (ki >= qi)
    case = workloads.make_case([8], [5], 2, 2, 8, "bf16", False, seed=214)
    out, lse = oracle.run_case(case, window_left=0)
    assert np.all(out[5:] == 0.0) and np.all(np.isneginf(lse[5:]))
    assert np.all(np.isfinite(lse[:5]))


def test_rows_mode_with_mask():
    case = workloads.make_case([30, 7], [25, 40], 4, 2, 16, "bf16", True, seed=215)
    mask = dict(window_left=6, window_right=3, seqused_k=[20, 33])
    out, lse = oracle.run_case(case, **mask)
    rows = workloads.sample_rows(case, 40)
    ro, rl = oracle.run_case_rows(case, rows, **mask)
    assert np.array_equal(ro, out[rows[:, 0], rows[:, 1]])
    assert np.array_equal(rl, lse[rows[:, 0], rows[:, 1]])


MUTANTS = {
    "left_window_off_by_one": ("ki < qi - c->win_left) return 1;",
                               "ki <= qi - c->win_left) return 1;"),
    "right_window_ignored": ("if (c->win_right >= 0 && ki > qi + c->win_right) return 1;",
                             "if (0) return 1;"),
    "seqused_ignored": ("if (u < Lk) Lk = u;", "(void)u;"),
}


def _window_pins_pass(lib) -> bool:
    try:
        for (left, right) in [(3, -1), (-1, 2), (0, 4)]:
            case = workloads.make_case([9, 17], [12, 17], 4, 2, 8, "bf16", False, seed=220)
            out, lse = oracle.run_case(case, lib=lib, window_left=left, window_right=right)
            ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v), case.cu_q.numpy(),
                                         case.cu_k.numpy(), False, case.scale, left, right)
            if np.max(np.abs(out - ob)) > 1e-12:
                return False
        case = workloads.make_case([7, 12], [10, 12], 6, 3, 8, "fp16", True, seed=221)
        out, lse = oracle.run_case(case, lib=lib, seqused_k=[3, 12])
        ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v), case.cu_q.numpy(),
                                     case.cu_k.numpy(), True, case.scale, seqused_k=[3, 12])
        return np.max(np.abs(out - ob)) <= 1e-12
    except Exception:
        return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_window_mistakes(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "varlen_attn_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor missing"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load_variant(path, os.path.join(tmp, "mutant.so"))
        assert not _window_pins_pass(lib), "planted mistake %s was not caught" % name
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
