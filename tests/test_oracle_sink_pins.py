"""Pins of the oracle's attention-sink extension.

Reading (the Ascend sparse shared-KV attention page lists a FLOAT32 per-head
``sinks`` input without a formula): sinks[h] is one extra logit, in score
units, in the softmax of every row of query head h, with no value row.  So
O = sum_ki exp(s_ki - m) V_ki / (sum_ki exp(s_ki - m) + exp(sink - m)) and
LSE = ln(sum_ki exp(s_ki) + exp(sink)).
"""
import math
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
from oracle import brute
import workloads


def f64(t):
    import torch
    return t.to(torch.float64).numpy()


def sinks_for(H, seed, lo=-3.0, hi=3.0):
    return np.random.default_rng(seed).uniform(lo, hi, H).tolist()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mask", [{}, dict(window_left=3), dict(window_left=2, window_right=1),
                                  dict(seqused_k=[5, 1, 0, 9])])
def test_sinks_match_brute_force(causal, mask):
    case = workloads.make_case([9, 1, 17, 6], [12, 3, 17, 9], 4, 2, 8, "bf16", causal,
                               seed=500 + causal + 3 * len(mask))
    sinks = sinks_for(4, 501)
    out, lse = oracle.run_case(case, sinks=sinks, **mask)
    ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v), case.cu_q.numpy(),
                                 case.cu_k.numpy(), causal, case.scale, sinks=sinks, **mask)
    assert np.max(np.abs(out - ob)) <= 1e-12
    assert np.max(np.abs(lse - lb)) <= 1e-12


def test_minus_infinity_sinks_equal_no_sinks():
    case = workloads.make_case([9, 20], [15, 20], 4, 4, 8, "fp16", True, seed=510)
    ref = oracle.run_case(case)
    got = oracle.run_case(case, sinks=[-math.inf] * 4)
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_single_key_closed_form():
    """One key: O = v0 / (1 + exp(sink - s00)), LSE = logaddexp(s00, sink)."""
    case = workloads.make_case([1, 1], [1, 1], 2, 2, 16, "bf16", False, seed=511)
    sinks = [0.7, -1.9]
    out, lse = oracle.run_case(case, sinks=sinks)
    q, k, v = f64(case.q), f64(case.k), f64(case.v)
    for tok in range(2):
        for h in range(2):
            s = math.fsum(q[tok, h] * k[tok, h]) * case.scale
            w = 1.0 / (1.0 + math.exp(sinks[h] - s))
            assert np.max(np.abs(out[tok, h] - w * v[tok, h])) <= 1e-14
            assert abs(lse[tok, h] - np.logaddexp(s, sinks[h])) <= 1e-13


def test_equal_scores_closed_form():
    """Q = 0: every visible score is 0, so O = n / (n + e^sink) * mean(V) and
    LSE = ln(n + e^sink)."""
    import torch
    L, sink = 11, 1.3
    case = workloads.make_case([L], None, 1, 1, 8, "bf16", False, seed=512)
    case.q = torch.zeros_like(case.q)
    out, lse = oracle.run_case(case, sinks=[sink])
    v = f64(case.v)[:, 0]
    want = v.mean(axis=0) * (L / (L + math.exp(sink)))
    for tok in range(L):
        assert np.max(np.abs(out[tok, 0] - want)) <= 1e-14
        assert abs(lse[tok, 0] - math.log(L + math.exp(sink))) <= 1e-14


def test_rows_without_keys_get_the_sink_as_lse():
    case = workloads.make_case([4, 3], [0, 5], 2, 1, 8, "bf16", False, seed=513)
    out, lse = oracle.run_case(case, sinks=[0.25, -4.0], window_left=0)
    # sequence 0 has no key; in sequence 1 (left = 0, non-causal) every query sees keys >= qi
    assert np.all(out[:4] == 0.0)
    assert np.array_equal(lse[:4], np.array([[0.25, -4.0]] * 4))
    assert np.all(np.isfinite(lse[4:]))


def test_sink_only_rescales_the_plain_result():
    """O_sink = O_plain * exp(LSE_plain - LSE_sink), LSE_sink =
    logaddexp(LSE_plain, sink): the sink changes the normalisation only."""
    case = workloads.make_case([30, 7], [25, 40], 4, 2, 16, "bf16", True, seed=514)
    sinks = sinks_for(4, 515, -1.0, 4.0)
    op, lp = oracle.run_case(case)
    os_, ls = oracle.run_case(case, sinks=sinks)
    for h in range(4):
        assert np.max(np.abs(ls[:, h] - np.logaddexp(lp[:, h], sinks[h]))) <= 1e-12
        ratio = np.exp(lp[:, h] - ls[:, h])[:, None]
        assert np.max(np.abs(os_[:, h] - op[:, h] * ratio)) <= 1e-12


def test_rows_mode_with_sinks():
    case = workloads.make_case([30, 7], [25, 40], 4, 2, 16, "bf16", True, seed=516)
    sinks = sinks_for(4, 517)
    out, lse = oracle.run_case(case, sinks=sinks, window_left=5)
    rows = workloads.sample_rows(case, 40)
    ro, rl = oracle.run_case_rows(case, rows, sinks=sinks, window_left=5)
    assert np.array_equal(ro, out[rows[:, 0], rows[:, 1]])
    assert np.array_equal(rl, lse[rows[:, 0], rows[:, 1]])


MUTANTS = {
    "sink_left_out_of_sum": ("    double acc = exp(extra - m);", "    double acc = 0.0;"),
    "sink_left_out_of_max": ("    double m = extra;", "    double m = -INFINITY;"),
    "sink_scaled": ("    return c->sinks ? c->sinks[h] : -INFINITY;",
                    "    return c->sinks ? c->sinks[h] * c->scale : -INFINITY;"),
    "sink_of_wrong_head": ("    return c->sinks ? c->sinks[h] : -INFINITY;",
                           "    return c->sinks ? c->sinks[h / (c->H / c->Hkv)] : -INFINITY;"),
}


def _sink_pins_pass(lib) -> bool:
    try:
        for causal in (False, True):
            case = workloads.make_case([9, 1, 17, 6], [12, 3, 17, 0], 4, 2, 8, "bf16", causal,
                                       seed=520)
            sinks = [0.5, -2.0, 80.0, 1.5]  # one large sink: exercises the max
            out, lse = oracle.run_case(case, lib=lib, sinks=sinks)
            ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v),
                                         case.cu_q.numpy(), case.cu_k.numpy(), causal,
                                         case.scale, sinks=sinks)
            if not (np.max(np.abs(out - ob)) <= 1e-12 and np.max(np.abs(lse - lb)) <= 1e-12):
                return False
        return True
    except Exception:
        return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_sink_mistakes(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "varlen_attn_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor missing"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load_variant(path, os.path.join(tmp, "mutant.so"))
        assert not _sink_pins_pass(lib), "planted mistake %s was not caught" % name
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
