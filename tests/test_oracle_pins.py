"""Pins of the fp64 oracle against facts that do not come from the oracle.

The oracle computes the packed attention forward defined by the boostr 0.2.0
source page src/ops/cpu/attention/varlen_attention.rs
(``varlen_attention_fwd``).  These tests tie it to: exact format decoding, the dense brute-force definition, a
library softmax, closed forms (single key, equal scores, two keys), the
causal rule (one-hot values), packing/permutation/GQA invariances, convexity,
the log-sum-exp definition and the empty cases.  ``test_planted_mistakes``
plants plausible mistakes in a copy of the oracle source and checks that the
pins catch every one.
"""
import math
import os
import shutil
import tempfile

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import brute
import workloads


def f64(t):
    return t.to(torch.float64).numpy()


def small_cases():
    yield workloads.make_case([5, 9, 1, 12], None, 4, 2, 16, "bf16", True, seed=11)
    yield workloads.make_case([7, 3], [11, 4], 6, 3, 8, "fp16", False, seed=12)
    yield workloads.make_case([20, 1, 13], None, 8, 1, 64, "bf16", True, seed=13)
    yield workloads.make_case([4, 17], [9, 2], 4, 4, 4, "bf16", True, seed=14)   # Lq != Lk causal
    yield workloads.make_case([6], [6], 2, 2, 8, "fp16", True, seed=15, sigma_q=3, sigma_k=3)


# --- exact widening of the 16-bit formats -------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_decode_all_bit_patterns(dtype):
    lib = oracle._load()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(workloads.DTYPES[dtype]).to(torch.float64).numpy()
    got = np.array([lib.oracle_decode16(int(b), oracle.DTYPE_CODE[dtype]) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(got[~nan]))


# --- against the dense brute force ------------------------------------------------

@pytest.mark.parametrize("idx", range(5))
def test_matches_brute_force(idx):
    case = list(small_cases())[idx]
    out, lse = oracle.run_case(case)
    ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v), case.cu_q.numpy(),
                                 case.cu_k.numpy(), case.causal, case.scale)
    assert np.max(np.abs(out - ob)) <= 1e-12
    assert np.max(np.abs(lse - lb)) <= 1e-12


def test_rows_mode_equals_full_mode():
    case = workloads.make_case([40, 3, 129], None, 4, 2, 32, "bf16", True, seed=21)
    out, lse = oracle.run_case(case)
    rows = workloads.sample_rows(case, 50)
    ro, rl = oracle.run_case_rows(case, rows)
    assert np.array_equal(ro, out[rows[:, 0], rows[:, 1]])
    assert np.array_equal(rl, lse[rows[:, 0], rows[:, 1]])


def test_textbook_softmax_single_sequence():
    """B=1, non-causal: O = softmax(Q K^T * scale) V with scipy's softmax."""
    case = workloads.make_case([23], [31], 3, 3, 16, "bf16", False, seed=22)
    out, lse = oracle.run_case(case)
    q, k, v = f64(case.q), f64(case.k), f64(case.v)
    for h in range(3):
        s = q[:, h, :] @ k[:, h, :].T * case.scale
        ref = scipy.special.softmax(s, axis=1) @ v[:, h, :]
        assert np.max(np.abs(out[:, h, :] - ref)) <= 1e-12
        assert np.max(np.abs(lse[:, h] - scipy.special.logsumexp(s, axis=1))) <= 1e-12


# --- closed forms --------------------------------------------------------------------

def test_single_key_gives_v0_and_score():
    case = workloads.make_case([1, 1, 1], [1, 1, 1], 4, 2, 32, "bf16", False, seed=23)
    out, lse = oracle.run_case(case)
    q, k, v = f64(case.q), f64(case.k), f64(case.v)
    for t in range(3):
        for h in range(4):
            assert np.array_equal(out[t, h], v[t, h // 2])
            s = math.fsum(q[t, h] * k[t, h // 2]) * case.scale
            assert abs(lse[t, h] - s) <= 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_equal_scores_give_mean_of_visible_values(causal):
    case = workloads.make_case([9, 14], None, 2, 1, 8, "bf16", causal, seed=24)
    case.q.zero_()                       # every score is exactly 0
    out, lse = oracle.run_case(case)
    v = f64(case.v)
    cu = case.cu_q.tolist()
    for b in range(2):
        L = cu[b + 1] - cu[b]
        for qi in range(L):
            n = qi + 1 if causal else L
            keys = v[cu[b]:cu[b] + n, 0, :]
            for h in range(2):
                ref = np.array([math.fsum(keys[:, d]) / n for d in range(8)])
                assert np.max(np.abs(out[cu[b] + qi, h] - ref)) <= 1e-14
                assert abs(lse[cu[b] + qi, h] - math.log(n)) <= 1e-14


def test_two_keys_closed_form():
    # q = e0 * a, keys e0 and 2*e0 -> scores a*scale*(1, 2)
    D = 4
    q = torch.zeros((1, 1, D), dtype=torch.bfloat16)
    k = torch.zeros((2, 1, D), dtype=torch.bfloat16)
    v = torch.zeros((2, 1, D), dtype=torch.bfloat16)
    q[0, 0, 0] = 3.0
    k[0, 0, 0] = 1.0
    k[1, 0, 0] = 2.0
    v[0, 0, :] = torch.tensor([1.0, 0.0, -2.0, 0.5])
    v[1, 0, :] = torch.tensor([0.0, 1.0, 4.0, -0.5])
    scale = 0.5
    out, lse = oracle.varlen_attn_fwd(q, k, v, [0, 1], [0, 2], 1, 1, D, False, scale, "bf16")
    s0, s1 = 1.5, 3.0
    w1 = 1.0 / (1.0 + math.exp(s0 - s1))
    w0 = 1.0 - w1
    ref = w0 * f64(v[0, 0]) + w1 * f64(v[1, 0])
    assert np.max(np.abs(out[0, 0] - ref)) <= 1e-15
    assert abs(lse[0, 0] - (s1 + math.log1p(math.exp(s0 - s1)))) <= 1e-15
    # causal: query 0 sees only key 0
    out_c, lse_c = oracle.varlen_attn_fwd(q, k, v, [0, 1], [0, 2], 1, 1, D, True, scale, "bf16")
    assert np.array_equal(out_c[0, 0], f64(v[0, 0]))
    assert lse_c[0, 0] == s0


# --- the causal rule ---------------------------------------------------------------

def test_causal_rows_see_exactly_their_prefix():
    """V = one-hot of the key index: O[qi, d] > 0 exactly for d <= qi."""
    L, D = 12, 16
    case = workloads.make_case([L, 5], None, 2, 2, D, "bf16", True, seed=25)
    v = torch.zeros_like(case.v)
    cu = case.cu_k.tolist()
    for b in range(2):
        for ki in range(cu[b + 1] - cu[b]):
            v[cu[b] + ki, :, ki] = 1.0
    case.v = v
    out, _ = oracle.run_case(case)
    for b in range(2):
        Lb = cu[b + 1] - cu[b]
        for qi in range(Lb):
            row = out[cu[b] + qi]
            assert np.all(row[:, :qi + 1] > 0)
            assert np.all(row[:, qi + 1:] == 0)
            assert np.allclose(row.sum(axis=1), 1.0, atol=1e-14, rtol=0)


def test_causal_first_row_is_v0():
    case = workloads.make_case([8, 3, 30], None, 4, 2, 32, "bf16", True, seed=26)
    out, _ = oracle.run_case(case)
    v = f64(case.v)
    cu = case.cu_q.tolist()
    for b in range(3):
        for h in range(4):
            assert np.array_equal(out[cu[b], h], v[cu[b], h // 2])


# --- invariances ---------------------------------------------------------------------

def test_packed_equals_separate_runs_and_permutation():
    lens = [13, 1, 27, 6]
    case = workloads.make_case(lens, None, 4, 2, 16, "bf16", True, seed=27)
    out, lse = oracle.run_case(case)
    cu = case.cu_q.tolist()
    for b, L in enumerate(lens):
        sl = slice(cu[b], cu[b + 1])
        o1, l1 = oracle.varlen_attn_fwd(case.q[sl], case.k[sl], case.v[sl], [0, L], [0, L],
                                        4, 2, 16, True, case.scale, "bf16")
        assert np.array_equal(o1, out[sl])
        assert np.array_equal(l1, lse[sl])
    perm = [2, 0, 3, 1]
    qs = torch.cat([case.q[cu[b]:cu[b + 1]] for b in perm])
    ks = torch.cat([case.k[cu[b]:cu[b + 1]] for b in perm])
    vs = torch.cat([case.v[cu[b]:cu[b + 1]] for b in perm])
    cp = workloads.cu_seqlens([lens[b] for b in perm]).tolist()
    op, lp = oracle.varlen_attn_fwd(qs, ks, vs, cp, cp, 4, 2, 16, True, case.scale, "bf16")
    for i, b in enumerate(perm):
        assert np.array_equal(op[cp[i]:cp[i + 1]], out[cu[b]:cu[b + 1]])
        assert np.array_equal(lp[cp[i]:cp[i + 1]], lse[cu[b]:cu[b + 1]])


def test_gqa_equals_mha_with_replicated_kv():
    case = workloads.make_case([10, 21], [15, 21], 8, 2, 16, "bf16", False, seed=28)
    out, lse = oracle.run_case(case)
    k_rep = case.k.repeat_interleave(4, dim=1)
    v_rep = case.v.repeat_interleave(4, dim=1)
    om, lm = oracle.varlen_attn_fwd(case.q, k_rep, v_rep, case.cu_q.numpy(), case.cu_k.numpy(),
                                    8, 8, 16, False, case.scale, "bf16")
    assert np.array_equal(om, out)
    assert np.array_equal(lm, lse)


def test_convexity_and_lse_bounds():
    case = workloads.make_case([19, 33], [40, 33], 4, 4, 8, "fp16", True, seed=29,
                               sigma_q=3.0, sigma_k=3.0)
    out, lse = oracle.run_case(case)
    q, k, v = f64(case.q), f64(case.k), f64(case.v)
    cq, ck = case.cu_q.tolist(), case.cu_k.tolist()
    for b in range(2):
        for qi in range(cq[b + 1] - cq[b]):
            n = min(qi + 1, ck[b + 1] - ck[b])
            vis = slice(ck[b], ck[b] + n)
            for h in range(4):
                row = out[cq[b] + qi, h]
                assert np.all(row >= v[vis, h].min(axis=0) - 1e-12)
                assert np.all(row <= v[vis, h].max(axis=0) + 1e-12)
                s = np.array([math.fsum(q[cq[b] + qi, h] * k[ck[b] + j, h]) * case.scale
                              for j in range(n)])
                m = s.max()
                ref = m + math.log(math.fsum(np.exp(s - m)))
                assert abs(lse[cq[b] + qi, h] - ref) <= 1e-12
                assert m - 1e-12 <= lse[cq[b] + qi, h] <= m + math.log(n) + 1e-12


def test_default_scale():
    case = workloads.make_case([7, 5], None, 2, 1, 16, "bf16", True, seed=30)
    ref = oracle.varlen_attn_fwd(case.q, case.k, case.v, case.cu_q, case.cu_k, 2, 1, 16, True,
                                 1.0 / math.sqrt(16), "bf16")
    for s in (0.0, -1.0, float("nan")):
        got = oracle.varlen_attn_fwd(case.q, case.k, case.v, case.cu_q, case.cu_k, 2, 1, 16,
                                     True, s, "bf16")
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_large_logits_are_finite():
    case = workloads.make_case([64, 64], None, 2, 2, 256, "fp16", True, seed=31,
                               sigma_q=3.0, sigma_k=3.0)
    out, lse = oracle.run_case(case)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


# --- empty cases ------------------------------------------------------------------------

def test_empty_key_set_and_empty_query():
    # sequence 0: 3 queries, 0 keys; sequence 1: 0 queries, 4 keys; sequence 2: normal
    lens_q, lens_k = [3, 0, 2], [0, 4, 2]
    case = workloads.make_case(lens_q, lens_k, 2, 2, 8, "bf16", False, seed=32)
    out, lse = oracle.run_case(case)
    assert np.all(out[0:3] == 0.0)
    assert np.all(np.isneginf(lse[0:3]))
    ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v), case.cu_q.numpy(),
                                 case.cu_k.numpy(), False, case.scale)
    assert np.max(np.abs(out[3:] - ob[3:])) <= 1e-12
    assert np.max(np.abs(lse[3:] - lb[3:])) <= 1e-12


# --- the pins catch planted mistakes ------------------------------------------------------

MUTANTS = {
    "causal_off_by_one": ("if (c->causal && qi < ki) return 1;", "if (c->causal && qi <= ki) return 1;"),
    "gqa_map_modulo": ("int kv_h = h / G;\n        int q0", "int kv_h = h % G;\n        int q0"),
    "dropped_scale": ("s[i] = c->scale * dot_d(qrow,", "s[i] = dot_d(qrow,"),
    "lse_without_max": ("return m + log(acc);", "return log(acc);"),
    "unnormalised_weights": ("const double w = exp(s[i] - lse);", "const double w = exp(s[i]);"),
    "k_v_swapped": ("kd[(size_t)ki * D + d] = oracle_decode16(c->k[off + d], c->dtype);",
                    "kd[(size_t)ki * D + d] = oracle_decode16(c->v[off + d], c->dtype);"),
    "fp16_bias_wrong": ("expo - 25", "expo - 24"),
}


def _pins_pass(lib) -> bool:
    """A compact run of the pins above against a given oracle build."""
    try:
        for case in small_cases():
            out, lse = oracle.run_case(case, lib=lib)
            ob, lb = brute.dense_forward(f64(case.q), f64(case.k), f64(case.v),
                                         case.cu_q.numpy(), case.cu_k.numpy(), case.causal,
                                         case.scale)
            if not (np.max(np.abs(out - ob)) <= 1e-12 and np.max(np.abs(lse - lb)) <= 1e-12):
                return False
        case = workloads.make_case([9, 14], None, 2, 1, 8, "bf16", False, seed=24)
        case.q.zero_()
        out, lse = oracle.run_case(case, lib=lib)
        v = f64(case.v)
        if abs(out[0, 0, 0] - v[0:9, 0, 0].mean()) > 1e-14:
            return False
        return True
    except Exception:
        return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "varlen_attn_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, "mutation anchor missing"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load_variant(path, os.path.join(tmp, "mutant.so"))
        assert not _pins_pass(lib), "planted mistake %s was not caught" % name
        good = os.path.join(tmp, "good.c")
        with open(good, "w") as f:
            f.write(src)
        assert _pins_pass(oracle.load_variant(good, os.path.join(tmp, "good.so")))
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
