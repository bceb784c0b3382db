"""Pins of the oracle's backward (the gradient that the boostr 0.2.0 source
page src/ops/cpu/attention/varlen_attention.rs defines in varlen_attention_bwd,
in fp64).

The references here do not share its arithmetic: PyTorch autograd through an
independent dense fp64 forward (block-diagonal + causal mask), central finite
differences of the NumPy brute-force forward, and closed forms.
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
    return t.to(torch.float64)


def dense_autograd(case, dout):
    """dQ, dK, dV of L = sum(O * dO) by autograd through a dense fp64
    forward; also returns the exact O and LSE."""
    q = f64(case.q).clone().requires_grad_(True)
    k = f64(case.k).clone().requires_grad_(True)
    v = f64(case.v).clone().requires_grad_(True)
    G = case.H // case.Hkv
    cq, ck = case.cu_q.tolist(), case.cu_k.tolist()
    Tq, Tk = case.Tq, case.Tk
    seg_q = torch.empty(Tq, dtype=torch.long)
    pos_q = torch.empty(Tq, dtype=torch.long)
    seg_k = torch.empty(Tk, dtype=torch.long)
    pos_k = torch.empty(Tk, dtype=torch.long)
    for b in range(case.B):
        seg_q[cq[b]:cq[b + 1]] = b
        pos_q[cq[b]:cq[b + 1]] = torch.arange(cq[b + 1] - cq[b])
        seg_k[ck[b]:ck[b + 1]] = b
        pos_k[ck[b]:ck[b + 1]] = torch.arange(ck[b + 1] - ck[b])
    vis = seg_q[:, None] == seg_k[None, :]
    if case.causal:
        vis &= ~(pos_q[:, None] < pos_k[None, :])
    kk = k.repeat_interleave(G, dim=1)
    vv = v.repeat_interleave(G, dim=1)
    s = torch.einsum("qhd,khd->hqk", q, kk) * case.scale
    s = s.masked_fill(~vis[None], float("-inf"))
    lse = torch.logsumexp(s, dim=-1)                       # [H, Tq]
    p = torch.exp(s - lse[..., None])
    o = torch.einsum("hqk,khd->qhd", p, vv)
    loss = (o * f64(dout)).sum()
    dq, dk, dv = torch.autograd.grad(loss, (q, k, v))
    return dq.numpy(), dk.numpy(), dv.numpy(), o.detach(), lse.detach().T.contiguous()


def rand_dout(case, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(case.q.shape, generator=g).to(case.q.dtype)


CASES = [
    ([9, 1, 17, 6], None, 4, 2, 8, "bf16", True),
    ([9, 1, 17, 6], [12, 3, 17, 2], 4, 2, 8, "fp16", False),
    ([20, 5], [7, 30], 6, 3, 16, "bf16", True),     # causal with Lq != Lk (top-left)
    ([13], None, 2, 2, 32, "bf16", False),
]


@pytest.mark.parametrize("i", range(len(CASES)))
def test_backward_matches_autograd(i):
    lq, lk, H, Hkv, D, dt, causal = CASES[i]
    case = workloads.make_case(lq, lk, H, Hkv, D, dt, causal, seed=700 + i)
    dout = rand_dout(case, 710 + i)
    dq_r, dk_r, dv_r, o, lse = dense_autograd(case, dout)
    dq, dk, dv = oracle.run_case_bwd(case, dout, o, lse)
    for got, ref in ((dq, dq_r), (dk, dk_r), (dv, dv_r)):
        assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_backward_matches_finite_differences_of_brute_force():
    """Central differences of L = sum(O * dO), O from the NumPy brute force."""
    case = workloads.make_case([5, 3], [4, 6], 2, 1, 4, "bf16", True, seed=720)
    dout = rand_dout(case, 721)
    q, k, v = (f64(t).numpy() for t in (case.q, case.k, case.v))
    cq, ck = case.cu_q.numpy(), case.cu_k.numpy()
    o, lse = brute.dense_forward(q, k, v, cq, ck, True, case.scale)
    dq, dk, dv = oracle.run_case_bwd(case, dout, o, lse)
    do = f64(dout).numpy()

    def loss(q_, k_, v_):
        return float((brute.dense_forward(q_, k_, v_, cq, ck, True, case.scale)[0] * do).sum())

    eps = 1e-6
    rng = np.random.default_rng(722)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = {"q": (plus, k, v), "k": (q, plus, v), "v": (q, k, plus)}[name]
            args_m = {"q": (minus, k, v), "k": (q, minus, v), "v": (q, k, minus)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7, (name, idx, fd, grad[idx])


def test_single_key_closed_form():
    """Lk = 1: p = 1 and dp = delta, so dQ = dK = 0 and dV = sum of dO over
    the queries (and query heads) of the key's sequence."""
    case = workloads.make_case([4, 2], [1, 1], 4, 2, 8, "bf16", False, seed=730)
    dout = rand_dout(case, 731)
    o, lse = brute.dense_forward(*(f64(t).numpy() for t in (case.q, case.k, case.v)),
                                 case.cu_q.numpy(), case.cu_k.numpy(), False, case.scale)
    dq, dk, dv = oracle.run_case_bwd(case, dout, o, lse)
    assert np.max(np.abs(dq)) <= 1e-14 and np.max(np.abs(dk)) <= 1e-14
    do = f64(dout).numpy()
    for b, (q0, q1) in enumerate([(0, 4), (4, 6)]):
        for kvh in range(2):
            want = do[q0:q1, 2 * kvh:2 * kvh + 2].sum(axis=(0, 1))
            assert np.max(np.abs(dv[b, kvh] - want)) <= 1e-13


def test_gqa_equals_summed_mha():
    """dK/dV of a GQA key head = the sum of the dK/dV of its replicas when
    K/V are replicated to every query head (MHA)."""
    case = workloads.make_case([9, 14], None, 4, 2, 8, "bf16", True, seed=740)
    dout = rand_dout(case, 741)
    _, _, _, o, lse = dense_autograd(case, dout)
    dq, dk, dv = oracle.run_case_bwd(case, dout, o, lse)
    mha = workloads.make_case([9, 14], None, 4, 4, 8, "bf16", True, seed=740)
    mha.q = case.q
    mha.k = case.k.repeat_interleave(2, dim=1)
    mha.v = case.v.repeat_interleave(2, dim=1)
    dq2, dk2, dv2 = oracle.run_case_bwd(mha, dout, o, lse)
    assert np.max(np.abs(dq - dq2)) <= 1e-13
    assert np.max(np.abs(dk - (dk2[:, 0::2] + dk2[:, 1::2]))) <= 1e-13
    assert np.max(np.abs(dv - (dv2[:, 0::2] + dv2[:, 1::2]))) <= 1e-13


def test_dv_rows_sum_to_dout_sums():
    """sum over keys of dV = sum over queries of dO (each query's weights sum
    to 1), per sequence and key/value head group."""
    case = workloads.make_case([30, 7], [25, 40], 2, 1, 16, "fp16", True, seed=750)
    dout = rand_dout(case, 751)
    _, _, _, o, lse = dense_autograd(case, dout)
    dq, dk, dv = oracle.run_case_bwd(case, dout, o, lse)
    do = f64(dout).numpy()
    assert np.max(np.abs(dv[:25].sum(axis=(0, 1)) - do[:30].sum(axis=(0, 1)))) <= 1e-12
    # and sum over keys of dK = 0 per query head set: sum_k ds = 0 for every query
    assert np.max(np.abs(dk[:25].sum(axis=0))) <= 1e-11


MUTANTS = {
    "delta_dropped": ("ds[i] = p[i] * (dp[i] - delta);", "ds[i] = p[i] * dp[i];"),
    "dq_without_scale": ("c->dq[qoff + d] = c->scale * acc;", "c->dq[qoff + d] = acc;"),
    "dk_uses_k": ("dk_row[d] += c->scale * ds[i] * qd[d];",
                  "dk_row[d] += c->scale * ds[i] * kd[(size_t)idx[i] * D + d];"),
    "dv_uses_ds": ("dv_row[d] += p[i] * dod[d];", "dv_row[d] += ds[i] * dod[d];"),
    "causal_ignored": ("if (c->causal && qi < ki) continue;", "if (0) continue;"),
    "lse_not_subtracted": ("p[i] = exp(c->scale * dot_d(qd, krow, D) - lse);",
                           "p[i] = exp(c->scale * dot_d(qd, krow, D));"),
}


def _bwd_pins_pass(lib) -> bool:
    try:
        for i in (0, 2):
            lq, lk, H, Hkv, D, dt, causal = CASES[i]
            case = workloads.make_case(lq, lk, H, Hkv, D, dt, causal, seed=700 + i)
            dout = rand_dout(case, 710 + i)
            dq_r, dk_r, dv_r, o, lse = dense_autograd(case, dout)
            dq, dk, dv = oracle.run_case_bwd(case, dout, o, lse, lib=lib)
            for got, ref in ((dq, dq_r), (dk, dk_r), (dv, dv_r)):
                if not np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref))):
                    return False
        return True
    except Exception:
        return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_backward_mistakes(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "varlen_attn_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor missing"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load_variant(path, os.path.join(tmp, "mutant.so"))
        assert not _bwd_pins_pass(lib), "planted mistake %s was not caught" % name
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
