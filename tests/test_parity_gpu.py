"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Tolerances (bf16/fp16 output against fp64): O max abs err <= 1.5e-2, O mean
abs err <= 2e-3, LSE max abs err <= 5e-3.  Indexing is checked exactly: the
output buffers carry guard rows before and after the packed extents, filled
with a canary, and must come back with every packed row written (no NaN
pre-fill left) and every guard row untouched.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import (O_MAX, O_MEAN, LSE_MAX, GUARD, check_close, full_check,  # noqa: F401
                            require_gpu, run_gpu, sampled_check, stratified_check)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


# --- the benchmark configurations ----------------------------------------------------

def test_tiny_full():
    full_check(workloads.make_workload("tiny"))


def test_gqa_prefill_full():
    full_check(workloads.make_workload("gqa"))


def test_long_ragged_stratified():
    # one oracle row of every (sequence, 128-query tile, head): ~33,900 rows
    n = stratified_check(workloads.make_workload("long"))
    assert n >= 33216


def test_short_query_long_kv_full():
    # every row (1,267 tokens x 32 heads) against the oracle
    full_check(workloads.make_workload("shortq"))


def test_wide_head_fp16_stratified():
    # four oracle rows of every (sequence, 128-query tile, head)
    n = stratified_check(workloads.make_workload("wide"), per_tile=4)
    assert n >= 2048 * 3


# --- several tiles plus ragged tails, every head dim and dtype ------------------------

@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("causal", [True, False])
def test_ragged_tiles(D, dtype, causal):
    lens = [300, 1, 129, 128, 77, 513]
    case = workloads.make_case(lens, None, 4, 2, D, dtype, causal, seed=D + len(dtype) + causal)
    full_check(case)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_q_and_k_lengths_differ(D):
    # causal with Lq != Lk uses the top-left (sequence-local) rule
    case = workloads.make_case([70, 200, 5, 131], [250, 64, 1, 300], 6, 3, D, "bf16", True,
                               seed=40 + D)
    full_check(case)
    case2 = workloads.make_case([70, 200, 5, 131], [250, 64, 1, 300], 6, 3, D, "bf16", False,
                                seed=41 + D)
    full_check(case2)


def test_empty_sequences_and_empty_keys():
    # Lq=0 sequences write nothing; Lk=0 sequences give O = 0, LSE = -inf
    case = workloads.make_case([0, 50, 3, 0, 140], [10, 0, 7, 0, 140], 4, 4, 128, "bf16", False,
                               seed=50)
    out, lse = full_check(case)
    cu = case.cu_q.tolist()
    assert np.all(out[cu[1]:cu[2]] == 0.0) and np.all(np.isneginf(lse[cu[1]:cu[2]]))


def test_single_kv_head_and_many_sequences():
    rng = np.random.default_rng(60)
    lens = [int(x) for x in rng.integers(1, 300, 97)]
    case = workloads.make_case(lens, None, 16, 1, 128, "bf16", True, seed=60)
    full_check(case)


def test_explicit_scale_and_default_scale():
    case = workloads.make_case([200, 31], None, 4, 4, 64, "bf16", True, seed=61, scale=0.05)
    full_check(case)
    case.scale = 1.0 / math.sqrt(64)
    out_a, lse_a, _, _ = run_gpu(case, scale=0.0)
    out_b, lse_b, _, _ = run_gpu(case, scale=1.0 / math.sqrt(64))
    assert np.array_equal(out_a, out_b) and np.array_equal(lse_a, lse_b)


def test_understated_max_seqlen_still_covers_all_rows():
    case = workloads.make_case([700, 20], None, 2, 2, 128, "bf16", True, seed=62)
    out, lse, _, _ = run_gpu(case, max_q=1, max_k=1)
    ref_out, ref_lse = oracle.run_case(case)
    check_close(out, lse, ref_out, ref_lse, "understated max_seqlen")


def test_deterministic():
    case = workloads.make_workload("gqa")
    _, _, o1, l1 = run_gpu(case)
    _, _, o2, l2 = run_gpu(case)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_large_logit_stability_fp16():
    case = workloads.make_case([1024, 333], None, 4, 4, 256, "fp16", True, seed=63,
                               sigma_q=3.0, sigma_k=3.0)
    out, lse = full_check(case)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def _ramped(case, slope):
    """Scales key row i by (1 + i/slope): scores grow along the key axis, so
    the running max keeps rising by more than 2^8 and O is rescaled often."""
    Tk = case.k.shape[0]
    ramp = (1.0 + torch.arange(Tk, dtype=torch.float32) / slope).view(Tk, 1, 1)
    case.k = (case.k.float() * ramp).to(case.k.dtype)
    return case


@pytest.mark.parametrize("D", [64, 128, 256])
def test_running_max_growth_rescales_fp16(D):
    # Extreme logits (up to ~9x growth): fp16 keeps P's rounding (2^-11)
    # inside the tolerance even for a softmax dominated by a few keys.
    case = workloads.make_case([900, 300], None, 4, 2, D, "fp16", True, seed=70 + D,
                               sigma_q=2.0, sigma_k=2.0)
    full_check(_ramped(case, 150.0))


@pytest.mark.parametrize("D", [64, 128, 256])
def test_running_max_growth_rescales_bf16(D):
    # Milder growth that still forces rescales, in bf16, with V ~ N(0, 1).  A
    # peaked softmax makes O close to a single V row; a bf16 value with
    # |O| >= 4 has an ulp of 2^-5, so rounding the exact result alone can miss
    # by 2^-6 > 1.5e-2: the check allows that rounding on top of the tolerance.
    case = workloads.make_case([900, 300], None, 4, 2, D, "bf16", True, seed=90 + D)
    full_check(_ramped(case, 300.0), round_to="bf16")


@pytest.mark.parametrize("D", [64, 128])
def test_large_logits_fp16(D):
    # The wide-head configuration's logit scale (std(s) = 9) on the D = 64/128
    # kernels, GQA pairs included.
    case = workloads.make_case([700, 129, 64], None, 8, 2, D, "fp16", True, seed=80 + D,
                               sigma_q=3.0, sigma_k=3.0)
    full_check(case)


# --- short queries: GQA-packed tiles (query heads of one key/value head share a tile) ----

@pytest.mark.parametrize("G", [2, 4, 8, 16])
@pytest.mark.parametrize("causal", [False, True])
def test_short_queries_gqa_packed(G, causal):
    rng = np.random.default_rng(100 + G + 10 * causal)
    lq = [int(x) for x in rng.integers(1, 65, 9)]
    lk = [int(x) for x in rng.integers(1, 700, 9)]
    Hkv = 2
    case = workloads.make_case(lq, lk, Hkv * G, Hkv, 128, "bf16", causal, seed=110 + G)
    full_check(case)


@pytest.mark.parametrize("D", [64, 128])
def test_short_queries_gqa_packed_fp16(D):
    lq = [64, 1, 33, 17, 2]
    lk = [900, 129, 64, 1, 300]
    case = workloads.make_case(lq, lk, 16, 2, D, "fp16", True, seed=120 + D)
    full_check(case)


@pytest.mark.parametrize("splits", [1, 3, None])
def test_sequence_table_past_the_buffers_is_clamped(splits):
    # the last sequence claims 500 more queries and 1000 more keys than the
    # buffers hold; the kernels clamp every extent to the buffers (total_q,
    # total_k), so the result is that of the table cut at the buffer ends, and
    # nothing outside them is read or written (guard rows intact)
    import dataclasses
    # (query lengths, max_seqlen_q passed): per-head pairs, GQA-packed, and
    # decode-like rows (replicated rows with a workspace)
    for lq, max_q, H, Hkv in (([40, 1, 200], 700, 8, 2), ([40, 1, 200], 700, 32, 8),
                              ([4, 1, 8], 8, 32, 8)):
        lk = [300, 5, 1700]
        case = workloads.make_case(lq, lk, H, Hkv, 128, "bf16", False, seed=1500 + H + max_q)
        ref_out, ref_lse = oracle.run_case(case)
        cq = case.cu_q.clone()
        ck = case.cu_k.clone()
        cq[-1] += 500
        ck[-1] += 1000
        bad = dataclasses.replace(case, cu_q=cq, cu_k=ck)
        out, lse, _, _ = run_gpu(bad, max_q=max_q, max_k=2700, num_splits=splits)
        check_close(out, lse, ref_out, ref_lse, "table past the buffers")


def _off16(shape, dtype, dev):
    """A contiguous tensor whose data starts 16 bytes past a 32-byte boundary
    (the entry points require 16-byte alignment only)."""
    n = 1
    for s in shape:
        n *= s
    e = torch.empty((), dtype=dtype).element_size()
    buf = torch.empty(n + 64 // e, dtype=dtype, device=dev)
    k = ((-buf.data_ptr()) % 32 + 16) % 32 // e
    t = buf[k:k + n].view(shape)
    assert t.data_ptr() % 32 == 16
    return t


@pytest.mark.parametrize("D", [64, 128, 256])
def test_rows_written_with_16_byte_alignment(D):
    # rows are stored 32 bytes at a time when the output starts on a 32-byte
    # boundary, 16 bytes at a time otherwise: both give the same bits
    import flash_attention_fwd_b200 as fa
    case = workloads.make_case([300, 77, 129], None, 4, 2, D, "bf16", True, seed=1700 + D)
    dev = torch.device("cuda", 0)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    cq, ck = case.cu_q.to(dev), case.cu_k.to(dev)
    o32, l32 = fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q, case.max_k, True)
    o16 = _off16(q.shape, q.dtype, dev)
    _, l16 = fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q, case.max_k, True, out=o16)
    torch.cuda.synchronize()
    assert o32.data_ptr() % 32 == 0
    assert torch.equal(o32.view(torch.int16), o16.view(torch.int16)) and torch.equal(l32, l16)
    # key-range pieces in a workspace that starts 16 bytes past a 32-byte boundary
    dec = workloads.make_case([1, 3, 2], [3000, 1700, 2500], 8, 2, D, "bf16", False, seed=1710)
    q, k, v = dec.q.to(dev), dec.k.to(dev), dec.v.to(dev)
    cq, ck = dec.cu_q.to(dev), dec.cu_k.to(dev)
    nbytes = fa.fwd_workspace_size(dec.Tq, dec.H, dec.Hkv, D, dec.max_q, dec.max_k, 4)
    ws = _off16((nbytes,), torch.uint8, dev)
    a, la = fa.varlen_attn_fwd(q, k, v, cq, ck, dec.max_q, dec.max_k, num_splits=4)
    b, lb = fa.varlen_attn_fwd(q, k, v, cq, ck, dec.max_q, dec.max_k, num_splits=4, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la, lb)
    # the backward's gradients
    g = torch.Generator("cpu").manual_seed(1720)
    dout = torch.randn(case.q.shape, generator=g).to(case.q.dtype).to(dev)
    args = [t.to(dev) for t in (case.q, case.k, case.v)]
    grads = fa.varlen_attn_bwd(dout, *args, o32, l32, case.cu_q.to(dev), case.cu_k.to(dev),
                               case.max_q, case.max_k, True)
    offs = [_off16(t.shape, t.dtype, dev) for t in grads]
    fa.varlen_attn_bwd(dout, *args, o32, l32, case.cu_q.to(dev), case.cu_k.to(dev),
                       case.max_q, case.max_k, True, dq=offs[0], dk=offs[1], dv=offs[2])
    torch.cuda.synchronize()
    for x, y in zip(grads, offs):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
