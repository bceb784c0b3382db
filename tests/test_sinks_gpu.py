"""GPU parity of attention sinks (varlen_attn_fwd_v3's ``sinks``) against the
fp64 oracle: sinks[h] is one extra logit, in score units, in the softmax of
every row of query head h, with no value row (the per-head FLOAT32 sinks
input of the Ascend sparse shared-KV attention page)."""
import math

import numpy as np
import pytest
import torch

import workloads
from parity_helpers import full_check, require_gpu, run_gpu

pytestmark = pytest.mark.gpu

LENS = [300, 1, 129, 128, 77, 513]


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


def sinks_for(H, seed, lo=-2.0, hi=4.0):
    # sinks of the size of typical row maxima (scores are ~N(0,1) here), so
    # that they change the result visibly
    return np.random.default_rng(seed).uniform(lo, hi, H).astype(np.float32).tolist()


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("causal", [True, False])
def test_sinks(D, causal):
    case = workloads.make_case(LENS, None, 4, 2, D, "bf16", causal, seed=600 + D + causal)
    full_check(case, mask=dict(sinks=sinks_for(4, D)))


def test_sinks_odd_group_single_kernel_fp16():
    case = workloads.make_case(LENS, None, 3, 1, 128, "fp16", True, seed=610)
    full_check(case, mask=dict(sinks=sinks_for(3, 611)))


@pytest.mark.parametrize("G", [4, 8])
def test_sinks_packed_short_queries(G):
    gen = np.random.default_rng(620 + G)
    lq = gen.integers(1, 17, size=30).tolist()
    lk = (gen.integers(1, 1500, size=30) + np.array(lq)).tolist()
    case = workloads.make_case(lq, lk, 2 * G, 2, 128, "bf16", False, seed=621 + G)
    full_check(case, mask=dict(sinks=sinks_for(2 * G, 622)))


def test_sinks_with_window_rows_without_keys():
    # left = 0, non-causal, Lk < Lq: rows qi >= Lk see no key and get LSE = sink
    case = workloads.make_case([300, 50], [130, 50], 4, 2, 128, "bf16", False, seed=630)
    sinks = sinks_for(4, 631)
    out, lse = full_check(case, mask=dict(window_left=0, sinks=sinks))
    assert np.all(out[130:300] == 0.0)
    assert np.allclose(lse[130:300], np.array(sinks)[None, :], atol=1e-6)


def test_large_and_very_negative_sinks():
    case = workloads.make_case(LENS, None, 4, 2, 128, "bf16", True, seed=640)
    full_check(case, mask=dict(sinks=[40.0, -60.0, 9.0, -1e30]))


def test_sinks_with_paged_kv():
    case = workloads.make_case(LENS, None, 8, 2, 128, "bf16", True, seed=650)
    full_check(case, mask=dict(sinks=sinks_for(8, 651)),
               paged=workloads.to_paged(case, 16, seed=652))


def test_minus_infinity_sinks_equal_plain_bitwise():
    case = workloads.make_case(LENS, None, 4, 2, 128, "bf16", True, seed=660)
    _, _, o1, l1 = run_gpu(case)
    _, _, o2, l2 = run_gpu(case, mask=dict(sinks=[-math.inf] * 4))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_gqa_prefill_with_sinks_full():
    case = workloads.make_workload("gqa")
    full_check(case, mask=dict(sinks=sinks_for(case.H, 670)))
