"""GPU parity of the sliding-window / used-key entry point (varlen_attn_fwd_v2)
against the fp64 oracle's extension of the same rule: key ki is visible to
query qi iff ki < min(Lk, seqused_k[b]), qi - left <= ki (left >= 0),
ki <= qi + right (right >= 0) and not (causal and qi < ki); rows without a
visible key give O = 0 and LSE = -inf (the window_size_left/right and
seqused_k arguments of PyTorch pull request #176015's varlen forward, read
with boostr's sequence-local indices).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import check_close, full_check, require_gpu, run_gpu, stratified_check

pytestmark = pytest.mark.gpu

LENS = [300, 1, 129, 128, 77, 513]


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


def poison_unused_keys(case, used, value):
    """Writes a large finite value into the key/value rows past seqused_k, so
    that any weight they received would show."""
    cu = case.cu_k.tolist()
    k, v = case.k.clone(), case.v.clone()
    for b, u in enumerate(used):
        lo = cu[b] + max(0, min(u, cu[b + 1] - cu[b]))
        k[lo:cu[b + 1]] = value
        v[lo:cu[b + 1]] = value
    case.k, case.v = k, v
    return case


# --- windows on several tiles and ragged tails --------------------------------------

WINDOWS = [(3, -1), (200, -1), (-1, 100), (64, 64), (0, 0), (127, 0), (128, 5), (1000, 1000)]


@pytest.mark.parametrize("left,right", WINDOWS)
@pytest.mark.parametrize("causal", [True, False])
def test_window_pair_kernel(left, right, causal):
    # H / Hkv = 2: two query heads share K/V tiles (D = 128)
    case = workloads.make_case(LENS, None, 4, 2, 128, "bf16", causal,
                               seed=300 + 7 * left + right + causal)
    full_check(case, mask=dict(window_left=left, window_right=right))


@pytest.mark.parametrize("D", [64, 256])
@pytest.mark.parametrize("causal", [True, False])
def test_window_other_head_dims(D, causal):
    case = workloads.make_case(LENS, None, 4, 2, D, "fp16", causal, seed=320 + D + causal)
    full_check(case, mask=dict(window_left=150, window_right=40))


@pytest.mark.parametrize("causal", [True, False])
def test_window_odd_group_single_kernel(causal):
    # H / Hkv = 3 is odd: one query tile per item
    case = workloads.make_case(LENS, None, 3, 1, 128, "bf16", causal, seed=330 + causal)
    full_check(case, mask=dict(window_left=90, window_right=17))


def test_window_q_and_k_lengths_differ():
    case = workloads.make_case([70, 200, 5, 131], [250, 64, 1, 300], 6, 3, 128, "bf16", True,
                               seed=340)
    full_check(case, mask=dict(window_left=33, window_right=-1))
    case2 = workloads.make_case([70, 200, 5, 131], [250, 64, 1, 300], 6, 3, 128, "bf16", False,
                                seed=341)
    full_check(case2, mask=dict(window_left=10, window_right=45))


# --- used-key counts ---------------------------------------------------------------

@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("causal", [True, False])
def test_seqused_k(D, causal):
    lq = [300, 1, 129, 128, 77, 513]
    lk = [300, 40, 200, 128, 77, 600]
    used = [250, 0, 129, 128, 1, 999]      # 0: no key; 999 > Lk: clipped to Lk
    case = workloads.make_case(lq, lk, 4, 2, D, "bf16", causal, seed=350 + D + causal)
    poison_unused_keys(case, used, 3.0e3)
    full_check(case, mask=dict(seqused_k=used))


def test_seqused_k_and_window_together():
    lq, lk = [400, 33, 260], [512, 300, 260]
    used = [450, 10, 200]
    case = workloads.make_case(lq, lk, 8, 2, 128, "fp16", True, seed=360)
    poison_unused_keys(case, used, 2.0e4)
    full_check(case, mask=dict(window_left=100, window_right=-1, seqused_k=used))


# --- rows without a visible key ------------------------------------------------------

def test_rows_without_visible_key():
    # left = 0, non-causal, Lk < Lq: queries qi >= Lk see no key
    case = workloads.make_case([300, 50], [130, 50], 4, 2, 128, "bf16", False, seed=370)
    out, lse = full_check(case, mask=dict(window_left=0, window_right=-1))
    assert np.all(np.isneginf(lse[130:300])) and np.all(out[130:300] == 0.0)


def test_first_visited_tile_masked_for_late_rows():
    # left = 3: in the item of queries 128..255 the first visited key tile
    # (keys 0..127) holds no visible key for queries >= 131
    case = workloads.make_case([1000], None, 2, 2, 64, "bf16", True, seed=371)
    full_check(case, mask=dict(window_left=3))


# --- GQA-packed short queries (decode-style) -----------------------------------------

@pytest.mark.parametrize("G", [4, 8])
def test_packed_short_queries_with_window_and_seqused(G):
    gen = np.random.default_rng(380 + G)
    B = 40
    lq = gen.integers(1, 17, size=B).tolist()
    lk = (gen.integers(1, 2000, size=B) + np.array(lq)).tolist()
    used = [int(max(x, 1) - gen.integers(0, 30)) for x in lk]
    case = workloads.make_case(lq, lk, 2 * G, 2, 128, "bf16", True, seed=381 + G)
    poison_unused_keys(case, used, 1.0e3)
    full_check(case, mask=dict(window_left=256, seqused_k=used))


# --- identities through the v2 entry point -------------------------------------------

def test_unreachable_window_equals_v1_bitwise():
    """Window bounds no query can reach go through varlen_attn_fwd_v2 and must
    give exactly the bytes of varlen_attn_fwd_v1."""
    case = workloads.make_case(LENS, None, 4, 2, 128, "bf16", True, seed=390)
    _, _, o1, l1 = run_gpu(case)
    _, _, o2, l2 = run_gpu(case, mask=dict(window_left=case.Tq + 5, window_right=case.Tk + 5))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_full_seqused_equals_v1_bitwise():
    case = workloads.make_case(LENS, [310, 5, 129, 128, 80, 513], 4, 2, 64, "fp16", False,
                               seed=391)
    _, _, o1, l1 = run_gpu(case)
    _, _, o2, l2 = run_gpu(case, mask=dict(seqused_k=[310, 5, 129, 128, 80, 513]))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# --- a large case, one oracle row per work item ---------------------------------------

def test_long_prefill_sliding_window_stratified():
    """The long ragged prefill workload with a 4096-key causal sliding window
    (the bench's long_swa workload): one oracle row of every (sequence,
    128-query tile, head)."""
    case = workloads.make_workload("long_swa")
    n = stratified_check(case, mask=case.mask)
    assert n >= 33216
