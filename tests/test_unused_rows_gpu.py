"""GPU parity with non-finite values in key/value rows that no query may see.

The last key tile a work item visits can run past its sequence's used keys:
into the next sequence's rows of the packed buffers, into the slots
[seqused_k[b], Lk) of a KV cache, or into the rest of a sequence's last page.
Those keys get a softmax weight of exactly 0, and the oracle never reads
them; but a product 0 * NaN or 0 * Inf is NaN, so the kernels must not feed
such rows to the PV product.  Here they hold NaN, +Inf and -Inf (uninitialised
cache memory can hold anything), and every output row must still match the
oracle (the varlen forward schema of PyTorch pull request #176015 for
seqused_k and page_table; the PageAttention cache layout of the Ascend sparse
shared-KV attention page).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import check_close, full_check, require_gpu, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


def _poison(t):
    """NaN, +Inf and -Inf in turn over the elements of t (in place)."""
    flat = t.view(-1)
    pattern = torch.tensor([float("nan"), float("inf"), float("-inf")], dtype=t.dtype)
    flat.copy_(pattern.repeat(flat.numel() // 3 + 1)[:flat.numel()])


def _with_poisoned_neighbours(lens, H, Hkv, D, dtype, causal, seed, dummy=77):
    """Real sequences `lens` separated by key-only sequences (no queries) of
    `dummy` keys whose K and V rows are non-finite; returns the case."""
    lq, lk = [], []
    for L in lens:
        lq += [L, 0]
        lk += [L, dummy]
    case = workloads.make_case(lq, lk, H, Hkv, D, dtype, causal, seed=seed)
    cu = case.cu_k.tolist()
    for b in range(1, len(lq), 2):
        _poison(case.k[cu[b]:cu[b + 1]])
        _poison(case.v[cu[b]:cu[b + 1]])
    return case


# (H, Hkv): pair kernel (even group), single kernel (odd group / MHA)
HEADS = [(8, 2), (6, 6)]


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("heads", HEADS)
@pytest.mark.parametrize("causal", [True, False])
def test_next_sequence_rows_non_finite(D, heads, causal):
    H, Hkv = heads
    case = _with_poisoned_neighbours([200, 129, 1, 300], H, Hkv, D, "bf16", causal,
                                     seed=2000 + D + H + causal)
    full_check(case)


@pytest.mark.parametrize("D", [64, 128])
def test_next_sequence_rows_non_finite_gqa_packed(D):
    # short queries: GQA-packed tiles (4 query heads of a KV head per tile)
    lq, lk = [], []
    for L, K in ((12, 300), (5, 129), (40, 77)):
        lq += [L, 0]
        lk += [K, 50]
    case = workloads.make_case(lq, lk, 8, 2, D, "fp16", False, seed=2100 + D)
    cu = case.cu_k.tolist()
    for b in range(1, len(lq), 2):
        _poison(case.v[cu[b]:cu[b + 1]])
        _poison(case.k[cu[b]:cu[b + 1]])
    full_check(case)


@pytest.mark.parametrize("splits", [None, 1, 3])
def test_next_sequence_rows_non_finite_decode(splits):
    # decode-like calls: replicated rows and key-range pieces (library's
    # choice), plain (1), three pieces
    lq, lk = [], []
    for K in (3000, 1500, 2201):
        lq += [1, 0]
        lk += [K, 90]
    case = workloads.make_case(lq, lk, 32, 8, 128, "bf16", False, seed=2200)
    cu = case.cu_k.tolist()
    for b in range(1, len(lq), 2):
        _poison(case.v[cu[b]:cu[b + 1]])
    full_check(case, num_splits=splits)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("heads", HEADS)
def test_unused_cache_slots_non_finite(D, heads):
    # keys [seqused_k[b], Lk) of each sequence are unused cache slots
    H, Hkv = heads
    lens = [300, 200, 513, 64, 130]
    case = workloads.make_case(lens, None, H, Hkv, D, "bf16", False, seed=2300 + D + H)
    used = [250, 129, 1, 64, 0]
    cu = case.cu_k.tolist()
    for b, u in enumerate(used):
        _poison(case.v[cu[b] + u:cu[b + 1]])
        _poison(case.k[cu[b] + u:cu[b + 1]])
    full_check(case, mask={"seqused_k": used})
    # causal, and a sliding window, over the same cache
    case.causal = True
    full_check(case, mask={"seqused_k": used})
    full_check(case, mask={"seqused_k": used, "window_left": 100})


@pytest.mark.parametrize("page_size", [16, 64, 256])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_paged_last_page_non_finite(page_size, D):
    # the rest of each sequence's last page and the spare pages are non-finite
    lens_q = [3, 17, 1, 40]
    lens_k = [700, 129, 1, 1000]
    H, Hkv = (8, 2) if D != 256 else (4, 4)
    case = workloads.make_case(lens_q, lens_k, H, Hkv, D, "bf16", False,
                               seed=2400 + page_size + D)
    paged = workloads.to_paged(case, page_size, seed=page_size, fill=float("nan"))
    out, lse, _, _ = run_gpu(case, paged=paged)
    ref_out, ref_lse = oracle.run_case(case)
    check_close(out, lse, ref_out, ref_lse, "paged, NaN past the used keys")
    assert np.isfinite(out).all()
    # the same cache with -Inf / +Inf in the unused rows
    for fill in (float("inf"), float("-inf")):
        paged = workloads.to_paged(case, page_size, seed=page_size, fill=fill)
        out, lse, _, _ = run_gpu(case, paged=paged)
        check_close(out, lse, ref_out, ref_lse, "paged, %r past the used keys" % fill)
