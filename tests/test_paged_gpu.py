"""GPU parity of the paged-K/V entry point (varlen_attn_fwd_v3) against the
fp64 oracle.

The cache layout is the PageAttention form of the Ascend sparse shared-KV
attention page ([num_pages, page_size, Hkv, D] blocks, a block table with one
row per sequence, key counts from seqused) and the argument is the page_table
of PyTorch pull request #176015's varlen forward schema.  The oracle reads the
packed K/V that each page cache is scattered from (workloads.to_paged), so a
wrong page, row or chunk shows up as a parity failure; rows of the cache that
hold no key carry a finite filler and table entries past a sequence's pages
are -1, which must never be read.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import check_close, full_check, require_gpu, run_gpu

pytestmark = pytest.mark.gpu

LENS = [300, 1, 129, 128, 77, 513]


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


@pytest.mark.parametrize("page_size", [16, 32, 48, 64, 80, 128, 256])
@pytest.mark.parametrize("causal", [True, False])
def test_paged_pair_kernel(page_size, causal):
    case = workloads.make_case(LENS, None, 4, 2, 128, "bf16", causal,
                               seed=400 + page_size + causal)
    full_check(case, paged=workloads.to_paged(case, page_size, seed=page_size))


@pytest.mark.parametrize("D,page_size", [(64, 16), (64, 144), (256, 16), (256, 48), (256, 128)])
def test_paged_other_head_dims(D, page_size):
    case = workloads.make_case(LENS, None, 4, 2, D, "fp16", True, seed=420 + D + page_size)
    full_check(case, paged=workloads.to_paged(case, page_size, seed=1))


def test_paged_odd_group_single_kernel():
    case = workloads.make_case(LENS, None, 3, 1, 128, "bf16", False, seed=430)
    full_check(case, paged=workloads.to_paged(case, 32, seed=2))


def test_paged_q_and_k_lengths_differ():
    case = workloads.make_case([70, 200, 5, 131], [250, 64, 1, 300], 6, 3, 128, "bf16", True,
                               seed=440)
    full_check(case, paged=workloads.to_paged(case, 16, seed=3))


def test_paged_with_window_and_fewer_used_keys():
    lq, lk = [400, 33, 260], [512, 300, 260]
    used = [450, 10, 200]
    case = workloads.make_case(lq, lk, 8, 2, 128, "bf16", True, seed=450)
    mask = dict(window_left=100, window_right=-1, seqused_k=used)
    full_check(case, mask=mask, paged=workloads.to_paged(case, 32, seed=4))


@pytest.mark.parametrize("G", [4, 8])
def test_paged_decode_style_packed_queries(G):
    gen = np.random.default_rng(460 + G)
    B = 40
    lq = gen.integers(1, 17, size=B).tolist()
    lk = (gen.integers(1, 3000, size=B) + np.array(lq)).tolist()
    case = workloads.make_case(lq, lk, 2 * G, 2, 128, "bf16", False, seed=461 + G)
    full_check(case, paged=workloads.to_paged(case, 16, seed=5))


def test_paged_equals_packed_bitwise():
    """The same keys through the page cache and packed: identical bytes."""
    case = workloads.make_case(LENS, None, 8, 2, 128, "bf16", True, seed=470)
    _, _, o1, l1 = run_gpu(case, mask=dict(seqused_k=case.lens_k))
    for ps in (16, 128):
        _, _, o2, l2 = run_gpu(case, paged=workloads.to_paged(case, ps, seed=ps))
        assert torch.equal(o1, o2) and torch.equal(l1, l2), "page size %d" % ps


def test_shared_prefix_pages():
    """Two sequences whose first pages are the same cache pages (a shared
    prompt prefix) and one that repeats a page."""
    ps = 16
    lq, lk = [20, 35, 9], [70, 50, 40]
    case = workloads.make_case(lq, lk, 4, 2, 64, "bf16", False, seed=480)
    cu = case.cu_k.tolist()
    k, v = case.k.clone(), case.v.clone()
    # sequence 1's first 32 keys = sequence 0's first 32 keys
    k[cu[1]:cu[1] + 32] = k[cu[0]:cu[0] + 32]
    v[cu[1]:cu[1] + 32] = v[cu[0]:cu[0] + 32]
    # sequence 2's keys 16..31 = its keys 0..15
    k[cu[2] + 16:cu[2] + 32] = k[cu[2]:cu[2] + 16]
    v[cu[2] + 16:cu[2] + 32] = v[cu[2]:cu[2] + 16]
    case.k, case.v = k, v
    pk = workloads.to_paged(case, ps, seed=6)
    pk.page_table[1, 0:2] = pk.page_table[0, 0:2]
    pk.page_table[2, 1] = pk.page_table[2, 0]
    full_check(case, paged=pk)


def test_out_of_range_page_entry_reads_zeros_and_sets_status():
    """A table entry outside [0, num_pages) is never dereferenced: its keys
    read as zeros (scores 0, values 0) and bit 2 of the status word is set."""
    import flash_attention_fwd_b200 as fa
    case = workloads.make_case([40], [64], 2, 2, 64, "bf16", False, seed=490)
    pk = workloads.to_paged(case, 16, seed=7)
    pk.page_table[0, 2] = 1 << 20                     # keys 32..47
    fa.device_status(clear=True)
    out, lse, _, _ = run_gpu(case, paged=pk)
    assert fa.device_status(clear=True) & 2
    k, v = case.k.clone(), case.v.clone()
    k[32:48] = 0
    v[32:48] = 0
    case.k, case.v = k, v
    ref_out, ref_lse = oracle.run_case(case)
    check_close(out, lse, ref_out, ref_lse, "zero page")
