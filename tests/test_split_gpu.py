"""GPU parity of the key-range split (varlen_attn_fwd_v4's num_splits)
against the fp64 oracle.

Without a causal rule or a window, the key range of a long sequence is cut
into pieces, each computed as its own work item (partial O / l and LSE in a
float32 workspace), and a second kernel merges the pieces by their LSE.  The
result is the same softmax regrouped, so the oracle and the tolerances are
those of the unsplit forward.  The cases cover every kernel layout
(GQA-packed pair, per-head pair, single), both dtypes and head dims, uneven
pieces (key counts not divisible by the piece size), sequences without keys
or queries, sinks (which enter only in the merge), used-key counts, paged
K/V, and an understated max_seqlen_k (more key tiles than the piece plan
assumed: the device clamps the piece count, pieces grow).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import check_close, full_check, require_gpu, run_gpu

pytestmark = pytest.mark.gpu

# short queries, long ragged keys; one sequence without keys, one without queries
LQ = [1, 40, 64, 0, 17, 3, 64, 33]
LK = [3000, 700, 129, 500, 0, 1, 5000, 2048]


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


@pytest.mark.parametrize("splits", [2, 3, 7, 32])
@pytest.mark.parametrize("D", [64, 128])
def test_split_gqa_packed(D, splits):
    case = workloads.make_case(LQ, LK, 16, 2, D, "bf16", False, seed=1000 + D + splits)
    full_check(case, num_splits=splits)


@pytest.mark.parametrize("D", [64, 128])
def test_split_gqa_packed_fp16(D):
    case = workloads.make_case(LQ, LK, 8, 2, D, "fp16", False, seed=1010 + D)
    full_check(case, num_splits=5)


def test_split_per_head_pairs_long_queries():
    # max_seqlen_q > 64: no GQA packing, two heads of one KV head per item
    case = workloads.make_case([200, 1, 300, 129], [4000, 900, 2500, 130], 4, 2, 128, "bf16",
                               False, seed=1020)
    full_check(case, num_splits=3)


@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "fp16")])
def test_split_single_kernel_odd_group(D, dtype):
    case = workloads.make_case(LQ, LK, 3, 1, D, dtype, False, seed=1030 + D)
    full_check(case, num_splits=4)


def test_split_single_kernel_wide_head_large_logits():
    # D = 256 (the single-tile kernel: K/V tiles in two column slices, two
    # softmax halves per row), std of the scaled scores about 9
    case = workloads.make_case([5, 64, 30], [3000, 1500, 257], 2, 2, 256, "fp16", False,
                               seed=1040, sigma_q=3.0, sigma_k=3.0)
    full_check(case, num_splits=6)


def test_split_with_sinks():
    case = workloads.make_case(LQ, LK, 16, 2, 128, "bf16", False, seed=1050)
    sinks = np.random.default_rng(1051).uniform(-2.0, 4.0, 16).astype(np.float32).tolist()
    out, lse = full_check(case, mask=dict(sinks=sinks), num_splits=4)
    # the sequence without keys: O = 0 and LSE = the sink of each head
    cu = case.cu_q.tolist()
    rows = slice(cu[4], cu[5])
    assert np.all(out[rows] == 0.0)
    assert np.allclose(lse[rows], np.array(sinks)[None, :], atol=1e-6)


def test_split_with_seqused_k():
    case = workloads.make_case(LQ, LK, 16, 2, 128, "bf16", False, seed=1060)
    used = [2999, 0, 129, 7, 0, 1, 1025, 4000]
    full_check(case, mask=dict(seqused_k=used), num_splits=3)


@pytest.mark.parametrize("page_size", [16, 256])
def test_split_paged(page_size):
    case = workloads.make_case(LQ, LK, 16, 2, 128, "bf16", False, seed=1070 + page_size)
    paged = workloads.to_paged(case, page_size, seed=1071)
    full_check(case, paged=paged, num_splits=4)


def test_split_understated_max_seqlen_k():
    # the plan assumes 2 key tiles at most; sequences of up to 40 tiles clamp
    # the piece count to the plan's maximum and every row is still written
    case = workloads.make_case(LQ, LK, 16, 2, 128, "bf16", False, seed=1080)
    full_check(case, max_k=256, num_splits=2)
    full_check(case, max_k=1000, num_splits=4)


def test_split_equals_unsplit_up_to_rounding():
    case = workloads.make_case(LQ, LK, 16, 2, 128, "fp16", False, seed=1090)
    o1, l1, _, _ = run_gpu(case, num_splits=1)
    o4, l4, _, _ = run_gpu(case, num_splits=4)
    fin = np.isfinite(l1)
    assert np.array_equal(fin, np.isfinite(l4))
    assert np.abs(o1 - o4).max() <= 4e-3
    assert np.abs(l1[fin] - l4[fin]).max() <= 1e-4


def test_split_deterministic():
    case = workloads.make_case(LQ, LK, 16, 2, 128, "bf16", False, seed=1100)
    _, _, a_o, a_l = run_gpu(case, num_splits=7)
    _, _, b_o, b_l = run_gpu(case, num_splits=7)
    assert torch.equal(a_o, b_o) and torch.equal(a_l, b_l)


def raw_forward(case, num_splits, window_left=-1):
    """The C entry point v4 without a workspace; returns (status, out, lse)."""
    import flash_attention_fwd_b200 as fa
    dev = torch.device("cuda", 0)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    cq, ck = case.cu_q.to(dev), case.cu_k.to(dev)
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device=dev)
    Tq, H, D = q.shape
    rc = fa.varlen_attn_fwd_raw(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), cq.data_ptr(), ck.data_ptr(),
        len(case.lens_q), Tq, k.shape[0], case.max_q, case.max_k, H, k.shape[1], D, case.causal,
        0.0, fa.DTYPE_CODES[q.dtype], out.data_ptr(), lse.data_ptr(),
        torch.cuda.current_stream().cuda_stream, window_left=window_left, num_splits=num_splits)
    torch.cuda.synchronize()
    return rc, out.cpu().to(torch.float64).numpy(), lse.cpu().to(torch.float64).numpy()


def test_split_ignored_with_causal_and_window():
    # the piece count is ignored (no split, so no workspace is needed) under
    # a causal rule or a window
    case = workloads.make_case([300, 40], [300, 3000], 8, 2, 128, "bf16", True, seed=1110)
    rc, out, lse = raw_forward(case, 8)
    assert rc == 0
    check_close(out, lse, *oracle.run_case(case), "causal, num_splits ignored")
    case = workloads.make_case([30, 40], [3000, 3000], 8, 2, 128, "bf16", False, seed=1111)
    # (a left bound below the query count: a bound no query can reach would
    # be dropped, and the call would be an unmasked one)
    rc, out, lse = raw_forward(case, 8, window_left=10)
    assert rc == 0
    check_close(out, lse, *oracle.run_case(case, window_left=10), "window, num_splits ignored")
    # without either, the same call needs the workspace
    rc, _, _ = raw_forward(case, 8)
    assert rc == -8


def test_split_auto_choice_decode_batch():
    # 8 sequences of 1-4 queries against up to 20k keys, 8 KV heads: 64 work
    # items for 148 SMs, so the library cuts the key ranges
    import flash_attention_fwd_b200 as fa
    lq = [1, 4, 2, 1, 3, 1, 4, 1]
    lk = [20000, 9000, 17000, 3000, 12000, 20000, 640, 15000]
    case = workloads.make_case(lq, lk, 32, 8, 128, "bf16", False, seed=1130)
    n = fa.fwd_num_splits(len(lq), sum(lq), sum(lk), case.max_q, case.max_k, 32, 8, 128)
    if torch.cuda.get_device_properties(0).multi_processor_count >= 100:
        assert n > 1
    full_check(case)


def test_split_workspace_errors():
    import flash_attention_fwd_b200 as fa
    case = workloads.make_case(LQ, LK, 16, 2, 128, "bf16", False, seed=1120)
    need = fa.fwd_workspace_size(case.q.shape[0], 16, 2, 128, case.max_q, case.max_k, 4)
    assert need > 0
    dev = torch.device("cuda", 0)
    args = (case.q.to(dev), case.k.to(dev), case.v.to(dev), case.cu_q.to(dev),
            case.cu_k.to(dev), case.max_q, case.max_k)
    small = torch.empty(need - 16, dtype=torch.uint8, device=dev)
    with pytest.raises(ValueError):
        fa.varlen_attn_fwd(*args, num_splits=4, workspace=small)
    out = torch.empty_like(args[0])
    lse = torch.empty(case.q.shape[:2], dtype=torch.float32, device=dev)
    # straight through the C entry point: too small, misaligned, missing
    ws = torch.empty(need + 64, dtype=torch.uint8, device=dev)
    base = dict(window_left=-1, window_right=-1, num_splits=4)
    for ptr, nbytes in ((ws.data_ptr(), need - 1), (ws.data_ptr() + 4, need), (0, need)):
        rc = fa.varlen_attn_fwd_raw(
            args[0].data_ptr(), args[1].data_ptr(), args[2].data_ptr(), args[3].data_ptr(),
            args[4].data_ptr(), len(LQ), case.q.shape[0], case.k.shape[0], case.max_q,
            case.max_k, 16, 2, 128, False, 0.0, fa.VARLEN_BF16, out.data_ptr(), lse.data_ptr(),
            torch.cuda.current_stream().cuda_stream, workspace_ptr=ptr, workspace_bytes=nbytes,
            **base)
        assert rc == -8
    torch.cuda.synchronize()


# ---- replicated rows: decode-like calls (at most 32 query rows per KV head)
# The pair kernel puts four copies of an item's <= 32 rows in the four TMEM
# lane quarters and gives copy c keys [32c, 32c + 32) of every key tile; the
# copies are merged like key-range pieces.  Eligible: non-causal, no window,
# H/Hkv a power of two >= 2, max_seqlen_q * H/Hkv <= 32, max_seqlen_k >= 1024,
# and a workspace (the binding passes one unless num_splits=1).

DEC_LK = [5000, 1025, 0, 3000, 17, 2048, 1999, 40]


@pytest.mark.parametrize("H,Hkv,max_q", [(4, 2, 16), (32, 8, 8), (16, 2, 4), (32, 2, 2),
                                         (32, 1, 1)])
def test_rep_group_sizes(H, Hkv, max_q):
    gen = np.random.default_rng(1200 + H + Hkv)
    lq = [int(x) for x in gen.integers(1, max_q + 1, len(DEC_LK))]
    lq[1] = max_q
    case = workloads.make_case(lq, DEC_LK, H, Hkv, 128, "bf16", False, seed=1201 + H)
    full_check(case)


@pytest.mark.parametrize("splits", [None, 2, 3, 8, 32])
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "fp16"), (128, "fp16")])
def test_rep_with_key_pieces(D, dtype, splits):
    lq = [1, 2, 1, 4, 3, 1, 2, 1]
    case = workloads.make_case(lq, DEC_LK, 32, 8, D, dtype, False, seed=1210 + D)
    full_check(case, num_splits=splits)


def test_rep_empty_query_and_key_sequences():
    lq = [1, 0, 2, 1, 0, 3]
    lk = [0, 3000, 1500, 0, 0, 2000]
    case = workloads.make_case(lq, lk, 32, 8, 128, "bf16", False, seed=1220)
    out, lse = full_check(case)
    cu = case.cu_q.tolist()
    assert np.all(out[cu[0]:cu[1]] == 0.0) and np.all(np.isneginf(lse[cu[0]:cu[1]]))


def test_rep_with_sinks_and_seqused_k():
    lq = [1, 2, 1, 4, 3, 1, 2, 1]
    case = workloads.make_case(lq, DEC_LK, 32, 8, 128, "bf16", False, seed=1230)
    sinks = np.random.default_rng(1231).uniform(-2.0, 4.0, 32).astype(np.float32).tolist()
    used = [4000, 1025, 0, 1, 17, 1100, 33, 40]
    full_check(case, mask=dict(sinks=sinks, seqused_k=used))


@pytest.mark.parametrize("page_size", [16, 64])
def test_rep_paged(page_size):
    lq = [1, 2, 1, 4, 3, 1, 2, 1]
    case = workloads.make_case(lq, DEC_LK, 32, 8, 128, "bf16", False, seed=1240 + page_size)
    paged = workloads.to_paged(case, page_size, seed=1241)
    full_check(case, paged=paged, num_splits=4)


def test_rep_understated_max_seqlen_k():
    lq = [1, 2, 1, 4, 3, 1, 2, 1]
    case = workloads.make_case(lq, DEC_LK, 32, 8, 128, "bf16", False, seed=1250)
    full_check(case, max_k=1024, num_splits=2)


def test_rep_equals_plain_path_up_to_rounding():
    lq = [1, 2, 1, 4, 3, 1, 2, 1]
    case = workloads.make_case(lq, DEC_LK, 32, 8, 128, "fp16", False, seed=1260)
    o1, l1, _, _ = run_gpu(case, num_splits=1)      # no workspace: the plain kernel path
    o2, l2, _, _ = run_gpu(case, num_splits=None)   # replicated rows (+ key pieces)
    fin = np.isfinite(l1)
    assert np.array_equal(fin, np.isfinite(l2))
    assert np.abs(o1 - o2).max() <= 4e-3
    assert np.abs(l1[fin] - l2[fin]).max() <= 1e-4


def test_rep_deterministic():
    lq = [1, 2, 1, 4, 3, 1, 2, 1]
    case = workloads.make_case(lq, DEC_LK, 32, 8, 128, "bf16", False, seed=1270)
    _, _, a_o, a_l = run_gpu(case)
    _, _, b_o, b_l = run_gpu(case)
    assert torch.equal(a_o, b_o) and torch.equal(a_l, b_l)
