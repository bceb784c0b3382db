"""Shared pieces of the GPU parity tests: run the CUDA path through the C ABI
with guard rows around the outputs, and compare with the fp64 oracle.

Tolerances (bf16/fp16 output against fp64): O max abs err <= 1.5e-2, O mean
abs err <= 2e-3, LSE max abs err <= 5e-3.  Indexing is checked exactly: the
output buffers carry guard rows before and after the packed extents, filled
with a canary, and must come back with every packed row written (no NaN
pre-fill left) and every guard row untouched.

``mask`` (optional dict: window_left, window_right, seqused_k, sinks) selects
the sliding-window / used-key / sink form of the forward; the same dict goes
to the oracle.
"""
import numpy as np
import torch

import oracle
import workloads

O_MAX, O_MEAN, LSE_MAX = 1.5e-2, 2e-3, 5e-3
GUARD = 3


def run_gpu(case, scale=None, guard=GUARD, max_q=None, max_k=None, mask=None, paged=None,
            num_splits=None):
    """Runs the CUDA forward with NaN-filled outputs inside guard rows.
    ``paged`` (a workloads.PagedKV) replaces the packed K/V by its page cache,
    page table and key counts (mask's seqused_k, if any, wins).
    ``num_splits``: key-range pieces (None: the library's choice).
    Returns (out float64 [Tq,H,D], lse float64 [Tq,H], raw out, raw lse)."""
    import flash_attention_fwd_b200 as fa
    mask = mask or {}
    dev = torch.device("cuda", 0)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    cq, ck = case.cu_q.to(dev), case.cu_k.to(dev)
    Tq, H, D = case.q.shape
    tdt = case.q.dtype
    out_buf = torch.full((Tq + 2 * guard, H, D), float("nan"), dtype=tdt, device=dev)
    lse_buf = torch.full((Tq + 2 * guard, H), float("nan"), dtype=torch.float32, device=dev)
    canary = torch.tensor(-12345.0, dtype=tdt)
    out_buf[:guard] = canary
    out_buf[guard + Tq:] = canary
    lse_buf[:guard] = -777.0
    lse_buf[guard + Tq:] = -777.0
    out = out_buf[guard:guard + Tq]
    lse = lse_buf[guard:guard + Tq]
    used = mask.get("seqused_k")
    table = None
    if paged is not None:
        k, v = paged.k_cache.to(dev), paged.v_cache.to(dev)
        table = paged.page_table.to(dev)
        ck = None
        if used is None:
            used = paged.seqused_k
    used_t = None if used is None else torch.tensor(list(used), dtype=torch.int32, device=dev)
    sinks = mask.get("sinks")
    sinks_t = None if sinks is None else torch.tensor(list(sinks), dtype=torch.float32,
                                                      device=dev)
    fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q if max_q is None else max_q,
                       case.max_k if max_k is None else max_k, case.causal,
                       scale if scale is not None else case.scale, out=out, lse=lse,
                       window_size_left=mask.get("window_left", -1),
                       window_size_right=mask.get("window_right", -1), seqused_k=used_t,
                       page_table=table, sinks=sinks_t, num_splits=num_splits)
    torch.cuda.synchronize()
    ob, lb = out_buf.cpu(), lse_buf.cpu()
    assert torch.all(ob[:guard] == canary) and torch.all(ob[guard + Tq:] == canary), \
        "guard rows of out written"
    assert torch.all(lb[:guard] == -777.0) and torch.all(lb[guard + Tq:] == -777.0), \
        "guard rows of lse written"
    return (ob[guard:guard + Tq].to(torch.float64).numpy(),
            lb[guard:guard + Tq].to(torch.float64).numpy(),
            ob[guard:guard + Tq], lb[guard:guard + Tq])


def half_ulp(x, dtype):
    """Half a unit in the last place of the bf16 / fp16 value nearest to each
    element of x: the error of rounding an exact result to the output dtype."""
    frac_bits, min_exp = {"bf16": (7, -126), "fp16": (10, -14)}[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** min_exp)))
    return 0.5 * 2.0 ** (e - frac_bits)


def check_close(out, lse, ref_out, ref_lse, what="", round_to=None):
    """``round_to`` ("bf16" / "fp16"): each O element may also differ by the
    rounding of the exact result to that dtype (half an ulp of the reference)
    on top of the absolute tolerance; for outputs of magnitude >= 4 in bf16
    that rounding alone (up to 2^-6) exceeds 1.5e-2."""
    assert not np.isnan(out).any(), "%s: NaN left in out (row not written)" % what
    assert not np.isnan(lse).any(), "%s: NaN left in lse (row not written)" % what
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin), "%s: -inf pattern of lse differs" % what
    assert np.all(np.isneginf(lse[~fin])), "%s: rows without keys need lse = -inf" % what
    assert np.all(out[~fin] == 0.0), "%s: rows without keys need O = 0" % what
    err = np.abs(out - ref_out)
    if round_to is not None:
        excess = err - half_ulp(ref_out, round_to)
        assert excess.max() <= O_MAX, "%s: O max abs err beyond rounding %.3e" % (
            what, excess.max())
    else:
        assert err.max() <= O_MAX, "%s: O max abs err %.3e" % (what, err.max())
    assert err.mean() <= O_MEAN, "%s: O mean abs err %.3e" % (what, err.mean())
    if fin.any():
        lerr = np.abs(lse[fin] - ref_lse[fin]).max()
        assert lerr <= LSE_MAX, "%s: LSE max abs err %.3e" % (what, lerr)


def full_check(case, mask=None, round_to=None, **kw):
    """Whole output against the oracle (with a page cache, the oracle reads
    the packed K/V the cache was built from)."""
    out, lse, _, _ = run_gpu(case, mask=mask, **kw)
    ref_out, ref_lse = oracle.run_case(case, **(mask or {}))
    check_close(out, lse, ref_out, ref_lse, case.name, round_to=round_to)
    return out, lse


def sampled_check(case, n=2000, seed=7, mask=None, **kw):
    out, lse, _, _ = run_gpu(case, mask=mask, **kw)
    assert not np.isnan(out).any() and not np.isnan(lse).any(), "a packed row was not written"
    rows = workloads.sample_rows(case, n, seed=seed)
    ref_out, ref_lse = oracle.run_case_rows(case, rows, **(mask or {}))
    check_close(out[rows[:, 0], rows[:, 1]], lse[rows[:, 0], rows[:, 1]], ref_out, ref_lse,
                case.name)


def stratified_check(case, per_tile=1, seed=4321, mask=None, **kw):
    """At least `per_tile` oracle-checked rows of every (sequence, 128-query
    tile, head) — so every work item of the kernels' schedule is compared —
    plus each (sequence, head)'s last row; every other row must be written."""
    out, lse, _, _ = run_gpu(case, mask=mask, **kw)
    assert not np.isnan(out).any() and not np.isnan(lse).any(), "a packed row was not written"
    rows = workloads.stratified_rows(case, seed=seed, per_tile=per_tile)
    ref_out, ref_lse = oracle.run_case_rows(case, rows, **(mask or {}))
    check_close(out[rows[:, 0], rows[:, 1]], lse[rows[:, 0], rows[:, 1]], ref_out, ref_lse,
                case.name)
    return rows.shape[0]


def require_gpu():
    """Body of the module fixtures: skip without a device, clear the device
    status word before and check it after the module's tests."""
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import flash_attention_fwd_b200 as fa
    fa.load_library()
    fa.device_status(clear=True)
    yield
    assert fa.device_status(clear=True) == 0, "a bounded pipeline wait timed out on the device"
