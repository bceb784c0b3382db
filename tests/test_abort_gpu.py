"""The kernels' abort path, exercised without a fault.

Every wait inside the kernels is bounded; when one runs out, the CTA raises an
abort flag, sets bit 1 of the device status word, drains the copies and
tensor-core work it has in flight, frees its TMEM and returns.  Here the
pipeline-wait limit is lowered to 20 microseconds (varlen_attn_set_wait_limit,
a testing hook), and the batch holds 200,000 sequences, all but a few of them
empty: the scheduling warp walks the whole sequence table before it hands out
the first work item, which takes far longer than the limit, so the other
roles' first waits run out and the kernels take the abort path.  The test
checks that the call returns, that the status word reports it, and that the
context stays usable: with the default limit restored, the next calls on
fresh buffers match the oracle and leave the word clear.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import check_close, require_gpu, run_gpu

pytestmark = pytest.mark.gpu

SHORT_NS = 20000
EMPTY_SEQUENCES = 200000


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


def _with_empty_sequences(case):
    """The case's sequence table with EMPTY_SEQUENCES empty sequences in
    front (same tokens, same results)."""
    pad = torch.zeros(EMPTY_SEQUENCES, dtype=torch.int32)
    return torch.cat([pad, case.cu_q]), torch.cat([pad, case.cu_k])


def _aborted_call(fn):
    """Runs fn() with the short wait limit; returns the status word."""
    import flash_attention_fwd_b200 as fa
    fa.device_status(clear=True)
    torch.cuda.synchronize()
    fa.set_wait_limit(SHORT_NS)
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        fa.set_wait_limit(0)
    return fa.device_status(clear=True)


# (lens, H, Hkv, D, dtype, causal): pair kernel, single kernel (D = 256),
# GQA-packed short queries
CASES = [
    ([1736, 630, 337, 701], None, 32, 8, 128, "bf16", True),
    ([700, 1300], None, 8, 8, 256, "fp16", True),
    ([12, 40, 5], [3000, 900, 4000], 32, 8, 128, "bf16", False),
]


@pytest.mark.parametrize("i", range(len(CASES)))
def test_forward_abort_then_recover(i):
    import flash_attention_fwd_b200 as fa
    lq, lk, H, Hkv, D, dt, causal = CASES[i]
    case = workloads.make_case(lq, lk, H, Hkv, D, dt, causal, seed=4000 + i)
    dev = torch.device("cuda", 0)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    cq, ck = (t.to(dev) for t in _with_empty_sequences(case))
    status = _aborted_call(lambda: fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q, case.max_k,
                                                      case.causal, num_splits=1))
    assert status & 1, "no pipeline wait ran out under a %d ns limit" % SHORT_NS
    # the default limit is back: fresh buffers, full parity, clear status
    out, lse, _, _ = run_gpu(case)
    ref_out, ref_lse = oracle.run_case(case)
    check_close(out, lse, ref_out, ref_lse, "after an aborted launch")
    assert fa.device_status(clear=True) == 0


def test_backward_abort_then_recover():
    import flash_attention_fwd_b200 as fa
    case = workloads.make_case([900, 300, 77], None, 8, 2, 128, "bf16", True, seed=4100)
    dev = torch.device("cuda", 0)
    ref_out, ref_lse = oracle.run_case(case)
    o16 = torch.from_numpy(ref_out).to(case.q.dtype)
    lse32 = torch.from_numpy(ref_lse).to(torch.float32)
    g = torch.Generator("cpu").manual_seed(4101)
    dout = torch.randn(case.q.shape, generator=g).to(case.q.dtype)
    args = [t.to(dev) for t in (dout, case.q, case.k, case.v, o16, lse32, case.cu_q, case.cu_k)]
    long_table = [t.to(dev) for t in _with_empty_sequences(case)]
    status = _aborted_call(lambda: fa.varlen_attn_bwd(*args[:6], *long_table, case.max_q,
                                                      case.max_k, case.causal, case.scale))
    assert status & 1, "no pipeline wait ran out under a %d ns limit" % SHORT_NS
    dq, dk, dv = fa.varlen_attn_bwd(*args, case.max_q, case.max_k, case.causal, case.scale)
    torch.cuda.synchronize()
    refs = oracle.run_case_bwd(case, dout, o16, lse32)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        err = np.abs(got.cpu().to(torch.float64).numpy() - ref)
        assert err.max() <= 1.5e-2 * np.abs(ref).max(), name
        assert err.mean() <= 2.0 ** -8 * np.abs(ref).mean(), name
    assert fa.device_status(clear=True) == 0


def test_opt_in_status_check_raises(monkeypatch):
    """With VARLEN_ATTN_CHECK_STATUS set, the binding waits for each call and
    raises VARLEN_ERR_DEVICE when a bounded wait ran out; a normal call does
    not raise."""
    import flash_attention_fwd_b200 as fa
    lq, lk, H, Hkv, D, dt, causal = CASES[0]
    case = workloads.make_case(lq, lk, H, Hkv, D, dt, causal, seed=4200)
    dev = torch.device("cuda", 0)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    cq, ck = case.cu_q.to(dev), case.cu_k.to(dev)
    long_q, long_k = (t.to(dev) for t in _with_empty_sequences(case))
    monkeypatch.setenv(fa.STATUS_CHECK_ENV, "1")
    fa.device_status(clear=True)
    fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q, case.max_k, case.causal, num_splits=1)
    torch.cuda.synchronize()
    fa.set_wait_limit(SHORT_NS)
    try:
        with pytest.raises(fa.VarlenAttnError) as err:
            fa.varlen_attn_fwd(q, k, v, long_q, long_k, case.max_q, case.max_k, case.causal,
                               num_splits=1)
        assert err.value.code == fa.VARLEN_ERR_DEVICE
    finally:
        torch.cuda.synchronize()
        fa.set_wait_limit(0)
    fa.device_status(clear=True)
    # the check stays on: a normal call on fresh buffers passes it and matches
    out, lse, _, _ = run_gpu(case)
    ref_out, ref_lse = oracle.run_case(case)
    check_close(out, lse, ref_out, ref_lse, "after the raised check")
