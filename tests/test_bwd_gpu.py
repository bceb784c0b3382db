"""GPU parity of the backward (varlen_attn_bwd_v1) against the fp64 oracle's
backward (the gradient the page's varlen_attention_bwd defines).

Both sides get the same inputs: Q, K, V, a seeded dO, and O / LSE taken from
the oracle's forward and rounded to the storage types the GPU path reads
(O to bf16/fp16, LSE to float32); the oracle widens those rounded values
exactly.

Tolerance (derived from the arithmetic; the pages state none for the
backward): the GPU rounds the results to bf16 (relative error up to 2^-9,
mean 2^-10) and, before that, every P and dS term of the dV, dK and dQ
products (2^-9 each); every gradient element sums many such terms with mixed
signs, so its error is measured against the scale of the tensor: mean |err|
<= 2^-8 * mean |ref| (the output rounding plus as much again from the
rounded terms) and max |err| <= 1.5e-2 * max |ref| for bf16; fp16 has three
more fraction bits, so both bounds are divided by 8.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import require_gpu

pytestmark = pytest.mark.gpu

LENS = [300, 1, 129, 128, 77, 513]
TOL = {"bf16": (1.5e-2, 2.0 ** -8), "fp16": (1.5e-2 / 8, 2.0 ** -8 / 8)}
GUARD = 3


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


def rand_dout(case, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(case.q.shape, generator=g).to(case.q.dtype)


def forward_inputs(case):
    """O (storage dtype) and LSE (float32) of the oracle's forward."""
    o, lse = oracle.run_case(case)
    return torch.from_numpy(o).to(case.q.dtype), torch.from_numpy(lse).to(torch.float32)


def run_gpu_bwd(case, dout, o, lse):
    """dq, dk, dv from the CUDA path, with guard rows around every output."""
    import flash_attention_fwd_b200 as fa
    dev = torch.device("cuda", 0)
    Tq, H, D = case.q.shape
    Tk, Hkv, _ = case.k.shape
    canary = torch.tensor(-4321.0, dtype=case.q.dtype)

    def guarded(rows, heads):
        buf = torch.full((rows + 2 * GUARD, heads, D), float("nan"), dtype=case.q.dtype,
                         device=dev)
        buf[:GUARD] = canary
        buf[GUARD + rows:] = canary
        return buf, buf[GUARD:GUARD + rows]

    dq_buf, dq = guarded(Tq, H)
    dk_buf, dk = guarded(Tk, Hkv)
    dv_buf, dv = guarded(Tk, Hkv)
    fa.varlen_attn_bwd(dout.to(dev), case.q.to(dev), case.k.to(dev), case.v.to(dev), o.to(dev),
                       lse.to(dev), case.cu_q.to(dev), case.cu_k.to(dev), case.max_q,
                       case.max_k, case.causal, case.scale, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    res = []
    for buf, rows in ((dq_buf, Tq), (dk_buf, Tk), (dv_buf, Tk)):
        b = buf.cpu()
        assert torch.all(b[:GUARD] == canary) and torch.all(b[GUARD + rows:] == canary), \
            "guard rows written"
        res.append(b[GUARD:GUARD + rows])
    return res


def check_bwd(case, dout_seed=0, what=None):
    dout = rand_dout(case, 900 + dout_seed)
    o, lse = forward_inputs(case)
    got = run_gpu_bwd(case, dout, o, lse)
    ref = oracle.run_case_bwd(case, dout, o, lse)
    tmax, tmean = TOL[case.dtype]
    stats = []
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.to(torch.float64).numpy()
        assert not np.isnan(g).any(), "%s: NaN left (row not written)" % name
        err = np.abs(g - r)
        scale_max = max(np.max(np.abs(r)), 1e-30)
        scale_mean = max(np.mean(np.abs(r)), 1e-30)
        stats.append("%s max %.2e (rel %.2e) mean rel %.2e" % (
            name, err.max(), err.max() / scale_max, err.mean() / scale_mean))
        if r.size == 0:
            continue
        assert err.max() <= tmax * scale_max, "%s %s" % (what or case.name, stats[-1])
        assert err.mean() <= tmean * scale_mean, "%s %s" % (what or case.name, stats[-1])
    print(what or case.name, "; ".join(stats))
    return got


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("causal", [True, False])
def test_backward_ragged_tiles(D, dtype, causal):
    case = workloads.make_case(LENS, None, 4, 2, D, dtype, causal, seed=800 + D + causal)
    check_bwd(case, D + causal)


@pytest.mark.parametrize("H,Hkv", [(8, 8), (6, 2), (3, 1)])
def test_backward_head_dim_256_head_layouts(H, Hkv):
    # head dim 256: 32-key tiles in the dQ pass, dK / dV in two column halves
    case = workloads.make_case([200, 77, 130, 1], None, H, Hkv, 256, "bf16", True,
                               seed=860 + H + Hkv)
    check_bwd(case, 7 + H)


def test_backward_head_dim_256_wide_logits_fp16():
    # the wide-head configuration's shape and logit scale (Q, K ~ N(0, 3^2)),
    # on two sequences of 1024 so that the fp64 oracle stays quick
    case = workloads.make_case([1024, 1024], None, 4, 4, 256, "fp16", True, seed=870,
                               sigma_q=3.0, sigma_k=3.0)
    check_bwd(case, 11)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_head_dim_256_q_and_k_lengths_differ(causal):
    case = workloads.make_case([70, 200, 5, 131], [250, 64, 1, 300], 4, 2, 256, "fp16", causal,
                               seed=880 + causal)
    check_bwd(case, 13)


@pytest.mark.parametrize("H,Hkv", [(8, 2), (3, 1), (3, 3)])
def test_backward_head_layouts(H, Hkv):
    case = workloads.make_case([200, 77, 130], None, H, Hkv, 128, "bf16", True,
                               seed=810 + H + Hkv)
    check_bwd(case, H)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_q_and_k_lengths_differ(causal):
    # causal top-left with Lq < Lk: keys past Lq are seen by no query -> dK = dV = 0
    case = workloads.make_case([70, 200, 5, 131], [250, 64, 1, 300], 6, 3, 128, "bf16", causal,
                               seed=820 + causal)
    got = check_bwd(case, 3)
    if causal:
        cu = case.cu_k.tolist()
        assert torch.all(got[1][cu[0] + 70:cu[1]] == 0) and torch.all(got[2][cu[0] + 70:cu[1]] == 0)


def test_backward_empty_sequences():
    case = workloads.make_case([0, 50, 3, 0, 140], [10, 0, 7, 0, 140], 4, 4, 128, "bf16", False,
                               seed=830)
    got = check_bwd(case, 4)
    # sequence 0 has keys but no queries: dK = dV = 0; sequence 1 has no keys: dQ = 0
    assert torch.all(got[1][:10] == 0) and torch.all(got[2][:10] == 0)
    assert torch.all(got[0][0:50] == 0)


def test_backward_medium_gqa():
    case = workloads.make_case([1000, 600, 37], None, 8, 2, 128, "bf16", True, seed=840)
    check_bwd(case, 5)


def test_backward_deterministic():
    case = workloads.make_case(LENS, None, 8, 2, 128, "bf16", True, seed=850)
    dout = rand_dout(case, 851)
    o, lse = forward_inputs(case)
    a = run_gpu_bwd(case, dout, o, lse)
    b = run_gpu_bwd(case, dout, o, lse)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
