"""varlen_attn_bwd_noalloc (the backward with the library's fixed 16 MiB
scratch instead of a caller workspace) against varlen_attn_bwd_v1 with a
workspace: two calls in a row must give the same bytes as the workspace
entry point, and problems whose scratch would not fit are rejected on the
host.  Kept in a file of its own, collected last, so that the fixed scratch
is first touched after every other GPU test has run."""
import pytest
import torch

import workloads
from parity_helpers import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_workspace_entry_point_twice(causal):
    import flash_attention_fwd_b200 as fa
    dev = torch.device("cuda", 0)
    case = workloads.make_case([300, 1, 129, 128, 77, 513], None, 8, 2, 128, "bf16", causal,
                               seed=950 + causal)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    cq, ck = case.cu_q.to(dev), case.cu_k.to(dev)
    out, lse = fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q, case.max_k, causal, case.scale)
    g = torch.Generator(device="cuda").manual_seed(951)
    dout = torch.randn(q.shape, generator=g, device=dev).to(q.dtype)
    ref = fa.varlen_attn_bwd(dout, q, k, v, out, lse, cq, ck, case.max_q, case.max_k, causal,
                             case.scale)
    for _ in range(2):
        dq = torch.full_like(q, float("nan"))
        dk = torch.full_like(k, float("nan"))
        dv = torch.full_like(v, float("nan"))
        rc = fa.varlen_attn_bwd_noalloc(dout, q, k, v, out, lse, cq, ck, case.max_q, case.max_k,
                                        dq, dk, dv, causal, case.scale)
        torch.cuda.synchronize()
        assert rc == 0, fa.strerror(rc)
        for got, want in zip((dq, dk, dv), ref):
            assert torch.equal(got, want)


def test_noalloc_rejects_scratch_beyond_its_size():
    import flash_attention_fwd_b200 as fa
    dev = torch.device("cuda", 0)
    # 2^20 tokens x 8 heads x 4 bytes = 32 MiB of scratch > 16 MiB: rejected before any launch
    T, H = 1 << 20, 8
    q = torch.empty((T, H, 64), dtype=torch.bfloat16, device=dev)
    k = torch.empty((16, 1, 64), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, H), dtype=torch.float32, device=dev)
    cu = torch.tensor([0, T], dtype=torch.int32, device=dev)
    cuk = torch.tensor([0, 16], dtype=torch.int32, device=dev)
    rc = fa.varlen_attn_bwd_noalloc(q, q, k, k, q, lse, cu, cuk, T, 16, q, k, k, True)
    assert rc == -8
