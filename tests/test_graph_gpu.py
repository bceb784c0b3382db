"""The forward inside a CUDA graph: the C entry points make no host
synchronisation and allocate nothing, so a call (and its merge launch, with
a caller workspace) can be captured once and replayed on new contents of the
same buffers.  Checked for the plain path, the key-range split and the
replicated-rows form: each replay must equal an eager call on the same
inputs bit for bit."""
import pytest
import torch

import workloads
from parity_helpers import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


CASES = {
    # (lens_q, lens_k, H, Hkv, D, causal, num_splits)
    "plain causal": ([300, 1, 129, 513], None, 8, 2, 128, True, 1),
    "key-range split": ([40, 64, 1, 17], [3000, 700, 5000, 2048], 16, 2, 128, False, 4),
    "replicated rows": ([1, 2, 1, 4], [5000, 1025, 3000, 2048], 32, 8, 128, False, None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_replays_in_a_cuda_graph(name):
    import flash_attention_fwd_b200 as fa
    lq, lk, H, Hkv, D, causal, splits = CASES[name]
    dev = torch.device("cuda", 0)
    cases = [workloads.make_case(lq, lk, H, Hkv, D, "bf16", causal, seed=1300 + i)
             for i in range(3)]
    c0 = cases[0]
    q, k, v = c0.q.to(dev), c0.k.to(dev), c0.v.to(dev)
    cq, ck = c0.cu_q.to(dev), c0.cu_k.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    ws = None
    if not causal:
        n = splits if splits is not None else fa.fwd_num_splits(
            len(lq), q.shape[0], k.shape[0], c0.max_q, c0.max_k, H, Hkv, D)
        nbytes = fa.fwd_workspace_size(q.shape[0], H, Hkv, D, c0.max_q, c0.max_k, n)
        assert nbytes > 0
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def call(stream):
        fa.varlen_attn_fwd(q, k, v, cq, ck, c0.max_q, c0.max_k, causal, None, out=out, lse=lse,
                           stream=stream, num_splits=splits, workspace=ws)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        call(side)  # attributes and one-time setup outside the capture
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(torch.cuda.current_stream(dev))
    for c in cases[1:]:
        q.copy_(c.q.to(dev))
        k.copy_(c.k.to(dev))
        v.copy_(c.v.to(dev))
        graph.replay()
        torch.cuda.synchronize()
        got_o, got_l = out.clone(), lse.clone()
        call(torch.cuda.current_stream(dev))
        torch.cuda.synchronize()
        assert torch.equal(got_o, out) and torch.equal(got_l, lse), name
        assert not torch.isnan(got_o).any()
    del graph
