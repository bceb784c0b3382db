"""Concurrent first calls from several host threads.

The library keeps per-device host state (the SM count, which kernels have had
their shared-memory limit raised, the tensor-map encoder's address), set up by
the first call in each CUDA context under a mutex.  Here a fresh process
starts eight threads that make their first forward calls at the same moment,
each on its own stream and buffers, in a mix of kernel forms; every result
must equal, bit for bit, the same call made alone afterwards (the forward is
deterministic), and the device status word must stay clear.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys, threading
sys.path.insert(0, sys.argv[1])
import torch
import flash_attention_fwd_b200 as fa
import workloads

dev = torch.device("cuda", 0)
torch.cuda.init()
shapes = [  # (lens_q, lens_k, H, Hkv, D, dtype, causal): pair, single, packed, wide
    ([300, 1, 129], None, 8, 2, 128, "bf16", True),
    ([200, 77], None, 6, 6, 64, "fp16", False),
    ([12, 5, 40], [300, 129, 700], 16, 2, 128, "bf16", False),
    ([256, 3], None, 4, 4, 256, "fp16", True),
]
cases = []
for i in range(8):
    lq, lk, H, Hkv, D, dt, causal = shapes[i % len(shapes)]
    c = workloads.make_case(lq, lk, H, Hkv, D, dt, causal, seed=3000 + i)
    cases.append([t.to(dev) if isinstance(t, torch.Tensor) else t
                  for t in (c.q, c.k, c.v, c.cu_q, c.cu_k)] + [c.max_q, c.max_k, causal])
torch.cuda.synchronize()
go = threading.Barrier(len(cases))
results = [None] * len(cases)
errors = []

def work(i):
    try:
        q, k, v, cq, ck, mq, mk, causal = cases[i]
        s = torch.cuda.Stream(device=dev)
        go.wait()
        with torch.cuda.stream(s):
            out, lse = fa.varlen_attn_fwd(q, k, v, cq, ck, mq, mk, causal, stream=s)
        s.synchronize()
        results[i] = (out.cpu(), lse.cpu())
    except Exception as e:  # reported by the parent
        errors.append(repr(e))

threads = [threading.Thread(target=work, args=(i,)) for i in range(len(cases))]
for t in threads:
    t.start()
for t in threads:
    t.join()
assert not errors, errors
for i, (q, k, v, cq, ck, mq, mk, causal) in enumerate(cases):
    out, lse = fa.varlen_attn_fwd(q, k, v, cq, ck, mq, mk, causal)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu().view(torch.int16), results[i][0].view(torch.int16)), i
    assert torch.equal(lse.cpu(), results[i][1]), i
assert fa.device_status(clear=True) == 0
print("threads ok")
"""


def test_first_calls_from_many_host_threads():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "threads ok" in r.stdout, r.stdout + r.stderr
