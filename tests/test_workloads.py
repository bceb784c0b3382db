"""The seeded generators reproduce the benchmark configurations' lengths."""
import json
import os

import numpy as np
import pytest
import torch

import workloads

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "workload_lengths.json")))


@pytest.mark.parametrize("name", ["tiny", "gqa", "long", "wide"])
def test_lengths(name):
    lq, lk = workloads.seqlens(name)
    assert lq == GOLDEN[name]["lens_q"]
    assert lk == lq


def test_tiny_cu_seqlens():
    lq, _ = workloads.seqlens("tiny")
    assert workloads.cu_seqlens(lq).tolist() == GOLDEN["tiny"]["cu_seqlens"]


def test_shortq_totals():
    lq, lk = workloads.seqlens("shortq")
    assert len(lq) == 32 and len(lk) == 32
    assert sum(lq) == GOLDEN["shortq"]["Tq"] and sum(lk) == GOLDEN["shortq"]["Tk"]
    assert min(lq) >= 1 and max(lq) <= 64 and min(lk) >= 512 and max(lk) <= 8192


def test_long_total_is_exact():
    lq, _ = workloads.seqlens("long")
    assert sum(lq) == 65536 and len(lq) == 16 and min(lq) >= 1


def test_tensor_recipe_is_deterministic_and_cast():
    a = workloads.make_case([5, 3], None, 4, 2, 16, "fp16", True, seed=7, sigma_q=3.0)
    b = workloads.make_case([5, 3], None, 4, 2, 16, "fp16", True, seed=7, sigma_q=3.0)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    assert a.q.dtype == torch.float16 and a.q.shape == (8, 4, 16) and a.k.shape == (8, 2, 16)
    g = torch.Generator("cpu").manual_seed(7)
    q = (torch.randn((8, 4, 16), generator=g) * 3.0).to(torch.float16)
    assert torch.equal(q, a.q)


def test_half_ulp_bounds_rounding_to_16_bit():
    # the GPU tests' allowance for rounding the exact result to bf16 / fp16:
    # every value lies within half_ulp of its rounded form, and the bound is
    # tight (reached at midpoints between neighbours)
    import torch
    from parity_helpers import half_ulp
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 50, 20000),
                        rng.uniform(-1e-3, 1e-3, 5000)])
    # float32 values, so that the cast to 16 bits is a single rounding
    x = x.astype(np.float32).astype(np.float64)
    for name, tdt in (("bf16", torch.bfloat16), ("fp16", torch.float16)):
        r = torch.from_numpy(x).to(tdt).to(torch.float64).numpy()
        assert np.all(np.abs(x - r) <= half_ulp(x, name))
        one = np.array([1.0])
        step = 2.0 ** -(7 if name == "bf16" else 10)
        assert half_ulp(one, name)[0] == step / 2
