"""Scheduler and indexing at scale: thousands of sequences (the
warp-cooperative walk over cu_seqlens, 32 sequences at a time, many cost
levels, many items per CTA) and one very long sequence (hundreds of key
tiles per item, a long causal diagonal walk)."""
import numpy as np
import pytest

import oracle
import workloads
from parity_helpers import check_close, full_check, require_gpu, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    yield from require_gpu()


def many_lengths(seed, n, hi):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, hi, n)
    lens[rng.integers(0, n, n // 20)] = 0  # some empty sequences
    return [int(x) for x in lens]


@pytest.mark.parametrize("causal", [True, False])
def test_four_thousand_short_sequences(causal):
    lq = many_lengths(1400 + causal, 4000, 40)
    lk = many_lengths(1401 + causal, 4000, 300) if not causal else None
    case = workloads.make_case(lq, lk, 8, 2, 64, "bf16", causal, seed=1402 + causal)
    full_check(case)


def test_four_thousand_sequences_key_range_split():
    lq = many_lengths(1410, 4000, 6)
    lk = many_lengths(1411, 4000, 3000)
    case = workloads.make_case(lq, lk, 8, 2, 128, "bf16", False, seed=1412)
    full_check(case, num_splits=4)


def test_one_long_causal_sequence_sampled():
    case = workloads.make_case([131072], None, 2, 1, 128, "bf16", True, seed=1420)
    out, lse, _, _ = run_gpu(case)
    assert not np.isnan(out).any() and not np.isnan(lse).any()
    rows = workloads.sample_rows(case, 300, seed=1421)
    ref_out, ref_lse = oracle.run_case_rows(case, rows)
    check_close(out[rows[:, 0], rows[:, 1]], lse[rows[:, 0], rows[:, 1]], ref_out, ref_lse,
                "131072-token causal sequence")
