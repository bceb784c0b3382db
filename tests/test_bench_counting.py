"""The benchmark's work counts (unmasked pairs -> FLOPs, algorithmic bytes)
against brute-force enumeration of the visibility rule: key ki is visible to
query qi iff ki < min(Lk, seqused_k), qi - left <= ki (left >= 0),
ki <= qi + right (right >= 0) and not (causal and qi < ki)."""
import numpy as np
import pytest

import bench
import workloads


def brute(lq, lk, causal, left, right, used):
    lim = lk if used is None else min(lk, max(used, 0))
    return sum(1 for qi in range(lq) for ki in range(lk)
               if ki < lim and (left < 0 or ki >= qi - left) and (right < 0 or ki <= qi + right)
               and not (causal and qi < ki))


@pytest.mark.parametrize("seed", range(40))
def test_visible_keys_brute_force(seed):
    rng = np.random.default_rng(seed)
    lq, lk = int(rng.integers(0, 40)), int(rng.integers(0, 40))
    causal = bool(rng.integers(0, 2))
    left = int(rng.integers(-1, 12))
    right = int(rng.integers(-1, 12))
    used = None if rng.integers(0, 2) else int(rng.integers(-2, 45))
    assert bench.visible_keys(lq, lk, causal, left, right, used) == \
        brute(lq, lk, causal, left, right, used)


def test_plain_counts_match_closed_form():
    for lq, lk in [(1, 1), (7, 3), (3, 7), (128, 128), (300, 129)]:
        assert bench.visible_keys(lq, lk, True) == brute(lq, lk, True, -1, -1, None)
        assert bench.visible_keys(lq, lk, False) == lq * lk


def test_sampled_row_flops_agree_with_per_row_counts():
    case = workloads.make_case([40, 9, 70], [50, 9, 64], 4, 2, 16, "bf16", True, seed=3)
    case.mask = dict(window_left=5, seqused_k=[30, 9, 100])
    rows, fl = bench.oracle_sample_rows(case, 50, seed=1)
    cu = case.cu_q.tolist()
    want = 0
    for tok, h in rows.tolist():
        b = max(i for i in range(case.B) if cu[i] <= tok)
        qi = tok - cu[b]
        want += brute(qi + 1, case.lens_k[b], True, 5, -1, case.mask["seqused_k"][b]) - \
            brute(qi, case.lens_k[b], True, 5, -1, case.mask["seqused_k"][b])
    assert fl == 4 * case.D * want


def test_used_keys_bytes():
    case = workloads.make_workload("tiny")
    plain = bench.algorithmic_bytes(case)
    case.mask = dict(seqused_k=[17, 0, 1])
    # 64 keys of sequence 1 are not used: K and V rows of Hkv heads x D dropped
    assert plain - bench.algorithmic_bytes(case) == 2 * 64 * case.Hkv * case.D * 2 - 4 * case.B


def test_named_masked_workloads():
    assert workloads.make_workload("long_swa").mask == {"window_left": 4095}
    used = workloads.seqused_k("shortq_used")
    _, lk = workloads.seqlens("shortq_used")
    assert len(used) == 32 and all(k // 2 <= u <= k for u, k in zip(used, lk))


def test_traffic_entries_follow_their_kernel_family(tmp_path, monkeypatch):
    # an entry counts only while the sources of the family it names hash to
    # the value it was captured on; an edit to another family leaves it valid
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(
        '{"a": {"kernel_kind": "pair", "kernel_hash": "P1", "bytes_per_launch": 10},'
        ' "b": {"kernel_kind": "single", "kernel_hash": "S0", "bytes_per_launch": 20},'
        ' "c": {"kernel_hash": "F1", "bytes_per_launch": 30},'
        ' "c:bwd": {"kernel_hash": "B1", "bytes_per_launch": 40}}')
    hashes = {"pair": "P1", "single": "S1", "fwd": "F1", "bwd": "B1"}
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_hash", lambda read=None, kind="fwd": hashes[kind])
    assert bench.traffic_for("a") == 10
    assert bench.traffic_for("b") is None       # single-kernel source changed since
    assert bench.traffic_for("c") == 30         # no family named: all forward kernels
    assert bench.traffic_for("c:bwd") == 40     # backward by the key's suffix
    assert bench.traffic_for("missing") is None


def test_committed_traffic_entries_name_known_families():
    import json
    import os
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for key, ent in d.items():
        assert ent["kernel_kind"] in bench.KERNEL_SOURCES, key
        assert len(ent["kernel_hash"]) == 16 and ent["bytes_per_launch"] > 0, key


def test_strong_scaling_shards_add_up_to_the_batch():
    # --shard: each rank's FLOPs (from its own shard) add up to the batch's,
    # for both splits and with the window / used-key masks
    import argparse
    for name in ("gqa", "shortq_used", "long_swa"):
        full = workloads.make_workload(name)
        total = bench.step_flops(full)
        for mode in ("kv_heads", "sequences"):
            args = argparse.Namespace(shard=mode)
            parts = []
            for r in range(2):
                sub, plan = bench.shard_for_rank(full, args, r, 2)
                assert plan["mode"] == mode
                parts.append(bench.step_flops(sub))
                assert plan["pairs"][r] * 4 * full.D == parts[-1]
            assert sum(parts) == total, (name, mode)
    # one rank, or no --shard: the whole batch
    full = workloads.make_workload("tiny")
    sub, plan = bench.shard_for_rank(full, argparse.Namespace(shard="auto"), 0, 1)
    assert plan is None and sub is full
