"""World-size-2 checks of the multi-rank host path on CPU (gloo): timings are
reduced with a max over ranks, the whole-job value counts every rank's
batch, and the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = [10.0 + rank * 5.0, 40.0 - rank * 10.0]
    got = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
    results[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    assert results[0] == [15.0, 40.0] and results[1] == [15.0, 40.0]


def test_whole_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(1, 10 ** 12, 100.0)
    two = bench.whole_job_tflops(2, 10 ** 12, 100.0)
    assert abs(one - 10.0) < 1e-9 and abs(two - 20.0) < 1e-9


def test_reference_arm_rank0_only():
    """Under torchrun the reference arm prints on rank 0; other ranks exit 0 silently."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--reference-seconds", "2",
                        "--workload", "tiny"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


# --- one batch split over two ranks (the forward has no exchange step) -----------------

def _shard_worker(rank, world, port, results):
    """Each rank plans the split, computes its shard with the fp64 oracle and
    gathers every rank's part; rank 0 reassembles them."""
    import datetime
    import numpy as np
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import flash_attention_fwd_b200 as fa
    import oracle
    import workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        out = {}
        # pair balance of the split on the long ragged prefill's lengths
        lq, lk = workloads.seqlens("long")
        plan = fa.plan_shards(workloads.cu_seqlens(lq).tolist(), workloads.cu_seqlens(lk).tolist(),
                              64, 8, world, "auto", causal=True)
        out["long_plan"] = plan
        # small cases, both splits, with and without a mask: oracle parts
        case = workloads.make_case([37, 5, 130, 1, 64, 200, 9], [37, 50, 130, 1, 64, 200, 90],
                                   8, 4, 16, "bf16", True, seed=31)
        masks = [{}, {"window_left": 20, "seqused_k": [30, 5, 100, 1, 64, 150, 0],
                      "sinks": [0.5 * h - 1.0 for h in range(8)]}]
        for mi, mask in enumerate(masks):
            case.mask = mask
            for mode in ("kv_heads", "sequences"):
                plan = fa.plan_shards(case.cu_q.tolist(), case.cu_k.tolist(), case.H, case.Hkv,
                                      world, mode, causal=case.causal,
                                      window_size_left=mask.get("window_left", -1),
                                      seqused_k=mask.get("seqused_k"))
                sub = workloads.shard_case(case, plan, rank)
                o, l = oracle.run_case(sub, **sub.mask)
                parts = [None] * world
                dist.all_gather_object(parts, (o, l))
                plans = [None] * world
                dist.all_gather_object(plans, plan)
                if rank == 0:
                    full_o, full_l, count = workloads.unshard(case, plan, parts)
                    ref_o, ref_l = oracle.run_case(case, **mask)
                    out[(mi, mode)] = dict(
                        same_plan=all(p == plan for p in plans),
                        once=bool(np.all(count == 1)),
                        bitwise=bool(np.array_equal(full_o, ref_o)
                                     and np.array_equal(full_l, ref_l)),
                        pairs=plan["pairs"])
        results[rank] = out
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shards_cover_every_row_once_and_reassemble_bitwise():
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    r0 = results[0]
    # the long ragged prefill splits by key/value-head groups, 4 of 8 per rank:
    # equal pair counts that add up to the batch's
    plan = r0["long_plan"]
    lq, lk = workloads.seqlens("long")
    total = bench.unmasked_pairs(lq, lk, 64, True)
    assert plan["mode"] == "kv_heads" and plan["kv_heads"] == [(0, 4), (4, 8)]
    assert sum(plan["pairs"]) == total
    assert max(plan["pairs"]) <= 1.05 * min(plan["pairs"])
    for key, got in r0.items():
        if key == "long_plan":
            continue
        assert got["same_plan"], key
        assert got["once"], "%s: a (token, head) row is not covered exactly once" % (key,)
        assert got["bitwise"], "%s: shards do not reassemble into the whole result" % (key,)


def test_sequence_split_balances_pairs():
    """The sequence split: longest processing time first over unmasked pairs
    (host planner; no device needed)."""
    sys.path.insert(0, ROOT)
    import bench
    import flash_attention_fwd_b200 as fa
    import workloads
    for name in ("gqa", "shortq"):
        lq, lk = workloads.seqlens(name)
        w = workloads.WORKLOADS[name]
        total = bench.unmasked_pairs(lq, lk, w.H, w.causal)
        for world in (2, 3):
            p = fa.plan_shards(workloads.cu_seqlens(lq).tolist(), workloads.cu_seqlens(lk).tolist(),
                               w.H, w.Hkv, world, "sequences", causal=w.causal)
            assert sum(p["pairs"]) == total
            assert max(p["pairs"]) <= 1.05 * total / world, (name, world, p["pairs"])
            assert sorted(set(p["seq_rank"])) == list(range(world))
    # more ranks than key/value heads: the automatic choice falls back to sequences
    lq, lk = workloads.seqlens("shortq")
    p = fa.plan_shards(workloads.cu_seqlens(lq).tolist(), workloads.cu_seqlens(lk).tolist(),
                       32, 4, 8, "auto")
    assert p["mode"] == "sequences"
    import pytest as _pytest
    with _pytest.raises(fa.VarlenAttnError):
        fa.plan_shards([0, 5], [0, 5], 32, 4, 8, "kv_heads")
