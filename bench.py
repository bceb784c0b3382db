"""Benchmark of the B200 varlen attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long]
    python bench.py --impl reference ...     # the fp64 CPU oracle arm

One step = one call of the C-ABI entry point ``varlen_attn_fwd`` over one
batch of the workload (inputs resident in HBM).  The default workload is the
long ragged prefill (16 causal sequences, 65536 tokens, H=64, Hkv=8, D=128,
bf16), the configuration the throughput target is stated on.  The metric is
TFLOP/s with FLOPs = 4 * D * (unmasked query-key pairs summed over heads).

Prints ONE JSON line on rank 0.  With N > 1 (launched by torchrun) every rank
runs its own batch of the workload (weak scaling, no collective on the data
path); with ``--shard kv_heads|sequences|auto`` the ranks instead split ONE
batch (strong scaling): by key/value-head groups (each rank holds contiguous
head slices, the tensor-parallel layout) or by sequences balanced by
unmasked pairs, as ``varlen_attn_plan_shards`` plans it.  The forward has no
exchange step, so no collective touches the data path either way; the time
is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "varlen attn fwd TFLOP/s (unmasked FLOPs) and % of B200 dense bf16 peak"
METRIC_BWD = ("varlen attn bwd TFLOP/s (10*D per unmasked pair: the backward's five products) "
              "and % of B200 dense bf16 peak")
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_DIR = "flash_attention_fwd_b200/csrc"


# ----------------------------------------------------------------------------- counting

def visible_keys(lq: int, lk: int, causal: bool, window_left: int = -1,
                 window_right: int = -1, used=None) -> int:
    """Unmasked (query, key) pairs of one sequence and one head: key ki is
    visible to query qi iff ki < min(lk, used), qi - left <= ki (left >= 0),
    ki <= qi + right (right >= 0) and not (causal and qi < ki)."""
    if used is not None:
        lk = min(lk, max(int(used), 0))
    if window_left >= 0 or window_right >= 0:
        qi = np.arange(lq, dtype=np.int64)
        lo = np.maximum(0, qi - window_left) if window_left >= 0 else np.zeros_like(qi)
        r = 0 if causal else window_right
        hi = np.minimum(lk, qi + r + 1) if r >= 0 else np.full_like(qi, lk)
        return int(np.maximum(0, hi - lo).sum())
    if not causal:
        return lq * lk
    # query qi sees keys 0..min(qi, lk-1): min(qi+1, lk) keys
    n = min(lq, lk)
    full = n * (n + 1) // 2
    return full + max(0, lq - lk) * lk


def unmasked_pairs(lens_q, lens_k, H: int, causal: bool, mask=None) -> int:
    mask = mask or {}
    used = mask.get("seqused_k") or [None] * len(lens_q)
    return H * sum(visible_keys(a, b, causal, mask.get("window_left", -1),
                                mask.get("window_right", -1), u)
                   for a, b, u in zip(lens_q, lens_k, used))


def step_flops(case) -> int:
    return 4 * case.D * unmasked_pairs(case.lens_q, case.lens_k, case.H, case.causal, case.mask)


def used_keys(case) -> int:
    """Keys a step must read: all of them, or the used counts with seqused_k."""
    used = case.mask.get("seqused_k")
    if used is None:
        return case.Tk
    return sum(min(lk, max(u, 0)) for lk, u in zip(case.lens_k, used))


L2_BYTES = 126 * 1000 * 1000
FLUSH_BYTES = 256 << 20


def input_bytes(case, backward: bool = False) -> int:
    """Bytes of the step's inputs: Q, K, V (and dO, O for the backward)."""
    e = 2
    q = case.Tq * case.H * case.D * e
    kv = 2 * case.Tk * case.Hkv * case.D * e
    return q * (3 if backward else 1) + kv


def timed_steps(step, steps, stream, dev, flush: bool):
    """Runs `steps` steps with a pair of CUDA events around each on `stream`;
    with `flush`, a FLUSH_BYTES buffer (twice the L2) is written before every
    step, outside the events.  Returns the per-step device times (ms)."""
    import torch
    buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    # one untimed step first: the GPU has idled while the clock sampler started
    step()
    torch.cuda.synchronize()
    # keep the GPU busy for about a millisecond while the host queues the first
    # steps, so that no step waits for the host between its events
    torch.cuda._sleep(2_000_000)
    for i in range(steps):
        if buf is not None:
            buf.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [starts[i].elapsed_time(ends[i]) for i in range(steps)]


def l2_note(case, backward: bool = False) -> str:
    nbytes = input_bytes(case, backward)
    if nbytes < 2 * L2_BYTES:
        return ("flush: a %d MB buffer written before every timed step (inputs %.1f MB, under "
                "twice the 126 MB L2)" % (FLUSH_BYTES >> 20, nbytes / 1e6))
    return "no flush: inputs (%.0f MB) exceed twice the 126 MB L2" % (nbytes / 1e6)


def algorithmic_bytes(case) -> int:
    e = 2
    return (case.Tq * case.H * case.D * e * 2 + 2 * used_keys(case) * case.Hkv * case.D * e
            + 4 * case.Tq * case.H + 8 * (case.B + 1)
            + (4 * case.B if "seqused_k" in case.mask else 0))


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# Device-code sources of each kernel family (the host code does not change a
# kernel's traffic): all forward kernels, the pair kernel and the single-tile
# kernel alone, the merge of split key ranges, the backward.
KERNEL_SOURCES = {
    "fwd": ("sm100_ptx.cuh", "fwd_common.cuh", "fwd_pair.cuh", "fwd_single.cuh"),
    "pair": ("sm100_ptx.cuh", "fwd_common.cuh", "fwd_pair.cuh"),
    "single": ("sm100_ptx.cuh", "fwd_common.cuh", "fwd_single.cuh"),
    "combine": ("fwd_common.cuh", "fwd_combine.cuh"),
    "bwd": ("sm100_ptx.cuh", "fwd_common.cuh", "bwd_common.cuh", "bwd_dq.cuh", "bwd_dkdv.cuh"),
}


def kernel_hash(read=None, kind: str = "fwd") -> str:
    """Hash of the device-code sources of the forward or backward kernels."""
    d = os.path.join(ROOT, KERNEL_DIR)
    names = sorted(KERNEL_SOURCES[kind])
    h = hashlib.sha256()
    for n in names:
        h.update(n.encode())
        h.update(read(n) if read else open(os.path.join(d, n), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(workload: str):
    """DRAM bytes per launch from the committed ncu summary, only if it was
    taken on the current source of the kernel family the entry names
    (``kernel_kind``, a key of KERNEL_SOURCES)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d.get(workload)
        default = "bwd" if workload.endswith(":bwd") else "fwd"
        kind = ent.get("kernel_kind", default) if ent else default
        if ent and ent.get("kernel_hash") == kernel_hash(kind=kind):
            return ent.get("bytes_per_launch")
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons, taken while
    the timed region runs."""
    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.bus_id:
                cmd += ["-i", self.bus_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        try:
            rows = [l.strip().split(", ") for l in open(self.path) if l.strip()]
            os.unlink(self.path)
        except Exception:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 10:
                continue
            try:
                sm.append(float(r[2]))
                mx.append(float(r[3]))
            except ValueError:
                continue
            for name, val in zip(names, r[6:10]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def gpu_bus_id(dev_index: int):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev_index)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        return None


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample_rows(case, n_rows: int, seed: int = 99):
    rows = workloads.sample_rows(case, n_rows, seed=seed)
    G = case.H // case.Hkv
    cu = case.cu_q.numpy()
    b = np.searchsorted(cu, rows[:, 0], side="right") - 1
    order = np.lexsort((rows[:, 0], rows[:, 1], rows[:, 1] // G, b))
    rows = rows[order]
    b = b[order]
    qi = rows[:, 0] - cu[b]
    lk = np.asarray(case.lens_k)[b]
    m = case.mask
    if m.get("seqused_k") is not None:
        lk = np.minimum(lk, np.maximum(np.asarray(m["seqused_k"])[b], 0))
    left, right = m.get("window_left", -1), m.get("window_right", -1)
    if case.causal:
        right = 0
    lo = np.maximum(0, qi - left) if left >= 0 else np.zeros_like(qi)
    hi = np.minimum(lk, qi + right + 1) if right >= 0 else lk
    vis = np.maximum(0, hi - lo)
    flops = int(4 * case.D * int(vis.sum()))
    return rows, flops


def time_oracle(case, seconds: float, nthreads: int | None = None):
    """Times the fp64 oracle (as it stands) on a seeded row sample sized for
    about ``seconds`` of CPU work.  Returns (TFLOP/s, rows, flops, secs)."""
    import oracle
    nthreads = nthreads or oracle.default_threads()
    # a small run sizes the sample; it is rescaled from the measured time
    # until a run reaches 60 % of the target (a small run underestimates the
    # rate: fixed costs per call), at most three runs
    n = 256
    for attempt in range(3):
        rows, fl = oracle_sample_rows(case, n, seed=98 + attempt)
        t0 = time.perf_counter()
        oracle.run_case_rows(case, rows, nthreads=nthreads, **case.mask)
        dt = time.perf_counter() - t0
        if dt >= 0.6 * seconds or n >= 2_000_000:
            break
        n = int(max(64, min(2_000_000, n * seconds / max(dt, 1e-3))))
    return fl / dt / 1e12, len(rows), fl, dt, nthreads


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (every rank calls it)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def sum_over_ranks(values, dist, device):
    """Element-wise sum of per-rank counts (every rank calls it)."""
    import torch
    t = torch.tensor([int(v) for v in values], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [int(x) for x in t.tolist()]


def whole_job_tflops(world: int, flops_per_rank_step: int, ms_per_step: float) -> float:
    """Aggregate throughput: every rank processes one batch per step."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def shard_for_rank(case, args, rank: int, world: int):
    """Strong scaling (``--shard``): the rank's part of the one batch, and the
    plan.  Weak scaling: the whole batch, no plan."""
    if args.shard == "none" or world == 1:
        return case, None
    import flash_attention_fwd_b200 as fa
    m = case.mask
    plan = fa.plan_shards(case.cu_q.tolist(), case.cu_k.tolist(), case.H, case.Hkv, world,
                          args.shard, causal=case.causal,
                          window_size_left=m.get("window_left", -1),
                          window_size_right=m.get("window_right", -1),
                          seqused_k=m.get("seqused_k"))
    return workloads.shard_case(case, plan, rank), plan


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args, rank: int, world: int):
    import torch
    import flash_attention_fwd_b200 as fa

    if args.pass_ == "bwd":
        return run_gpu_bwd(args, rank, world)

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    full_case = workloads.make_workload(args.workload)
    case, plan = shard_for_rank(full_case, args, rank, world)
    flops = step_flops(case)
    args.job_flops = step_flops(full_case) if plan else world * flops
    args.plan = plan
    wl = workloads.WORKLOADS[args.workload]
    table_t = None
    if wl.page_size:
        # the same keys in a page cache; the oracle legs read the packed copy
        pk = workloads.to_paged(case, wl.page_size, seed=wl.seed)
        q, k, v = case.q.to(dev), pk.k_cache.to(dev), pk.v_cache.to(dev)
        table_t = pk.page_table.to(dev)
        ck = None
    else:
        q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
        ck = case.cu_k.to(dev)
    cq = case.cu_q.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((case.Tq, case.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    fa.load_library()
    fa.device_status(clear=True)

    used = case.mask.get("seqused_k")
    if table_t is not None and used is None:
        used = case.lens_k
    used_t = None if used is None else torch.tensor(used, dtype=torch.int32, device=dev)
    wl, wr = case.mask.get("window_left", -1), case.mask.get("window_right", -1)
    sinks = case.mask.get("sinks")
    sinks_t = None if sinks is None else torch.tensor(sinks, dtype=torch.float32, device=dev)

    # key-range split: the library's choice for these sizes, with the
    # workspace allocated once, outside the timed region
    splits, ws = 1, None
    if not case.causal and wl < 0 and wr < 0:
        rows_k = k.shape[0] * k.shape[1] if table_t is not None else k.shape[0]
        splits = fa.fwd_num_splits(case.B, case.Tq, rows_k, case.max_q, case.max_k, case.H,
                                   case.Hkv, case.D, paged=table_t is not None, device=dev)
        nbytes = fa.fwd_workspace_size(case.Tq, case.H, case.Hkv, case.D, case.max_q,
                                       case.max_k, splits)
        if nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        else:
            splits = 1
    args.num_splits = splits
    args.workspace_bytes = nbytes if ws is not None else 0

    def step_on(q, k, v, cq, ck, used_t, table_t, sinks_t, out, lse):
        fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q, case.max_k, case.causal, case.scale,
                           out=out, lse=lse, stream=stream, window_size_left=wl,
                           window_size_right=wr, seqused_k=used_t, page_table=table_t,
                           sinks=sinks_t, num_splits=None if ws is not None else 1,
                           workspace=ws)

    set0 = (q, k, v, cq, ck, used_t, table_t, sinks_t)

    def step():
        step_on(*set0, out, lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(gpu_bus_id(local))
    clocks.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    args.l2 = l2_note(case)
    per_launch = timed_steps(step, args.steps, stream, dev, input_bytes(case) < 2 * L2_BYTES)
    if dist:
        dist.barrier()
    clk = clocks.stop()
    total_ms = sum(per_launch)
    status = fa.device_status(clear=True)
    if status != 0:
        raise RuntimeError("device status word set: %d" % status)

    # ---- end to end: pinned host inputs -> device -> kernel -> host results
    if args.no_e2e:
        e2e_ms, h2d, d2h = float("nan"), 0, 0
    else:
        ins0 = [t for t in set0 if t is not None]
        host_in = [pinned(t) for t in ins0]
        for h, d in zip(host_in, ins0):
            h.copy_(d)
        set1 = tuple(None if t is None else torch.empty_like(t) for t in set0)
        outs = [(out, lse), (torch.empty_like(out), torch.empty_like(lse))]
        sets = [set0, set1]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
        e2e_ms = pipelined_e2e(
            lambda b: step_on(*sets[b], *outs[b]),
            [[t for t in st if t is not None] for st in sets], host_in, outs,
            [[pinned(t) for t in o] for o in outs], e2e_steps(args), stream, dist)

    if dist:
        total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist, dev)
        h2d, d2h = sum_over_ranks([h2d, d2h], dist, dev)
        dist.barrier()
    emit(args, rank, world, full_case, flops, total_ms, per_launch, e2e_ms, h2d, d2h, clk,
         launches_per_step=2 if ws is not None else 1, rank_case=case)
    if dist:
        dist.destroy_process_group()


def pipelined_e2e(run_step, dev_in, host_in, dev_out, host_out, steps, stream, dist):
    """End-to-end time per step through the public API: every step copies all
    of its inputs from pinned host memory to the device, runs the call and
    copies all of its results back.  Two device buffer sets take the steps in
    turn, with the host-to-device and device-to-host copies on streams of
    their own, so that the copies of one step overlap the call of the other
    (as a serving loop would run them); a set is refilled only once its
    previous call has read it, and rewritten only once its results have left.
    run_step(b) runs the call on buffer set b on `stream`.  Returns ms per
    step (device time from the first copy to the last result)."""
    import torch
    dev = stream.device
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def one(i):
        b = i % 2
        if used[b]:
            h2d_s.wait_event(comp_done[b])
        with torch.cuda.stream(h2d_s):
            for d, h in zip(dev_in[b], host_in):
                d.copy_(h, non_blocking=True)
        h2d_done[b].record(h2d_s)
        stream.wait_event(h2d_done[b])
        if used[b]:
            stream.wait_event(d2h_done[b])
        run_step(b)
        comp_done[b].record(stream)
        d2h_s.wait_event(comp_done[b])
        with torch.cuda.stream(d2h_s):
            for h, d in zip(host_out[b], dev_out[b]):
                h.copy_(d, non_blocking=True)
        d2h_done[b].record(d2h_s)
        used[b] = True

    one(0)
    one(1)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_s.wait_event(e0)
    d2h_s.wait_event(e0)
    for i in range(steps):
        one(i)
    stream.wait_event(d2h_done[(steps - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def e2e_steps(args) -> int:
    """Steps of the end-to-end leg: the timed steps, at least 2 and at most 20
    (the pipeline's first copy and last read-back are spread over them, as in
    a serving loop that runs on)."""
    return max(2, min(args.steps, 20))


def pinned(t):
    import torch
    return torch.empty(t.shape, dtype=t.dtype).pin_memory()


def hbm_line(case, avg_launch_ms: float, peaks: dict, peak_src: str, traffic_key: str,
             flops: int):
    """HBM side of the roofline: algorithmic bytes per launch (Q, K, V read
    once, O and LSE written once) / launch time against the measured copy
    bandwidth, and the arithmetic intensity against the ridge point."""
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    nbytes = algorithmic_bytes(case)
    gbs = nbytes / (avg_launch_ms * 1e-3) / 1e9
    return {"achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
            "algorithmic_bytes": nbytes, "traffic": traffic_for(traffic_key),
            "flop_per_byte": round(flops / nbytes, 1),
            "ridge_flop_per_byte": round(peak * 1e12 / (hbm * 1e9), 1),
            "peak_source": "%s copy bandwidth" % peak_src}


def parallelism_note(world: int, plan) -> str:
    if plan is None:
        return "dp%d (one independent batch per GPU)" % world
    if plan["mode"] == "kv_heads":
        return ("one batch split over %d GPUs by key/value-head groups %s (contiguous head "
                "slices per GPU; no collective)" % (world, plan["kv_heads"]))
    return ("one batch split over %d GPUs by sequences, balanced by unmasked pairs %s "
            "(no collective)" % (world, plan["pairs"]))


def emit(args, rank, world, case, flops, total_ms, per_launch, e2e_ms, h2d, d2h, clk,
         metric=METRIC, cpu_fn=None, launches_per_step=1, traffic_key=None, rank_case=None):
    """One JSON line on rank 0.  ``case`` is the whole batch, ``flops`` and
    ``per_launch`` are rank 0's (its shard's, with --shard); the whole-job
    value divides the job's FLOPs per step (args.job_flops: every rank's
    batch, or the one batch that the ranks split) by the max-over-ranks time.
    h2d / d2h are whole-job bytes per step."""
    if rank == 0:
        ms = total_ms / args.steps
        job_flops = getattr(args, "job_flops", None) or world * flops
        plan = getattr(args, "plan", None)
        value = job_flops / (ms * 1e-3) / 1e12
        rcase = rank_case if rank_case is not None else case
        peaks, peak_src = load_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        avg_launch_ms = sum(per_launch) / len(per_launch)
        achieved = flops / (avg_launch_ms * 1e-3) / 1e12
        cpu = None
        if world == 1 and not args.no_cpu_baseline and cpu_fn is not None:
            cpu = cpu_fn()
        elif world == 1 and not args.no_cpu_baseline:
            tfs, nrows, fl, dt, thr = time_oracle(case, args.cpu_seconds)
            cpu = {"value": tfs, "unit": UNIT, "cores": thr, "kind": "oracle",
                   "sample": "%d seeded random (token, head) rows of the %s workload, "
                             "%.2f GFLOP of its %.2f TFLOP step, %.1f s on %d threads"
                             % (nrows, args.workload, fl / 1e9, flops / 1e12, dt, thr)}
        line = {
            "metric": metric, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "strong" if plan else "weak",
            "vs_baseline": None,
            "dtype": case.dtype, "data": "synthetic (seeded N(0,1) Q/K/V, seeded lengths)",
            "config": {
                "workload": workloads.WORKLOADS[args.workload].description,
                "name": args.workload, "batch_sequences": case.B, "total_q": case.Tq,
                "total_k": case.Tk, "max_seqlen": case.max_q, "H": case.H, "Hkv": case.Hkv,
                "D": case.D, "causal": case.causal, "flops_per_step": flops,
                "window": [case.mask.get("window_left", -1), case.mask.get("window_right", -1)],
                "seqused_k": "seqused_k" in case.mask,
                "page_size": workloads.WORKLOADS[args.workload].page_size or None,
                "sinks": "sinks" in case.mask,
                "num_splits": getattr(args, "num_splits", 1),
                "workspace_bytes": getattr(args, "workspace_bytes", 0),
                "l2": getattr(args, "l2", l2_note(rcase)),
                "parallelism": parallelism_note(world, plan),
                "job_flops_per_step": job_flops},
            "pct_of_peak": round(100.0 * achieved / peak, 2),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 3), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic_for(traffic_key or args.workload),
                         "peak_source": "%s burst bf16 (sustained %.1f -> frac %.4f)"
                                        % (peak_src, peak_sus, achieved / peak_sus)},
            "hbm": hbm_line(rcase, avg_launch_ms, peaks, peak_src, traffic_key or args.workload,
                            flops),
            "launch_ms": {"min": round(min(per_launch), 4),
                          "median": round(statistics.median(per_launch), 4),
                          "max": round(max(per_launch), 4)},
            "e2e": {"value": round(job_flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps(args),
                    "schedule": "every step copies all its inputs from pinned host memory and "
                                "reads all its results back; two device buffer sets take the "
                                "steps in turn, the copies on streams of their own overlapping "
                                "the other set's call"},
            "gpu_launches": args.steps * launches_per_step,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        if args.no_e2e:
            line["e2e"] = None
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- backward

def bwd_flops(case) -> int:
    """10 * D per unmasked (query, key, head) pair: S = QK^T and dP = dO V^T
    (recomputed), dV += P^T dO, dK += dS^T Q, dQ += dS K, 2 * D each."""
    return 10 * case.D * unmasked_pairs(case.lens_q, case.lens_k, case.H, case.causal)


def prefix_case(case, m: int):
    """The workload's first m sequences (a packed prefix) as a case of its own."""
    cq, ck = case.cu_q.tolist(), case.cu_k.tolist()
    return workloads.Case(case.q[:cq[m]], case.k[:ck[m]], case.v[:ck[m]], case.cu_q[:m + 1].clone(),
                          case.cu_k[:m + 1].clone(), case.lens_q[:m], case.lens_k[:m], case.H,
                          case.Hkv, case.D, case.causal, case.dtype, case.scale,
                          name=case.name + "[:%d]" % m, seed=case.seed)


def time_oracle_bwd(case, seconds: float, nthreads: int | None = None):
    """Times the fp64 oracle backward (as it stands) on the workload's first
    sequences, as many as fit in about ``seconds`` of CPU work (O and LSE from
    the oracle forward of the same sample, not timed).  Returns the
    cpu_baseline object."""
    import torch
    import oracle
    nthreads = nthreads or oracle.default_threads()

    def run(m):
        sub = prefix_case(case, m)
        g = torch.Generator("cpu").manual_seed(97)
        dout = torch.randn(sub.q.shape, generator=g).to(sub.q.dtype)
        o, lse = oracle.run_case(sub, nthreads=nthreads)
        t0 = time.perf_counter()
        oracle.run_case_bwd(sub, dout, o, lse, nthreads=nthreads)
        return time.perf_counter() - t0, bwd_flops(sub)

    dt, fl = run(1)
    m = 1
    rate = fl / max(dt, 1e-6)
    while m < case.B and bwd_flops(prefix_case(case, m + 1)) / rate < seconds:
        m += 1
    if m > 1:
        dt, fl = run(m)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": "backward of the workload's first %d sequences (%.2f GFLOP of its %.2f "
                      "TFLOP step), %.1f s on %d threads"
                      % (m, fl / 1e9, bwd_flops(case) / 1e12, dt, nthreads)}


def run_gpu_bwd(args, rank: int, world: int):
    """One step = one varlen_attn_bwd call (its two kernels) over the workload,
    with dO seeded and O / LSE from one forward call before the timing."""
    import torch
    import flash_attention_fwd_b200 as fa

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    case = workloads.make_workload(args.workload)
    if case.mask or workloads.WORKLOADS[args.workload].page_size:
        raise SystemExit("the backward covers the plain forward (no window, paged K/V or sinks)")
    flops = bwd_flops(case)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    cq, ck = case.cu_q.to(dev), case.cu_k.to(dev)
    fa.load_library()
    fa.device_status(clear=True)
    out, lse = fa.varlen_attn_fwd(q, k, v, cq, ck, case.max_q, case.max_k, case.causal,
                                  case.scale)
    g = torch.Generator("cpu").manual_seed(case.seed + 7)
    dout = torch.randn(case.q.shape, generator=g).to(case.q.dtype).to(dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(fa.bwd_workspace_size(case.Tq, case.H), 1), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step_on(dout, q, k, v, out, lse, cq, ck, dq, dk, dv):
        fa.varlen_attn_bwd(dout, q, k, v, out, lse, cq, ck, case.max_q, case.max_k, case.causal,
                           case.scale, dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)

    set0 = (dout, q, k, v, out, lse, cq, ck)

    def step():
        step_on(*set0, dq, dk, dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_bus_id(local))
    clocks.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    args.l2 = l2_note(case, backward=True)
    per_launch = timed_steps(step, args.steps, stream, dev,
                             input_bytes(case, backward=True) < 2 * L2_BYTES)
    if dist:
        dist.barrier()
    clk = clocks.stop()
    total_ms = sum(per_launch)
    status = fa.device_status(clear=True)
    if status != 0:
        raise RuntimeError("device status word set: %d" % status)

    e2e_ms, h2d, d2h = float("nan"), 0, 0
    if not args.no_e2e:
        host_in = [pinned(t) for t in set0]
        for h, d in zip(host_in, set0):
            h.copy_(d)
        sets = [set0, tuple(torch.empty_like(t) for t in set0)]
        outs = [(dq, dk, dv), tuple(torch.empty_like(t) for t in (dq, dk, dv))]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = sum(t.numel() * t.element_size() for t in outs[0])
        e2e_ms = pipelined_e2e(lambda b: step_on(*sets[b], *outs[b]), [list(st) for st in sets],
                               host_in, outs, [[pinned(t) for t in o] for o in outs],
                               e2e_steps(args), stream, dist)
    if dist:
        total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist, dev)
        h2d, d2h = sum_over_ranks([h2d, d2h], dist, dev)
        dist.barrier()
    emit(args, rank, world, case, flops, total_ms, per_launch, e2e_ms, h2d, d2h, clk,
         metric=METRIC_BWD, cpu_fn=lambda: time_oracle_bwd(case, args.cpu_seconds),
         launches_per_step=2, traffic_key=args.workload + ":bwd")
    if dist:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- reference arm

def run_reference_bwd(args, world, case, nthreads, budget):
    """Reference arm of the backward: the oracle backward on the workload's
    first sequences (as many as fit the per-step budget), every step."""
    import torch
    import oracle
    m = 1
    calib = time_oracle_bwd(prefix_case(case, 1), 0.0, nthreads)
    rate = calib["value"] * 1e12
    while m < case.B and bwd_flops(prefix_case(case, m + 1)) / rate < budget:
        m += 1
    sub = prefix_case(case, m)
    g = torch.Generator("cpu").manual_seed(97)
    dout = torch.randn(sub.q.shape, generator=g).to(sub.q.dtype)
    o, lse = oracle.run_case(sub, nthreads=nthreads)
    for _ in range(args.warmup):
        oracle.run_case_bwd(sub, dout, o, lse, nthreads=nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.run_case_bwd(sub, dout, o, lse, nthreads=nthreads)
    dt = (time.perf_counter() - t0) / args.steps
    fl = bwd_flops(sub)
    value = fl / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC_BWD, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) Q/K/V/dO, seeded lengths)",
        "config": {"workload": workloads.WORKLOADS[args.workload].description,
                   "name": args.workload, "pass": "bwd", "sample_sequences": m,
                   "sample_flops": fl},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": "backward of the first %d sequences per step, %.2f GFLOP"
                                   % (m, fl / 1e9)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_reference(args, rank: int, world: int):
    """The fp64 CPU oracle as it stands, on the host cores, one bounded row
    sample of the workload per step."""
    if rank != 0:
        return
    import oracle
    case = workloads.make_workload(args.workload)
    nthreads = oracle.default_threads()
    budget = max(0.5, min(30.0, args.reference_seconds / max(1, args.steps + args.warmup)))
    if args.pass_ == "bwd":
        return run_reference_bwd(args, world, case, nthreads, budget)
    rows0, fl0 = oracle_sample_rows(case, 256, seed=98)
    t0 = time.perf_counter()
    oracle.run_case_rows(case, rows0, nthreads=nthreads, **case.mask)
    rate = fl0 / max(time.perf_counter() - t0, 1e-6)
    n = int(max(64, budget * rate / max(fl0 / len(rows0), 1)))
    rows, fl = oracle_sample_rows(case, n, seed=99)
    for _ in range(args.warmup):
        oracle.run_case_rows(case, rows, nthreads=nthreads, **case.mask)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.run_case_rows(case, rows, nthreads=nthreads, **case.mask)
    dt = (time.perf_counter() - t0) / args.steps
    value = fl / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) Q/K/V, seeded lengths)",
        "config": {"workload": workloads.WORKLOADS[args.workload].description,
                   "name": args.workload, "sample_rows": len(rows), "sample_flops": fl},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": "%d seeded random (token, head) rows per step, %.2f GFLOP"
                                   % (len(rows), fl / 1e9)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="long", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd"],
                    help="time the forward (default) or the backward (dQ, dK, dV)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--shard", default="none", choices=["none", "auto", "kv_heads", "sequences"],
                    help="N > 1: split one batch over the GPUs (strong scaling) instead of one "
                         "batch per GPU (weak scaling, the default)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.pass_ == "bwd" and args.shard != "none":
        ap.error("--shard applies to the forward")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_gpu(args, rank, world)


if __name__ == "__main__":
    main()
