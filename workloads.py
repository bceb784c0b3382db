"""Seeded synthetic inputs for the varlen attention forward.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  It is the one module that both the oracle side (tests,
CPU baseline) and the CUDA side (tests, bench) use, so both see identical
inputs.

Workloads (sequence lengths, head counts, head dim, dtype, mask) follow the
five benchmark configurations of the varlen attention forward:

  tiny      3 packed sequences {17, 64, 1}, H=Hkv=4, D=64, bf16, causal
  gqa       8 sequences, q_len=k_len uniform-int [128, 2048], H=32, Hkv=8,
            D=128, bf16, causal
  long      16 sequences, log-uniform lengths in [64, 16384] rescaled to a
            total of exactly 65536 tokens, H=64, Hkv=8, D=128, bf16, causal
  shortq    32 sequences, q_len uniform-int [1, 64], k_len uniform-int
            [512, 8192], H=32, Hkv=4, D=128, bf16, non-causal
  wide      4 sequences of 4096, H=Hkv=16, D=256, fp16, Q/K ~ N(0, 3^2),
            V ~ N(0, 1), causal

and, beyond them, variants for the window / used-key / paged / sink forms
and one long-KV decode batch (8 single-query sequences, k_len uniform-int
[16384, 32768], H=32, Hkv=8: fewer work items than SMs, the case for the
key-range split).

Length recipe: numpy ``default_rng(seed)`` (PCG64).  Tensor recipe:
``torch.Generator('cpu').manual_seed(seed)``, fp32 ``randn`` drawn in the
order Q [Tq,H,D], K [Tk,Hkv,D], V [Tk,Hkv,D], multiplied by sigma, then cast
to the storage dtype (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    H: int
    Hkv: int
    D: int
    dtype: str
    causal: bool
    sigma_q: float = 1.0
    sigma_k: float = 1.0
    sigma_v: float = 1.0
    description: str = ""
    window_left: int = -1   # sliding window (negative = unbounded)
    window_right: int = -1
    seqused: bool = False   # draw a per-sequence used-key count
    page_size: int = 0      # > 0: K/V held in a page cache of this many keys per page
    sinks: bool = False     # draw one attention-sink logit per query head


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 4, 64, "bf16", True,
                     description="3 packed sequences {17,64,1}, H=Hkv=4, D=64, bf16, causal"),
    "gqa": Workload("gqa", 2, 32, 8, 128, "bf16", True,
                    description="GQA prefill: 8 sequences in [128,2048], H=32, Hkv=8, D=128, bf16, causal"),
    "long": Workload("long", 3, 64, 8, 128, "bf16", True,
                     description="long ragged prefill: 16 log-uniform sequences totalling 65536 tokens, "
                                 "H=64, Hkv=8, D=128, bf16, causal"),
    "shortq": Workload("shortq", 4, 32, 4, 128, "bf16", False,
                       description="short-query/long-KV: 32 sequences q in [1,64], k in [512,8192], "
                                   "H=32, Hkv=4, D=128, bf16, non-causal"),
    "wide": Workload("wide", 5, 16, 16, 256, "fp16", True, sigma_q=3.0, sigma_k=3.0, sigma_v=1.0,
                     description="wide-head MHA: 4x4096, H=Hkv=16, D=256, fp16, Q/K sigma 3, causal"),
    # Sliding window and used-key counts (the window_size_left/right and
    # seqused_k arguments of PyTorch pull request #176015's varlen forward)
    # on the shapes above.
    "long_swa": Workload("long_swa", 3, 64, 8, 128, "bf16", True, window_left=4095,
                         description="long ragged prefill lengths with a causal sliding window of "
                                     "4096 keys (left 4095), H=64, Hkv=8, D=128, bf16"),
    "shortq_used": Workload("shortq_used", 4, 32, 4, 128, "bf16", False, seqused=True,
                            description="short-query/long-KV lengths with per-sequence used-key "
                                        "counts seqused_k in [Lk/2, Lk], H=32, Hkv=4, D=128, "
                                        "bf16, non-causal"),
    "shortq_paged": Workload("shortq_paged", 4, 32, 4, 128, "bf16", False, page_size=16,
                             description="short-query/long-KV lengths with K/V in a page cache of "
                                         "16-key pages in seeded random order, H=32, Hkv=4, "
                                         "D=128, bf16, non-causal"),
    "gqa_sinks": Workload("gqa_sinks", 2, 32, 8, 128, "bf16", True, sinks=True,
                          description="GQA prefill lengths with one attention-sink logit per "
                                      "query head (uniform in [-2, 4]), H=32, Hkv=8, D=128, bf16, "
                                      "causal"),
    # Long-KV decode: one query token per sequence against long ragged key
    # ranges; 64 work items (one per sequence and KV head) for 148 SMs.
    "decode": Workload("decode", 6, 32, 8, 128, "bf16", False,
                       description="long-KV decode: 8 sequences of 1 query token, k_len "
                                   "uniform-int [16384, 32768], H=32, Hkv=8, D=128, bf16, "
                                   "non-causal"),
    # Profiling case only (not a benchmark configuration): the long ragged
    # prefill lengths with a quarter of its heads, so that a many-pass profiler
    # capture stays small while its inputs still exceed the L2 cache.
    "long_h16": Workload("long_h16", 3, 16, 2, 128, "bf16", True,
                         description="profiling case: long ragged prefill lengths, H=16, Hkv=2, "
                                     "D=128, bf16, causal"),
}


def _long_lengths(seed: int, n: int = 16, total: int = 65536,
                  lo: int = 64, hi: int = 16384) -> List[int]:
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), n)
    raw = np.exp(u)
    raw = raw * (total / raw.sum())
    base = np.maximum(1, np.floor(raw)).astype(np.int64)
    remainder = total - int(base.sum())
    frac = raw - np.floor(raw)
    # remainder goes to the largest fractional parts; ties go to the lower index
    order = sorted(range(n), key=lambda i: (-frac[i], i))
    for i in order[:remainder]:
        base[i] += 1
    return [int(x) for x in base]


def seqlens(name: str):
    """Per-sequence (q_lens, k_lens) of a named workload."""
    w = WORKLOADS[name]
    if name == "tiny":
        q = [17, 64, 1]
        return q, list(q)
    if name in ("gqa", "gqa_sinks"):
        rng = np.random.default_rng(w.seed)
        q = [int(x) for x in rng.integers(128, 2049, 8)]
        return q, list(q)
    if name in ("long", "long_h16", "long_swa"):
        q = _long_lengths(w.seed)
        return q, list(q)
    if name in ("shortq", "shortq_used", "shortq_paged"):
        rng = np.random.default_rng(w.seed)
        q = [int(x) for x in rng.integers(1, 65, 32)]
        k = [int(x) for x in rng.integers(512, 8193, 32)]
        return q, k
    if name == "wide":
        q = [4096] * 4
        return q, list(q)
    if name == "decode":
        rng = np.random.default_rng(w.seed)
        k = [int(x) for x in rng.integers(16384, 32769, 8)]
        return [1] * 8, k
    raise KeyError(name)


def seqused_k(name: str) -> Optional[List[int]]:
    """Per-sequence used-key counts of a named workload (None if it has none):
    drawn uniformly in [Lk // 2, Lk] by the length generator's stream, after
    the lengths."""
    w = WORKLOADS[name]
    if not w.seqused:
        return None
    if name != "shortq_used":
        raise KeyError(name)
    rng = np.random.default_rng(w.seed)
    rng.integers(1, 65, 32)
    k = rng.integers(512, 8193, 32)
    return [int(x) for x in rng.integers(k // 2, k + 1)]


def mask_of(name: str) -> dict:
    """Window / used-key arguments of a named workload, in the keyword form
    the oracle takes (empty for the plain forward)."""
    w = WORKLOADS[name]
    m = {}
    if w.window_left >= 0:
        m["window_left"] = w.window_left
    if w.window_right >= 0:
        m["window_right"] = w.window_right
    used = seqused_k(name)
    if used is not None:
        m["seqused_k"] = used
    if w.sinks:
        # float32 values, so that the oracle and the kernels see the same logits
        g = np.random.default_rng(w.seed + 1000)
        m["sinks"] = [float(x) for x in g.uniform(-2.0, 4.0, w.H).astype(np.float32)]
    return m


def cu_seqlens(lens: Sequence[int]) -> torch.Tensor:
    """Exclusive prefix sums [0, l0, l0+l1, ...] as int32."""
    out = [0]
    for x in lens:
        out.append(out[-1] + int(x))
    return torch.tensor(out, dtype=torch.int32)


@dataclass
class Case:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    cu_q: torch.Tensor
    cu_k: torch.Tensor
    lens_q: List[int]
    lens_k: List[int]
    H: int
    Hkv: int
    D: int
    causal: bool
    dtype: str
    scale: float
    name: str = "custom"
    seed: int = 0
    mask: dict = field(default_factory=dict)  # window_left / window_right / seqused_k

    @property
    def B(self) -> int:
        return len(self.lens_q)

    @property
    def max_q(self) -> int:
        return max(self.lens_q) if self.lens_q else 0

    @property
    def max_k(self) -> int:
        return max(self.lens_k) if self.lens_k else 0

    @property
    def Tq(self) -> int:
        return int(self.cu_q[-1])

    @property
    def Tk(self) -> int:
        return int(self.cu_k[-1])


def make_case(lens_q: Sequence[int], lens_k: Optional[Sequence[int]], H: int, Hkv: int, D: int,
              dtype: str = "bf16", causal: bool = True, seed: int = 0,
              sigma_q: float = 1.0, sigma_k: float = 1.0, sigma_v: float = 1.0,
              scale: Optional[float] = None, name: str = "custom") -> Case:
    """Seeded random packed inputs for arbitrary lengths and head shapes."""
    lens_q = [int(x) for x in lens_q]
    lens_k = [int(x) for x in (lens_k if lens_k is not None else lens_q)]
    assert len(lens_q) == len(lens_k)
    Tq, Tk = sum(lens_q), sum(lens_k)
    g = torch.Generator("cpu").manual_seed(seed)
    tdt = DTYPES[dtype]
    q = (torch.randn((Tq, H, D), generator=g, dtype=torch.float32) * sigma_q).to(tdt)
    k = (torch.randn((Tk, Hkv, D), generator=g, dtype=torch.float32) * sigma_k).to(tdt)
    v = (torch.randn((Tk, Hkv, D), generator=g, dtype=torch.float32) * sigma_v).to(tdt)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return Case(q, k, v, cu_seqlens(lens_q), cu_seqlens(lens_k), lens_q, lens_k,
                H, Hkv, D, causal, dtype, float(scale), name=name, seed=seed)


def make_workload(name: str) -> Case:
    """Full-size inputs of a named workload (CPU tensors)."""
    w = WORKLOADS[name]
    lq, lk = seqlens(name)
    case = make_case(lq, lk, w.H, w.Hkv, w.D, w.dtype, w.causal, w.seed,
                     w.sigma_q, w.sigma_k, w.sigma_v, name=name)
    case.mask = mask_of(name)
    return case


def sample_rows(case: Case, n: int, seed: int = 1234) -> np.ndarray:
    """A seeded sample of (token, head) output rows that always includes the
    first and last row of every sequence (ragged edges) plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    cu = case.cu_q.tolist()
    for b in range(case.B):
        if cu[b + 1] > cu[b]:
            for tok in (cu[b], cu[b + 1] - 1, min(cu[b] + 127, cu[b + 1] - 1),
                        min(cu[b] + 128, cu[b + 1] - 1)):
                rows.add((tok, int(rng.integers(0, case.H))))
    if case.Tq > 0:
        toks = rng.integers(0, case.Tq, n)
        hs = rng.integers(0, case.H, n)
        rows.update(zip(toks.tolist(), hs.tolist()))
    arr = np.array(sorted(rows), dtype=np.int64).reshape(-1, 2)
    return arr


def stratified_rows(case: Case, seed: int = 4321, tile: int = 128,
                    per_tile: int = 1) -> np.ndarray:
    """Seeded (token, head) rows of every (sequence, query tile of `tile`
    rows, head): with per_tile = 1 one row, the tile's first, its last or a
    random one, chosen at random; with per_tile > 1 the first and the last
    row and per_tile - 2 random rows.  Plus the last query row of every
    (sequence, head), whose visible keys reach the sequence's last key tile.
    Duplicates are dropped.  Sorted by (head, token), so that rows sharing a
    key/value head and a sequence are adjacent."""
    rng = np.random.default_rng(seed)
    cu = case.cu_q.tolist()
    H = case.H
    toks, heads = [], []
    for b in range(case.B):
        q0, L = cu[b], cu[b + 1] - cu[b]
        if L <= 0:
            continue
        starts = np.arange(0, L, tile)
        ends = np.minimum(starts + tile, L)
        n_t = len(starts)
        for i in range(per_tile):
            kind = rng.integers(0, 3, (n_t, H)) if per_tile == 1 else np.full((n_t, H), min(i, 2))
            rnd = starts[:, None] + (rng.random((n_t, H)) * (ends - starts)[:, None]).astype(
                np.int64)
            pick = np.where(kind == 0, starts[:, None],
                            np.where(kind == 1, (ends - 1)[:, None], rnd))
            toks.append((q0 + pick).reshape(-1))
            heads.append(np.tile(np.arange(H), n_t))
        toks.append(np.full(H, q0 + L - 1))
        heads.append(np.arange(H))
    if not toks:
        return np.zeros((0, 2), dtype=np.int64)
    rows = np.unique(np.stack([np.concatenate(heads), np.concatenate(toks)], axis=1), axis=0)
    return np.ascontiguousarray(rows[:, ::-1]).astype(np.int64)


# ----------------------------------------------------------------------------- paged K/V

@dataclass
class PagedKV:
    k_cache: torch.Tensor      # [num_pages, page_size, Hkv, D]
    v_cache: torch.Tensor
    page_table: torch.Tensor   # int32 [B, pages_per_seq], -1 past each sequence's pages
    seqused_k: List[int]       # keys of each sequence
    page_size: int


def to_paged(case: Case, page_size: int, seed: int = 0, spare_pages: int = 3,
             fill: float = 7.0, table_pad: int = 1) -> PagedKV:
    """Scatters the packed keys/values of ``case`` into a page cache: each
    sequence's keys fill ceil(Lk / page_size) pages taken in a seeded random
    order from a pool with ``spare_pages`` unused pages; key ki of sequence b
    goes to row ki % page_size of page page_table[b, ki // page_size].  Rows
    that hold no key (the tail of a sequence's last page, the spare pages) get
    the finite value ``fill``; table entries past a sequence's pages are -1
    (``table_pad`` extra columns of them)."""
    rng = np.random.default_rng(seed)
    need = [-(-lk // page_size) for lk in case.lens_k]
    num_pages = sum(need) + spare_pages
    order = rng.permutation(num_pages)
    width = max(need + [0]) + table_pad
    table = torch.full((case.B, max(width, 1)), -1, dtype=torch.int32)
    shape = (num_pages, page_size, case.Hkv, case.D)
    kc = torch.full(shape, fill, dtype=case.k.dtype)
    vc = torch.full(shape, fill, dtype=case.v.dtype)
    cu = case.cu_k.tolist()
    nxt = 0
    for b in range(case.B):
        for j in range(need[b]):
            pg = int(order[nxt])
            nxt += 1
            table[b, j] = pg
            lo = cu[b] + j * page_size
            hi = min(cu[b + 1], lo + page_size)
            kc[pg, :hi - lo] = case.k[lo:hi]
            vc[pg, :hi - lo] = case.v[lo:hi]
    return PagedKV(kc, vc, table, list(case.lens_k), page_size)


# ----------------------------------------------------------------------------- shards

def shard_case(case: Case, plan: dict, rank: int) -> Case:
    """The part of ``case`` that rank ``rank`` computes under ``plan`` (the
    dict ``flash_attention_fwd_b200.plan_shards`` returns), laid out as that
    rank would hold it: with the key/value-head split, contiguous head slices
    [T, heads_r, D] of q, k, v (all sequences); with the sequence split, the
    rank's sequences packed in their original order (all heads).  The mask
    arguments (window, seqused_k, sinks) follow."""
    G = case.H // case.Hkv
    mask = dict(case.mask)
    if plan["mode"] == "kv_heads":
        lo, hi = plan["kv_heads"][rank]
        q = case.q[:, lo * G:hi * G].contiguous()
        k = case.k[:, lo:hi].contiguous()
        v = case.v[:, lo:hi].contiguous()
        if "sinks" in mask:
            mask["sinks"] = list(mask["sinks"][lo * G:hi * G])
        sub = Case(q, k, v, case.cu_q.clone(), case.cu_k.clone(), list(case.lens_q),
                   list(case.lens_k), (hi - lo) * G, hi - lo, case.D, case.causal, case.dtype,
                   case.scale, name="%s[kv heads %d:%d]" % (case.name, lo, hi), seed=case.seed)
        sub.mask = mask
        return sub
    mine = [b for b, r in enumerate(plan["seq_rank"]) if r == rank]
    cq, ck = case.cu_q.tolist(), case.cu_k.tolist()
    q = torch.cat([case.q[cq[b]:cq[b + 1]] for b in mine]) if mine else case.q[:0]
    k = torch.cat([case.k[ck[b]:ck[b + 1]] for b in mine]) if mine else case.k[:0]
    v = torch.cat([case.v[ck[b]:ck[b + 1]] for b in mine]) if mine else case.v[:0]
    lq = [case.lens_q[b] for b in mine]
    lk = [case.lens_k[b] for b in mine]
    if "seqused_k" in mask:
        mask["seqused_k"] = [mask["seqused_k"][b] for b in mine]
    sub = Case(q.contiguous(), k.contiguous(), v.contiguous(), cu_seqlens(lq), cu_seqlens(lk),
               lq, lk, case.H, case.Hkv, case.D, case.causal, case.dtype, case.scale,
               name="%s[%d sequences]" % (case.name, len(mine)), seed=case.seed)
    sub.mask = mask
    return sub


def shard_rows(case: Case, plan: dict, rank: int):
    """(token indices, query heads) of the full output that rank ``rank``'s
    shard output covers, in the shard's own row and head order."""
    G = case.H // case.Hkv
    if plan["mode"] == "kv_heads":
        lo, hi = plan["kv_heads"][rank]
        return np.arange(case.Tq), np.arange(lo * G, hi * G)
    cq = case.cu_q.tolist()
    mine = [b for b, r in enumerate(plan["seq_rank"]) if r == rank]
    toks = [np.arange(cq[b], cq[b + 1]) for b in mine]
    return (np.concatenate(toks) if toks else np.zeros(0, dtype=np.int64)), np.arange(case.H)


def unshard(case: Case, plan: dict, parts) -> tuple:
    """Places the ranks' shard outputs ``parts`` (per rank (out [T_r, H_r, D],
    lse [T_r, H_r]) NumPy arrays) back into full [Tq, H, D] / [Tq, H] arrays;
    also returns how many ranks wrote each (token, head) row."""
    out = np.zeros((case.Tq, case.H, case.D), dtype=np.float64)
    lse = np.zeros((case.Tq, case.H), dtype=np.float64)
    count = np.zeros((case.Tq, case.H), dtype=np.int64)
    for r, (o, l) in enumerate(parts):
        toks, heads = shard_rows(case, plan, r)
        out[np.ix_(toks, heads)] = o
        lse[np.ix_(toks, heads)] = l
        count[np.ix_(toks, heads)] += 1
    return out, lse, count
