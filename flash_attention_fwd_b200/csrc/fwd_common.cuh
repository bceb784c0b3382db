/*
 * fwd_common.cuh — pieces shared by the attention forward kernels: launch
 * parameters, the cu_seqlens-driven work scheduler, bounded mbarrier waits,
 * packing and TMEM move helpers.
 *
 * The work decomposition follows the per-sequence loop of boostr 0.2.0,
 * src/ops/cpu/attention/varlen_attention.rs (varlen_attention_fwd): sequence
 * b owns query rows [cu_q[b], cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]);
 * here a sequence is cut into query tiles of BM rows, and each (sequence,
 * query tile, head unit) is one work item.  With the causal rule (key ki
 * hidden from query qi when qi < ki, sequence-local indices) a query tile
 * starting at row qi0 needs the keys [0, min(Lk, min(Lq, qi0 + BM))), so key
 * tiles above the diagonal are never visited.
 */
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace vattn {

constexpr int BM = 128;                             // query rows per tile = TMEM lanes
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;           // log2 units: rescale O only when max grows > 2^8
constexpr uint64_t WAIT_TIMEOUT_NS = 2000000000ull; // 2 s: far beyond any legitimate wait
constexpr unsigned STATUS_TIMEOUT = 1u;
constexpr unsigned STATUS_BAD_PAGE = 2u;  // a page-table entry outside [0, num_pages)

// Device-side status word (bit STATUS_TIMEOUT: a bounded wait gave up).
__device__ unsigned int g_device_status = 0;
// Limit of the pipeline waits (wait_bar) on this device: WAIT_TIMEOUT_NS,
// unless a test lowers it (varlen_attn_set_wait_limit) so that the waits run
// out and the kernels take their abort path.  Each CTA copies it into shared
// memory at start (AbortState).  The end-of-kernel drains keep
// WAIT_TIMEOUT_NS: they wait for work already issued.
__device__ unsigned long long g_wait_limit_ns = WAIT_TIMEOUT_NS;

// Per-CTA abort state in shared memory: the flag a role raises when one of
// its waits runs out (every other pipeline wait then gives up too), and the
// CTA's copy of the wait limit.
struct AbortState {
  unsigned long long limit_ns;
  int flag;
  __device__ void init() {
    limit_ns = g_wait_limit_ns;
    flag = 0;
  }
  __device__ bool raised() const { return *reinterpret_cast<const volatile int *>(&flag) != 0; }
  __device__ void raise() { *reinterpret_cast<volatile int *>(&flag) = 1; }
};

struct KParams {
  const int *cu_q;
  const int *cu_k;
  void *out;
  float *lse;
  int B, H, Hkv, group;  // group = H / Hkv
  int head_units;        // head units per (sequence, token range): H, H/2 (head pairs) or Hkv (packed)
  int unit_tokens;       // query tokens per work item (divides BM)
  int pack_log2;         // 0: a tile's rows are BM tokens of one head; k > 0: a tile's rows are
                         // BM >> k tokens x the 2^k query heads of one key/value head
  int total_q, total_k;
  int causal;
  float scale_log2;      // scale * log2(e)
  const int *seqused_k;  // optional [B]: keys of sequence b used = min(Lk_b, seqused_k[b])
  int win_left;          // key ki visible to query qi only if ki >= qi - win_left (-1: no bound)
  int win_right;         // ... and ki <= qi + win_right (-1: no bound); the causal rule is
                         // folded in by the host (causal => win_right = 0)
  // Paged K/V (page_table != nullptr): k and v are [num_pages * page_size, Hkv, D]
  // (i.e. [num_pages, page_size, Hkv, D]); key ki of sequence b lives in row
  // page_table[b * pt_stride + ki / page_size] * page_size + ki % page_size, and
  // sequence b has seqused_k[b] keys (cu_k is not read).
  const int *page_table;
  int pt_stride;   // entries per sequence in page_table
  int page_size;   // keys per page, a multiple of 16
  int num_pages;
  int page_chunk;  // rows per TMA box of a paged K/V tile (divides page_size and the key tile)
  const float *sinks;  // optional [H]: one extra logit per query head in the softmax normalisation
  // Key-range split (only without the causal rule and without a window): a
  // work item whose sequence has more than split_tiles key tiles of BM keys is
  // cut into P = min(ceil(nk / split_tiles), max_parts) pieces of near-equal
  // tile counts.  Piece i of row `row` (= token * H + head) writes O / l as
  // float32 to part_o[(i * part_rows + row) * D ...] and its log2-domain LSE to
  // part_lse[i * part_rows + row]; the combine kernel merges the pieces.
  int split_tiles;  // 0: no item is split
  int max_parts;
  // Replicated rows (pair kernel, GQA-packed, rep = 4; 1 otherwise): an item
  // holds at most 32 query rows; tile A carries four copies of them, one per
  // TMEM lane quarter, copy c keeps keys [32c, 32c + 32) of every key tile,
  // and each copy is a piece of its own for the combine kernel (piece index
  // part * rep + c).  Tile B is not used.
  int rep;
  // Folded causal units (single kernel, query ranges of BM tokens, Lq = Lk, no
  // window): query ranges u and nq - 1 - u of a sequence form one unit of
  // nq + 1 key tiles, handed to one CTA as two consecutive work items (the
  // second reads K/V the first just brought into L2); an odd nq leaves the
  // middle range on its own.
  int fold;
  long long part_rows;  // total_q * H
  float *part_o;
  float *part_lse;
  // out / part_o start on a 32-byte boundary (their rows then do too: a row
  // is a multiple of 128 bytes), so rows are written in 32-byte stores, one
  // whole sector each; otherwise in 16-byte stores
  int out_v8, part_v8;
};

// 16 words (32 bf16 / fp16 values) to dst: two 32-byte stores when v8 (dst
// 32-byte aligned), four 16-byte stores otherwise.
__device__ __forceinline__ void store16w(void *dst, const uint32_t (&w)[16], bool v8) {
  if (v8) {
    ptx::st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    ptx::st_global_v8(static_cast<uint32_t *>(dst) + 8, w[8], w[9], w[10], w[11], w[12], w[13],
                      w[14], w[15]);
  } else {
    uint4 *d = static_cast<uint4 *>(dst);
#pragma unroll
    for (int v4 = 0; v4 < 4; ++v4) d[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
  }
}

// Pieces of a key range of nk tiles: P pieces, the first r of base + 1 tiles
// and the other P - r of base tiles (P = 1, base = nk when it is not split).
__device__ __forceinline__ void kv_pieces(int nk, int split_tiles, int max_parts, int &P,
                                          int &base, int &r) {
  P = (split_tiles > 0 && nk > split_tiles) ? min((nk + split_tiles - 1) / split_tiles, max_parts)
                                            : 1;
  if (P < 1) P = 1;
  base = nk / P;
  r = nk - base * P;
}

// Query and key extents of sequence b, clamped into the buffers (so that an
// inconsistent sequence table can never address memory outside them): queries
// [qs, qs + lq) of the packed q, keys [ks, ks + lk) of the packed k/v (paged:
// ks = 0 and lk = the used keys, at most paged_keys).
__device__ __forceinline__ void seq_extents(const int *cu_q, const int *cu_k,
                                            const int *seqused_k, bool paged, int paged_keys,
                                            int total_q, int total_k, int b, int &qs, int &lq,
                                            int &ks, int &lk) {
  qs = __ldg(cu_q + b);
  int qe = __ldg(cu_q + b + 1);
  qs = min(max(qs, 0), total_q);
  qe = min(max(qe, qs), total_q);
  lq = qe - qs;
  if (paged) {
    ks = 0;
    lk = min(max(__ldg(seqused_k + b), 0), paged_keys);
    return;
  }
  ks = __ldg(cu_k + b);
  int ke = __ldg(cu_k + b + 1);
  ks = min(max(ks, 0), total_k);
  ke = min(max(ke, ks), total_k);
  lk = ke - ks;
  if (seqused_k) lk = min(lk, max(__ldg(seqused_k + b), 0));
}
__device__ __forceinline__ int paged_key_extent(const KParams &p) {
  return (int)min((long long)p.pt_stride * p.page_size, (long long)INT32_MAX);
}

// Sink logit of query head h in log2 units (-inf: none).
__device__ __forceinline__ float sink_log2(const KParams &p, int h) {
  return p.sinks ? __ldg(p.sinks + h) * 1.4426950408889634f : -INFINITY;
}

// Visible keys [key_lo, key_hi) of the sequence-local query qi in a sequence
// with Lk used keys (empty when key_hi <= key_lo).
__device__ __forceinline__ int key_lo(const KParams &p, int qi) {
  return p.win_left >= 0 ? max(0, qi - p.win_left) : 0;
}
__device__ __forceinline__ int key_hi(const KParams &p, int qi, int Lk) {
  return p.win_right >= 0 ? (int)min((long long)Lk, (long long)qi + p.win_right + 1) : Lk;
}

struct WorkItem {
  int b;        // sequence
  int hu;       // head unit (a head, a pair of heads 2hu, 2hu+1, or a key/value head)
  int q0;       // packed index of the item's first query token
  int q_rows;   // valid query tokens in the item (<= unit_tokens)
  int qi0;      // sequence-local index of the item's first query
  int part;     // piece of a split key range (-1: the item covers all its keys)
  int k0;       // packed index of the first key of the first visited key tile
  int kofs;     // sequence-local index of that key (a multiple of the key tile)
  int Lk;       // used keys in the sequence
  int n_kv;     // key tiles to visit
  int min_hi;   // smallest per-row visible-key end, relative to kofs
  int max_lo;   // largest per-row visible-key start, relative to kofs
};

// ---------------------------------------------------------------------------
// Work scheduler.  A work item is (sequence b, query range qt of U tokens,
// head unit hu), U = unit_tokens dividing BM.  Its cost is measured in 128-key
// tiles: with the causal rule the range needs the keys
// [0, min(Lk, min(Lq, (qt+1) * U))), i.e. min(nk, ceil((qt+1) / R)) tiles
// where nk = ceil(Lk / BM) and R = BM / U; without it, nk tiles.  Items
// are listed by cost level, highest first ("longest processing time first"),
// and within a level by sequence, query tile, head unit (the head units that
// share K/V tiles are adjacent, so they run at the same time on neighbouring
// CTAs and the K/V tiles are served from L2).  Item i goes to CTA i mod G, the
// direction reversed every round, so each CTA gets a near-equal sum of costs.
//
// With per-sequence used-key counts Lk means the used keys.  A sliding
// window changes which key tiles an item visits (the range [lo, hi) spanned
// by its rows' visible keys) but not the ordering, which stays the one above:
// the windowed cost is nearly the same for all ranges of a sequence, so the
// dealing still balances.
//
// The walk is warp-cooperative (all 32 lanes of the calling warp call
// init/next together): sequences are examined 32 at a time.  Lengths are
// clamped into the buffers' extents, so an inconsistent sequence table can
// never address memory outside them.
template <int BN>
struct Scheduler {
  const int *cu_q, *cu_k, *seqused_k;
  int B, HU, U, R, causal, total_q, total_k;
  bool paged;
  int paged_keys;  // keys addressable through one page-table row
  int cta, grid, lane;
  long long round;
  int level;              // current cost level; -1 once the list is exhausted
  long long level_base;   // index of the first item of the level
  long long level_items;  // items in the level
  int cur_b;              // cursor inside the level: first sequence not passed yet
  long long cur_units;    // (sequence, query tile) units before cur_b in this level
  int split_tiles, max_parts;
  int fold;               // KParams::fold
  bool pending;           // the second range of a folded unit is still to be handed out
  WorkItem pend;

  __device__ void extents(int b, int &qs, int &lq, int &ks, int &lk) const {
    seq_extents(cu_q, cu_k, seqused_k, paged, paged_keys, total_q, total_k, b, qs, lq, ks, lk);
  }
  // (sequence, query range[, key piece]) units of a sequence at cost level c;
  // nq ranges of U tokens, nk tiles of BM keys.  Without the causal rule a
  // split key range gives each query range P pieces, at levels base + 1 and
  // base.
  // folded: the sequence is cut into folded units (fold, causal, Lq = Lk)
  __device__ bool folded(int lq, int lk) const { return fold && causal && lq == lk && lq > 0; }
  __device__ int units_at(int nq, int nk, int c, bool fd = false) const {
    if (fd) return (c == nq + 1 ? nq / 2 : 0) + ((nq & 1) && c == (nq + 1) / 2 ? 1 : 0);
    if (!causal || nk == 0) {
      int P, base, r;
      kv_pieces(nk, split_tiles, max_parts, P, base, r);
      return nq * ((c == base ? P - r : 0) + (r > 0 && c == base + 1 ? r : 0));
    }
    if (c >= 1 && c < nk) return max(0, min(c * R, nq) - (c - 1) * R);
    if (c == nk) return max(0, nq - (nk - 1) * R);
    return 0;
  }
  __device__ int top_level(int nq, int nk, bool fd = false) const {
    if (nq == 0) return -1;
    if (fd) return nq >= 2 ? nq + 1 : 1;
    if (causal && nk > 0) return min(nk, (nq + R - 1) / R);
    int P, base, r;
    kv_pieces(nk, split_tiles, max_parts, P, base, r);
    return r > 0 ? base + 1 : base;
  }
  __device__ long long count_level(int c) const {
    long long u = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      int b = b0 + lane, v = 0;
      if (b < B) {
        int qs, lq, ks, lk;
        extents(b, qs, lq, ks, lk);
        v = units_at((lq + U - 1) / U, (lk + BM - 1) / BM, c, folded(lq, lk));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      u += v;
    }
    return u * HU;
  }

  __device__ void init(const KParams &p) {
    cu_q = p.cu_q;
    cu_k = p.cu_k;
    seqused_k = p.seqused_k;
    paged = p.page_table != nullptr;
    paged_keys = paged_key_extent(p);
    split_tiles = p.split_tiles;
    max_parts = p.max_parts;
    fold = p.fold;
    pending = false;
    B = p.B;
    HU = p.head_units;
    U = p.unit_tokens;
    R = BM / U;
    causal = p.causal;
    total_q = p.total_q;
    total_k = p.total_k;
    cta = blockIdx.x;
    grid = gridDim.x;
    lane = threadIdx.x & 31;
    round = 0;
    int top = -1;
    for (int b0 = 0; b0 < B; b0 += 32) {
      int b = b0 + lane;
      if (b < B) {
        int qs, lq, ks, lk;
        extents(b, qs, lq, ks, lk);
        top = max(top, top_level((lq + U - 1) / U, (lk + BM - 1) / BM, folded(lq, lk)));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) top = max(top, __shfl_xor_sync(0xffffffffu, top, o));
    level = top;
    level_base = 0;
    level_items = (level >= 0) ? count_level(level) : 0;
    cur_b = 0;
    cur_units = 0;
  }

  // the query range qt of a sequence whose keys are not split: its queries
  // and the key tiles spanned by their visible keys
  __device__ void fill_range(WorkItem &w, const KParams &p, int qt, int qs, int lq, int ks,
                             int lk) const {
    w.part = -1;
    w.qi0 = qt * U;
    w.q0 = qs + w.qi0;
    w.q_rows = min(U, lq - w.qi0);
    w.Lk = lk;
    const int qa = w.qi0, qb = w.qi0 + w.q_rows - 1;
    const int lo_a = key_lo(p, qa), hi_b = key_hi(p, qb, lk);
    w.kofs = (lo_a / BN) * BN;
    w.k0 = ks + w.kofs;
    w.n_kv = hi_b > lo_a ? (hi_b - w.kofs + BN - 1) / BN : 0;
    w.min_hi = key_hi(p, qa, lk) - w.kofs;
    w.max_lo = key_lo(p, qb) - w.kofs;
  }

  __device__ bool next(WorkItem &w, const KParams &p) {
    if (pending) {
      pending = false;
      w = pend;
      return true;
    }
    const long long idx = round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
    ++round;
    while (level >= 0 && idx >= level_base + level_items) {
      level_base += level_items;
      --level;
      if (level >= 0) {
        level_items = count_level(level);
        cur_b = 0;
        cur_units = 0;
      }
    }
    if (level < 0) return false;
    const long long local = idx - level_base;
    const long long unit = local / HU;
    w.hu = (int)(local % HU);
    for (;;) {
      const int b = cur_b + lane;
      int qs = 0, lq = 0, ks = 0, lk = 0, u = 0;
      if (b < B) {
        extents(b, qs, lq, ks, lk);
        u = units_at((lq + U - 1) / U, (lk + BM - 1) / BM, level, folded(lq, lk));
      }
      int incl = u;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (cur_units + total > unit) {
        const unsigned hit = __ballot_sync(0xffffffffu, cur_units + incl > unit);
        const int src = __ffs(hit) - 1;
        const int before = __shfl_sync(0xffffffffu, incl - u, src);
        const int u_b = __shfl_sync(0xffffffffu, u, src);
        qs = __shfl_sync(0xffffffffu, qs, src);
        lq = __shfl_sync(0xffffffffu, lq, src);
        ks = __shfl_sync(0xffffffffu, ks, src);
        lk = __shfl_sync(0xffffffffu, lk, src);
        cur_b += src;
        cur_units += before;
        w.b = cur_b;
        int k = (int)(unit - cur_units);
        const int nk = (lk + BM - 1) / BM;
        int qt, t0 = 0, nt = 0;
        w.part = -1;
        if (folded(lq, lk)) {
          // folded unit: ranges k and nq - 1 - k, or the middle range alone.
          // The sequence's u_b units x HU head units at this level are taken
          // unit fastest: the units in flight then cover few (sequence, head)
          // pairs, whose K/V stays in L2 while all their query ranges read it.
          const long long o = local - (long long)cur_units * HU;
          k = (int)(o % u_b);
          w.hu = (int)(o / u_b);
          const int nq = (lq + U - 1) / U;
          if (level == nq + 1 && nq >= 2) {
            qt = k;
            pend = w;
            fill_range(pend, p, nq - 1 - k, qs, lq, ks, lk);
            pending = true;
          } else {
            qt = (nq - 1) / 2;
          }
        } else if (causal && nk > 0) {
          qt = (min(level, nk) - 1) * R + k;
        } else {
          // units of the level: (piece, query range) with the range fastest, so
          // the query ranges that share a piece's K/V tiles run side by side
          int P, base, r;
          kv_pieces(nk, split_tiles, max_parts, P, base, r);
          const int nq = (lq + U - 1) / U;
          qt = k % nq;
          int i = k / nq;
          if (r > 0 && level == base + 1) {
            t0 = i * (base + 1);
            nt = base + 1;
          } else {
            i += r;
            t0 = r * (base + 1) + (i - r) * base;
            nt = base;
          }
          if (P > 1) w.part = i;
        }
        if (w.part < 0) {
          fill_range(w, p, qt, qs, lq, ks, lk);
        } else {
          w.qi0 = qt * U;
          w.q0 = qs + w.qi0;
          w.q_rows = min(U, lq - w.qi0);
          w.Lk = lk;
          // keys [t0 * BM, min((t0 + nt) * BM, lk)); every row sees all keys
          // (a split range has no window and no causal rule)
          const int kend = min((t0 + nt) * BM, lk);
          w.kofs = t0 * BM;
          w.k0 = ks + w.kofs;
          w.n_kv = (kend - w.kofs + BN - 1) / BN;
          w.min_hi = lk - w.kofs;
          w.max_lo = -w.kofs;
        }
        return true;
      }
      cur_b += 32;
      cur_units += total;
    }
  }
};

// Keys of the item's last visited key tile (of BN keys) that lie inside the
// sequence's used keys (at least 1); the tile's other rows hold whatever
// follows them in the buffer (the next sequence, unused cache slots, the rest
// of a page).
template <int BN>
__device__ __forceinline__ int last_tile_keys(const WorkItem &w) {
  return min(BN, w.Lk - (w.kofs + (w.n_kv - 1) * BN));
}

// Work items travel from the scheduling (producer) warp to the other roles
// through a small ring in shared memory.  An item with hu < 0 ends the list.
constexpr int ITEM_RING = 4;
struct ItemRing {
  WorkItem items[ITEM_RING];
  uint64_t full[ITEM_RING];
  uint64_t empty[ITEM_RING];
};

// Bounded wait; on timeout raises the CTA abort flag and the device status.
// The clock and the abort flag are looked at every 64 polls (about 2 us).
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, AbortState *abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort_flag->raised()) return false;
      if (ptx::globaltimer_ns() - t0 > abort_flag->limit_ns) {
        abort_flag->raise();
        atomicOr(&g_device_status, STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait of the end-of-kernel drains: the copies and MMAs a CTA issued
// must finish before it exits or frees TMEM, after an abort too, so this wait
// does not stop at the abort flag; it gives up only after WAIT_TIMEOUT_NS
// (status bit STATUS_TIMEOUT).  Every drain waits on work already issued,
// which always completes.
__device__ __forceinline__ bool drain_wait(uint64_t *bar, uint32_t parity) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && ptx::globaltimer_ns() - t0 > WAIT_TIMEOUT_NS) {
      atomicOr(&g_device_status, STATUS_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// Producer side of the K/V shared-memory ring: NSLOT slots of one BN-key tile
// (D / 64 swizzled 128-byte column blocks) each, slot s guarded by full[s]
// (TMA bytes landed) and empty[s] (the MMAs that read it completed).  Used by
// one warp; lane 0 issues the copies.
//
// Packed K/V: a key tile is BN consecutive rows of k/v.  Paged K/V: a key tile
// is BN / chunk boxes of `chunk` rows (chunk divides the page size and BN, so a
// box never crosses a page); lane c of the warp looks up the page of box c.
// A box past the sequence's used keys, or whose page-table entry is out of
// range, is read at a row beyond the buffer, which the TMA fills with zeros.
//
// With SPLIT > 1 a slot holds one D-wide column slice of a key tile (the
// tensor's head dim is SPLIT * D) and a tile takes SPLIT consecutive slots,
// slice 0 first.
//
// Rows past the used keys.  The last key tile of an item may run past the
// sequence's used keys (into the next sequence's rows, the unused slots of a
// KV cache, or the rest of a page).  Their scores are masked, so P is 0
// there, but 0 times a non-finite value is NaN.  So the copies of that V tile
// complete on `tail` (an mbarrier of SPLIT arrivals) instead of the slot's
// `full` barrier; once they have landed, the warp overwrites the rows past the
// used keys with zeros, fences the writes for the async proxy and then
// arrives on `full` itself, which is what the MMA warp waits for: the
// consumers see an ordinary slot.  The fix is deferred until the next item's
// first K tile is queued (so that the wait for the V tile to land overlaps
// that load, and the slot it needs is never held by the fix), and it runs
// before that item's Q tile, whose buffer frees only once the current item's
// last S products complete.
template <int BN, int D, int NSLOT, int SPLIT = 1>
struct KVProducer {
  static constexpr int DB = D / 64;
  static constexpr uint32_t KV_BYTES = BN * D * 2;
  uint8_t *sKV;
  uint64_t *full, *empty, *tail;
  AbortState *abort_flag;
  uint64_t pol;
  uint32_t slot, phase;
  uint32_t fills[NSLOT];
  int lane;
  // pending tail fix: first ring slot of the last V tile, the number of its
  // rows that hold used keys (BN: nothing to fix), tail fills so far
  uint32_t fix_slot;
  int fix_keys;
  uint32_t tails;

  __device__ void init(uint8_t *s, uint64_t *f, uint64_t *e, uint64_t *tl, AbortState *abort) {
    sKV = s;
    full = f;
    empty = e;
    tail = tl;
    tails = 0;
    abort_flag = abort;
    pol = ptx::policy_evict_last();
    slot = 0;
    phase = 0;
    for (int i = 0; i < NSLOT; ++i) fills[i] = 0;
    lane = threadIdx.x & 31;
    fix_keys = BN;
  }
  // Whole warp: once the pending last V tile has landed on `tail`, zero its
  // rows [fix_keys, BN) in every slice and complete the slices' `full`
  // barriers.  False when the wait gave up.
  __device__ bool fix_tail() {
    if (fix_keys >= BN) return true;
    // on a wait that gave up the fix stays pending, for drain_tail
    if (!__all_sync(0xffffffffu, wait_bar(tail, (tails - 1) & 1u, abort_flag))) return false;
    const int keys = fix_keys;
    fix_keys = BN;
    const int per_block = (BN - keys) * 8;  // 16-byte chunks of one column block
    uint32_t s = fix_slot;
#pragma unroll
    for (int i = 0; i < SPLIT; ++i) {
#pragma unroll
      for (int db = 0; db < DB; ++db) {
        // rows [keys, BN) of a column block are one contiguous range
        uint4 *dst = reinterpret_cast<uint4 *>(sKV + s * KV_BYTES + db * (BN * 128) + keys * 128);
        for (int c = lane; c < per_block; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (++s == NSLOT) s = 0;
    }
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      s = fix_slot;
#pragma unroll
      for (int i = 0; i < SPLIT; ++i) {
        ptx::mbar_arrive(&full[s]);
        if (++s == NSLOT) s = 0;
      }
    }
    return true;
  }
  // lane 0, end of kernel: a tail tile whose fix never ran (the CTA gave up)
  // still has copies in flight; wait for them, then complete its slots'
  // `full` barriers so that the ring drain below sees every fill done.
  __device__ void drain_tail() {
    if (fix_keys >= BN) return;
    drain_wait(tail, (tails - 1) & 1u);
    uint32_t s = fix_slot;
    for (int i = 0; i < SPLIT; ++i) {
      ptx::mbar_arrive(&full[s]);
      if (++s == NSLOT) s = 0;
    }
    fix_keys = BN;
  }
  __device__ void advance() {
    ++fills[slot];
    if (++slot == NSLOT) {
      slot = 0;
      phase ^= 1u;
    }
  }
  // lane 0: key rows [row, row + BN) of a packed k/v (columns [col0, col0 + D)
  // of the tensor; col0 a multiple of 64), completing on `bar`
  __device__ bool load_packed(const CUtensorMap *tm, int kv_h, int row, int col0 = 0,
                              uint64_t *bar = nullptr) {
    if (!wait_bar(&empty[slot], phase ^ 1u, abort_flag)) return false;
    uint8_t *dst = sKV + slot * KV_BYTES;
    if (bar == nullptr) bar = &full[slot];
    ptx::mbar_arrive_expect_tx(bar, KV_BYTES);
#pragma unroll
    for (int db = 0; db < DB; ++db)
      ptx::tma_load_3d_hint(dst + db * (BN * 128), tm, bar, col0 + db * 64, kv_h, row, pol);
    advance();
    return true;
  }
  __device__ bool tile_packed(const CUtensorMap *tm, int kv_h, int row, uint64_t *bar = nullptr) {
#pragma unroll
    for (int s = 0; s < SPLIT; ++s)
      if (!load_packed(tm, kv_h, row, s * D, bar)) return false;
    return true;
  }
  // paged: source row of box `lane` of the key tile that starts at key0
  __device__ int chunk_row(const KParams &p, const WorkItem &w, int key0) const {
    int row = p.total_k;  // beyond the buffer: zero fill
    const int ch = p.page_chunk;
    if (lane * ch < BN) {
      const int key = key0 + lane * ch;
      if (key < w.Lk) {
        const int pg = __ldg(p.page_table + (size_t)w.b * p.pt_stride + key / p.page_size);
        if (pg >= 0 && pg < p.num_pages)
          row = pg * p.page_size + key % p.page_size;
        else
          atomicOr(&g_device_status, STATUS_BAD_PAGE);
      }
    }
    return row;
  }
  // Whole warp: one paged key tile; lane c copies box c from row my_row.
  // Lane 0 waits for the slot and posts the byte count first, so the lanes'
  // copies (one warp instruction per column block) complete into a phase
  // that already expects them.
  __device__ bool load_paged(const CUtensorMap *tm, int kv_h, int my_row, int ch, int col0 = 0,
                             uint64_t *bar = nullptr) {
    bool ok = true;
    if (bar == nullptr) bar = &full[slot];
    if (lane == 0) {
      ok = wait_bar(&empty[slot], phase ^ 1u, abort_flag);
      if (ok) ptx::mbar_arrive_expect_tx(bar, KV_BYTES);
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) return false;
    if (lane * ch < BN) {
      uint8_t *dst = sKV + slot * KV_BYTES + lane * ch * 128;
#pragma unroll
      for (int db = 0; db < DB; ++db)
        ptx::tma_load_3d_hint(dst + db * (BN * 128), tm, bar, col0 + db * 64, kv_h, my_row, pol);
    }
    advance();
    return true;
  }
  __device__ bool tile_paged(const CUtensorMap *tm, int kv_h, int my_row, int ch,
                             uint64_t *bar = nullptr) {
#pragma unroll
    for (int s = 0; s < SPLIT; ++s)
      if (!load_paged(tm, kv_h, my_row, ch, s * D, bar)) return false;
    return true;
  }
  // The item's last V tile, about to be loaded: when some of its rows lie
  // past the used keys, records its ring position and returns the barrier
  // its copies complete on (`tail`); otherwise its slot's own `full`.
  __device__ uint64_t *note_tail(const WorkItem &w) {
    const int keys = last_tile_keys<BN>(w);
    if (keys >= BN) return nullptr;
    fix_keys = keys;
    fix_slot = slot;
    ++tails;
    return tail;
  }
  // Whole warp: the K/V tiles of one item in the order the MMA warp consumes
  // them (K0, K1, V0, K2, V1, K3, ..., V(n-1)), with the item's Q tile(s) after
  // K0 through load_q (called by lane 0, returns false when a wait gave up).
  // The previous item's pending tail fix runs between K0 and the Q load.
  template <class LoadQ>
  __device__ bool load_item(const KParams &p, const WorkItem &w, int kv_h, const CUtensorMap *tm_k,
                            const CUtensorMap *tm_v, LoadQ &&load_q) {
    const int n = w.n_kv;
    if (p.page_table == nullptr) {
      bool ok = true;
      if (lane == 0) ok = tile_packed(tm_k, kv_h, w.k0);
      ok = __shfl_sync(0xffffffffu, ok, 0) && fix_tail();
      if (lane == 0) {
        if (ok) ok = load_q();
        if (ok && n >= 2) ok = tile_packed(tm_k, kv_h, w.k0 + BN);
        for (int j = 0; ok && j < n; ++j) {
          ok = tile_packed(tm_v, kv_h, w.k0 + j * BN, j == n - 1 ? note_tail(w) : nullptr);
          if (ok && j + 2 < n) ok = tile_packed(tm_k, kv_h, w.k0 + (j + 2) * BN);
        }
      }
      // lane 0 issued the copies; the whole warp runs the fix
      ok = __shfl_sync(0xffffffffu, ok, 0);
      fix_keys = __shfl_sync(0xffffffffu, fix_keys, 0);
      fix_slot = __shfl_sync(0xffffffffu, fix_slot, 0);
      tails = __shfl_sync(0xffffffffu, tails, 0);
      return ok;
    }
    const int ch = p.page_chunk;
    int r0 = chunk_row(p, w, w.kofs), r1 = 0;
    bool ok = tile_paged(tm_k, kv_h, r0, ch) && fix_tail();
    if (ok) {
      bool q = true;
      if (lane == 0) q = load_q();
      ok = __shfl_sync(0xffffffffu, q, 0);
    }
    if (ok && n >= 2) {
      r1 = chunk_row(p, w, w.kofs + BN);
      ok = tile_paged(tm_k, kv_h, r1, ch);
    }
    for (int j = 0; ok && j < n; ++j) {
      // look up K(j+2) before waiting for V(j)'s slot, so that the two overlap
      const int rn = (j + 2 < n) ? chunk_row(p, w, w.kofs + (j + 2) * BN) : 0;
      ok = tile_paged(tm_v, kv_h, (j & 1) ? r1 : r0, ch, j == n - 1 ? note_tail(w) : nullptr);
      if (ok && j + 2 < n) {
        if (j & 1)
          r1 = rn;
        else
          r0 = rn;
        ok = tile_paged(tm_k, kv_h, rn, ch);
      }
    }
    return ok;
  }
  // lane 0: every copy issued has landed (before the CTA exits)
  __device__ void drain() {
    drain_tail();
    for (int i = 0; i < NSLOT; ++i)
      if (fills[i] > 0) drain_wait(&full[i], (fills[i] - 1) & 1u);
  }
};

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  }
}

template <int N>
__device__ __forceinline__ void tmem_ld_wait(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_wait<16>(uint32_t taddr, uint32_t (&r)[16]) {
  ptx::tmem_ld_x16_wait(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_wait<32>(uint32_t taddr, uint32_t (&r)[32]) {
  ptx::tmem_ld_x32_wait(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_wait<64>(uint32_t taddr, uint32_t (&r)[64]) {
  ptx::tmem_ld_x64_wait(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_wait<128>(uint32_t taddr, uint32_t (&r)[128]) {
  ptx::tmem_ld_x128_wait(taddr, r);
}

template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_st<16>(uint32_t taddr, const uint32_t (&r)[16]) {
  ptx::tmem_st_x16(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_st<32>(uint32_t taddr, const uint32_t (&r)[32]) {
  ptx::tmem_st_x32(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_st<64>(uint32_t taddr, const uint32_t (&r)[64]) {
  ptx::tmem_st_x64(taddr, r);
}

// Running-max update of one row for key tile j, mx = the tile's row max in
// log2 units (-inf when every key of the tile is hidden from the row).  m
// stays -inf until the row has seen a visible key; the first finite max then
// "rescales" O and l by exp2(-inf) = 0, which is exact because both are 0.
// s[c] = -inf for every column whose key offset c0 + c lies outside
// [lo, hi), as one select per column: the bounds differ from row to row, and
// an `if` per column made the warp take both paths of 128 branches.
template <int N>
__device__ __forceinline__ void mask_outside(float (&s)[N], int lo, int hi, int c0 = 0) {
#pragma unroll
  for (int c = 0; c < N; ++c)
    s[c] = ptx::slct_f32(s[c], -INFINITY, min(c0 + c - lo, hi - 1 - (c0 + c)));
}

__device__ __forceinline__ void update_max(int j, float mx, float &m, float &alpha, bool &need) {
  if (j == 0) {
    m = mx;
  } else if (mx > m + RESCALE_THRESHOLD) {
    alpha = ptx::ex2_approx(m - mx);
    m = mx;
    need = true;
  }
}
// Offset added to the scaled scores before exp2: -m, or 0 while m = -inf (the
// row has no visible key yet, every score is -inf and exp2 gives 0).
__device__ __forceinline__ float exp_offset(float m) { return m == -INFINITY ? 0.f : -m; }

// Epilogue of one row: O / l -> out (bf16/fp16, 16-byte stores), LSE -> lse.
// A sink logit (sink_l2 > -inf, log2 units) joins the normalisation: with
// M = max(m, sink), l' = l 2^(m-M) + 2^(sink-M) and O' = O 2^(m-M), so the
// row gets O / (l + 2^(sink-m)) and LSE = M + log2 l' without overflow.  A
// row that saw no visible key (l = 0; O is then 0 too) gets O = 0 and
// LSE = the sink, or -inf without one.  Arrives on o_free (one arrival per
// warp) as soon as O has been read.  D is the number of columns this thread
// writes (a column slice of the row when several threads share it; only one
// of them writes the LSE).
template <int D, bool BF16>
__device__ __forceinline__ void epilogue_row(uint32_t tO, float m, float l, float sink_l2,
                                             bool row_valid, uint16_t *orow_ptr, float *lse_ptr,
                                             uint64_t *o_free, int lane, bool v8,
                                             bool write_lse = true) {
  float o_scale = 1.f;
  if (sink_l2 != -INFINITY) {
    const float M = fmaxf(m, sink_l2);
    o_scale = ptx::ex2_approx(m - M);  // 0 when m = -inf
    l = l * o_scale + ptx::ex2_approx(sink_l2 - M);
    m = M;
  }
  const bool any = l > 0.f;
  const float inv_l = any ? o_scale / l : 0.f;
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t o[32];
    tmem_ld_wait<32>(tO + c0, o);
    if (c0 + 32 == D) {
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(o_free);
    }
    if (row_valid) {
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2)
        pk[c / 2] = pack2<BF16>(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
      store16w(orow_ptr + c0, pk, v8);
    }
  }
  if (row_valid && write_lse)
    *lse_ptr = any ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
}

// Epilogue of one row of a piece of a split key range: O / l as float32 and
// the piece's LSE in log2 units (m + log2 l; -inf and O = 0 when the piece has
// no visible key for the row).  Sinks are left to the combine.
template <int D>
__device__ __forceinline__ void epilogue_part(uint32_t tO, float m, float l, bool row_valid,
                                              float *part_o_row, float *part_lse, uint64_t *o_free,
                                              int lane, bool v8, bool write_lse = true) {
  const bool any = l > 0.f;
  const float inv_l = any ? 1.f / l : 0.f;
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t o[32];
    tmem_ld_wait<32>(tO + c0, o);
    if (c0 + 32 == D) {
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(o_free);
    }
    if (row_valid) {
      uint32_t w[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(__uint_as_float(o[c]) * inv_l);
      const uint32_t(&lo)[16] = *reinterpret_cast<const uint32_t(*)[16]>(&w[0]);
      const uint32_t(&hi)[16] = *reinterpret_cast<const uint32_t(*)[16]>(&w[16]);
      store16w(part_o_row + c0, lo, v8);
      store16w(part_o_row + c0 + 16, hi, v8);
    }
  }
  if (row_valid && write_lse) *part_lse = any ? m + log2f(l) : -INFINITY;
}

// A query row of an item without visible keys: O = 0, LSE = the sink logit
// (natural log units) or -inf without one.
template <int D>
__device__ __forceinline__ void empty_row(uint16_t *orow_ptr, float *lse_ptr, float sink_l2) {
  uint4 *dst = reinterpret_cast<uint4 *>(orow_ptr);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
  *lse_ptr = sink_l2 * 0.69314718055994530942f;
}

}  // namespace vattn
