/*
 * bwd_dkdv.cuh — backward, dK/dV pass: one 128-key tile of one key/value
 * head per work item (at head dim 256: one column half of its dK / dV, see
 * below); the item streams every query tile (BQ = 64 queries, 32 at D = 256)
 * of each of the head's H / Hkv query heads that sees the tile:
 *
 *   S^T  = K Q^T,  dP^T = V dO^T          tcgen05 (keys on the TMEM lanes)
 *   P^T  = exp2(S^T scale log2e - LSE log2e),  dS^T = P^T (dP^T - delta)
 *                                          one thread per key row, written back
 *                                          as bf16/fp16 over the first columns
 *                                          of S^T and dP^T in TMEM
 *   dV  += P^T dO,  dK += dS^T Q           tcgen05, A operand from TMEM,
 *                                          accumulated in TMEM
 *
 * and at the end dV -> dv, dK * scale -> dk.  This is the key side of the
 * page's backward loop (see bwd_common.cuh); dK and dV of a key/value head sum
 * over its query heads inside one item, so no accumulation crosses CTAs.
 * delta comes from the dQ pass (workspace), LSE from the forward.
 *
 * One persistent CTA per SM, 320 threads: two warpgroups of row threads
 * (warps 0-3 and 4-7, one key row per thread each) that take the steps in
 * turn — even global steps to the first, odd to the second, matching the
 * double-buffered S^T / dP^T in TMEM and P^T / dS^T in shared memory — so one
 * computes while the tensor cores serve the other; warp 8 scheduler + TMA
 * producer, warp 9 TMEM owner + MMA issuer.  TMEM:
 * dV (DO) | dK (DO) | S^T[2] (BQ) | dP^T[2] (BQ).  Shared memory: K and V
 * tiles of the item and NST stages of (Q, dO) query tiles; a stage is held
 * from its load until the step's dV / dK products complete, so the depth is
 * what hides the load latency.
 *
 * Head dim 256: dK and dV of a 128-key tile would take all 512 TMEM columns,
 * so an item computes one column half of them (DO = 128 output columns; the
 * two halves of a key tile are two items, side by side in the schedule so
 * that they share the K / V tiles in L2).  S^T and dP^T still contract over
 * all 256 columns, so each half recomputes them.  K and V take 128 KB of
 * shared memory, which leaves three stages of 32 queries.
 */
#pragma once
#include "bwd_common.cuh"

namespace vattn {
namespace bwd_dkdv {

constexpr int NUM_THREADS = 320;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int RING_CONSUMERS = 1 + 8;
constexpr int BK = 128;  // keys per item (TMEM lanes)
// Queries per step BQ, (Q, dO) stages NST and output column halves NH per
// head dim.
template <int D>
struct Cfg {
  static constexpr int BQ = 64, NST = 5, NH = 1;
};
template <>
struct Cfg<256> {
  static constexpr int BQ = 32, NST = 3, NH = 2;
};
constexpr int MAX_STAGES = 5;
constexpr int MAX_BQ = 64;

struct KeyItem {
  int b;       // sequence; < 0 ends the list
  int kvh;     // key/value head
  int kt;      // key tile in the sequence
  int k0;      // packed index of the tile's first key
  int Lk, Lq;  // keys / queries of the sequence
  int q0;      // packed index of the sequence's first query
  int qt0;     // first query tile (BQ queries) that sees the key tile
  int nqt;     // query tiles per query head
  int nsteps;  // (query head, query tile) steps = (H / Hkv) * nqt
  int half;    // column half of dK / dV (0 when NH = 1)
};

struct KeyRing {
  KeyItem items[ITEM_RING];
  uint64_t full[ITEM_RING];
  uint64_t empty[ITEM_RING];
};

// Items are (sequence b, key tile kt, key/value head[, column half]); an
// item's cost is its number of query tiles per query head,
// nqt = ceil(Lq / BQ) - R kt with the causal rule (R = BK / BQ: key tile kt is
// first seen by query tile R kt) and ceil(Lq / BQ) without it.  Items are
// listed by cost level, highest first ("longest processing time first", as
// in the forward scheduler), then by sequence, head and half, and dealt to
// CTA i mod G with the direction reversed every round.  The walk is
// warp-cooperative over 32 sequences at a time.
template <int BQ, int NH>
struct KeyScheduler {
  static constexpr int R = BK / BQ;
  const int *cu_q, *cu_k;
  int B, Hkv, group, causal, total_q, total_k;
  int cta, grid, lane;
  long long round;
  int level;  // current cost level; -1 once the list is exhausted
  long long level_base, level_items;
  int cur_b;
  long long cur_units;

  __device__ void extents(int b, int &qs, int &lq, int &ks, int &lk) const {
    qs = __ldg(cu_q + b);
    int qe = __ldg(cu_q + b + 1);
    ks = __ldg(cu_k + b);
    int ke = __ldg(cu_k + b + 1);
    qs = min(max(qs, 0), total_q);
    qe = min(max(qe, qs), total_q);
    ks = min(max(ks, 0), total_k);
    ke = min(max(ke, ks), total_k);
    lq = qe - qs;
    lk = ke - ks;
  }
  // key tiles of a sequence (nq query tiles, nk key tiles) at cost level c
  __device__ int units_at(int nq, int nk, int c) const {
    if (!causal) return (c == nq) ? nk : 0;
    if (c == 0) return max(0, nk - (nq + R - 1) / R);
    const int d = nq - c;
    return (d >= 0 && d % R == 0 && d / R < nk) ? 1 : 0;
  }
  // key tile of the k-th unit of a sequence at cost level c
  __device__ int tile_of(int nq, int c, int k) const {
    if (!causal) return k;
    if (c == 0) return (nq + R - 1) / R + k;
    return (nq - c) / R;
  }
  __device__ long long count_level(int c) const {
    long long u = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      int v = 0;
      if (b < B) {
        int qs, lq, ks, lk;
        extents(b, qs, lq, ks, lk);
        v = units_at((lq + BQ - 1) / BQ, (lk + BK - 1) / BK, c);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      u += v;
    }
    return u * Hkv * NH;
  }
  __device__ void init(const KParams &p) {
    cu_q = p.cu_q;
    cu_k = p.cu_k;
    B = p.B;
    Hkv = p.Hkv;
    group = p.group;
    causal = p.causal;
    total_q = p.total_q;
    total_k = p.total_k;
    cta = blockIdx.x;
    grid = gridDim.x;
    lane = threadIdx.x & 31;
    round = 0;
    // the top level: the largest query-tile count of a sequence with keys
    int top = -1;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      if (b < B) {
        int qs, lq, ks, lk;
        extents(b, qs, lq, ks, lk);
        if (lk > 0) top = max(top, (lq + BQ - 1) / BQ);
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
  __device__ bool next(KeyItem &w) {
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
    const long long unit = local / (Hkv * NH);
    w.kvh = (int)((local / NH) % Hkv);
    w.half = (int)(local % NH);
    for (;;) {
      const int b = cur_b + lane;
      int qs = 0, lq = 0, ks = 0, lk = 0, u = 0;
      if (b < B) {
        extents(b, qs, lq, ks, lk);
        u = units_at((lq + BQ - 1) / BQ, (lk + BK - 1) / BK, level);
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
        qs = __shfl_sync(0xffffffffu, qs, src);
        lq = __shfl_sync(0xffffffffu, lq, src);
        ks = __shfl_sync(0xffffffffu, ks, src);
        lk = __shfl_sync(0xffffffffu, lk, src);
        cur_b += src;
        cur_units += before;
        const int nq = (lq + BQ - 1) / BQ;
        const int kt = tile_of(nq, level, (int)(unit - cur_units));
        w.b = cur_b;
        w.kt = kt;
        w.k0 = ks + kt * BK;
        w.Lk = lk;
        w.Lq = lq;
        w.q0 = qs;
        // causal (sequence-local, top-left): key kk is seen by the queries qi >= kk
        w.qt0 = causal ? R * kt : 0;
        w.nqt = max(0, nq - w.qt0);
        w.nsteps = group * w.nqt;
        return true;
      }
      cur_b += 32;
      cur_units += total;
    }
  }
};

struct Barriers {
  uint64_t kv_full, kv_empty;
  uint64_t st_full[MAX_STAGES], st_empty[MAX_STAGES];
  uint64_t s_full[2];    // S^T and dP^T of a step in TMEM buffer
  uint64_t pd_full[2];   // P^T and dS^T written to TMEM (one arrival per row warp)
  uint64_t acc_ready, acc_free;
  uint64_t lsd_full[2];  // [warpgroup]: a step's LSE / delta values written (one arrival per warp)
  uint64_t drain;
  KeyRing ring;
  alignas(16) float lsd[2][2][MAX_BQ];  // [warpgroup]: LSE * log2e and delta of the step's queries
  uint32_t tmem_base;
  AbortState abort;
};

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)2 * BK * D * 2 + (size_t)Cfg<D>::NST * 2 * Cfg<D>::BQ * D * 2 +
         sizeof(Barriers) + 1024;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const BwdParams bp) {
  constexpr int BQ = Cfg<D>::BQ;
  constexpr int NST = Cfg<D>::NST;
  constexpr int NH = Cfg<D>::NH;
  constexpr int DO = D / NH;  // dK / dV columns of an item
  static_assert(NST <= MAX_STAGES && BQ <= MAX_BQ && BQ % 32 == 0, "stage layout");
  constexpr int DB = D / 64;
  constexpr uint32_t KV_BYTES = BK * D * 2;
  constexpr uint32_t QS_BYTES = BQ * D * 2;
  constexpr uint32_t DV_COL = 0, DK_COL = DO;
  constexpr uint32_t ST_COL = 2 * DO, DPT_COL = 2 * DO + 2 * BQ;
  static_assert(DPT_COL + 2 * BQ <= TMEM_COLS, "TMEM budget");
  constexpr uint32_t IDESC_ST = ptx::idesc_f16(BK, BQ, BF16, false);
  constexpr uint32_t IDESC_ACC = ptx::idesc_f16(BK, DO, BF16, true);
  const KParams &p = bp.kp;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = smem;
  uint8_t *sV = sK + KV_BYTES;
  uint8_t *sQs = sV + KV_BYTES;  // stage s: Q at sQs + s * 2 * QS_BYTES, dO after it
  Barriers *bars = reinterpret_cast<Barriers *>(sQs + NST * 2 * QS_BYTES);
  AbortState *abort_flag = &bars->abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->kv_full, 1);
    ptx::mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < NST; ++s) {
      ptx::mbar_init(&bars->st_full[s], 1);
      ptx::mbar_init(&bars->st_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->pd_full[i], 4);
    }
    ptx::mbar_init(&bars->acc_ready, 1);
    ptx::mbar_init(&bars->acc_free, 8);
    ptx::mbar_init(&bars->lsd_full[0], 4);
    ptx::mbar_init(&bars->lsd_full[1], 4);
    ptx::mbar_init(&bars->drain, 1);
    for (int i = 0; i < ITEM_RING; ++i) {
      ptx::mbar_init(&bars->ring.full[i], 1);
      ptx::mbar_init(&bars->ring.empty[i], RING_CONSUMERS);
    }
    bars->abort.init();
    ptx::mbar_init_fence();
  }
  if (warp == PRODUCER_WARP && lane == 0) {
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_do);
    ptx::tma_prefetch_desc(&tm_k);
    ptx::tma_prefetch_desc(&tm_v);
  }
  if (warp == MMA_WARP) {
    ptx::tmem_alloc(&bars->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    KeyScheduler<BQ, NH> sched;
    sched.init(p);
    uint32_t rs = 0, rph = 0, kv_count = 0, gs = 0;
    bool ok = true;
    for (;;) {
      KeyItem w;
      const bool have = sched.next(w);
      if (!have) w.b = -1;
      if (lane == 0) {
        ok = wait_bar(&bars->ring.empty[rs], rph ^ 1u, abort_flag);
        if (ok) {
          bars->ring.items[rs] = w;
          ptx::mbar_arrive(&bars->ring.full[rs]);
        }
      }
      if (++rs == ITEM_RING) {
        rs = 0;
        rph ^= 1u;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!have || !ok) break;
      if (lane == 0 && w.nsteps > 0) {
        ok = wait_bar(&bars->kv_empty, (kv_count & 1u) ^ 1u, abort_flag);
        if (ok) {
          ptx::mbar_arrive_expect_tx(&bars->kv_full, 2 * KV_BYTES);
#pragma unroll
          for (int db = 0; db < DB; ++db) {
            ptx::tma_load_3d(sK + db * (BK * 128), &tm_k, &bars->kv_full, db * 64, w.kvh, w.k0);
            ptx::tma_load_3d(sV + db * (BK * 128), &tm_v, &bars->kv_full, db * 64, w.kvh, w.k0);
          }
          ++kv_count;
        }
        for (int s = 0; ok && s < w.nsteps; ++s, ++gs) {
          const int h = w.kvh * p.group + s / w.nqt;
          const int qrow = w.q0 + (w.qt0 + s % w.nqt) * BQ;
          const uint32_t st = gs % NST;
          if (!(ok = wait_bar(&bars->st_empty[st], ((gs / NST) & 1u) ^ 1u, abort_flag))) break;
          uint8_t *dq_ = sQs + st * 2 * QS_BYTES;
          ptx::mbar_arrive_expect_tx(&bars->st_full[st], 2 * QS_BYTES);
#pragma unroll
          for (int db = 0; db < DB; ++db) {
            ptx::tma_load_3d(dq_ + db * (BQ * 128), &tm_q, &bars->st_full[st], db * 64, h, qrow);
            ptx::tma_load_3d(dq_ + QS_BYTES + db * (BQ * 128), &tm_do, &bars->st_full[st],
                             db * 64, h, qrow);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      gs = __shfl_sync(0xffffffffu, gs, 0);
      if (!ok) break;
    }
    if (lane == 0) {
      // Drain: every copy issued has landed before the CTA exits.
      if (kv_count > 0) drain_wait(&bars->kv_full, (kv_count - 1) & 1u);
      for (uint32_t k = (gs > NST ? gs - NST : 0); k < gs; ++k)
        drain_wait(&bars->st_full[k % NST], (k / NST) & 1u);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t rs = 0, rph = 0, g = 0, items = 0, kv_items = 0;
      bool ok = true;
      const uint32_t sK_addr = ptx::smem_u32(sK);
      const uint32_t sV_addr = ptx::smem_u32(sV);
      const uint32_t sQs_addr = ptx::smem_u32(sQs);
      // S^T and dP^T of global step gs into TMEM buffer gs & 1
      auto issue_st = [&](uint32_t gs) -> bool {
        const uint32_t st = gs % NST;
        if (!wait_bar(&bars->st_full[st], (gs / NST) & 1u, abort_flag)) return false;
        ptx::tc_fence_after();
        const uint32_t qa = sQs_addr + st * 2 * QS_BYTES;
        const uint32_t buf = gs & 1u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (BK * 128) + (kk % 4) * 32u;
          const uint32_t boff = (kk / 4) * (BQ * 128) + (kk % 4) * 32u;
          uint64_t bq = ptx::sdesc_sw128(qa + boff, 16, 1024);
          uint64_t bdo = ptx::sdesc_sw128(qa + QS_BYTES + boff, 16, 1024);
          ptx::mma_ss(tmem + ST_COL + buf * BQ, ptx::sdesc_sw128(sK_addr + off, 16, 1024), bq,
                      IDESC_ST, kk > 0 ? 1u : 0u);
          ptx::mma_ss(tmem + DPT_COL + buf * BQ, ptx::sdesc_sw128(sV_addr + off, 16, 1024), bdo,
                      IDESC_ST, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(&bars->s_full[buf]);
        return true;
      };
      // dV += P^T dO, dK += dS^T Q for global step gs: P^T / dS^T from TMEM
      // (bf16/fp16 pairs over the first BQ / 2 columns of S^T / dP^T), dO and
      // Q MN-major from the stage (columns [half * DO, (half + 1) * DO): the
      // column blocks from half * DO / 64 on), in steps of 16 queries
      auto issue_acc = [&](uint32_t gs, bool acc, int half) {
        const uint32_t st = gs % NST;
        const uint32_t qa = sQs_addr + st * 2 * QS_BYTES + half * (DO / 64) * (BQ * 128);
        const uint32_t buf = gs & 1u;
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          uint64_t bdo = ptx::sdesc_sw128(qa + QS_BYTES + kk * (16 * 128), BQ * 128, 1024);
          uint64_t bq = ptx::sdesc_sw128(qa + kk * (16 * 128), BQ * 128, 1024);
          const uint32_t a = (acc || kk > 0) ? 1u : 0u;
          ptx::mma_ts(tmem + DV_COL, tmem + ST_COL + buf * BQ + kk * 8, bdo, IDESC_ACC, a);
          ptx::mma_ts(tmem + DK_COL, tmem + DPT_COL + buf * BQ + kk * 8, bq, IDESC_ACC, a);
        }
      };
      while (ok) {
        if (!(ok = wait_bar(&bars->ring.full[rs], rph, abort_flag))) break;
        const KeyItem w = bars->ring.items[rs];
        ptx::mbar_arrive(&bars->ring.empty[rs]);
        if (++rs == ITEM_RING) {
          rs = 0;
          rph ^= 1u;
        }
        if (w.b < 0) break;
        const int n = w.nsteps;
        if (n == 0) continue;
        if (!(ok = wait_bar(&bars->kv_full, kv_items & 1u, abort_flag))) break;
        ++kv_items;
        ptx::tc_fence_after();
        for (int ss = 0; ok && ss < 2 && ss < n; ++ss) ok = issue_st(g + ss);
        for (int s = 0; ok && s < n; ++s) {
          const uint32_t gs = g + s;
          const uint32_t buf = gs & 1u;
          if (!(ok = wait_bar(&bars->pd_full[buf], (gs >> 1) & 1u, abort_flag))) break;
          ptx::tc_fence_after();
          if (s == 0 && items > 0) {
            if (!(ok = wait_bar(&bars->acc_free, (items - 1) & 1u, abort_flag))) break;
            ptx::tc_fence_after();
          }
          issue_acc(gs, s > 0, w.half);
          ptx::mma_commit(&bars->st_empty[gs % NST]);
          if (s == n - 1) {
            ptx::mma_commit(&bars->acc_ready);
            ptx::mma_commit(&bars->kv_empty);
          }
          if (s + 2 < n) ok = issue_st(gs + 2);
        }
        g += n;
        ++items;
      }
      ptx::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ key rows
    const int t = warp / 4;             // warpgroup: takes the global steps gs with gs & 1 == t
    const int r = threadIdx.x - 128 * t;  // key row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tST = tmem + lane_base + ST_COL + t * BQ;
    const uint32_t tDPT = tmem + lane_base + DPT_COL + t * BQ;
    const float sl2 = p.scale_log2;
    uint32_t rs = 0, rph = 0, g = 0, items = 0;
    bool ok = true;
    // LSE (log2 units) or delta of query c of step s: thread r < BQ loads LSE
    // of query r, thread BQ + c delta of query c
    auto load_lsd = [&](const KeyItem &w, int s) -> float {
      if (r >= 2 * BQ) return 0.f;  // no value to publish
      const int c = r & (BQ - 1);
      const int h = w.kvh * p.group + s / w.nqt;
      const int qi = (w.qt0 + s % w.nqt) * BQ + c;
      const bool valid = qi < w.Lq;
      const size_t row = (size_t)(w.q0 + qi) * p.H + h;
      if (r < BQ) return valid ? __ldg(bp.lse + row) * LOG2E : INFINITY;
      return valid ? bp.delta[row] : 0.f;
    };
    while (ok) {
      bool have = wait_bar(&bars->ring.full[rs], rph, abort_flag);
      if (!__all_sync(0xffffffffu, have)) break;
      const KeyItem w = bars->ring.items[rs];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->ring.empty[rs]);
      if (++rs == ITEM_RING) {
        rs = 0;
        rph ^= 1u;
      }
      if (w.b < 0) break;
      const int n = w.nsteps;
      const int kk = w.kt * BK + r;  // sequence-local key
      const bool key_valid = kk < w.Lk;
      const size_t drow = ((size_t)(w.k0 + r) * p.Hkv + w.kvh) * D + w.half * DO;
      // warpgroup 0 writes dV, warpgroup 1 dK (the item's column half)
      uint16_t *out_row = (t == 0 ? bp.dv : bp.dk) + drow;
      if (n == 0) {
        if (key_valid) zero_row<DO>(out_row);
        continue;
      }
      const int s0 = (int)((t - g) & 1u);  // this warpgroup's first step of the item
      float pre = s0 < n ? load_lsd(w, s0) : 0.f;
      for (int s = s0; ok && s < n; s += 2) {
        const uint32_t gs = g + s;
        bool got = wait_bar(&bars->s_full[t], (gs >> 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // Exchange of the step's LSE / delta values among the warpgroup's
        // warps.  S^T(gs) arriving means the MMA warp saw all four warps'
        // P^T / dS^T of this warpgroup's previous step, so every warp has
        // finished reading the previous values and the buffer can be reused.
        // (S^T(gs) also overwrote the previous step's P^T in TMEM only after
        // the dV / dK products that read it: the tensor core runs in order.)
        if (r < 2 * BQ) bars->lsd[t][r / BQ][r & (BQ - 1)] = pre;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->lsd_full[t]);
        if (s + 2 < n) pre = load_lsd(w, s + 2);
        got = wait_bar(&bars->lsd_full[t], (gs >> 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        // queries of this step that see key kk: qi < Lq (lse = +inf otherwise)
        // and, with the causal rule, qi >= kk
        const int qbase = (w.qt0 + s % w.nqt) * BQ;
        const int cmin = p.causal ? kk - qbase : 0;  // first visible column
        const float *lse2 = bars->lsd[t][0];
        const float *dl = bars->lsd[t][1];
#pragma unroll
        for (int piece = 0; piece < BQ / 32; ++piece) {
          uint32_t sv[32], dpv[32];
          tmem_ld_wait<32>(tST + piece * 32, sv);
          tmem_ld_wait<32>(tDPT + piece * 32, dpv);
          uint32_t ppk[16], dpk[16];
#pragma unroll
          for (int c2 = 0; c2 < 32; c2 += 2) {
            float pr[2], ds[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = piece * 32 + c2 + e;
              const float x = __uint_as_float(sv[c2 + e]) * sl2 - lse2[c];
              pr[e] = (key_valid && c >= cmin) ? ptx::ex2_approx(x) : 0.f;
              ds[e] = pr[e] * (__uint_as_float(dpv[c2 + e]) - dl[c]);
            }
            ppk[c2 / 2] = pack2<BF16>(pr[0], pr[1]);
            dpk[c2 / 2] = pack2<BF16>(ds[0], ds[1]);
          }
          // columns [16 piece, 16 piece + 16): S^T / dP^T columns already read
          tmem_st<16>(tST + piece * 16, ppk);
          tmem_st<16>(tDPT + piece * 16, dpk);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->pd_full[t]);
      }
      if (!ok) break;
      g += n;
      bool got = wait_bar(&bars->acc_ready, items & 1u, abort_flag);
      ++items;
      if (!__all_sync(0xffffffffu, got)) break;
      ptx::tc_fence_after();
      store_tmem_row<DO, BF16>(tmem + lane_base + (t == 0 ? DV_COL : DK_COL),
                               t == 0 ? 1.f : bp.scale, key_valid, out_row, bp.v8 != 0);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->acc_free);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == MMA_WARP) {
    __syncwarp();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace bwd_dkdv
}  // namespace vattn
