/*
 * bwd_dkdv.cuh — backward, dK/dV pass: one 128-key tile of one key/value
 * head per work item; the item streams every query tile (BQ = 64 queries)
 * of each of the head's H / Hkv query heads that sees the tile:
 *
 *   S^T  = K Q^T,  dP^T = V dO^T          tcgen05 (keys on the TMEM lanes)
 *   P^T  = exp2(S^T scale log2e - LSE log2e),  dS^T = P^T (dP^T - delta)
 *                                          one thread per key row, written as
 *                                          bf16/fp16 MMA operands in shared memory
 *   dV  += P^T dO,  dK += dS^T Q           tcgen05, accumulated in TMEM
 *
 * and at the end dV -> dv, dK * scale -> dk.  This is the key side of the
 * page's backward loop (see bwd_common.cuh); dK and dV of a key/value head sum
 * over its query heads inside one item, so no accumulation crosses CTAs.
 * delta comes from the dQ pass (workspace), LSE from the forward.
 *
 * One persistent CTA per SM, 192 threads: warps 0-3 one key row per thread,
 * warp 4 scheduler + TMA producer, warp 5 TMEM owner + MMA issuer.  TMEM:
 * dV (D) | dK (D) | S^T[2] (BQ) | dP^T[2] (BQ).  Shared memory: K and V
 * tiles of the item, NST stages of (Q, dO) query tiles, and two buffers each
 * of P^T and dS^T.
 */
#pragma once
#include "bwd_common.cuh"

namespace vattn {
namespace bwd_dkdv {

constexpr int NUM_THREADS = 192;
constexpr int PRODUCER_WARP = 4;
constexpr int MMA_WARP = 5;
constexpr int RING_CONSUMERS = 1 + 4;
constexpr int BK = 128;  // keys per item (TMEM lanes)
constexpr int BQ = 64;   // queries per step
constexpr int NST = 3;   // (Q, dO) stages

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
};

struct KeyRing {
  KeyItem items[ITEM_RING];
  uint64_t full[ITEM_RING];
  uint64_t empty[ITEM_RING];
};

// Items are (key tile kt, sequence b, key/value head), listed by kt, then b,
// then head, and dealt to CTA i mod G with the direction reversed every round.
// With the causal rule the first key tiles see the most queries, so the list
// runs roughly from the largest item to the smallest.  The walk is
// warp-cooperative over 32 sequences at a time, like the forward scheduler.
struct KeyScheduler {
  const int *cu_q, *cu_k;
  int B, Hkv, group, causal, total_q, total_k;
  int cta, grid, lane;
  long long round;
  int level;  // current key tile index; max_kt + 1 once exhausted
  int max_kt;
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
  __device__ long long count_level(int kt) const {
    long long u = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      int v = 0;
      if (b < B) {
        int qs, lq, ks, lk;
        extents(b, qs, lq, ks, lk);
        v = (lk + BK - 1) / BK > kt ? 1 : 0;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      u += v;
    }
    return u * Hkv;
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
    int top = -1;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      if (b < B) {
        int qs, lq, ks, lk;
        extents(b, qs, lq, ks, lk);
        top = max(top, (lk + BK - 1) / BK - 1);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) top = max(top, __shfl_xor_sync(0xffffffffu, top, o));
    max_kt = top;
    level = 0;
    level_base = 0;
    level_items = (max_kt >= 0) ? count_level(0) : 0;
    cur_b = 0;
    cur_units = 0;
  }
  __device__ bool next(KeyItem &w) {
    const long long idx = round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
    ++round;
    while (level <= max_kt && idx >= level_base + level_items) {
      level_base += level_items;
      ++level;
      if (level <= max_kt) {
        level_items = count_level(level);
        cur_b = 0;
        cur_units = 0;
      }
    }
    if (level > max_kt) return false;
    const long long local = idx - level_base;
    const long long unit = local / Hkv;
    w.kvh = (int)(local % Hkv);
    for (;;) {
      const int b = cur_b + lane;
      int qs = 0, lq = 0, ks = 0, lk = 0, u = 0;
      if (b < B) {
        extents(b, qs, lq, ks, lk);
        u = (lk + BK - 1) / BK > level ? 1 : 0;
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
        w.b = cur_b;
        w.kt = level;
        w.k0 = ks + level * BK;
        w.Lk = lk;
        w.Lq = lq;
        w.q0 = qs;
        // causal (sequence-local, top-left): key kk is seen by the queries qi >= kk
        w.qt0 = causal ? (level * BK) / BQ : 0;
        w.nqt = max(0, (lq + BQ - 1) / BQ - w.qt0);
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
  uint64_t st_full[NST], st_empty[NST];
  uint64_t s_full[2];    // S^T and dP^T of a step in TMEM buffer
  uint64_t pd_full[2];   // P^T and dS^T written (one arrival per row warp)
  uint64_t pd_free[2];   // the MMAs that read them completed
  uint64_t acc_ready, acc_free;
  uint64_t lsd_full[2];  // a step's LSE / delta values written (one arrival per row warp)
  uint64_t drain;
  KeyRing ring;
  alignas(16) float lsd[2][2][BQ];  // per step parity: LSE * log2e and delta of the step's queries
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)2 * BK * D * 2 + (size_t)NST * 2 * BQ * D * 2 + (size_t)4 * BK * BQ * 2 +
         sizeof(Barriers) + 1024;
}

// Writes one 64-value row (8 x 16 bytes) of a K-major operand tile with the
// 128-byte swizzle: row r, 16-byte chunk c at chunk position c ^ (r & 7).
__device__ __forceinline__ void store_sw128_row(uint8_t *tile, int r, const uint32_t (&v)[32]) {
  uint8_t *row = tile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4 *>(row + ((c ^ (r & 7)) << 4)) =
        make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const BwdParams bp) {
  constexpr int DB = D / 64;
  constexpr uint32_t KV_BYTES = BK * D * 2;
  constexpr uint32_t QS_BYTES = BQ * D * 2;
  constexpr uint32_t PT_BYTES = BK * BQ * 2;
  constexpr uint32_t DV_COL = 0, DK_COL = D;
  constexpr uint32_t ST_COL = 2 * D, DPT_COL = 2 * D + 2 * BQ;
  static_assert(DPT_COL + 2 * BQ <= TMEM_COLS, "TMEM budget");
  constexpr uint32_t IDESC_ST = ptx::idesc_f16(BK, BQ, BF16, false);
  constexpr uint32_t IDESC_ACC = ptx::idesc_f16(BK, D, BF16, true);
  const KParams &p = bp.kp;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = smem;
  uint8_t *sV = sK + KV_BYTES;
  uint8_t *sQs = sV + KV_BYTES;               // stage s: Q at sQs + s * 2 * QS_BYTES, dO after it
  uint8_t *sPT = sQs + NST * 2 * QS_BYTES;    // P^T[2]
  uint8_t *sDST = sPT + 2 * PT_BYTES;         // dS^T[2]
  Barriers *bars = reinterpret_cast<Barriers *>(sDST + 2 * PT_BYTES);
  volatile int *abort_flag = &bars->abort_flag;

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
      ptx::mbar_init(&bars->pd_free[i], 1);
    }
    ptx::mbar_init(&bars->acc_ready, 1);
    ptx::mbar_init(&bars->acc_free, 4);
    ptx::mbar_init(&bars->lsd_full[0], 4);
    ptx::mbar_init(&bars->lsd_full[1], 4);
    ptx::mbar_init(&bars->drain, 1);
    for (int i = 0; i < ITEM_RING; ++i) {
      ptx::mbar_init(&bars->ring.full[i], 1);
      ptx::mbar_init(&bars->ring.empty[i], RING_CONSUMERS);
    }
    bars->abort_flag = 0;
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
    KeyScheduler sched;
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
      if (kv_count > 0) wait_bar(&bars->kv_full, (kv_count - 1) & 1u, abort_flag);
      for (uint32_t k = (gs > NST ? gs - NST : 0); k < gs; ++k)
        wait_bar(&bars->st_full[k % NST], (k / NST) & 1u, abort_flag);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t rs = 0, rph = 0, g = 0, items = 0, kv_items = 0;
      bool ok = true;
      const uint32_t sK_addr = ptx::smem_u32(sK);
      const uint32_t sV_addr = ptx::smem_u32(sV);
      const uint32_t sQs_addr = ptx::smem_u32(sQs);
      const uint32_t sPT_addr = ptx::smem_u32(sPT);
      const uint32_t sDST_addr = ptx::smem_u32(sDST);
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
      // dV += P^T dO, dK += dS^T Q for global step gs (operands in shared memory)
      auto issue_acc = [&](uint32_t gs, bool acc) {
        const uint32_t st = gs % NST;
        const uint32_t qa = sQs_addr + st * 2 * QS_BYTES;
        const uint32_t buf = gs & 1u;
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          uint64_t apt = ptx::sdesc_sw128(sPT_addr + buf * PT_BYTES + kk * 32u, 16, 1024);
          uint64_t adst = ptx::sdesc_sw128(sDST_addr + buf * PT_BYTES + kk * 32u, 16, 1024);
          uint64_t bdo = ptx::sdesc_sw128(qa + QS_BYTES + kk * (16 * 128), BQ * 128, 1024);
          uint64_t bq = ptx::sdesc_sw128(qa + kk * (16 * 128), BQ * 128, 1024);
          const uint32_t a = (acc || kk > 0) ? 1u : 0u;
          ptx::mma_ss(tmem + DV_COL, apt, bdo, IDESC_ACC, a);
          ptx::mma_ss(tmem + DK_COL, adst, bq, IDESC_ACC, a);
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
          issue_acc(gs, s > 0);
          ptx::mma_commit(&bars->pd_free[buf]);
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
      wait_bar(&bars->drain, 0, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ key rows
    const int r = threadIdx.x;  // key row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tST0 = tmem + lane_base + ST_COL;
    const uint32_t tDPT0 = tmem + lane_base + DPT_COL;
    const float sl2 = p.scale_log2;
    uint32_t rs = 0, rph = 0, g = 0, items = 0;
    bool ok = true;
    // LSE (log2 units) or delta of query c of step s: thread t < BQ loads LSE
    // of query t, thread BQ + t delta of query t
    auto load_lsd = [&](const KeyItem &w, int s) -> float {
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
      const size_t drow = ((size_t)(w.k0 + r) * p.Hkv + w.kvh) * D;
      if (n == 0) {
        if (key_valid) {
          zero_row<D>(bp.dk + drow);
          zero_row<D>(bp.dv + drow);
        }
        continue;
      }
      float pre = load_lsd(w, 0);
      for (int s = 0; ok && s < n; ++s) {
        const uint32_t gs = g + s;
        const uint32_t buf = gs & 1u;
        // Exchange of the step's LSE / delta values among the row warps.  The
        // buffer of parity buf is written again two steps later, only after
        // every warp has arrived for the step in between, i.e. finished this one.
        bars->lsd[buf][r / BQ][r & (BQ - 1)] = pre;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->lsd_full[buf]);
        if (s + 1 < n) pre = load_lsd(w, s + 1);
        bool got = wait_bar(&bars->lsd_full[buf], (gs >> 1) & 1u, abort_flag) &&
                   wait_bar(&bars->s_full[buf], (gs >> 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        uint32_t sv[BQ], dpv[BQ];
        tmem_ld_wait<BQ>(tST0 + buf * BQ, sv);
        tmem_ld_wait<BQ>(tDPT0 + buf * BQ, dpv);
        // queries of this step that see key kk: qi < Lq (lse = +inf otherwise)
        // and, with the causal rule, qi >= kk
        const int qbase = (w.qt0 + s % w.nqt) * BQ;
        const int cmin = p.causal ? kk - qbase : 0;  // first visible column
        const float *lse2 = bars->lsd[buf][0];
        const float *dl = bars->lsd[buf][1];
        uint32_t ppk[BQ / 2], dpk[BQ / 2];
#pragma unroll
        for (int c = 0; c < BQ; c += 2) {
          float pr[2], ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x = __uint_as_float(sv[c + e]) * sl2 - lse2[c + e];
            pr[e] = (key_valid && c + e >= cmin) ? ptx::ex2_approx(x) : 0.f;
            ds[e] = pr[e] * (__uint_as_float(dpv[c + e]) - dl[c + e]);
          }
          ppk[c / 2] = pack2<BF16>(pr[0], pr[1]);
          dpk[c / 2] = pack2<BF16>(ds[0], ds[1]);
        }
        // P^T / dS^T buffer free once the MMAs of step gs - 2 completed
        got = wait_bar(&bars->pd_free[buf], ((gs >> 1) & 1u) ^ 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        store_sw128_row(sPT + buf * PT_BYTES, r, ppk);
        store_sw128_row(sDST + buf * PT_BYTES, r, dpk);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->pd_full[buf]);
      }
      if (!ok) break;
      g += n;
      bool got = wait_bar(&bars->acc_ready, items & 1u, abort_flag);
      ++items;
      if (!__all_sync(0xffffffffu, got)) break;
      ptx::tc_fence_after();
      store_tmem_row<D, BF16>(tmem + lane_base + DV_COL, 1.f, key_valid, bp.dv + drow);
      store_tmem_row<D, BF16>(tmem + lane_base + DK_COL, bp.scale, key_valid, bp.dk + drow);
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
