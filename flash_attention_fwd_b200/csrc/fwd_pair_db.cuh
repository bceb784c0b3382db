/*
 * fwd_pair_db.cuh — attention forward, two query tiles per work item (the
 * same 128 query rows of query heads 2u and 2u+1, which share a key/value
 * head when H / Hkv is even) with 64-key tiles and a DOUBLE-BUFFERED S per
 * query tile.  Head dims 64 and 128.
 *
 * TMEM (512 columns): S_A0, S_A1, S_B0, S_B1 (64 columns each; P of a buffer
 * aliases its first 32 columns), O_A, O_B (D columns each).  The MMA warp
 * issues, after the prologue S_A(0), S_B(0), S_A(1), S_B(1), for every key
 * tile j:
 *     PV_A(j), S_A(j+2), PV_B(j), S_B(j+2)
 * S_T(j+2) goes into the buffer that held S_T(j)/P_T(j) and is issued after
 * PV_T(j) read that P.  When a softmax warpgroup finishes tile j, S_T(j+1)
 * was issued a whole tile earlier, so the softmax runs back to back instead
 * of waiting for its own PV and S MMAs; the tensor cores fill the time with
 * both tiles' MMAs.  Because S_T(j) is issued after PV_T(j-2), not PV_T(j-1),
 * an in-place rescale of O_T waits for PV_T(j-1) on a per-PV barrier (the
 * parity wait is exact: the barrier is in phase j-1 or j).
 *
 * One persistent CTA per SM, 384 threads (three warpgroups):
 *   warps 0-3  softmax warpgroup A (query head 2u; thread t = row t = TMEM lane t)
 *   warps 4-7  softmax warpgroup B (query head 2u+1)
 *   warp 8     scheduler + TMA producer (Q tiles, K/V ring)
 *   warp 9     TMEM owner and MMA issuer
 *   warps 10-11 idle
 * Registers are rebalanced with setmaxnreg as in fwd_pair.cuh.
 */
#pragma once
#include "fwd_common.cuh"

namespace vattn {
namespace pairdb {

constexpr int NUM_THREADS = 384;
constexpr int PRODUCER_WARP = 8;
constexpr int RING_CONSUMERS = 1 + 8;  // MMA thread + one arrival per softmax warp
constexpr int MMA_WARP = 9;
constexpr uint32_t REG_LAUNCH = 168;  // 65536 / 384 rounded down to a multiple of 8
constexpr uint32_t REG_LOW = 120;
constexpr uint32_t REG_HIGH = 192;
static_assert(128 * REG_LOW + 256 * REG_HIGH == NUM_THREADS * REG_LAUNCH, "register split");
constexpr int BN = 64;

template <int D>
struct Cfg;
template <>
struct Cfg<64> {
  static constexpr int NSLOT = 12;
};
template <>
struct Cfg<128> {
  static constexpr int NSLOT = 10;
};

struct Barriers {
  uint64_t full[12];
  uint64_t empty[12];
  uint64_t q_full, q_empty;
  uint64_t s_full[2][2], p_full[2][2];  // [query tile A/B][S buffer]
  uint64_t pv_done[2], o_ready[2], o_free[2];
  uint64_t drain;
  ItemRing ring;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)2 * BM * D * 2 + (size_t)Cfg<D>::NSLOT * BN * D * 2 + sizeof(Barriers) + 1024;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const KParams p) {
  constexpr int NSLOT = Cfg<D>::NSLOT;
  constexpr int DB = D / 64;
  constexpr uint32_t Q_BYTES = BM * D * 2;  // one query tile
  constexpr uint32_t KV_BYTES = BN * D * 2;
  // TMEM columns: S_t,b at [(2t+b)*BN, (2t+b+1)*BN), O_t at [4*BN + t*D, ...)
  constexpr uint32_t O_COL0 = 4 * BN;
  static_assert(O_COL0 + 2 * D <= TMEM_COLS, "TMEM budget");
  constexpr uint32_t IDESC_S = ptx::idesc_f16(BM, BN, BF16, false);
  constexpr uint32_t IDESC_PV = ptx::idesc_f16(BM, D, BF16, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;  // tile A at sQ, tile B at sQ + Q_BYTES
  uint8_t *sKV = smem + 2 * Q_BYTES;
  Barriers *bars = reinterpret_cast<Barriers *>(sKV + NSLOT * KV_BYTES);
  volatile int *abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->q_full, 1);
    ptx::mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&bars->s_full[i][b], 1);
        ptx::mbar_init(&bars->p_full[i][b], 4);
      }
      ptx::mbar_init(&bars->pv_done[i], 1);
      ptx::mbar_init(&bars->o_ready[i], 1);
      ptx::mbar_init(&bars->o_free[i], 4);
    }
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

  // Each branch below keeps its register budget to the end of the kernel; the
  // branches meet only at the named end-of-kernel barrier.
  auto end_of_kernel = [&]() {
    ptx::tc_fence_before();
    ptx::named_bar_sync(1, NUM_THREADS);
    ptx::tc_fence_after();
  };
  if (warp >= 8) {
  ptx::setmaxnreg_dec<REG_LOW>();
  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the scheduler and publishes items on the ring;
    // lane 0 issues the TMA copies.
    {
      Scheduler<BN> sched;
      sched.init(p);
      uint32_t rs = 0, rph = 0;
      uint32_t slot = 0, phase = 0, q_count = 0;
      uint32_t slot_fills[NSLOT];
      for (int s = 0; s < NSLOT; ++s) slot_fills[s] = 0;
      bool ok = true;
      const uint64_t pol_kv = ptx::policy_evict_last();
      auto load_kv = [&](const CUtensorMap *tm, int kv_h, int row) -> bool {
        if (!wait_bar(&bars->empty[slot], phase ^ 1u, abort_flag)) return false;
        uint8_t *dst = sKV + slot * KV_BYTES;
        ptx::mbar_arrive_expect_tx(&bars->full[slot], KV_BYTES);
#pragma unroll
        for (int db = 0; db < DB; ++db)
          ptx::tma_load_3d_hint(dst + db * (BN * 128), tm, &bars->full[slot], db * 64, kv_h, row,
                                pol_kv);
        ++slot_fills[slot];
        if (++slot == NSLOT) {
          slot = 0;
          phase ^= 1u;
        }
        return true;
      };
      // Ring order per item: K0, K1, V0, K2, V1, K3, ..., V(n-1) — the order
      // in which the MMA warp consumes them.
      // Loads of one item, issued by lane 0; false when a bounded wait gave up.
      auto load_item = [&](const WorkItem &w) -> bool {
        const int n = w.n_kv;
        bool ok = true;
        const int h0 = 2 * w.hu;
        const int kv_h = h0 / p.group;
        if (!load_kv(&tm_k, kv_h, w.k0)) return false;
        if (!wait_bar(&bars->q_empty, (q_count & 1u) ^ 1u, abort_flag)) return false;
        ptx::mbar_arrive_expect_tx(&bars->q_full, 2 * Q_BYTES);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int db = 0; db < DB; ++db)
            ptx::tma_load_3d(sQ + t * Q_BYTES + db * (BM * 128), &tm_q, &bars->q_full, db * 64,
                             h0 + t, w.q0);
        ++q_count;
        if (n >= 2) ok = load_kv(&tm_k, kv_h, w.k0 + BN);
        for (int j = 0; ok && j < n; ++j) {
          ok = load_kv(&tm_v, kv_h, w.k0 + j * BN);
          if (ok && j + 2 < n) ok = load_kv(&tm_k, kv_h, w.k0 + (j + 2) * BN);
        }
        return ok;
      };
      for (;;) {
        WorkItem w;
        const bool have = sched.next(w);
        if (!have) w.hu = -1;
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
        if (lane == 0 && w.n_kv > 0) ok = load_item(w);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      if (lane == 0) {
        // Drain: every copy this thread issued has landed before the CTA exits.
        for (int s = 0; s < NSLOT; ++s)
          if (slot_fills[s] > 0) wait_bar(&bars->full[s], (slot_fills[s] - 1) & 1u, abort_flag);
        if (q_count > 0) wait_bar(&bars->q_full, (q_count - 1) & 1u, abort_flag);
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t rs = 0, rph = 0;
      uint32_t slot = 0, phase = 0, g = 0, items = 0;
      bool ok = true;
      const uint32_t sQ_addr = ptx::smem_u32(sQ);
      const uint32_t sKV_addr = ptx::smem_u32(sKV);
      auto take_slot = [&](uint32_t &s_out) -> bool {
        s_out = slot;
        if (!wait_bar(&bars->full[slot], phase, abort_flag)) return false;
        ptx::tc_fence_after();
        if (++slot == NSLOT) {
          slot = 0;
          phase ^= 1u;
        }
        return true;
      };
      auto issue_s = [&](int t, uint32_t buf, uint32_t kslot) {
        const uint32_t qbase = sQ_addr + t * Q_BYTES;
        const uint32_t kbase = sKV_addr + kslot * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk % 4) * 32u;
          uint64_t a = ptx::sdesc_sw128(qbase + (kk / 4) * (BM * 128) + off, 16, 1024);
          uint64_t bdesc = ptx::sdesc_sw128(kbase + (kk / 4) * (BN * 128) + off, 16, 1024);
          ptx::mma_ss(tmem + (2 * t + buf) * BN, a, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, uint32_t buf, uint32_t vslot, bool acc) {
        const uint32_t vbase = sKV_addr + vslot * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          uint64_t bdesc = ptx::sdesc_sw128(vbase + kk * (16 * 128), BN * 128, 1024);
          ptx::mma_ts(tmem + O_COL0 + t * D, tmem + (2 * t + buf) * BN + kk * 8, bdesc, IDESC_PV,
                      (acc || kk > 0) ? 1u : 0u);
        }
      };
      while (ok) {
        if (!(ok = wait_bar(&bars->ring.full[rs], rph, abort_flag))) break;
        const WorkItem w = bars->ring.items[rs];
        ptx::mbar_arrive(&bars->ring.empty[rs]);
        if (++rs == ITEM_RING) {
          rs = 0;
          rph ^= 1u;
        }
        if (w.hu < 0) break;
        const int n = w.n_kv;
        if (n == 0) continue;
        if (!wait_bar(&bars->q_full, items & 1u, abort_flag)) break;
        ptx::tc_fence_after();
        for (int jj = 0; ok && jj < 2 && jj < n; ++jj) {
          uint32_t ks;
          if (!(ok = take_slot(ks))) break;
          const uint32_t buf = (g + jj) & 1u;
          issue_s(0, buf, ks);
          ptx::mma_commit(&bars->s_full[0][buf]);
          issue_s(1, buf, ks);
          ptx::mma_commit(&bars->s_full[1][buf]);
          ptx::mma_commit(&bars->empty[ks]);
          if (jj == n - 1) ptx::mma_commit(&bars->q_empty);
        }
        for (int j = 0; ok && j < n; ++j) {
          const uint32_t gj = g + j;
          const uint32_t buf = gj & 1u;
          uint32_t vs;
          if (!(ok = take_slot(vs))) break;
          const bool more = j + 2 < n;
          uint32_t ks_next = 0;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!(ok = wait_bar(&bars->p_full[t][buf], (gj >> 1) & 1u, abort_flag))) break;
            ptx::tc_fence_after();
            if (j == 0 && items > 0) {
              if (!(ok = wait_bar(&bars->o_free[t], (items - 1) & 1u, abort_flag))) break;
              ptx::tc_fence_after();
            }
            issue_pv(t, buf, vs, j > 0);
            ptx::mma_commit(&bars->pv_done[t]);
            if (j == n - 1) ptx::mma_commit(&bars->o_ready[t]);
            if (t == 1) ptx::mma_commit(&bars->empty[vs]);
            if (more) {
              if (t == 0 && !(ok = take_slot(ks_next))) break;
              issue_s(t, buf, ks_next);
              ptx::mma_commit(&bars->s_full[t][buf]);
              if (t == 1) {
                ptx::mma_commit(&bars->empty[ks_next]);
                if (j + 2 == n - 1) ptx::mma_commit(&bars->q_empty);
              }
            }
          }
        }
        g += n;
        ++items;
      }
      ptx::mma_commit(&bars->drain);
      wait_bar(&bars->drain, 0, abort_flag);
    }
  }
  end_of_kernel();
  if (warp == MMA_WARP) {
    __syncwarp();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
  } else {
    ptx::setmaxnreg_inc<REG_HIGH>();
    // ------------------------------------------------------------ softmax WGs
    const int t = warp / 4;              // query tile A (0) or B (1)
    const int r = threadIdx.x - t * 128; // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS0 = tmem + lane_base + 2 * t * BN;
    const uint32_t tO = tmem + lane_base + O_COL0 + t * D;
    const float sl2 = p.scale_log2;
    uint32_t rs = 0, rph = 0;
    uint32_t g = 0, items = 0;
    bool ok = true;
    while (ok) {
      bool have = wait_bar(&bars->ring.full[rs], rph, abort_flag);
      if (!__all_sync(0xffffffffu, have)) break;
      const WorkItem w = bars->ring.items[rs];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->ring.empty[rs]);
      if (++rs == ITEM_RING) {
        rs = 0;
        rph ^= 1u;
      }
      if (w.hu < 0) break;
      const int n = w.n_kv;
      const int h = 2 * w.hu + t;
      const int qi = w.qi0 + r;
      const bool row_valid = r < w.q_rows;
      const size_t orow = (size_t)(w.q0 + r) * p.H + h;
      uint16_t *orow_ptr = reinterpret_cast<uint16_t *>(p.out) + orow * D;
      if (n == 0) {
        if (row_valid) empty_row<D>(orow_ptr, p.lse + orow);
        continue;
      }
      const int key_lim = p.causal ? min(w.Lk, qi + 1) : w.Lk;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const uint32_t gj = g + j;
        const uint32_t buf = gj & 1u;
        bool got = wait_bar(&bars->s_full[t][buf], (gj >> 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // O_T must hold PV_T(gj-1) before it is rescaled in place.
        auto wait_o = [&]() { return wait_bar(&bars->pv_done[t], (gj - 1) & 1u, abort_flag); };
        if (!softmax_tile<BN, D, BF16>(tS0 + buf * BN, tO, j, sl2, (j + 1) * BN > w.min_lim,
                                       key_lim - j * BN, m, l, wait_o)) {
          ok = false;
          break;
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->p_full[t][buf]);
      }
      if (!ok) break;
      g += n;
      bool got = wait_bar(&bars->o_ready[t], items & 1u, abort_flag);
      ++items;
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      epilogue_row<D, BF16>(tO, m, l, row_valid, orow_ptr, p.lse + orow, &bars->o_free[t], lane);
    }
    end_of_kernel();
  }
}

}  // namespace pairdb
}  // namespace vattn
