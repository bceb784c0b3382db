/*
 * fwd_pair.cuh — attention forward, two query tiles per work item that share
 * every K/V tile: the same 128 query rows of the two query heads 2u and 2u+1,
 * which map to the same key/value head whenever H / Hkv is even (GQA head map
 * kv_h = h / (H / Hkv)).  Head dims 64 and 128.
 *
 * One persistent CTA per SM, 384 threads (three warpgroups):
 *   warps 0-3  softmax warpgroup A (query head 2u; thread t = row t = TMEM lane t)
 *   warps 4-7  softmax warpgroup B (query head 2u+1)
 *   warp 8     TMA producer: both Q tiles, K/V tiles through a shared-memory ring
 *   warp 9     TMEM owner and MMA issuer
 *   warps 10-11 idle
 * The kernel is compiled for REG_LAUNCH registers per thread; the third
 * warpgroup gives registers back (REG_LOW) and the softmax warpgroups take
 * them (REG_HIGH): 128 * REG_LOW + 256 * REG_HIGH == 384 * REG_LAUNCH.  The
 * host refuses to launch a build whose register count is not REG_LAUNCH.
 * TMEM: S_A, S_B (BN columns each, P aliases their first BN/2 columns), O_A,
 * O_B (D columns each).  The MMA warp alternates between the tiles:
 *   S_A(0), S_B(0), then for each key tile j:
 *     PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)
 * so softmax A of tile j runs while the tensor cores do PV_B(j-1), S_B(j),
 * and softmax B while they do PV_A(j), S_A(j+1) ("ping-pong").  Each K/V tile
 * crosses L2 -> shared memory once for both query tiles.
 *
 * Because S_T(j) is issued after PV_T(j-1) and its tcgen05.commit tracks all
 * earlier MMAs of the issuing thread, the arrival of S_T(j) implies that
 * PV_T(j-1) has completed: the softmax may rescale O_T in place without a
 * further wait.
 */
#pragma once
#include "fwd_common.cuh"

namespace vattn {
namespace pair {

constexpr int NUM_THREADS = 384;
constexpr int PRODUCER_WARP = 8;
constexpr int RING_CONSUMERS = 1 + 8;  // MMA thread + one arrival per softmax warp
constexpr int MMA_WARP = 9;
constexpr uint32_t REG_LAUNCH = 168;  // 65536 / 384 rounded down to a multiple of 8
constexpr uint32_t REG_LOW = 120;
constexpr uint32_t REG_HIGH = 192;
static_assert(128 * REG_LOW + 256 * REG_HIGH == NUM_THREADS * REG_LAUNCH, "register split");
constexpr int BN = 128;

template <int D>
struct Cfg;
template <>
struct Cfg<64> {
  static constexpr int NSLOT = 8;
};
template <>
struct Cfg<128> {
  static constexpr int NSLOT = 5;
};

struct Barriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];  // per query tile (A, B)
  uint64_t o_ready[2], o_free[2];
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
  // TMEM columns: S_t at [t*BN, (t+1)*BN), O_t at [2*BN + t*D, 2*BN + (t+1)*D)
  constexpr uint32_t O_COL0 = 2 * BN;
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
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 4);
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
      // Ring order per item: K0, V0, K1, V1, ..., K(n-1), V(n-1).
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
        for (int j = 0; ok && j < n; ++j) {
          ok = load_kv(&tm_v, kv_h, w.k0 + j * BN);
          if (ok && j + 1 < n) ok = load_kv(&tm_k, kv_h, w.k0 + (j + 1) * BN);
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
      auto issue_s = [&](int t, uint32_t kslot) {
        const uint32_t qbase = sQ_addr + t * Q_BYTES;
        const uint32_t kbase = sKV_addr + kslot * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk % 4) * 32u;
          uint64_t a = ptx::sdesc_sw128(qbase + (kk / 4) * (BM * 128) + off, 16, 1024);
          uint64_t bdesc = ptx::sdesc_sw128(kbase + (kk / 4) * (BN * 128) + off, 16, 1024);
          ptx::mma_ss(tmem + t * BN, a, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, uint32_t vslot, bool acc) {
        const uint32_t vbase = sKV_addr + vslot * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          uint64_t bdesc = ptx::sdesc_sw128(vbase + kk * (16 * 128), BN * 128, 1024);
          ptx::mma_ts(tmem + O_COL0 + t * D, tmem + t * BN + kk * 8, bdesc, IDESC_PV,
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
        uint32_t ks;
        if (!(ok = take_slot(ks))) break;
        issue_s(0, ks);
        ptx::mma_commit(&bars->s_full[0]);
        issue_s(1, ks);
        ptx::mma_commit(&bars->s_full[1]);
        ptx::mma_commit(&bars->empty[ks]);
        if (n == 1) ptx::mma_commit(&bars->q_empty);
        for (int j = 0; ok && j < n; ++j) {
          const uint32_t gj = g + j;
          uint32_t vs;
          if (!(ok = take_slot(vs))) break;
          const bool more = j + 1 < n;
          uint32_t ks_next = 0;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!(ok = wait_bar(&bars->p_full[t], gj & 1u, abort_flag))) break;
            ptx::tc_fence_after();
            if (j == 0 && items > 0) {
              if (!(ok = wait_bar(&bars->o_free[t], (items - 1) & 1u, abort_flag))) break;
              ptx::tc_fence_after();
            }
            issue_pv(t, vs, j > 0);
            if (j == n - 1) ptx::mma_commit(&bars->o_ready[t]);
            if (t == 1) ptx::mma_commit(&bars->empty[vs]);
            if (more) {
              if (t == 0 && !(ok = take_slot(ks_next))) break;
              issue_s(t, ks_next);
              ptx::mma_commit(&bars->s_full[t]);
              if (t == 1) {
                ptx::mma_commit(&bars->empty[ks_next]);
                if (j + 1 == n - 1) ptx::mma_commit(&bars->q_empty);
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
    const uint32_t tS = tmem + lane_base + t * BN;
    const uint32_t tO = tmem + lane_base + O_COL0 + t * D;
    const float sl2 = p.scale_log2;
    uint32_t rs = 0, rph = 0;
    uint32_t g = 0, items = 0;
    bool ok = true;
    auto no_wait = []() { return true; };
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
        bool got = wait_bar(&bars->s_full[t], gj & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        softmax_tile<BN, D, BF16>(tS, tO, j, sl2, (j + 1) * BN > w.min_lim, key_lim - j * BN, m,
                                  l, no_wait);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->p_full[t]);
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

}  // namespace pair
}  // namespace vattn
