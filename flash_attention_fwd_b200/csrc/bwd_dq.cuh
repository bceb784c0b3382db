/*
 * bwd_dq.cuh — backward, dQ pass: one 128-row query tile (one query head) per
 * work item, streaming the sequence's visible key tiles of BN keys (96 at
 * head dims 64 and 128, 32 at 256):
 *
 *   S(j)  = Q K(j)^T                      tcgen05, into TMEM
 *   dP(j) = dO V(j)^T                     tcgen05, into TMEM
 *   P     = exp2(S scale log2e - LSE log2e)          one thread per query row
 *   dS    = P (dP - delta)  -> bf16/fp16 over S's first columns in TMEM
 *   dQ   += dS K(j)                       tcgen05, A = dS from TMEM, B = K MN-major
 *
 * and at the end dQ * scale -> dq.  delta = <dO, O> of each row is computed
 * here (before the first key tile) and also written to the workspace for the
 * dK/dV pass.  This is the query side of the page's backward loop (see
 * bwd_common.cuh); the work items and their order are the forward's.
 *
 * One persistent CTA per SM, 320 threads: two warpgroups of row threads
 * (warps 0-3 and 4-7, one query row per thread each) that take the key tiles
 * in turn — even global tiles to the first, odd to the second, matching the
 * double-buffered S / dP in TMEM — so one computes while the tensor cores
 * serve the other; warp 8 scheduler + TMA producer, warp 9 TMEM owner + MMA
 * issuer.  TMEM:
 * S[2] | dP[2] (BN columns each, double-buffered across key tiles) | dQ (D),
 * 4 * 96 + 128 = 512 columns at D = 128, 4 * 32 + 256 = 384 at D = 256.
 * (The S and dP products take about as long per instruction at N = 96 as at
 * N = 64, so the wider tile does half again as much work per instruction;
 * N = 128 would not fit.  At D = 256 shared memory, not TMEM, sets the
 * 32-key tile.)  The row
 * threads read S and dP in 32-column pieces.  The K/V ring holds K(j) and
 * V(j) in turn; V(j) is released after dP(j), K(j) after dQ(j).
 */
#pragma once
#include "bwd_common.cuh"

namespace vattn {
namespace bwd_dq {

constexpr int NUM_THREADS = 320;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int RING_CONSUMERS = 1 + 8;
// Key tile BN and K/V ring depth NSLOT per head dim.  At D = 256 the query
// and dO tiles take 128 KB of shared memory and dQ 256 TMEM columns, which
// leaves room for double-buffered S / dP of 32 keys and six 16 KB slots (the
// ring must hold K and V of two tiles ahead: the prologue computes S / dP of
// two tiles before the first dQ product releases a K tile).
template <int D>
struct Cfg {
  static constexpr int BN = 96, NSLOT = 6;
};
template <>
struct Cfg<256> {
  static constexpr int BN = 32, NSLOT = 6;
};
constexpr int MAX_SLOTS = 6;

struct Barriers {
  uint64_t full[MAX_SLOTS];
  uint64_t empty[MAX_SLOTS];
  uint64_t q_full, q_empty;  // Q and dO tiles of the item
  uint64_t s_full[2];        // S(j) and dP(j) in TMEM buffer j & 1
  uint64_t ds_full[2];       // dS(j) written (one arrival per row warp)
  uint64_t dq_ready, dq_free;
  uint64_t drain;
  ItemRing ring;
  uint32_t tmem_base;
  AbortState abort;
};

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)2 * BM * D * 2 + (size_t)Cfg<D>::NSLOT * Cfg<D>::BN * D * 2 + sizeof(Barriers) +
         1024;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const BwdParams bp) {
  constexpr int BN = Cfg<D>::BN;
  constexpr int NSLOT = Cfg<D>::NSLOT;
  static_assert(NSLOT <= MAX_SLOTS && NSLOT >= 4, "K/V ring depth");
  constexpr int DB = D / 64;
  constexpr uint32_t Q_BYTES = BM * D * 2;
  constexpr uint32_t KV_BYTES = BN * D * 2;
  constexpr uint32_t DP_COL = 2 * BN;
  constexpr uint32_t DQ_COL = 4 * BN;
  static_assert(DQ_COL + D <= TMEM_COLS, "TMEM budget");
  constexpr uint32_t IDESC_S = ptx::idesc_f16(BM, BN, BF16, false);
  constexpr uint32_t IDESC_DQ = ptx::idesc_f16(BM, D, BF16, true);
  const KParams &p = bp.kp;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sDO = smem + Q_BYTES;
  uint8_t *sKV = smem + 2 * Q_BYTES;
  Barriers *bars = reinterpret_cast<Barriers *>(sKV + NSLOT * KV_BYTES);
  AbortState *abort_flag = &bars->abort;

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
      ptx::mbar_init(&bars->ds_full[i], 4);
    }
    ptx::mbar_init(&bars->dq_ready, 1);
    ptx::mbar_init(&bars->dq_free, 8);
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
    Scheduler<BN> sched;
    sched.init(p);
    uint32_t rs = 0, rph = 0, q_count = 0;
    bool ok = true;
    KVProducer<BN, D, NSLOT> kv;
    kv.init(sKV, bars->full, bars->empty, nullptr, abort_flag);
    for (;;) {
      WorkItem w;
      const bool have = sched.next(w, p);
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
      if (lane == 0 && w.n_kv > 0) {
        // ring order: K0, Q+dO, V0, K1, V1, K2, V2, ...
        const int kv_h = w.hu / p.group;
        ok = kv.load_packed(&tm_k, kv_h, w.k0);
        if (ok) ok = wait_bar(&bars->q_empty, (q_count & 1u) ^ 1u, abort_flag);
        if (ok) {
          ptx::mbar_arrive_expect_tx(&bars->q_full, 2 * Q_BYTES);
#pragma unroll
          for (int db = 0; db < DB; ++db) {
            ptx::tma_load_3d(sQ + db * (BM * 128), &tm_q, &bars->q_full, db * 64, w.hu, w.q0);
            ptx::tma_load_3d(sDO + db * (BM * 128), &tm_do, &bars->q_full, db * 64, w.hu, w.q0);
          }
          ++q_count;
          ok = kv.load_packed(&tm_v, kv_h, w.k0);
        }
        for (int j = 1; ok && j < w.n_kv; ++j) {
          ok = kv.load_packed(&tm_k, kv_h, w.k0 + j * BN);
          if (ok) ok = kv.load_packed(&tm_v, kv_h, w.k0 + j * BN);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
    }
    if (lane == 0) {
      kv.drain();
      if (q_count > 0) drain_wait(&bars->q_full, (q_count - 1) & 1u);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t rs = 0, rph = 0;
      uint32_t slot = 0, phase = 0, g = 0, items = 0;
      uint32_t kslot[2] = {0, 0};
      bool ok = true;
      const uint32_t sQ_addr = ptx::smem_u32(sQ);
      const uint32_t sDO_addr = ptx::smem_u32(sDO);
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
      // dst = A K^T over D: A = Q or dO tile (K-major), K = the key tile (K-major)
      auto issue_qk = [&](uint32_t dst_col, uint32_t a_addr, uint32_t kvslot) {
        const uint32_t kbase = sKV_addr + kvslot * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk % 4) * 32u;
          uint64_t a = ptx::sdesc_sw128(a_addr + (kk / 4) * (BM * 128) + off, 16, 1024);
          uint64_t b = ptx::sdesc_sw128(kbase + (kk / 4) * (BN * 128) + off, 16, 1024);
          ptx::mma_ss(tmem + dst_col, a, b, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // S(j), dP(j) into buffer buf: takes K(j) (kept for dQ) and V(j) (released)
      auto issue_sdp = [&](uint32_t buf, bool last) -> bool {
        uint32_t ks, vs;
        if (!take_slot(ks)) return false;
        issue_qk(buf * BN, sQ_addr, ks);
        if (!take_slot(vs)) return false;
        issue_qk(DP_COL + buf * BN, sDO_addr, vs);
        ptx::mma_commit(&bars->s_full[buf]);
        ptx::mma_commit(&bars->empty[vs]);
        if (last) ptx::mma_commit(&bars->q_empty);
        kslot[buf] = ks;
        return true;
      };
      // dQ += dS K over the BN keys in steps of 16 (dS from TMEM, K MN-major)
      auto issue_dq = [&](uint32_t buf, bool acc) {
        const uint32_t kbase = sKV_addr + kslot[buf] * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          uint64_t b = ptx::sdesc_sw128(kbase + kk * (16 * 128), BN * 128, 1024);
          ptx::mma_ts(tmem + DQ_COL, tmem + buf * BN + kk * 8, b, IDESC_DQ,
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
        // K0 is ahead of Q in the ring; Q / dO land on q_full
        if (!(ok = wait_bar(&bars->q_full, items & 1u, abort_flag))) break;
        ptx::tc_fence_after();
        for (int jj = 0; ok && jj < 2 && jj < n; ++jj) ok = issue_sdp((g + jj) & 1u, jj == n - 1);
        for (int j = 0; ok && j < n; ++j) {
          const uint32_t gj = g + j;
          const uint32_t buf = gj & 1u;
          if (!(ok = wait_bar(&bars->ds_full[buf], (gj >> 1) & 1u, abort_flag))) break;
          ptx::tc_fence_after();
          if (j == 0 && items > 0) {
            if (!(ok = wait_bar(&bars->dq_free, (items - 1) & 1u, abort_flag))) break;
            ptx::tc_fence_after();
          }
          issue_dq(buf, j > 0);
          ptx::mma_commit(&bars->empty[kslot[buf]]);
          if (j == n - 1) ptx::mma_commit(&bars->dq_ready);
          if (j + 2 < n) ok = issue_sdp(buf, j + 2 == n - 1);
        }
        g += n;
        ++items;
      }
      ptx::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ query rows
    const int t = warp / 4;               // warpgroup: takes the global tiles gj with gj & 1 == t
    const int r = threadIdx.x - 128 * t;  // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * BN;
    const uint32_t tDP = tmem + lane_base + DP_COL + t * BN;
    const uint32_t tDQ = tmem + lane_base + DQ_COL;
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
      const int qi = w.qi0 + r;
      const bool row_valid = r < w.q_rows;
      const size_t row = (size_t)(w.q0 + r) * p.H + w.hu;  // into [total_q, H]
      // each warpgroup writes half of the dQ row's columns
      uint16_t *dq_half = bp.dq + row * D + t * (D / 2);
      float delta = 0.f, lse2 = INFINITY;  // invalid rows: p = exp2(-inf) = 0
      if (row_valid) {
        delta = row_delta<D, BF16>(bp.dout + row * D, bp.o + row * D);
        if (t == 0) bp.delta[row] = delta;
        lse2 = __ldg(bp.lse + row) * LOG2E;
      }
      if (n == 0) {
        if (row_valid) zero_row<D / 2>(dq_half);
        continue;
      }
      const int hi = key_hi(p, qi, w.Lk);  // visible keys [0, hi)
      for (int j = (int)((t - g) & 1u); ok && j < n; j += 2) {
        const uint32_t gj = g + j;
        bool got = wait_bar(&bars->s_full[t], (gj >> 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const int lim = hi - j * BN;
        // 32 keys at a time: dS of keys [c0, c0 + 32) goes to packed columns
        // [c0 / 2, c0 / 2 + 16) of S, which were read by an earlier piece
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t sv[32], dpv[32];
          tmem_ld_wait<32>(tS + c0, sv);
          tmem_ld_wait<32>(tDP + c0, dpv);
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float ds[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float x = __uint_as_float(sv[c + e]) * sl2 - lse2;
              const float pr = (c0 + c + e < lim) ? ptx::ex2_approx(x) : 0.f;
              ds[e] = pr * (__uint_as_float(dpv[c + e]) - delta);
            }
            pk[c / 2] = pack2<BF16>(ds[0], ds[1]);
          }
          tmem_st<16>(tS + c0 / 2, pk);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->ds_full[t]);
      }
      if (!ok) break;
      g += n;
      bool got = wait_bar(&bars->dq_ready, items & 1u, abort_flag);
      ++items;
      if (!__all_sync(0xffffffffu, got)) break;
      ptx::tc_fence_after();
      store_tmem_row<D / 2, BF16>(tDQ + t * (D / 2), bp.scale, row_valid, dq_half, bp.v8 != 0);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->dq_free);
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

}  // namespace bwd_dq
}  // namespace vattn
