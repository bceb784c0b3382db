/*
 * fwd_single.cuh — attention forward, one 128-row query tile per work item.
 *
 * Used for head dim 256 (TMEM holds one tile's O of 256 columns plus two S
 * buffers of 128 key columns) and for head layouts without query-head pairs
 * sharing a key/value head (H / Hkv odd, e.g. plain multi-head attention).
 *
 * At head dim 256 a 128-key K or V tile (64 KB) is staged as two 128-column
 * slices in consecutive ring slots of 32 KB: S = Q K^T runs at N = 128 (an
 * N = 64 MMA takes as long as an N = 128 one) and PV as two N = 128 products
 * into the two column halves of O.
 *
 * One persistent CTA per SM, 320 threads:
 *   warps 0-3  softmax, key columns [0, BN/2) of every S tile
 *   warps 4-7  softmax, key columns [BN/2, BN)
 *              (thread t of either warpgroup = query row t = TMEM lane t, and
 *              column half of O: [0, D/2) or [D/2, D))
 *   warp 8     TMA producer: Q tile, K/V tiles through a shared-memory ring
 *   warp 9     TMEM owner and MMA issuer
 * S is double-buffered in TMEM so that S(j+1) = Q K(j+1)^T runs on the tensor
 * cores while the softmax warps work on S(j); the MMA order per key tile is
 * S(0), S(1), then PV(j), S(j+2) for j = 0, 1, ...
 *
 * The two threads of a row share its running max: per tile each publishes its
 * half's max in shared memory and both continue with the larger one, so both
 * take the same rescaling decisions and their P halves carry one scale.  The
 * packed P of key c goes to column BN/4 + c/2, so the first half's P lands in
 * columns [BN/4, BN/2) and the second's in [BN/2, 3BN/4): each inside the S
 * columns that its own warps read, never over S that the other half has
 * still to load.
 */
#pragma once
#include "fwd_common.cuh"

namespace vattn {
namespace single {

constexpr int NUM_THREADS = 320;
constexpr int SOFTMAX_WARPS = 8;
constexpr int PRODUCER_WARP = 8;
constexpr int RING_CONSUMERS = 1 + SOFTMAX_WARPS;  // MMA thread + one arrival per softmax warp
constexpr int MMA_WARP = 9;

template <int D>
struct Cfg;
// BN = keys per tile, NSLOT = K/V shared-memory ring depth, SPLIT = column
// slices of a K/V tile (one ring slot each).
template <>
struct Cfg<64> {
  static constexpr int BN = 128, NSLOT = 8, SPLIT = 1;
};
template <>
struct Cfg<128> {
  static constexpr int BN = 128, NSLOT = 6, SPLIT = 1;
};
template <>
struct Cfg<256> {
  static constexpr int BN = 128, NSLOT = 5, SPLIT = 2;
};

struct Barriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_ready, o_free, drain;
  uint64_t v_tail;  // an item's last V tile that runs past the used keys has landed
  uint64_t xf[4], xr[4];  // row-pair exchange, per TMEM lane quarter: value written / read
  float xch[2][BM];       // exchanged value of row r from column half h
  ItemRing ring;
  uint32_t tmem_base;
  AbortState abort;
};

// Exchange of one float between the two threads of a row (one per column
// half; warps w and w + 4 cover the same TMEM lanes).  Each swap publishes v
// in its slot and returns the partner's.  xf completes when both have written,
// xr when both have read, and a slot is rewritten only after xr of the
// previous swap, so one slot per thread suffices.  Waits are bounded; false
// when one gave up (warp-uniform).
struct RowSwap {
  float *mine;
  const volatile float *other;
  uint64_t *xf, *xr;
  AbortState *abort_flag;
  uint32_t n;
  int lane;
  __device__ void init(float *a, const float *b, uint64_t *f, uint64_t *rd, int ln,
                       AbortState *abort) {
    mine = a;
    other = b;
    xf = f;
    xr = rd;
    lane = ln;
    abort_flag = abort;
    n = 0;
  }
  __device__ bool swap(float v, float &out) {
    if (n > 0 && !__all_sync(0xffffffffu, wait_bar(xr, (n - 1) & 1u, abort_flag))) return false;
    *mine = v;
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(xf);
    if (!__all_sync(0xffffffffu, wait_bar(xf, n & 1u, abort_flag))) return false;
    out = *other;
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(xr);
    ++n;
    return true;
  }
};

// Softmax of one key tile over this thread's half of its columns (HB keys,
// S at tS, packed P to tP, O columns [0, DC) at tO) for one row; the row's
// max over the whole tile comes from the swap with the other half.  Running
// state: m = the row's running max of the scaled scores in log2 units (the
// same in both halves; possibly stale by up to RESCALE_THRESHOLD), l = this
// half's sum of the rounded P values (what the PV product sees, so O / l
// carries one rounding).  When a tile raises m by more than the threshold, O
// (TMEM, this half's DC columns) is multiplied by exp2(m_old - m_new) in
// place, after `wait_o()` (called by the whole warp) has guaranteed that no
// PV product into O is in flight.  Returns false when a wait gave up.
template <int HB, int DC, bool BF16, class WaitO>
__device__ __forceinline__ bool softmax_half(uint32_t tS, uint32_t tP, uint32_t tO, int j,
                                             float sl2, bool need_mask, int lo, int hi, float &m,
                                             float &l, RowSwap &xs, WaitO &&wait_o) {
  uint32_t sr[HB];
  tmem_ld_wait<HB>(tS, sr);
  float s[HB];
#pragma unroll
  for (int c = 0; c < HB; ++c) s[c] = __uint_as_float(sr[c]);
  if (need_mask) mask_outside(s, lo, hi);
  float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
  for (int c = 4; c + 8 <= HB; c += 8) {
    mx0 = ptx::fmax3(mx0, s[c], s[c + 1]);
    mx1 = ptx::fmax3(mx1, s[c + 2], s[c + 3]);
    mx2 = ptx::fmax3(mx2, s[c + 4], s[c + 5]);
    mx3 = ptx::fmax3(mx3, s[c + 6], s[c + 7]);
  }
  mx0 = ptx::fmax3(mx0, s[HB - 4], s[HB - 3]);
  mx1 = ptx::fmax3(mx1, s[HB - 2], s[HB - 1]);
  const float mh = fmaxf(ptx::fmax3(mx0, mx1, mx2), mx3);
  float mo;
  if (!xs.swap(mh, mo)) return false;
  const float mx = fmaxf(mh, mo) * sl2;
  float alpha = 1.f;
  bool need = false;
  update_max(j, mx, m, alpha, need);
  const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
  const float negm = exp_offset(m);
  const uint64_t negm_2 = ptx::f2_pack(negm, negm);
  float sa = 0.f, sb = 0.f, sc = 0.f, sd = 0.f;
#pragma unroll
  for (int c0 = 0; c0 < HB; c0 += 32) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = c0 + 2 * i;
      const uint64_t x2 = ptx::f2_fma(ptx::f2_pack(s[c], s[c + 1]), sl2_2, negm_2);
      float x0, x1;
      ptx::f2_unpack(x2, x0, x1);
      pk[i] = pack2<BF16>(ptx::ex2_approx(x0), ptx::ex2_approx(x1));
      if (i & 1) {
        sc = ptx::add_lo16<BF16>(pk[i], sc);
        sd = ptx::add_hi16<BF16>(pk[i], sd);
      } else {
        sa = ptx::add_lo16<BF16>(pk[i], sa);
        sb = ptx::add_hi16<BF16>(pk[i], sb);
      }
    }
    ptx::tmem_st_x16(tP + c0 / 2, pk);
  }
  l = l * alpha + ((sa + sb) + (sc + sd));
  if (__any_sync(0xffffffffu, need)) {
    if (!__all_sync(0xffffffffu, wait_o())) return false;
    ptx::tc_fence_after();
    const uint64_t a2 = ptx::f2_pack(alpha, alpha);
#pragma unroll
    for (int c0 = 0; c0 < DC; c0 += 32) {
      uint32_t o[32];
      tmem_ld_wait<32>(tO + c0, o);
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float o0, o1;
        ptx::f2_unpack(
            ptx::f2_mul(ptx::f2_pack(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), a2), o0,
            o1);
        o[c] = __float_as_uint(o0);
        o[c + 1] = __float_as_uint(o1);
      }
      tmem_st<32>(tO + c0, o);
    }
  }
  ptx::tmem_st_wait();
  return true;
}

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)BM * D * 2 + (size_t)Cfg<D>::NSLOT * Cfg<D>::BN * (D / Cfg<D>::SPLIT) * 2 +
         sizeof(Barriers) + 1024;
}
static_assert(smem_bytes<256>() <= 232448 && smem_bytes<128>() <= 232448 &&
                  smem_bytes<64>() <= 232448,
              "shared memory per block");

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const KParams p) {
  constexpr int BN = Cfg<D>::BN;
  constexpr int NSLOT = Cfg<D>::NSLOT;
  constexpr int SPLIT = Cfg<D>::SPLIT;
  constexpr int DS = D / SPLIT;  // columns of a K/V slice (one ring slot)
  constexpr int DB = D / 64;     // 128-byte swizzle blocks along D
  constexpr uint32_t Q_BYTES = BM * D * 2;
  constexpr uint32_t KV_BYTES = BN * DS * 2;
  // TMEM columns: S buffer b at [b*BN, (b+1)*BN), P aliases its columns
  // [BN/4, 3*BN/4), O accumulator at [2*BN, 2*BN + D).
  constexpr uint32_t P_COL = BN / 4;
  constexpr uint32_t O_COL = 2 * BN;
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
  constexpr uint32_t IDESC_S = ptx::idesc_f16(BM, BN, BF16, false);
  constexpr uint32_t IDESC_PV = ptx::idesc_f16(BM, DS, BF16, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + Q_BYTES;
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
      ptx::mbar_init(&bars->p_full[i], SOFTMAX_WARPS);
    }
    ptx::mbar_init(&bars->pv_done, 1);
    ptx::mbar_init(&bars->o_ready, 1);
    ptx::mbar_init(&bars->o_free, SOFTMAX_WARPS);
    for (int i = 0; i < 4; ++i) {
      ptx::mbar_init(&bars->xf[i], 2);
      ptx::mbar_init(&bars->xr[i], 2);
    }
    ptx::mbar_init(&bars->drain, 1);
    ptx::mbar_init(&bars->v_tail, Cfg<D>::SPLIT);  // one arrival per V slice
    for (int i = 0; i < ITEM_RING; ++i) {
      ptx::mbar_init(&bars->ring.full[i], 1);
      ptx::mbar_init(&bars->ring.empty[i], RING_CONSUMERS);
    }
    bars->abort.init();
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

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the scheduler and publishes items on the ring;
    // lane 0 issues the TMA copies.
    {
      Scheduler<BN> sched;
      sched.init(p);
      uint32_t rs = 0, rph = 0, q_count = 0;
      bool ok = true;
      KVProducer<BN, DS, NSLOT, SPLIT> kv;
      kv.init(sKV, bars->full, bars->empty, &bars->v_tail, abort_flag);
      // Q tile of an item (lane 0)
      auto load_q = [&](const WorkItem &w) -> bool {
        if (!wait_bar(&bars->q_empty, (q_count & 1u) ^ 1u, abort_flag)) return false;
        ptx::mbar_arrive_expect_tx(&bars->q_full, Q_BYTES);
#pragma unroll
        for (int db = 0; db < DB; ++db)
          ptx::tma_load_3d(sQ + db * (BM * 128), &tm_q, &bars->q_full, db * 64, w.hu, w.q0);
        ++q_count;
        return true;
      };
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
        if (!ok) break;
        if (!have) {
          kv.fix_tail();
          break;
        }
        if (w.n_kv > 0)
          ok = kv.load_item(p, w, w.hu / p.group, &tm_k, &tm_v, [&]() { return load_q(w); });
        else
          ok = kv.fix_tail();
        if (!ok) break;
      }
      if (lane == 0) {
        // Drain: every copy this warp issued has landed before the CTA exits.
        kv.drain();
        if (q_count > 0) drain_wait(&bars->q_full, (q_count - 1) & 1u);
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
      // the SPLIT ring slots of the next K or V tile
      auto take_tile = [&](uint32_t (&s_out)[SPLIT]) -> bool {
#pragma unroll
        for (int i = 0; i < SPLIT; ++i) {
          s_out[i] = slot;
          if (!wait_bar(&bars->full[slot], phase, abort_flag)) return false;
          if (++slot == NSLOT) {
            slot = 0;
            phase ^= 1u;
          }
        }
        ptx::tc_fence_after();
        return true;
      };
      // S[buf] = Q K^T over D in steps of 16 (K-major A and B, 128B swizzle),
      // slice by slice; each slice's ring slot is released (commit) as soon
      // as the MMAs issued so far, which include all that read it, complete
      auto issue_s = [&](uint32_t buf, const uint32_t (&ks)[SPLIT]) {
#pragma unroll
        for (int i = 0; i < SPLIT; ++i) {
          const uint32_t kbase = sKV_addr + ks[i] * KV_BYTES;
#pragma unroll
          for (int ki = 0; ki < DS / 16; ++ki) {
            const int kk = i * (DS / 16) + ki;    // step along D
            const uint32_t off = (ki % 4) * 32u;  // 16 elements = 32 bytes inside a swizzle row
            uint64_t a = ptx::sdesc_sw128(sQ_addr + (kk / 4) * (BM * 128) + off, 16, 1024);
            uint64_t bdesc = ptx::sdesc_sw128(kbase + (ki / 4) * (BN * 128) + off, 16, 1024);
            ptx::mma_ss(tmem + buf * BN, a, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
          }
          if (i == SPLIT - 1) ptx::mma_commit(&bars->s_full[buf]);
          ptx::mma_commit(&bars->empty[ks[i]]);
        }
      };
      // O += P V over the BN keys in steps of 16 (P from TMEM, V MN-major);
      // slice i of V feeds O's columns [i * DS, (i + 1) * DS) and its slot is
      // released right after its MMAs
      auto issue_pv = [&](uint32_t buf, const uint32_t (&vs)[SPLIT], bool acc) {
#pragma unroll
        for (int i = 0; i < SPLIT; ++i) {
          const uint32_t vbase = sKV_addr + vs[i] * KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            uint64_t bdesc = ptx::sdesc_sw128(vbase + kk * (16 * 128), BN * 128, 1024);
            ptx::mma_ts(tmem + O_COL + i * DS, tmem + buf * BN + P_COL + kk * 8, bdesc, IDESC_PV,
                        (acc || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit(&bars->empty[vs[i]]);
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
          uint32_t ks[SPLIT];
          if (!(ok = take_tile(ks))) break;
          const uint32_t buf = (g + jj) & 1u;
          issue_s(buf, ks);
          if (jj == n - 1) ptx::mma_commit(&bars->q_empty);
        }
        for (int j = 0; ok && j < n; ++j) {
          const uint32_t gj = g + j;
          const uint32_t buf = gj & 1u;
          if (!(ok = wait_bar(&bars->p_full[buf], (gj >> 1) & 1u, abort_flag))) break;
          ptx::tc_fence_after();
          if (j == 0 && items > 0) {
            if (!(ok = wait_bar(&bars->o_free, (items - 1) & 1u, abort_flag))) break;
            ptx::tc_fence_after();
          }
          uint32_t vs[SPLIT];
          if (!(ok = take_tile(vs))) break;
          issue_pv(buf, vs, j > 0);
          ptx::mma_commit(&bars->pv_done);
          if (j == n - 1) ptx::mma_commit(&bars->o_ready);
          if (j + 2 < n) {
            uint32_t ks[SPLIT];
            if (!(ok = take_tile(ks))) break;
            issue_s(buf, ks);
            if (j + 2 == n - 1) ptx::mma_commit(&bars->q_empty);
          }
        }
        g += n;
        ++items;
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      ptx::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    constexpr int HB = BN / 2;  // key columns per half
    constexpr int DC = D / 2;   // O columns per half
    const int h = threadIdx.x / BM;  // column half
    const int r = threadIdx.x % BM;  // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS0 = tmem + lane_base + h * HB;
    const uint32_t tP0 = tmem + lane_base + P_COL + h * (HB / 2);
    const uint32_t tO = tmem + lane_base + O_COL + h * DC;
    RowSwap xs;
    xs.init(&bars->xch[h][r], &bars->xch[h ^ 1][r], &bars->xf[warp & 3], &bars->xr[warp & 3],
            lane, abort_flag);
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
      const size_t orow = (size_t)(w.q0 + r) * p.H + w.hu;  // row index into [total_q, H]
      uint16_t *orow_ptr = reinterpret_cast<uint16_t *>(p.out) + orow * D;
      if (n == 0) {
        if (row_valid && h == 0) empty_row<D>(orow_ptr, p.lse + orow, sink_log2(p, w.hu));
        continue;
      }
      // visible keys of this row, relative to the first key of this thread's
      // half of the first visited key tile
      const int lo = key_lo(p, qi) - w.kofs - h * HB;
      const int hi = key_hi(p, qi, w.Lk) - w.kofs - h * HB;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const uint32_t gj = g + j;
        const uint32_t buf = gj & 1u;
        bool got = wait_bar(&bars->s_full[buf], (gj >> 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // O must hold PV(gj-1) before it is rescaled in place.  The wait by
        // parity is exact: S(gj) completing implies PV(gj-2) did, and PV(gj)
        // cannot be issued before this iteration's P, so the barrier is in
        // phase gj-1 or gj.
        auto wait_o = [&]() { return wait_bar(&bars->pv_done, (gj - 1) & 1u, abort_flag); };
        const bool need_mask = j * BN < w.max_lo || (j + 1) * BN > w.min_hi;
        if (!softmax_half<HB, DC, BF16>(tS0 + buf * BN, tP0 + buf * BN, tO, j, sl2, need_mask,
                                        lo - j * BN, hi - j * BN, m, l, xs, wait_o)) {
          ok = false;
          break;
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->p_full[buf]);
      }
      if (!ok) break;
      g += n;
      // o_ready completes once per item, after the item's last PV; the next
      // item's first PV waits for o_free, so it is never a phase ahead.
      bool got = wait_bar(&bars->o_ready, items & 1u, abort_flag);
      ++items;
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // the row's sum over both halves (the same float in both threads)
      float l_other;
      if (!xs.swap(l, l_other)) {
        ok = false;
        break;
      }
      l += l_other;
      if (w.part < 0)
        epilogue_row<DC, BF16>(tO, m, l, sink_log2(p, w.hu), row_valid, orow_ptr + h * DC,
                               p.lse + orow, &bars->o_free, lane, p.out_v8 != 0, h == 0);
      else
        epilogue_part<DC>(tO, m, l, row_valid,
                          p.part_o + ((size_t)w.part * p.part_rows + orow) * D + h * DC,
                          p.part_lse + (size_t)w.part * p.part_rows + orow, &bars->o_free, lane,
                          p.part_v8 != 0, h == 0);
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

}  // namespace single
}  // namespace vattn
