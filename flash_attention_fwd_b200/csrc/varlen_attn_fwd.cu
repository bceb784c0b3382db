/*
 * varlen_attn_fwd.cu — sm_100a (B200) packed variable-length attention
 * forward and its C ABI (declared in include/varlen_attn.h).
 *
 * What is computed is the forward loop of boostr 0.2.0,
 * src/ops/cpu/attention/varlen_attention.rs (varlen_attention_fwd): per
 * (sequence b, query head h, query qi) a softmax over the scaled dot products
 * with the keys of the same sequence (GQA head map kv_h = h / (H/Hkv); with
 * causal, key ki is hidden from query qi when qi < ki), the softmax-weighted
 * sum of the values, and LSE = max + ln(sum).  The page computes the softmax
 * in two passes over a full row of scores; here the row is streamed in key
 * tiles with a running maximum and sum (the "online" form), which reaches
 * the same result up to rounding.
 *
 * Kernel design (one persistent CTA per SM, 192 threads):
 *   warps 0-3  softmax warpgroup: thread t owns query row t of the tile
 *              (TMEM lane t); reads S from TMEM, masks, keeps the running
 *              max/sum, writes P (bf16/fp16) back into TMEM over S, rescales
 *              O in TMEM when the running max grows by more than 2^8, and
 *              runs the epilogue (O / l -> global, LSE -> global).
 *   warp 4     TMA producer: Q tile per work item, K/V tiles through a ring
 *              of shared-memory slots (mbarrier full/empty pairs).
 *   warp 5     TMEM owner and MMA issuer: S = Q K^T (A and B from shared
 *              memory) into one of two TMEM S buffers, O += P V (A = P from
 *              TMEM, B = V from shared memory, MN-major) into the TMEM O
 *              accumulator; completion is signalled with tcgen05.commit.
 * Work items are (sequence, query tile of 128 rows, head), walked from the
 * device-resident cu_seqlens by every role independently and dealt to the
 * CTAs round-robin with the direction reversed every round, which keeps the
 * per-CTA sums of causal tile costs close.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "sm100_ptx.cuh"
#include "varlen_attn.h"

namespace vattn {

constexpr int BM = 128;              // query rows per tile = TMEM lanes
constexpr int NUM_THREADS = 192;     // 4 softmax warps + producer + MMA
constexpr int PRODUCER_WARP = 4;
constexpr int MMA_WARP = 5;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only when max grows > 2^8
constexpr uint64_t WAIT_TIMEOUT_NS = 2000000000ull;  // 2 s: far beyond any legitimate wait
constexpr unsigned STATUS_TIMEOUT = 1u;

__device__ unsigned int g_device_status = 0;

template <int D>
struct TileCfg;
// BN = keys per KV tile, NSLOT = K/V shared-memory ring depth.
template <>
struct TileCfg<64> {
  static constexpr int BN = 128, NSLOT = 8;
};
template <>
struct TileCfg<128> {
  static constexpr int BN = 128, NSLOT = 6;
};
template <>
struct TileCfg<256> {
  static constexpr int BN = 64, NSLOT = 4;
};

struct KParams {
  const int *cu_q;
  const int *cu_k;
  void *out;
  float *lse;
  int B, H, Hkv, group;  // group = H / Hkv
  int total_q, total_k;
  int causal;
  float scale_log2;  // scale * log2(e)
};

struct Barriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_ready, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct WorkItem {
  int h;
  int q0;      // packed index of the tile's first query token
  int q_rows;  // valid rows in the tile (<= BM)
  int qi0;     // sequence-local index of the tile's first query
  int k0;      // packed index of the sequence's first key
  int Lk;      // keys in the sequence
  int n_kv;    // KV tiles to visit
  int min_lim; // smallest per-row visible-key bound in the tile
};

// Walks the work list (b ascending, query tile descending, head ascending)
// and deals item idx to CTA (round-robin, direction reversed each round).
// Lengths are clamped into the buffers' extents so that an inconsistent
// sequence table cannot address memory outside them.
template <int BN>
struct Scheduler {
  const int *cu_q, *cu_k;
  int B, H, causal, total_q, total_k;
  int cta, grid, round;
  int b;
  long long base;
  int q_start, q_len, k_start, k_len, nq;

  __device__ void init(const KParams &p) {
    cu_q = p.cu_q;
    cu_k = p.cu_k;
    B = p.B;
    H = p.H;
    causal = p.causal;
    total_q = p.total_q;
    total_k = p.total_k;
    cta = blockIdx.x;
    grid = gridDim.x;
    round = 0;
    b = 0;
    base = 0;
    if (B > 0) load(0);
  }

  __device__ void load(int bb) {
    int qs = __ldg(cu_q + bb), qe = __ldg(cu_q + bb + 1);
    int ks = __ldg(cu_k + bb), ke = __ldg(cu_k + bb + 1);
    qs = min(max(qs, 0), total_q);
    qe = min(max(qe, qs), total_q);
    ks = min(max(ks, 0), total_k);
    ke = min(max(ke, ks), total_k);
    q_start = qs;
    q_len = qe - qs;
    k_start = ks;
    k_len = ke - ks;
    nq = (q_len + BM - 1) / BM;
  }

  __device__ bool next(WorkItem &w) {
    long long idx = (long long)round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
    ++round;
    while (b < B && idx >= base + (long long)nq * H) {
      base += (long long)nq * H;
      ++b;
      if (b < B) load(b);
    }
    if (b >= B) return false;
    long long local = idx - base;
    int qt = nq - 1 - (int)(local / H);
    w.h = (int)(local % H);
    w.qi0 = qt * BM;
    w.q0 = q_start + w.qi0;
    w.q_rows = min(BM, q_len - w.qi0);
    w.k0 = k_start;
    w.Lk = k_len;
    int kv_end = causal ? min(k_len, min(q_len, w.qi0 + BM)) : k_len;
    w.n_kv = (kv_end + BN - 1) / BN;
    w.min_lim = causal ? min(k_len, w.qi0 + 1) : k_len;
    return true;
  }
};

// Bounded wait; on timeout raises the CTA abort flag and the device status.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > WAIT_TIMEOUT_NS) {
        *abort_flag = 1;
        atomicOr(&g_device_status, STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

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
__device__ __forceinline__ void tmem_st<32>(uint32_t taddr, const uint32_t (&r)[32]) {
  ptx::tmem_st_x32(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_st<64>(uint32_t taddr, const uint32_t (&r)[64]) {
  ptx::tmem_st_x64(taddr, r);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    varlen_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const KParams p) {
  constexpr int BN = TileCfg<D>::BN;
  constexpr int NSLOT = TileCfg<D>::NSLOT;
  constexpr int DB = D / 64;                     // 128-byte swizzle blocks along D
  constexpr uint32_t Q_BYTES = BM * D * 2;
  constexpr uint32_t KV_BYTES = BN * D * 2;
  // TMEM columns: S buffer b at [b*BN, (b+1)*BN), P aliases its first BN/2
  // columns, O accumulator at [2*BN, 2*BN + D).
  constexpr uint32_t O_COL = 2 * BN;
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
  constexpr uint32_t IDESC_S = ptx::idesc_f16(BM, BN, BF16, false);
  constexpr uint32_t IDESC_PV = ptx::idesc_f16(BM, D, BF16, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + Q_BYTES;
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
    }
    ptx::mbar_init(&bars->pv_done, 1);
    ptx::mbar_init(&bars->o_ready, 1);
    ptx::mbar_init(&bars->o_free, 4);
    ptx::mbar_init(&bars->drain, 1);
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

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      Scheduler<BN> sched;
      sched.init(p);
      WorkItem w;
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
      while (ok && sched.next(w)) {
        const int n = w.n_kv;
        if (n == 0) continue;
        const int kv_h = w.h / p.group;
        ok = load_kv(&tm_k, kv_h, w.k0);
        if (!ok) break;
        if (!wait_bar(&bars->q_empty, (q_count & 1u) ^ 1u, abort_flag)) break;
        ptx::mbar_arrive_expect_tx(&bars->q_full, Q_BYTES);
#pragma unroll
        for (int db = 0; db < DB; ++db)
          ptx::tma_load_3d(sQ + db * (BM * 128), &tm_q, &bars->q_full, db * 64, w.h, w.q0);
        ++q_count;
        if (n >= 2) ok = load_kv(&tm_k, kv_h, w.k0 + BN);
        for (int j = 0; ok && j < n; ++j) {
          ok = load_kv(&tm_v, kv_h, w.k0 + j * BN);
          if (ok && j + 2 < n) ok = load_kv(&tm_k, kv_h, w.k0 + (j + 2) * BN);
        }
      }
      // Drain: every copy this thread issued has landed before the CTA exits.
      for (int s = 0; s < NSLOT; ++s)
        if (slot_fills[s] > 0) {
          uint32_t last_parity = (slot_fills[s] - 1) & 1u;
          wait_bar(&bars->full[s], last_parity, abort_flag);
        }
      if (q_count > 0) wait_bar(&bars->q_full, (q_count - 1) & 1u, abort_flag);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      Scheduler<BN> sched;
      sched.init(p);
      WorkItem w;
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
      // S[buf] = Q K^T over D in steps of 16 (K-major A and B, 128B swizzle)
      auto issue_s = [&](uint32_t buf, uint32_t kslot) {
        const uint32_t kbase = sKV_addr + kslot * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk % 4) * 32u;  // 16 elements = 32 bytes inside a swizzle row
          uint64_t a = ptx::sdesc_sw128(sQ_addr + (kk / 4) * (BM * 128) + off, 16, 1024);
          uint64_t bdesc = ptx::sdesc_sw128(kbase + (kk / 4) * (BN * 128) + off, 16, 1024);
          ptx::mma_ss(tmem + buf * BN, a, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // O += P V over the BN keys in steps of 16 (P from TMEM, V MN-major)
      auto issue_pv = [&](uint32_t buf, uint32_t vslot, bool acc) {
        const uint32_t vbase = sKV_addr + vslot * KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          uint64_t bdesc = ptx::sdesc_sw128(vbase + kk * (16 * 128), BN * 128, 1024);
          ptx::mma_ts(tmem + O_COL, tmem + buf * BN + kk * 8, bdesc, IDESC_PV,
                      (acc || kk > 0) ? 1u : 0u);
        }
      };
      while (ok && sched.next(w)) {
        const int n = w.n_kv;
        if (n == 0) continue;
        if (!wait_bar(&bars->q_full, items & 1u, abort_flag)) break;
        ptx::tc_fence_after();
        for (int jj = 0; ok && jj < 2 && jj < n; ++jj) {
          uint32_t ks;
          if (!(ok = take_slot(ks))) break;
          const uint32_t buf = (g + jj) & 1u;
          issue_s(buf, ks);
          ptx::mma_commit(&bars->s_full[buf]);
          ptx::mma_commit(&bars->empty[ks]);
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
          uint32_t vs;
          if (!(ok = take_slot(vs))) break;
          issue_pv(buf, vs, j > 0);
          ptx::mma_commit(&bars->empty[vs]);
          ptx::mma_commit(&bars->pv_done);
          if (j == n - 1) ptx::mma_commit(&bars->o_ready);
          if (j + 2 < n) {
            uint32_t ks;
            if (!(ok = take_slot(ks))) break;
            issue_s(buf, ks);
            ptx::mma_commit(&bars->s_full[buf]);
            ptx::mma_commit(&bars->empty[ks]);
            if (j + 2 == n - 1) ptx::mma_commit(&bars->q_empty);
          }
        }
        g += n;
        ++items;
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      ptx::mma_commit(&bars->drain);
      wait_bar(&bars->drain, 0, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ softmax WG
    const int r = threadIdx.x;  // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tS0 = tmem + lane_base;
    const uint32_t tO = tmem + lane_base + O_COL;
    const float sl2 = p.scale_log2;
    Scheduler<BN> sched;
    sched.init(p);
    WorkItem w;
    uint32_t g = 0, items = 0;
    bool ok = true;
    while (ok && sched.next(w)) {
      const int n = w.n_kv;
      const int qi = w.qi0 + r;
      const bool row_valid = r < w.q_rows;
      const size_t orow = (size_t)(w.q0 + r) * p.H + w.h;  // row index into [total_q, H]
      if (n == 0) {
        if (row_valid) {
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) + orow * D);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          p.lse[orow] = -INFINITY;
        }
        continue;
      }
      const int key_lim = p.causal ? min(w.Lk, qi + 1) : w.Lk;
      float m = -INFINITY;  // running max of scaled scores, log2 units
      float l = 0.f;        // running sum of exp2(x - m)
      for (int j = 0; j < n; ++j) {
        const uint32_t gj = g + j;
        const uint32_t buf = gj & 1u;
        bool got = wait_bar(&bars->s_full[buf], (gj >> 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        uint32_t sr[BN];
        tmem_ld_wait<BN>(tS0 + buf * BN, sr);
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(sr[c]);
        if ((j + 1) * BN > w.min_lim) {
          const int lim = key_lim - j * BN;
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < BN; c += 4) {
          mx0 = fmaxf(mx0, s[c]);
          mx1 = fmaxf(mx1, s[c + 1]);
          mx2 = fmaxf(mx2, s[c + 2]);
          mx3 = fmaxf(mx3, s[c + 3]);
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
        float alpha = 1.f;
        bool need = false;
        if (j == 0) {
          m = (mx == -INFINITY) ? 0.f : mx;
        } else if (mx > m + RESCALE_THRESHOLD) {
          alpha = ptx::ex2_approx(m - mx);
          m = mx;
          need = true;
        }
        if (__any_sync(0xffffffffu, need)) {
          // O must hold PV(gj-1) before it is rescaled in place.  The wait
          // by parity is exact here: S(gj) completing implies PV(gj-2) did,
          // and PV(gj) cannot be issued before this iteration's P, so the
          // barrier is in phase gj-1 or gj.
          bool got2 = wait_bar(&bars->pv_done, (gj - 1) & 1u, abort_flag);
          if (!__all_sync(0xffffffffu, got2)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld_wait<32>(tO + c0, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st<32>(tO + c0, o);
          }
        }
        l *= alpha;
        const float neg_m = -m;
        float sum0 = 0.f, sum1 = 0.f;
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const float p0 = ptx::ex2_approx(fmaf(s[c], sl2, neg_m));
          const float p1 = ptx::ex2_approx(fmaf(s[c + 1], sl2, neg_m));
          const uint32_t pp = pack2<BF16>(p0, p1);
          pk[c / 2] = pp;
          if constexpr (BF16) {
            // Sum the values the PV MMA actually sees (bf16-rounded), so the
            // numerator and the denominator of O / l carry the same rounding.
            sum0 += __uint_as_float(pp << 16);
            sum1 += __uint_as_float(pp & 0xFFFF0000u);
          } else {
            sum0 += p0;
            sum1 += p1;
          }
        }
        l += sum0 + sum1;
        tmem_st<BN / 2>(tS0 + buf * BN, pk);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->p_full[buf]);
      }
      if (!ok) break;
      g += n;
      // ---- epilogue: O / l -> out, LSE -> lse.  o_ready completes once per
      // item, after the item's last PV; the next item's first PV waits for
      // o_free, so this barrier is never more than one phase ahead.
      bool got = wait_bar(&bars->o_ready, items & 1u, abort_flag);
      ++items;
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const float inv_l = 1.f / l;
      uint16_t *orow_ptr = reinterpret_cast<uint16_t *>(p.out) + orow * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld_wait<32>(tO + c0, o);
        if (c0 + 32 == D) {
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&bars->o_free);
        }
        if (row_valid) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            pk[c / 2] = pack2<BF16>(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
          uint4 *dst = reinterpret_cast<uint4 *>(orow_ptr + c0);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (row_valid) p.lse[orow] = (m + log2f(l)) * 0.69314718055994530942f;
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

// ====================================================================== host

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [rows, heads, D] row-major 16-bit tensor; box = 64 elements x 1 head x box_rows.
static bool encode_qkv_map(EncodeTiledFn enc, CUtensorMap *map, const void *base, bool bf16,
                           int64_t rows, int heads, int D, int box_rows) {
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int g_last_cuda_error = 0;

struct DeviceInfo {
  int sms = 0;
  int major = 0, minor = 0;
  bool attr_set[3][2] = {{false, false}, {false, false}, {false, false}};
};
static DeviceInfo g_dev[64];

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)BM * D * 2 + (size_t)TileCfg<D>::NSLOT * TileCfg<D>::BN * D * 2 +
         sizeof(Barriers) + 1024;
}

template <int D, bool BF16>
static int launch(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                  const KParams &kp, int grid, cudaStream_t stream, DeviceInfo &dev, int didx) {
  constexpr size_t smem = smem_bytes<D>();
  static_assert(smem <= 232448, "shared memory budget");
  if (!dev.attr_set[didx][BF16 ? 0 : 1]) {
    cudaError_t e = cudaFuncSetAttribute(varlen_fwd_kernel<D, BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
      g_last_cuda_error = (int)e;
      return VARLEN_ERR_LAUNCH;
    }
    dev.attr_set[didx][BF16 ? 0 : 1] = true;
  }
  varlen_fwd_kernel<D, BF16><<<grid, NUM_THREADS, smem, stream>>>(tq, tk, tv, kp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_last_cuda_error = (int)e;
    return VARLEN_ERR_LAUNCH;
  }
  return VARLEN_OK;
}

static bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace vattn

using namespace vattn;

extern "C" int varlen_attn_fwd_v1(const void *q, const void *k, const void *v,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_kv_heads, int head_dim,
                                  int causal, float scale, varlen_dtype_t dtype, void *out,
                                  float *lse, varlen_stream_t stream) {
  // ---- host-side validation: nothing is launched or touched on error
  if (dtype != VARLEN_BF16 && dtype != VARLEN_FP16) return VARLEN_ERR_DTYPE;
  if (batch < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
    return VARLEN_ERR_SHAPE;
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return VARLEN_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return VARLEN_ERR_SHAPE;
  if (total_q >= (int64_t(1) << 31) || total_k >= (int64_t(1) << 31)) return VARLEN_ERR_SHAPE;
  if (num_heads > 65535) return VARLEN_ERR_SHAPE;
  if (batch > 0 && (!cu_seqlens_q || !cu_seqlens_k)) return VARLEN_ERR_NULL;
  if (total_q > 0 && (!q || !out || !lse)) return VARLEN_ERR_NULL;
  if (total_k > 0 && (!k || !v)) return VARLEN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return VARLEN_ERR_ALIGN;
  if (!aligned(lse, 4) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
    return VARLEN_ERR_ALIGN;
  if (batch == 0 || total_q == 0) return VARLEN_OK;

  int dev_id = 0;
  cudaError_t e = cudaGetDevice(&dev_id);
  if (e != cudaSuccess || dev_id < 0 || dev_id >= 64) {
    g_last_cuda_error = (int)e;
    return VARLEN_ERR_LAUNCH;
  }
  DeviceInfo &dev = g_dev[dev_id];
  if (dev.sms == 0) {
    int sms = 0, mj = 0, mn = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_id) != cudaSuccess ||
        cudaDeviceGetAttribute(&mj, cudaDevAttrComputeCapabilityMajor, dev_id) != cudaSuccess ||
        cudaDeviceGetAttribute(&mn, cudaDevAttrComputeCapabilityMinor, dev_id) != cudaSuccess)
      return VARLEN_ERR_LAUNCH;
    dev.major = mj;
    dev.minor = mn;
    dev.sms = sms;
  }
  if (dev.major != 10 || dev.minor != 0) return VARLEN_ERR_ARCH;

  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return VARLEN_ERR_LAUNCH;
  const bool bf16 = dtype == VARLEN_BF16;
  const int D = head_dim;
  const int BN = (D == 256) ? TileCfg<256>::BN : TileCfg<128>::BN;
  alignas(64) CUtensorMap tq, tk, tv;
  memset(&tk, 0, sizeof tk);
  memset(&tv, 0, sizeof tv);
  if (!encode_qkv_map(enc, &tq, q, bf16, total_q, num_heads, D, BM)) return VARLEN_ERR_LAUNCH;
  if (total_k > 0) {
    if (!encode_qkv_map(enc, &tk, k, bf16, total_k, num_kv_heads, D, BN) ||
        !encode_qkv_map(enc, &tv, v, bf16, total_k, num_kv_heads, D, BN))
      return VARLEN_ERR_LAUNCH;
  }

  KParams kp;
  kp.cu_q = cu_seqlens_q;
  kp.cu_k = cu_seqlens_k;
  kp.out = out;
  kp.lse = lse;
  kp.B = batch;
  kp.H = num_heads;
  kp.Hkv = num_kv_heads;
  kp.group = num_heads / num_kv_heads;
  kp.total_q = (int)total_q;
  kp.total_k = (int)total_k;
  kp.causal = causal ? 1 : 0;
  const float sc = (scale > 0.f) ? scale : 1.0f / sqrtf((float)D);  // NaN fails "> 0"
  kp.scale_log2 = sc * 1.4426950408889634f;

  // Upper bound of work items from max_seqlen_q; at least one CTA so that an
  // understated bound never drops work.
  long long max_items = (long long)batch * ((max_seqlen_q + BM - 1) / BM) * num_heads;
  int grid = dev.sms;
  if (max_items >= 1 && max_items < grid) grid = (int)max_items;
  if (grid < 1) grid = 1;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (D) {
    case 64:
      return bf16 ? launch<64, true>(tq, tk, tv, kp, grid, s, dev, 0)
                  : launch<64, false>(tq, tk, tv, kp, grid, s, dev, 0);
    case 128:
      return bf16 ? launch<128, true>(tq, tk, tv, kp, grid, s, dev, 1)
                  : launch<128, false>(tq, tk, tv, kp, grid, s, dev, 1);
    default:
      return bf16 ? launch<256, true>(tq, tk, tv, kp, grid, s, dev, 2)
                  : launch<256, false>(tq, tk, tv, kp, grid, s, dev, 2);
  }
}

extern "C" int varlen_attn_fwd(const void *q, const void *k, const void *v,
                               const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int batch,
                               int64_t total_q, int64_t total_k, int max_seqlen_q,
                               int max_seqlen_k, int num_heads, int num_kv_heads, int head_dim,
                               int causal, float scale, varlen_dtype_t dtype, void *out,
                               float *lse, varlen_stream_t stream) {
  return varlen_attn_fwd_v1(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                            max_seqlen_q, max_seqlen_k, num_heads, num_kv_heads, head_dim, causal,
                            scale, dtype, out, lse, stream);
}

extern "C" const char *varlen_attn_strerror(int code) {
  switch (code) {
    case VARLEN_OK:
      return "success";
    case VARLEN_ERR_NULL:
      return "a required pointer is NULL";
    case VARLEN_ERR_SHAPE:
      return "unsupported shape: need H % Hkv == 0, D in {64,128,256}, non-negative sizes, "
             "token counts < 2^31";
    case VARLEN_ERR_DTYPE:
      return "unsupported dtype: need VARLEN_BF16 or VARLEN_FP16";
    case VARLEN_ERR_ALIGN:
      return "misaligned pointer: q, k, v, out need 16-byte alignment; lse and cu_seqlens "
             "4-byte";
    case VARLEN_ERR_LAUNCH:
      return "CUDA launch or tensor-map setup failed";
    case VARLEN_ERR_DEVICE:
      return "device-side status word is set (a bounded pipeline wait timed out)";
    case VARLEN_ERR_ARCH:
      return "current device is not compute capability 10.0 (sm_100a build)";
    default:
      return "unknown status code";
  }
}

extern "C" int varlen_attn_device_status(unsigned int *status, int clear) {
  if (!status) return VARLEN_ERR_NULL;
  if (cudaMemcpyFromSymbol(status, g_device_status, sizeof(unsigned int)) != cudaSuccess)
    return VARLEN_ERR_LAUNCH;
  if (clear) {
    unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(unsigned int)) != cudaSuccess)
      return VARLEN_ERR_LAUNCH;
  }
  return VARLEN_OK;
}

extern "C" int varlen_attn_abi_version(void) { return 1; }
