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

// Device-side status word (bit STATUS_TIMEOUT: a bounded wait gave up).
__device__ unsigned int g_device_status = 0;

struct KParams {
  const int *cu_q;
  const int *cu_k;
  void *out;
  float *lse;
  int B, H, Hkv, group;  // group = H / Hkv
  int head_units;        // heads per work item row: H (one tile) or H/2 (head pairs)
  int total_q, total_k;
  int causal;
  float scale_log2;  // scale * log2(e)
};

struct WorkItem {
  int hu;       // head unit (a head, or a pair of heads 2hu, 2hu+1)
  int q0;       // packed index of the tile's first query token
  int q_rows;   // valid rows in the tile (<= BM)
  int qi0;      // sequence-local index of the tile's first query
  int k0;       // packed index of the sequence's first key
  int Lk;       // keys in the sequence
  int n_kv;     // key tiles to visit
  int min_lim;  // smallest per-row visible-key bound in the tile
};

// Walks the work list (sequence ascending, query tile descending, head unit
// ascending) and deals item idx to CTA round-robin with the direction
// reversed every round.  Every role of a CTA runs its own copy and sees the
// same sequence of items.  Lengths are clamped into the buffers' extents so
// that an inconsistent sequence table cannot address memory outside them.
template <int BN>
struct Scheduler {
  const int *cu_q, *cu_k;
  int B, HU, causal, total_q, total_k;
  int cta, grid, round;
  int b;
  long long base;
  int q_start, q_len, k_start, k_len, nq;

  __device__ void init(const KParams &p) {
    cu_q = p.cu_q;
    cu_k = p.cu_k;
    B = p.B;
    HU = p.head_units;
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
    while (b < B && idx >= base + (long long)nq * HU) {
      base += (long long)nq * HU;
      ++b;
      if (b < B) load(b);
    }
    if (b >= B) return false;
    long long local = idx - base;
    int qt = nq - 1 - (int)(local / HU);
    w.hu = (int)(local % HU);
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

// ---------------------------------------------------------------------------
// Softmax of one S tile held in TMEM (one row per thread), written back as P
// (bf16/fp16) over the first BN/2 columns of the same TMEM region.
//
// Running state per row: m = max of the scaled scores seen so far in log2
// units (possibly stale by up to RESCALE_THRESHOLD), l = sum of exp2(x - m).
// When a tile raises the max by more than the threshold, O (TMEM, D columns)
// is multiplied by exp2(m_old - m_new) in place; before that `wait_o()` is
// called by the whole warp and must guarantee that no PV MMA into O is in
// flight.  P is written in 32-column chunks and O is rescaled after P, so
// that the full S row, the packed P and an O chunk are never live together.
// Returns false when that wait gave up.
template <int BN, int D, bool BF16, class WaitO>
__device__ __forceinline__ bool softmax_tile(uint32_t tS, uint32_t tO, int j, float sl2,
                                             bool need_mask, int lim, float &m, float &l,
                                             WaitO &&wait_o) {
  uint32_t sr[BN];
  tmem_ld_wait<BN>(tS, sr);
  float s[BN];
#pragma unroll
  for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(sr[c]);
  if (need_mask) {
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
  const float neg_m = -m;
  float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      const float p0 = ptx::ex2_approx(fmaf(s[c0 + c], sl2, neg_m));
      const float p1 = ptx::ex2_approx(fmaf(s[c0 + c + 1], sl2, neg_m));
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
    ptx::tmem_st_x16(tS + c0 / 2, pk);
  }
  l = l * alpha + (sum0 + sum1);
  if (__any_sync(0xffffffffu, need)) {
    if (!__all_sync(0xffffffffu, wait_o())) return false;
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
  ptx::tmem_st_wait();
  return true;
}

// Epilogue of one row: O / l -> out (bf16/fp16, 16-byte stores), LSE -> lse.
// Arrives on o_free (one arrival per warp) as soon as O has been read.
template <int D, bool BF16>
__device__ __forceinline__ void epilogue_row(uint32_t tO, float m, float l, bool row_valid,
                                             uint16_t *orow_ptr, float *lse_ptr,
                                             uint64_t *o_free, int lane) {
  const float inv_l = 1.f / l;
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
      uint4 *dst = reinterpret_cast<uint4 *>(orow_ptr + c0);
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4)
        dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
    }
  }
  if (row_valid) *lse_ptr = (m + log2f(l)) * 0.69314718055994530942f;
}

// A query row whose sequence has no key: O = 0, LSE = -inf.
template <int D>
__device__ __forceinline__ void empty_row(uint16_t *orow_ptr, float *lse_ptr) {
  uint4 *dst = reinterpret_cast<uint4 *>(orow_ptr);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
  *lse_ptr = -INFINITY;
}

}  // namespace vattn
