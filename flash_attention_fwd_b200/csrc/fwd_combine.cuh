/*
 * fwd_combine.cuh — merge of the pieces of split key ranges.
 *
 * Without the causal rule a short-query / long-key sequence gives a handful of
 * long work items, and the persistent CTAs that draw them finish long after
 * the others.  The host then cuts the key range of such items into pieces
 * (KParams::split_tiles); each piece runs as its own work item and writes its
 * partial softmax result — O_i / l_i in float32 and lse_i = m_i + log2 l_i —
 * to the workspace.  This kernel forms, per query row, the softmax over the
 * union of the pieces' keys:
 *
 *     M   = max(max_i lse_i, sink)          (log2 units)
 *     L   = sum_i 2^(lse_i - M) + 2^(sink - M)
 *     O   = sum_i 2^(lse_i - M) / L * O_i
 *     LSE = (M + log2 L) * ln 2
 *
 * which is the same sum of exp(s - m) v over all visible keys, regrouped.
 * The sink term (a per-head extra logit in the normalisation) enters once,
 * here, not in the pieces.
 *
 * With replicated rows (KParams::rep) every key piece of a row comes in rep
 * copies over interleaved key subsets, each a piece of its own here.
 *
 * One warp per row (token, head); lane i reads piece i's LSE (at most 32
 * pieces), and lane c holds columns [c * D/32, (c + 1) * D/32) of O.  Rows of
 * sequences that are not split were written by the attention kernel and are
 * skipped.
 */
#pragma once
#include "fwd_common.cuh"

namespace vattn {
namespace combine {

constexpr int NUM_THREADS = 256;
constexpr int ROWS_PER_CTA = NUM_THREADS / 32;
constexpr int MAX_PARTS = 32;

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS) combine_kernel(const KParams p) {
  constexpr int E = D / 32;  // columns per lane
  static_assert(E == 2 || E == 4 || E == 8, "head dim");
  const int lane = threadIdx.x & 31;
  const bool paged = p.page_table != nullptr;
  const int paged_keys = paged_key_extent(p);
  const long long rows = p.part_rows;
  const long long stride = (long long)gridDim.x * ROWS_PER_CTA;
  for (long long row = (long long)blockIdx.x * ROWS_PER_CTA + threadIdx.x / 32; row < rows;
       row += stride) {
    const int tok = (int)(row / p.H);
    const int h = (int)(row % p.H);
    // the sequence holding token tok: the last b with cu_q[b] <= tok
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(p.cu_q + mid) <= tok)
        lo = mid;
      else
        hi = mid - 1;
    }
    int qs, lq, ks, lk;
    seq_extents(p.cu_q, p.cu_k, p.seqused_k, paged, paged_keys, p.total_q, p.total_k, lo, qs, lq,
                ks, lk);
    if (tok < qs || tok >= qs + lq) continue;  // not a row of any sequence
    int P, base, r;
    const int nk = (lk + BM - 1) / BM;
    kv_pieces(nk, p.split_tiles, p.max_parts, P, base, r);
    if (nk > 0 && p.rep > 1) P *= p.rep;  // every key piece in rep interleaved copies
    if (P <= 1) continue;  // written whole by the attention kernel
    const float lse_i = lane < P ? __ldcg(p.part_lse + (size_t)lane * rows + row) : -INFINITY;
    float M = lse_i;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float sink = sink_log2(p, h);
    M = fmaxf(M, sink);
    const float wgt = (M == -INFINITY || lse_i == -INFINITY) ? 0.f : exp2f(lse_i - M);
    float L = wgt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (sink != -INFINITY) L += exp2f(sink - M);
    const float inv_L = L > 0.f ? 1.f / L : 0.f;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    // UNROLL pieces at a time: their loads are all issued before the first
    // is used, so the latency of the partials is paid once per group
    constexpr int UNROLL = E <= 4 ? 8 : 4;
    const float *src0 = p.part_o + (size_t)row * D + lane * E;
    for (int i0 = 0; i0 < P; i0 += UNROLL) {
      float2 x[UNROLL][E / 2];
      float wi[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int i = i0 + u;
        wi[u] = __shfl_sync(0xffffffffu, wgt, i & 31) * inv_L;
        const float *src = src0 + (size_t)i * rows * D;
#pragma unroll
        for (int e = 0; e < E; e += 2)
          x[u][e / 2] = i < P ? __ldcg(reinterpret_cast<const float2 *>(src + e))
                              : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        if (i0 + u >= P) wi[u] = 0.f;
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          acc[e] += wi[u] * x[u][e / 2].x;
          acc[e + 1] += wi[u] * x[u][e / 2].y;
        }
      }
    }
    uint32_t pk[E / 2];
#pragma unroll
    for (int e = 0; e < E; e += 2) pk[e / 2] = pack2<BF16>(acc[e], acc[e + 1]);
    uint16_t *orow = reinterpret_cast<uint16_t *>(p.out) + (size_t)row * D + lane * E;
    if constexpr (E == 2) {
      *reinterpret_cast<uint32_t *>(orow) = pk[0];
    } else if constexpr (E == 4) {
      *reinterpret_cast<uint2 *>(orow) = make_uint2(pk[0], pk[1]);
    } else {
      *reinterpret_cast<uint4 *>(orow) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    if (lane == 0)
      p.lse[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
  }
}

}  // namespace combine
}  // namespace vattn
