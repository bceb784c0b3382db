/*
 * bwd_host.cuh — host side of the backward entry points declared in
 * include/varlen_attn.h (varlen_attn_bwd_workspace_size, varlen_attn_bwd_v1).
 * Included by varlen_attn_fwd.cu so that both directions share one device
 * status word and one set of host helpers.
 *
 * The computation is the page's varlen_attention_bwd (boostr 0.2.0,
 * src/ops/cpu/attention/varlen_attention.rs), split into two kernels that
 * run back to back on the caller's stream:
 *   1. bwd_dq::dq_kernel    dQ, and delta = <dO, O> into the workspace
 *   2. bwd_dkdv::dkdv_kernel dK and dV (reads delta)
 */
#pragma once
#include "bwd_dkdv.cuh"
#include "bwd_dq.cuh"

namespace vattn {

template <class Kernel>
static int launch_bwd_kernel(Kernel kernel, size_t smem, int threads, const CUtensorMap &t0,
                             const CUtensorMap &t1, const CUtensorMap &t2, const CUtensorMap &t3,
                             const BwdParams &bp, int grid, cudaStream_t stream, DeviceInfo &dev,
                             int slot) {
  if (const int rc = prepare_kernel(kernel, smem, dev, slot)) return rc;
  kernel<<<grid, threads, smem, stream>>>(t0, t1, t2, t3, bp);
  return cudaGetLastError() == cudaSuccess ? VARLEN_OK : VARLEN_ERR_LAUNCH;
}

template <int D, bool BF16>
static int launch_bwd(const CUtensorMap (&m_dq)[4], const CUtensorMap (&m_kv)[4],
                      const BwdParams &bp, int grid_q, int grid_k, bool run_dq, bool run_dkdv,
                      cudaStream_t s, DeviceInfo &dev, int slot) {
  constexpr size_t smem_q = bwd_dq::smem_bytes<D>();
  constexpr size_t smem_k = bwd_dkdv::smem_bytes<D>();
  static_assert(smem_q <= 232448 && smem_k <= 232448, "shared memory budget");
  int rc = VARLEN_OK;
  if (run_dq)
    rc = launch_bwd_kernel(bwd_dq::dq_kernel<D, BF16>, smem_q, bwd_dq::NUM_THREADS, m_dq[0],
                           m_dq[1], m_dq[2], m_dq[3], bp, grid_q, s, dev, slot);
  if (rc == VARLEN_OK && run_dkdv)
    rc = launch_bwd_kernel(bwd_dkdv::dkdv_kernel<D, BF16>, smem_k, bwd_dkdv::NUM_THREADS,
                           m_kv[0], m_kv[1], m_kv[2], m_kv[3], bp, grid_k, s, dev, slot + 1);
  return rc;
}

}  // namespace vattn

extern "C" size_t varlen_attn_bwd_workspace_size(int64_t total_q, int num_heads) {
  if (total_q <= 0 || num_heads <= 0) return 0;
  return ((size_t)total_q * (size_t)num_heads * sizeof(float) + 255) & ~(size_t)255;
}

namespace vattn {

// Host-side validation of the backward's arguments except the workspace:
// nothing is launched or touched on error.
static int bwd_check_args(const void *dout, const void *q, const void *k, const void *v,
                          const void *out, const float *lse, const int32_t *cu_seqlens_q,
                          const int32_t *cu_seqlens_k, int batch, int64_t total_q,
                          int64_t total_k, int max_seqlen_q, int max_seqlen_k, int num_heads,
                          int num_kv_heads, int head_dim, varlen_dtype_t dtype, const void *dq,
                          const void *dk, const void *dv) {
  if (dtype != VARLEN_BF16 && dtype != VARLEN_FP16) return VARLEN_ERR_DTYPE;
  if (batch < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
    return VARLEN_ERR_SHAPE;
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return VARLEN_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return VARLEN_ERR_SHAPE;
  if (total_q >= (int64_t(1) << 31) || total_k >= (int64_t(1) << 31)) return VARLEN_ERR_SHAPE;
  if (num_heads > 65535) return VARLEN_ERR_SHAPE;
  if (batch > 0 && (!cu_seqlens_q || !cu_seqlens_k)) return VARLEN_ERR_NULL;
  if (total_q > 0 && (!dout || !q || !out || !lse || !dq)) return VARLEN_ERR_NULL;
  if (total_k > 0 && (!k || !v || !dk || !dv)) return VARLEN_ERR_NULL;
  if (!aligned(dout, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
      !aligned(out, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
    return VARLEN_ERR_ALIGN;
  if (!aligned(lse, 4) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
    return VARLEN_ERR_ALIGN;
  return VARLEN_OK;
}

}  // namespace vattn

extern "C" int varlen_attn_bwd_v1(const void *dout, const void *q, const void *k, const void *v,
                                  const void *out, const float *lse,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_kv_heads, int head_dim,
                                  int causal, float scale, varlen_dtype_t dtype, void *dq,
                                  void *dk, void *dv, void *workspace, size_t workspace_bytes,
                                  varlen_stream_t stream) {
  using namespace vattn;
  int rc = bwd_check_args(dout, q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, batch, total_q,
                          total_k, max_seqlen_q, max_seqlen_k, num_heads, num_kv_heads, head_dim,
                          dtype, dq, dk, dv);
  if (rc != VARLEN_OK) return rc;
  if (!aligned(workspace, 16)) return VARLEN_ERR_ALIGN;
  if (total_q > 0 &&
      (!workspace || workspace_bytes < varlen_attn_bwd_workspace_size(total_q, num_heads)))
    return VARLEN_ERR_WORKSPACE;
  if (batch == 0 || (total_q == 0 && total_k == 0)) return VARLEN_OK;

  DeviceInfo *devp = nullptr;
  if (const int rc = device_state(devp)) return rc;
  DeviceInfo &dev = *devp;
  if (dev.major != 10 || dev.minor != 0) return VARLEN_ERR_ARCH;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return VARLEN_ERR_LAUNCH;
  const bool bf16 = dtype == VARLEN_BF16;
  const int D = head_dim;

  // tensor maps: dQ pass (Q, dO tiles of 128 rows; K, V tiles of its key
  // tile), dK/dV pass (Q, dO tiles of its query step; K, V tiles of 128)
  const int dq_bn = D == 256 ? bwd_dq::Cfg<256>::BN : bwd_dq::Cfg<128>::BN;
  const int kv_bq = D == 256 ? bwd_dkdv::Cfg<256>::BQ : bwd_dkdv::Cfg<128>::BQ;
  const int kv_nh = D == 256 ? bwd_dkdv::Cfg<256>::NH : bwd_dkdv::Cfg<128>::NH;
  alignas(64) CUtensorMap m_dq[4], m_kv[4];
  memset(m_dq, 0, sizeof m_dq);
  memset(m_kv, 0, sizeof m_kv);
  if (total_q > 0) {
    if (!encode_qkv_map(enc, &m_dq[0], q, bf16, total_q, num_heads, D, BM) ||
        !encode_qkv_map(enc, &m_dq[1], dout, bf16, total_q, num_heads, D, BM) ||
        !encode_qkv_map(enc, &m_kv[0], q, bf16, total_q, num_heads, D, kv_bq) ||
        !encode_qkv_map(enc, &m_kv[1], dout, bf16, total_q, num_heads, D, kv_bq))
      return VARLEN_ERR_LAUNCH;
  }
  if (total_k > 0) {
    if (!encode_qkv_map(enc, &m_dq[2], k, bf16, total_k, num_kv_heads, D, dq_bn) ||
        !encode_qkv_map(enc, &m_dq[3], v, bf16, total_k, num_kv_heads, D, dq_bn) ||
        !encode_qkv_map(enc, &m_kv[2], k, bf16, total_k, num_kv_heads, D, bwd_dkdv::BK) ||
        !encode_qkv_map(enc, &m_kv[3], v, bf16, total_k, num_kv_heads, D, bwd_dkdv::BK))
      return VARLEN_ERR_LAUNCH;
  }

  BwdParams bp;
  memset(&bp, 0, sizeof bp);
  KParams &kp = bp.kp;
  kp.cu_q = cu_seqlens_q;
  kp.cu_k = cu_seqlens_k;
  kp.B = batch;
  kp.H = num_heads;
  kp.Hkv = num_kv_heads;
  kp.group = num_heads / num_kv_heads;
  kp.head_units = num_heads;
  kp.unit_tokens = BM;
  kp.pack_log2 = 0;
  kp.total_q = (int)total_q;
  kp.total_k = (int)total_k;
  kp.causal = causal ? 1 : 0;
  const float sc = (scale > 0.f) ? scale : 1.0f / sqrtf((float)D);
  kp.scale_log2 = sc * 1.4426950408889634f;
  kp.win_left = -1;
  kp.win_right = causal ? 0 : -1;
  bp.dout = static_cast<const uint16_t *>(dout);
  bp.o = static_cast<const uint16_t *>(out);
  bp.lse = lse;
  bp.delta = static_cast<float *>(workspace);
  bp.dq = static_cast<uint16_t *>(dq);
  bp.dk = static_cast<uint16_t *>(dk);
  bp.dv = static_cast<uint16_t *>(dv);
  bp.scale = sc;
  bp.v8 = (aligned(dq, 32) && aligned(dk, 32) && aligned(dv, 32)) ? 1 : 0;

  long long items_q = (long long)batch * ((max_seqlen_q + BM - 1) / BM) * num_heads;
  long long items_k = (long long)batch * ((max_seqlen_k + bwd_dkdv::BK - 1) / bwd_dkdv::BK) *
                      num_kv_heads * kv_nh;
  int grid_q = dev.sms, grid_k = dev.sms;
  if (items_q >= 1 && items_q < grid_q) grid_q = (int)items_q;
  if (items_k >= 1 && items_k < grid_k) grid_k = (int)items_k;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool run_dq = total_q > 0, run_dkdv = total_k > 0;
  if (D == 64)
    return bf16 ? launch_bwd<64, true>(m_dq, m_kv, bp, grid_q, grid_k, run_dq, run_dkdv, s, dev,
                                       10)
                : launch_bwd<64, false>(m_dq, m_kv, bp, grid_q, grid_k, run_dq, run_dkdv, s,
                                        dev, 12);
  if (D == 256)
    return bf16 ? launch_bwd<256, true>(m_dq, m_kv, bp, grid_q, grid_k, run_dq, run_dkdv, s,
                                        dev, 22)
                : launch_bwd<256, false>(m_dq, m_kv, bp, grid_q, grid_k, run_dq, run_dkdv, s,
                                         dev, 24);
  return bf16 ? launch_bwd<128, true>(m_dq, m_kv, bp, grid_q, grid_k, run_dq, run_dkdv, s, dev,
                                      14)
              : launch_bwd<128, false>(m_dq, m_kv, bp, grid_q, grid_k, run_dq, run_dkdv, s, dev,
                                       16);
}

// ---------------------------------------------------------------------------
// varlen_attn_bwd_noalloc: the backward with its scratch (delta, float32
// [total_q, H]) in a fixed file-scope device array instead of a caller
// workspace.  NOALLOC_SCRATCH_BYTES bounds total_q * H * 4 (16 MiB: 4,194,304
// (token, head) rows, e.g. 65,536 tokens x 64 heads).  The array's device
// address is looked up with cudaGetSymbolAddress on the first call in each
// CUDA context (with the device current) and kept with the device's other
// per-context state, so a device reset leads to a fresh lookup.  Nothing in
// the scratch has to start at zero: every delta the dK/dV pass reads is
// written by the dQ pass of the same call.  All calls on a device share the
// array, so calls that overlap in time (other streams, other host threads)
// race on it.
namespace vattn {
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_bwd_scratch[NOALLOC_SCRATCH_BYTES];
}  // namespace vattn

extern "C" int varlen_attn_bwd_noalloc(const void *dout, const void *q, const void *k,
                                       const void *v, const void *out, const float *lse,
                                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                       int batch, int64_t total_q, int64_t total_k,
                                       int max_seqlen_q, int max_seqlen_k, int num_heads,
                                       int num_kv_heads, int head_dim, int causal, float scale,
                                       varlen_dtype_t dtype, void *dq, void *dk, void *dv,
                                       varlen_stream_t stream) {
  using namespace vattn;
  int rc = bwd_check_args(dout, q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, batch, total_q,
                          total_k, max_seqlen_q, max_seqlen_k, num_heads, num_kv_heads, head_dim,
                          dtype, dq, dk, dv);
  if (rc != VARLEN_OK) return rc;
  if (varlen_attn_bwd_workspace_size(total_q, num_heads) > NOALLOC_SCRATCH_BYTES)
    return VARLEN_ERR_WORKSPACE;
  if (batch == 0 || (total_q == 0 && total_k == 0)) return VARLEN_OK;
  DeviceInfo *devp = nullptr;
  if ((rc = device_state(devp)) != VARLEN_OK) return rc;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(devp->mu);
    if (!devp->bwd_scratch) {
      void *addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_bwd_scratch) != cudaSuccess || !addr)
        return VARLEN_ERR_LAUNCH;
      devp->bwd_scratch = addr;
    }
    scratch = devp->bwd_scratch;
  }
  return varlen_attn_bwd_v1(dout, q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, batch, total_q,
                            total_k, max_seqlen_q, max_seqlen_k, num_heads, num_kv_heads,
                            head_dim, causal, scale, dtype, dq, dk, dv, scratch,
                            NOALLOC_SCRATCH_BYTES, stream);
}
