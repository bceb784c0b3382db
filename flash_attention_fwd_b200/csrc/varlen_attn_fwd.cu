/*
 * varlen_attn_fwd.cu — sm_100a (B200) packed variable-length attention
 * forward: host side of the C ABI declared in include/varlen_attn.h.
 *
 * What is computed is the forward loop of boostr 0.2.0,
 * src/ops/cpu/attention/varlen_attention.rs (varlen_attention_fwd): per
 * (sequence b, query head h, query qi) a softmax over the scaled dot products
 * with the keys of the same sequence (GQA head map kv_h = h / (H/Hkv); with
 * causal, key ki is hidden from query qi when qi < ki), the softmax-weighted
 * sum of the values, and LSE = max + ln(sum).  The page computes the softmax
 * in two passes over a full row of scores; the kernels stream the row in key
 * tiles with a running maximum and sum (the "online" form), which reaches the
 * same result up to rounding.  The calling convention (output written into a
 * caller buffer, LSE returned, no dropout) is the out-variant of PyTorch pull
 * request #176015.
 *
 * Kernels (all persistent, one CTA per SM, warp-specialised, tcgen05 MMAs
 * into TMEM fed by TMA):
 *   fwd_pair.cuh    two 128-row query tiles per work item sharing every K/V
 *                   tile (two query heads of one GQA group, or GQA-packed rows
 *                   for short queries), D = 64 / 128, H / Hkv even
 *   fwd_single.cuh  one query tile per work item, every other case
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "fwd_combine.cuh"
#include "fwd_common.cuh"
#include "fwd_pair.cuh"
#include "fwd_single.cuh"
#include "varlen_attn.h"

namespace vattn {

// ====================================================================== host

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// A driver API entry point through the runtime (the library does not link
// libcuda directly); nullptr when the driver does not provide it.
static void *driver_entry(const char *name) {
  void *ptr = nullptr;
  cudaDriverEntryPointQueryResult qres;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
      qres == cudaDriverEntryPointSuccess)
    return ptr;
  return nullptr;
}

// Function-local statics: initialised once, thread-safely (C++11).
static EncodeTiledFn get_encode_fn() {
  static const EncodeTiledFn fn =
      reinterpret_cast<EncodeTiledFn>(driver_entry("cuTensorMapEncodeTiled"));
  return fn;
}

// Unique id of the calling thread's current CUDA context (0 when none is
// current yet, or the driver cannot tell).  Ids are never reused within a
// process, so a device reset, which destroys the context, changes the id.
static unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_cur =
      reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent"));
  static const CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_entry("cuCtxGetId"));
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// [rows, heads, D] row-major 16-bit tensor; box = 64 elements x box_heads
// heads x box_rows rows, written to shared memory (row-major over rows, then
// heads) with the 128-byte swizzle the MMA descriptors expect.
static bool encode_qkv_map(EncodeTiledFn enc, CUtensorMap *map, const void *base, bool bf16,
                           int64_t rows, int heads, int D, int box_rows, int box_heads = 1) {
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Per-device state kept across calls: the SM count and compute capability,
// which kernels have had their shared-memory limit raised, and the address
// of the no-allocation backward's scratch array.  All of it belongs to one
// CUDA context (function attributes and symbol addresses do not survive a
// device reset), so it is tied to the context's unique id and set up again
// when the calling thread's context differs.  Calls from several host
// threads are safe: the set-up runs under the device's mutex.
constexpr int MAX_DEVICES = 64;
constexpr int KERNEL_SLOTS = 26;  // forward 0..9, backward 10..17 and 22..25, replicated rows 18..21
struct DeviceInfo {
  std::mutex mu;
  std::atomic<unsigned long long> ctx_id;  // context the state below belongs to (0: none)
  int sms, major, minor;                   // written under mu before ctx_id is published
  std::atomic<bool> attr_set[KERNEL_SLOTS];
  void *bwd_scratch;                       // under mu
};
static DeviceInfo g_dev[MAX_DEVICES];  // static storage: zero-initialised

// The calling thread's device, its state brought up to date for the current
// context.
static int device_state(DeviceInfo *&dev_out) {
  int dev_id = 0;
  if (cudaGetDevice(&dev_id) != cudaSuccess || dev_id < 0 || dev_id >= MAX_DEVICES)
    return VARLEN_ERR_LAUNCH;
  DeviceInfo &dev = g_dev[dev_id];
  const unsigned long long id = current_context_id();
  if (id == 0 || dev.ctx_id.load(std::memory_order_acquire) != id) {
    std::lock_guard<std::mutex> lock(dev.mu);
    if (id == 0 || dev.ctx_id.load(std::memory_order_relaxed) != id) {
      int sms = 0, mj = 0, mn = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_id) != cudaSuccess ||
          cudaDeviceGetAttribute(&mj, cudaDevAttrComputeCapabilityMajor, dev_id) != cudaSuccess ||
          cudaDeviceGetAttribute(&mn, cudaDevAttrComputeCapabilityMinor, dev_id) != cudaSuccess)
        return VARLEN_ERR_LAUNCH;
      dev.sms = sms;
      dev.major = mj;
      dev.minor = mn;
      for (int i = 0; i < KERNEL_SLOTS; ++i) dev.attr_set[i].store(false, std::memory_order_relaxed);
      dev.bwd_scratch = nullptr;
      dev.ctx_id.store(id, std::memory_order_release);
    }
  }
  dev_out = &dev;
  return VARLEN_OK;
}

// Raises a kernel's dynamic shared-memory limit once per context.  min_regs:
// the kernel rebalances registers between its warpgroups with setmaxnreg and
// relies on the CTA having been launched with at least this many registers
// per thread; a build that reports fewer is never launched (the increase
// would wait for registers that do not exist).
template <class Kernel>
static int prepare_kernel(Kernel kernel, size_t smem, DeviceInfo &dev, int slot,
                          int min_regs = 0) {
  if (dev.attr_set[slot].load(std::memory_order_acquire)) return VARLEN_OK;
  std::lock_guard<std::mutex> lock(dev.mu);
  if (dev.attr_set[slot].load(std::memory_order_relaxed)) return VARLEN_OK;
  if (min_regs > 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || fa.numRegs < min_regs)
      return VARLEN_ERR_LAUNCH;
  }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return VARLEN_ERR_LAUNCH;
  dev.attr_set[slot].store(true, std::memory_order_release);
  return VARLEN_OK;
}

template <class Kernel>
static int launch_kernel(Kernel kernel, size_t smem, int threads, const CUtensorMap &tq,
                         const CUtensorMap &tk, const CUtensorMap &tv, const KParams &kp,
                         int grid, cudaStream_t stream, DeviceInfo &dev, int slot,
                         int min_regs = 0) {
  if (const int rc = prepare_kernel(kernel, smem, dev, slot, min_regs)) return rc;
  kernel<<<grid, threads, smem, stream>>>(tq, tk, tv, kp);
  return cudaGetLastError() == cudaSuccess ? VARLEN_OK : VARLEN_ERR_LAUNCH;
}

template <int D, bool BF16>
static int launch_single(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                         const KParams &kp, int grid, cudaStream_t s, DeviceInfo &dev, int slot) {
  constexpr size_t smem = single::smem_bytes<D>();
  static_assert(smem <= 232448, "shared memory budget");
  return launch_kernel(single::fwd_kernel<D, BF16>, smem, single::NUM_THREADS, tq, tk, tv, kp,
                       grid, s, dev, slot);
}

template <int D, bool BF16>
static int launch_pair(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                       const KParams &kp, int grid, cudaStream_t s, DeviceInfo &dev, int slot) {
  constexpr size_t smem = pair::smem_bytes<D>();
  static_assert(smem <= 232448, "shared memory budget");
  // replicated rows: its own instantiation, attribute slots 18..21 (the
  // forward uses 0..9, the backward 10..17)
  if (kp.rep > 1)
    return launch_kernel(pair::fwd_kernel<D, BF16, true>, smem, pair::NUM_THREADS, tq, tk, tv, kp,
                         grid, s, dev, slot + 18, (int)pair::REG_LAUNCH);
  return launch_kernel(pair::fwd_kernel<D, BF16, false>, smem, pair::NUM_THREADS, tq, tk, tv, kp,
                       grid, s, dev, slot, (int)pair::REG_LAUNCH);
}

static bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <int D, bool BF16>
static int launch_combine(const KParams &kp, int sms, cudaStream_t s) {
  const long long blocks = (kp.part_rows + combine::ROWS_PER_CTA - 1) / combine::ROWS_PER_CTA;
  const int grid = (int)(blocks < (long long)sms * 16 ? blocks : (long long)sms * 16);
  combine::combine_kernel<D, BF16><<<grid < 1 ? 1 : grid, combine::NUM_THREADS, 0, s>>>(kp);
  return cudaGetLastError() == cudaSuccess ? VARLEN_OK : VARLEN_ERR_LAUNCH;
}

// Which kernel serves a call, and how it cuts the queries into work items.
struct FwdLayout {
  bool use_pair;    // pair kernel (two query tiles per item sharing K/V)
  int pack_log2;    // GQA packing (see KParams::pack_log2)
  int head_units;   // head units per (sequence, token range)
  int unit_tokens;  // query tokens per work item
  int rep;          // replicated rows (see KParams::rep): 4, or 1
};
static FwdLayout fwd_layout(int max_seqlen_q, int num_heads, int num_kv_heads, int D,
                            bool rep = false) {
  FwdLayout L;
  const int group = num_heads / num_kv_heads;
  // Query-head pairs share a key/value head when the group size is even;
  // the pair kernel then covers D = 64 and 128 (TMEM holds 2 x (S + O)).
  L.use_pair = (group % 2 == 0) && (D == 64 || D == 128);
  // GQA packing: a tile's 128 rows = (128 / group) tokens x the group's query
  // heads.  It pays when query sequences are short next to a 128-row tile
  // (most rows of a per-head tile would be empty); group must be a power of
  // two dividing 128.
  L.pack_log2 = 0;
  if (L.use_pair && (group & (group - 1)) == 0 && group <= BM) {
    const bool short_q = (long long)max_seqlen_q * 2 <= BM;
    if (short_q)
      while ((1 << L.pack_log2) < group) ++L.pack_log2;
  }
  L.head_units = L.pack_log2 ? num_kv_heads : (L.use_pair ? num_heads / 2 : num_heads);
  L.unit_tokens = L.pack_log2 ? 2 * (BM >> L.pack_log2) : BM;
  L.rep = 1;
  if (rep && L.pack_log2 > 0) {  // replicated rows: 32 rows (32 >> pack tokens) per item
    L.rep = 4;
    L.unit_tokens = 32 >> L.pack_log2;
  }
  return L;
}

// The replicated-rows form (KParams::rep) applies to GQA-packed calls whose
// items have at most 32 query rows (max_seqlen_q x H / Hkv <= 32) and whose
// key ranges reach 8 tiles, so that the merge launch pays; without a causal
// rule or a window, and only when the caller gives a workspace.
static bool rep_eligible(int max_seqlen_q, int max_seqlen_k, int num_heads, int num_kv_heads,
                         int D) {
  const FwdLayout L = fwd_layout(max_seqlen_q, num_heads, num_kv_heads, D);
  return L.pack_log2 > 0 && L.pack_log2 <= 5 && ((long long)max_seqlen_q << L.pack_log2) <= 32 &&
         max_seqlen_k >= 8 * BM;
}

// Key tiles per piece and the largest piece count when a call asks for at
// most num_splits pieces per key range (no split: num_splits <= 1, a causal
// rule or a window, or no sequence long enough to be cut).
static void split_plan(int num_splits, int max_seqlen_k, bool masked, int &split_tiles,
                       int &max_parts) {
  split_tiles = 0;
  max_parts = 1;
  if (num_splits <= 1 || masked || max_seqlen_k <= 0) return;
  const int nk_max = (int)(((long long)max_seqlen_k + BM - 1) / BM);
  const int S = (nk_max + num_splits - 1) / num_splits;
  if (S < 1 || nk_max <= S) return;
  split_tiles = S;
  max_parts = (nk_max + S - 1) / S;
}

// Piece count chosen when the caller leaves it to the library.  A piece is a
// work item of its own (Q load, pipeline start, epilogue) and the merge is a
// second launch over float32 partials of every row, so a split pays only when
// the work items alone cannot fill the GPU (fewer than 3/4 as many items as
// SMs): then each key range is cut into up to 16 pieces of at least 16 key
// tiles, so that the pieces of the few long items spread over all SMs in
// several rounds that the cost-ordered dealing evens out (replicated-row
// calls: see below).  Measured on B200:
// 8 single-query sequences x 8 KV heads x 32k keys, 0.61 ms unsplit, 0.27 ms
// in 16 pieces; 208 short-query items over up to 63 key tiles (the
// short-query / long-KV batch), every split slower than none.
static int auto_num_splits(int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                           int max_seqlen_k, int num_heads, int num_kv_heads, int D, bool masked,
                           bool paged, int sms, bool rep) {
  (void)total_k;
  (void)paged;
  if (masked || batch <= 0 || max_seqlen_k <= 0 || max_seqlen_q <= 0 || sms <= 0) return 1;
  const FwdLayout L = fwd_layout(max_seqlen_q, num_heads, num_kv_heads, D, rep);
  const double nk_max = ceil((double)max_seqlen_k / BM);
  const double q_mean = fmin((double)total_q / batch, (double)max_seqlen_q);
  const double items = (double)batch * fmax(1.0, ceil(q_mean / L.unit_tokens)) * L.head_units;
  if (rep) {
    // replicated rows: items are short and the merge is cheap (few rows), so
    // pieces of about 32 key tiles even out ragged key ranges unless there are
    // plenty of items (measured: 64 ragged 1k-16k sequences, 512 items,
    // 0.441 ms in one piece, 0.397 ms in 4)
    // (pieces of 16 tiles when the items alone leave SMs idle)
    if (items >= 4.0 * sms) return 1;
    const double tiles = items < 0.75 * sms ? 16.0 : 32.0;
    const double ns = fmin((double)(combine::MAX_PARTS / 4), floor(nk_max / tiles));
    return ns < 2.0 ? 1 : (int)ns;
  }
  if (items >= 0.75 * sms) return 1;
  const double ns = fmin(16.0, floor(nk_max / 16.0));
  return ns < 2.0 ? 1 : (ns > combine::MAX_PARTS ? combine::MAX_PARTS : (int)ns);
}

static size_t split_workspace_bytes(int64_t total_q, int num_heads, int D, int max_parts) {
  return (size_t)max_parts * (size_t)total_q * (size_t)num_heads * (size_t)(D + 1) * 4u;
}

}  // namespace vattn

using namespace vattn;

static int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Common body of the entry points.  window_left / window_right < 0 mean "no
// bound"; seqused_k may be NULL unless page_table is given; page_table NULL =
// packed k/v.
static int fwd_impl(const void *q, const void *k, const void *v, const int32_t *cu_seqlens_q,
                    const int32_t *cu_seqlens_k, int batch, int64_t total_q, int64_t total_k,
                    int max_seqlen_q, int max_seqlen_k, int num_heads, int num_kv_heads,
                    int head_dim, int causal, float scale, int window_left, int window_right,
                    const int32_t *seqused_k, const int32_t *page_table, int page_table_stride,
                    int page_size, const float *sinks, int num_splits, void *workspace,
                    size_t workspace_bytes, varlen_dtype_t dtype, void *out, float *lse,
                    varlen_stream_t stream) {
  const bool paged = page_table != nullptr;
  // ---- host-side validation: nothing is launched or touched on error
  if (dtype != VARLEN_BF16 && dtype != VARLEN_FP16) return VARLEN_ERR_DTYPE;
  if (batch < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
    return VARLEN_ERR_SHAPE;
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return VARLEN_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return VARLEN_ERR_SHAPE;
  if (total_q >= (int64_t(1) << 31) || total_k >= (int64_t(1) << 31)) return VARLEN_ERR_SHAPE;
  if (num_heads > 65535) return VARLEN_ERR_SHAPE;
  if (paged && (page_size < 16 || page_size % 16 != 0 || page_table_stride < 1 ||
                total_k % page_size != 0))
    return VARLEN_ERR_SHAPE;
  if (batch > 0 && (!cu_seqlens_q || (!paged && !cu_seqlens_k))) return VARLEN_ERR_NULL;
  if (paged && batch > 0 && !seqused_k) return VARLEN_ERR_NULL;
  if (total_q > 0 && (!q || !out || !lse)) return VARLEN_ERR_NULL;
  if (total_k > 0 && (!k || !v)) return VARLEN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return VARLEN_ERR_ALIGN;
  if (!aligned(lse, 4) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4) ||
      !aligned(seqused_k, 4) || !aligned(page_table, 4) || !aligned(sinks, 4))
    return VARLEN_ERR_ALIGN;
  if (num_splits < 0 || num_splits > combine::MAX_PARTS) return VARLEN_ERR_SHAPE;
  if (batch == 0 || total_q == 0) return VARLEN_OK;

  DeviceInfo *devp = nullptr;
  if (const int rc = device_state(devp)) return rc;
  DeviceInfo &dev = *devp;
  if (dev.major != 10 || dev.minor != 0) return VARLEN_ERR_ARCH;

  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return VARLEN_ERR_LAUNCH;
  const bool bf16 = dtype == VARLEN_BF16;
  const int D = head_dim;
  const int group = num_heads / num_kv_heads;
  // Window bounds in canonical form: a bound that no query of the buffers can
  // reach is dropped (this also keeps qi - left and qi + right + 1 in range),
  // and the causal rule is the right bound 0.
  // (a sequence has at most total_k keys, or page_table_stride pages of keys when paged: pages
  // may be shared, so a paged sequence can hold more keys than the cache has rows)
  const int64_t key_extent = paged ? (int64_t)page_table_stride * page_size : total_k;
  int win_left = (window_left >= 0 && (int64_t)window_left < total_q) ? window_left : -1;
  int win_right = (window_right >= 0 && (int64_t)window_right < key_extent) ? window_right : -1;
  if (causal) win_right = 0;
  const bool masked = win_left >= 0 || win_right >= 0;
  const bool rep = !masked && workspace != nullptr &&
                   rep_eligible(max_seqlen_q, max_seqlen_k, num_heads, num_kv_heads, D);
  const FwdLayout layout = fwd_layout(max_seqlen_q, num_heads, num_kv_heads, D, rep);
  const bool use_pair = layout.use_pair;
  const int pack_log2 = layout.pack_log2;
  const int BN = use_pair ? pair::BN : (D == 256 ? single::Cfg<256>::BN : single::Cfg<128>::BN);
  alignas(64) CUtensorMap tq, tk, tv;
  memset(&tk, 0, sizeof tk);
  memset(&tv, 0, sizeof tv);
  // a query box is one tile of 128 rows, or one copy of 32 rows with replicated rows
  if (!encode_qkv_map(enc, &tq, q, bf16, total_q, num_heads, D,
                      (layout.rep > 1 ? 32 : BM) >> pack_log2, 1 << pack_log2))
    return VARLEN_ERR_LAUNCH;
  // paged: a key tile is fetched as boxes of `chunk` rows, which divide both
  // the page and the tile, so that no box crosses a page
  const int chunk = paged ? gcd_int(page_size, BN) : BN;
  if (total_k > 0) {
    if (!encode_qkv_map(enc, &tk, k, bf16, total_k, num_kv_heads, D, chunk) ||
        !encode_qkv_map(enc, &tv, v, bf16, total_k, num_kv_heads, D, chunk))
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
  kp.group = group;
  kp.head_units = layout.head_units;
  kp.unit_tokens = layout.unit_tokens;
  kp.pack_log2 = pack_log2;
  kp.total_q = (int)total_q;
  kp.total_k = (int)total_k;
  kp.causal = causal ? 1 : 0;
  const float sc = (scale > 0.f) ? scale : 1.0f / sqrtf((float)D);  // NaN fails "> 0"
  kp.scale_log2 = sc * 1.4426950408889634f;
  kp.seqused_k = seqused_k;
  kp.win_left = win_left;
  kp.win_right = win_right;
  // folded causal units for the single kernel (one query tile per item): the
  // query tiles of a sequence would otherwise run in different cost rounds, and
  // with no GQA sharing their K/V prefixes leave the L2 in between
  kp.fold = (!use_pair && causal && win_left < 0 && layout.unit_tokens == BM) ? 1 : 0;
  kp.page_table = page_table;
  kp.pt_stride = paged ? page_table_stride : 0;
  kp.page_size = paged ? page_size : 0;
  kp.num_pages = paged ? (int)(total_k / page_size) : 0;
  kp.page_chunk = chunk;
  kp.sinks = sinks;
  // Key-range split (non-causal, windowless calls) and replicated rows:
  // pieces merged by the combine kernel through the caller's workspace.
  kp.rep = layout.rep;
  if (num_splits == 0)
    num_splits = auto_num_splits(batch, total_q, total_k, max_seqlen_q, max_seqlen_k, num_heads,
                                 num_kv_heads, D, masked, paged, dev.sms, rep);
  if (num_splits > combine::MAX_PARTS / kp.rep) num_splits = combine::MAX_PARTS / kp.rep;
  split_plan(num_splits, max_seqlen_k, masked, kp.split_tiles, kp.max_parts);
  kp.part_rows = (long long)total_q * num_heads;
  kp.part_o = nullptr;
  kp.part_lse = nullptr;
  kp.out_v8 = aligned(out, 32) ? 1 : 0;
  kp.part_v8 = aligned(workspace, 32) ? 1 : 0;
  if (kp.split_tiles > 0 || kp.rep > 1) {
    const int slots = kp.max_parts * kp.rep;
    const size_t need = split_workspace_bytes(total_q, num_heads, D, slots);
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < need)
      return VARLEN_ERR_WORKSPACE;
    kp.part_o = static_cast<float *>(workspace);
    kp.part_lse = kp.part_o + (size_t)slots * (size_t)kp.part_rows * D;
  }

  // Upper bound of work items from max_seqlen_q; at least one CTA so that an
  // understated bound never drops work (the CTAs loop over all items).
  long long max_items =
      (long long)batch * ((max_seqlen_q + kp.unit_tokens - 1) / kp.unit_tokens) * kp.head_units *
      kp.max_parts;
  int grid = dev.sms;
  if (max_items >= 1 && max_items < grid) grid = (int)max_items;
  if (grid < 1) grid = 1;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int rc;
  if (use_pair) {
    if (D == 64)
      rc = bf16 ? launch_pair<64, true>(tq, tk, tv, kp, grid, s, dev, 0)
                : launch_pair<64, false>(tq, tk, tv, kp, grid, s, dev, 1);
    else
      rc = bf16 ? launch_pair<128, true>(tq, tk, tv, kp, grid, s, dev, 2)
                : launch_pair<128, false>(tq, tk, tv, kp, grid, s, dev, 3);
  } else {
    switch (D) {
      case 64:
        rc = bf16 ? launch_single<64, true>(tq, tk, tv, kp, grid, s, dev, 4)
                  : launch_single<64, false>(tq, tk, tv, kp, grid, s, dev, 5);
        break;
      case 128:
        rc = bf16 ? launch_single<128, true>(tq, tk, tv, kp, grid, s, dev, 6)
                  : launch_single<128, false>(tq, tk, tv, kp, grid, s, dev, 7);
        break;
      default:
        rc = bf16 ? launch_single<256, true>(tq, tk, tv, kp, grid, s, dev, 8)
                  : launch_single<256, false>(tq, tk, tv, kp, grid, s, dev, 9);
    }
  }
  if (rc != VARLEN_OK || (kp.split_tiles == 0 && kp.rep == 1)) return rc;
  switch (D) {
    case 64:
      return bf16 ? launch_combine<64, true>(kp, dev.sms, s) : launch_combine<64, false>(kp, dev.sms, s);
    case 128:
      return bf16 ? launch_combine<128, true>(kp, dev.sms, s)
                  : launch_combine<128, false>(kp, dev.sms, s);
    default:
      return bf16 ? launch_combine<256, true>(kp, dev.sms, s)
                  : launch_combine<256, false>(kp, dev.sms, s);
  }
}

extern "C" int varlen_attn_fwd_v1(const void *q, const void *k, const void *v,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_kv_heads, int head_dim,
                                  int causal, float scale, varlen_dtype_t dtype, void *out,
                                  float *lse, varlen_stream_t stream) {
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, num_heads, num_kv_heads, head_dim, causal, scale, -1, -1, nullptr,
                  nullptr, 0, 0, nullptr, 1, nullptr, 0, dtype, out, lse, stream);
}

extern "C" int varlen_attn_fwd_v2(const void *q, const void *k, const void *v,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_kv_heads, int head_dim,
                                  int causal, float scale, int window_left, int window_right,
                                  const int32_t *seqused_k, varlen_dtype_t dtype, void *out,
                                  float *lse, varlen_stream_t stream) {
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, num_heads, num_kv_heads, head_dim, causal, scale, window_left,
                  window_right, seqused_k, nullptr, 0, 0, nullptr, 1, nullptr, 0, dtype, out, lse,
                  stream);
}

extern "C" int varlen_attn_fwd_v3(const void *q, const void *k, const void *v,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_kv_heads, int head_dim,
                                  int causal, float scale, int window_left, int window_right,
                                  const int32_t *seqused_k, const int32_t *page_table,
                                  int page_table_stride, int page_size, const float *sinks,
                                  varlen_dtype_t dtype, void *out, float *lse,
                                  varlen_stream_t stream) {
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, num_heads, num_kv_heads, head_dim, causal, scale, window_left,
                  window_right, seqused_k, page_table, page_table_stride, page_size, sinks, 1,
                  nullptr, 0, dtype, out, lse, stream);
}

extern "C" int varlen_attn_fwd_v4(const void *q, const void *k, const void *v,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_kv_heads, int head_dim,
                                  int causal, float scale, int window_left, int window_right,
                                  const int32_t *seqused_k, const int32_t *page_table,
                                  int page_table_stride, int page_size, const float *sinks,
                                  int num_splits, void *workspace, size_t workspace_bytes,
                                  varlen_dtype_t dtype, void *out, float *lse,
                                  varlen_stream_t stream) {
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, num_heads, num_kv_heads, head_dim, causal, scale, window_left,
                  window_right, seqused_k, page_table, page_table_stride, page_size, sinks,
                  num_splits, workspace, workspace_bytes, dtype, out, lse, stream);
}

extern "C" int varlen_attn_fwd_num_splits(int batch, int64_t total_q, int64_t total_k,
                                          int max_seqlen_q, int max_seqlen_k, int num_heads,
                                          int num_kv_heads, int head_dim, int causal,
                                          int window_left, int window_right, int paged,
                                          int num_sms) {
  if (batch < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 ||
      num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      (head_dim != 64 && head_dim != 128 && head_dim != 256))
    return VARLEN_ERR_SHAPE;
  if (num_sms <= 0) {
    DeviceInfo *dev = nullptr;
    if (const int rc = device_state(dev)) return rc;
    num_sms = dev->sms;
  }
  const bool masked = causal || window_left >= 0 || window_right >= 0;
  const bool rep =
      !masked && rep_eligible(max_seqlen_q, max_seqlen_k, num_heads, num_kv_heads, head_dim);
  const int n = auto_num_splits(batch, total_q, total_k, max_seqlen_q, max_seqlen_k, num_heads,
                                num_kv_heads, head_dim, masked, paged != 0, num_sms, rep);
  return rep && n > combine::MAX_PARTS / 4 ? combine::MAX_PARTS / 4 : n;
}

extern "C" size_t varlen_attn_fwd_workspace_size(int64_t total_q, int num_heads,
                                                 int num_kv_heads, int head_dim, int max_seqlen_q,
                                                 int max_seqlen_k, int num_splits) {
  if (total_q <= 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      (head_dim != 64 && head_dim != 128 && head_dim != 256) || max_seqlen_q < 0 ||
      num_splits < 1 || num_splits > combine::MAX_PARTS)
    return 0;
  const int rep =
      rep_eligible(max_seqlen_q, max_seqlen_k, num_heads, num_kv_heads, head_dim) ? 4 : 1;
  if (num_splits > combine::MAX_PARTS / rep) num_splits = combine::MAX_PARTS / rep;
  int split_tiles, max_parts;
  split_plan(num_splits, max_seqlen_k, false, split_tiles, max_parts);
  return (split_tiles > 0 || rep > 1)
             ? split_workspace_bytes(total_q, num_heads, head_dim, max_parts * rep)
             : 0;
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
      return "device-side status word is set (a bounded pipeline wait timed out, or a page-table "
             "entry was out of range)";
    case VARLEN_ERR_ARCH:
      return "current device is not compute capability 10.0 (sm_100a build)";
    case VARLEN_ERR_WORKSPACE:
      return "workspace missing, not 16-byte aligned, or smaller than "
             "varlen_attn_fwd_workspace_size() / varlen_attn_bwd_workspace_size()";
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

extern "C" int varlen_attn_set_wait_limit(unsigned long long ns) {
  const unsigned long long v = ns ? ns : WAIT_TIMEOUT_NS;
  return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof v) == cudaSuccess ? VARLEN_OK
                                                                           : VARLEN_ERR_LAUNCH;
}

extern "C" int varlen_attn_abi_version(void) { return 6; }

// Backward entry points (same translation unit: one device status word).
#include "bwd_host.cuh"
