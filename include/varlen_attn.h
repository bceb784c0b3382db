/*
 * varlen_attn.h — C ABI of the B200 (sm_100a) variable-length attention
 * forward.
 *
 * The operation is the packed ("varlen") scaled-dot-product attention
 * forward of boostr 0.2.0, src/ops/cpu/attention/varlen_attention.rs
 * (VarLenAttentionOps::varlen_attention_fwd): for every sequence b, query
 * head h and sequence-local query index qi,
 *
 *   kv_h = h / (H / Hkv)                                   (GQA head map)
 *   s_ki = scale * <Q[cu_q[b]+qi, h, :], K[cu_k[b]+ki, kv_h, :]>
 *          for the keys ki in [0, Lk_b) that are visible: with causal != 0
 *          key ki is hidden from query qi when qi < ki (sequence-local
 *          indices, i.e. the mask is aligned at the top-left corner)
 *   O[cu_q[b]+qi, h, :] = sum_ki softmax(s)_ki * V[cu_k[b]+ki, kv_h, :]
 *   LSE[cu_q[b]+qi, h]  = max_ki s_ki + ln(sum_ki exp(s_ki - max))
 *
 * The calling convention follows the out-variant of PyTorch pull request
 * #176015 "[varlen_attn for inference] add out variant"
 * (_flash_attention_forward_no_dropout_inplace): the attention output is
 * written into a caller-provided buffer, the softmax log-sum-exp is returned
 * too, and there is no dropout, debug mask or RNG state.  That discussion
 * also sets the rule that a stable C ABI is never changed in place: a new
 * signature gets a new, versioned symbol.  varlen_attn_fwd is therefore an
 * alias of varlen_attn_fwd_v1, whose signature will not change.
 *
 * All pointers passed to varlen_attn_fwd are DEVICE pointers that the caller
 * allocates and owns.  The library allocates no memory per call, keeps no
 * reference to any buffer after the call returns, and the call is
 * asynchronous on `stream` (no host synchronisation, no host read of
 * cu_seqlens).
 */
#ifndef VARLEN_ATTN_H_
#define VARLEN_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as the CUDA runtime's cudaStream_t. */
struct CUstream_st;
typedef struct CUstream_st *varlen_stream_t;

typedef enum {
    VARLEN_BF16 = 0, /* q, k, v and out hold bfloat16 */
    VARLEN_FP16 = 1  /* q, k, v and out hold IEEE binary16 */
} varlen_dtype_t;

/* Status codes (0 = success, negative = error).  Every error except
 * VARLEN_ERR_LAUNCH is detected on the host before anything is launched,
 * and then no memory has been touched. */
#define VARLEN_OK 0
#define VARLEN_ERR_NULL (-1)        /* a required pointer is NULL */
#define VARLEN_ERR_SHAPE (-2)       /* H % Hkv != 0, unsupported D, negative size, ... */
#define VARLEN_ERR_DTYPE (-3)       /* dtype not VARLEN_BF16 / VARLEN_FP16 */
#define VARLEN_ERR_ALIGN (-4)       /* q, k, v or out not 16-byte aligned; lse or cu_seqlens not 4-byte aligned */
#define VARLEN_ERR_LAUNCH (-5)      /* the CUDA launch itself failed (see varlen_attn_strerror) */
#define VARLEN_ERR_DEVICE (-6)      /* device-side status word set (see varlen_attn_device_status) */
#define VARLEN_ERR_ARCH (-7)        /* current device is not compute capability 10.0 (B200/B100 class) */
#define VARLEN_ERR_WORKSPACE (-8)   /* workspace NULL, misaligned or smaller than the *_workspace_size */

/*
 * varlen_attn_fwd_v1 — packed attention forward, output written in place.
 *
 *   q            [total_q, H, D]   row-major, dtype, 16-byte aligned
 *   k, v         [total_k, Hkv, D] row-major, dtype, 16-byte aligned
 *   cu_seqlens_q [batch + 1] int32, device: cu_seqlens_q[0] = 0, non-decreasing,
 *                cu_seqlens_q[batch] <= total_q.  Sequence b owns query rows
 *                [cu_seqlens_q[b], cu_seqlens_q[b+1]).
 *   cu_seqlens_k [batch + 1] int32, device, same rules against total_k.
 *   batch        number of sequences B (>= 0; 0 is a no-op)
 *   total_q, total_k   number of token rows allocated in q/out/lse and in k/v.
 *                Every TMA read is bounded by these extents, so a sequence
 *                table that runs past them cannot make the kernel read or
 *                write outside the buffers.
 *   max_seqlen_q, max_seqlen_k   upper bounds of the per-sequence lengths
 *                (>= 0).  They only size the launch; the kernel walks the
 *                actual lengths from cu_seqlens, so an understated bound
 *                costs occupancy, never correctness.
 *   num_heads H, num_kv_heads Hkv   H % Hkv == 0; query head h reads
 *                key/value head h / (H / Hkv).
 *   head_dim D   64, 128 or 256.
 *   causal       0: every key of the sequence is visible; 1: key ki is hidden
 *                from query qi when qi < ki (sequence-local indices).
 *   scale        softmax scale; a value <= 0 or NaN selects 1/sqrt(D).
 *   dtype        element type of q, k, v and out.
 *   out          [total_q, H, D] dtype, written for rows [0, cu_seqlens_q[batch]).
 *                Rows outside the packed extents are not touched.
 *   lse          [total_q, H] float32, natural-log log-sum-exp of the scaled
 *                scores of each row; a query with no visible key (Lk_b = 0)
 *                gets out = 0 and lse = -inf.
 *   stream       CUDA stream of the launch (NULL = legacy default stream).
 *
 * Returns VARLEN_OK or one of the negative codes above.
 */
int varlen_attn_fwd_v1(const void *q, const void *k, const void *v,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int batch, int64_t total_q, int64_t total_k,
                       int max_seqlen_q, int max_seqlen_k,
                       int num_heads, int num_kv_heads, int head_dim,
                       int causal, float scale, varlen_dtype_t dtype,
                       void *out, float *lse, varlen_stream_t stream);

/* Unversioned name of the current stable entry point (same arguments and
 * behaviour as varlen_attn_fwd_v1). */
int varlen_attn_fwd(const void *q, const void *k, const void *v,
                    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                    int batch, int64_t total_q, int64_t total_k,
                    int max_seqlen_q, int max_seqlen_k,
                    int num_heads, int num_kv_heads, int head_dim,
                    int causal, float scale, varlen_dtype_t dtype,
                    void *out, float *lse, varlen_stream_t stream);

/*
 * varlen_attn_fwd_v2 — varlen_attn_fwd_v1 plus a sliding window and a
 * per-sequence count of used keys: the window_size_left, window_size_right
 * and seqused_k arguments of the varlen forward schema in PyTorch pull
 * request #176015 (whose rule on versioned symbols puts them in a new entry
 * point rather than into v1's signature).  The boostr page has no window; its
 * sequence-local indices are kept: key ki is visible to query qi iff
 *
 *   ki < Lk_used(b),  Lk_used(b) = min(Lk_b, seqused_k[b])  (Lk_b without seqused_k)
 *   ki >= qi - window_left    when window_left  >= 0
 *   ki <= qi + window_right   when window_right >= 0
 *   not (causal && qi < ki)
 *
 * A negative window bound means "no bound" on that side; window_left =
 * window_right = -1 with seqused_k = NULL is exactly varlen_attn_fwd_v1.
 *
 *   window_left, window_right   as above (any int; negative = unbounded).
 *   seqused_k    NULL, or [batch] int32 device array (4-byte aligned); a
 *                negative entry counts as 0, an entry above Lk_b as Lk_b.
 *                Keys in [Lk_used(b), Lk_b) take no part: their contents do
 *                not matter (they may be uninitialised, NaN or infinite).
 *
 * Every other argument, the ownership and the error behaviour are those of
 * varlen_attn_fwd_v1.  A query that sees no key (possible with a window, a
 * short seqused_k or Lk_b = 0) gets out = 0 and lse = -inf.
 */
int varlen_attn_fwd_v2(const void *q, const void *k, const void *v,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int batch, int64_t total_q, int64_t total_k,
                       int max_seqlen_q, int max_seqlen_k,
                       int num_heads, int num_kv_heads, int head_dim,
                       int causal, float scale, int window_left, int window_right,
                       const int32_t *seqused_k, varlen_dtype_t dtype,
                       void *out, float *lse, varlen_stream_t stream);

/*
 * varlen_attn_fwd_v3 — varlen_attn_fwd_v2 plus paged K/V and attention
 * sinks.  Paged K/V: the page_table
 * argument of the varlen forward schema in PyTorch pull request #176015 (its
 * follow-up #175924 "add page_table"), with the cache layout of the
 * PageAttention form of the Ascend sparse shared-KV attention page: a cache of
 * num_pages blocks of page_size tokens, [num_pages, page_size, Hkv, D], a
 * block table with one row per sequence, and the key lengths taken from the
 * used-key counts (cu_seqlens_k is not read in that form).
 *
 *   page_table   NULL: k and v are packed exactly as in v2 (the remaining two
 *                arguments are ignored).  Otherwise an int32 device array
 *                [batch, page_table_stride] (4-byte aligned): logical page j of
 *                sequence b is cache page page_table[b * page_table_stride + j],
 *                so key ki of sequence b is row
 *                  page_table[b * stride + ki / page_size] * page_size + ki % page_size
 *                of k and v viewed as [total_k, Hkv, D].  Pages may be shared
 *                between sequences.
 *   page_table_stride   entries per table row (>= 1); a sequence addresses at
 *                most page_table_stride * page_size keys.
 *   page_size    keys per page: a positive multiple of 16 dividing total_k
 *                (total_k = num_pages * page_size).
 *
 * With page_table != NULL, seqused_k is required and gives the number of keys
 * of each sequence (a negative entry counts as 0, one above
 * page_table_stride * page_size as that), cu_seqlens_k may be NULL, and only
 * the table entries of pages holding used keys are read.  A table entry
 * outside [0, num_pages) is never dereferenced: its keys read as zeros and
 * bit 2 of the device status word is set.  The rows of a page past the used
 * keys, and pages no used key lives in, take no part: their contents do not
 * matter (uninitialised, NaN or infinite values are fine).
 *
 * sinks        NULL, or a float32 device array [num_heads] (4-byte aligned):
 *              attention sinks, the FLOAT32 per-head "sinks" input of the
 *              Ascend sparse shared-KV attention page (which gives no
 *              formula).  sinks[h] is one more logit in the softmax of every
 *              row of query head h, in score units (not multiplied by scale),
 *              with no value row:
 *                m = max(max_ki s_ki, sinks[h]),
 *                l = sum_ki exp(s_ki - m) + exp(sinks[h] - m),
 *                out = sum_ki exp(s_ki - m) / l * V_ki,  lse = m + ln l.
 *              A row without visible keys then gets out = 0, lse = sinks[h].
 *
 * Everything else is as in v2 (window rule, empty rows, ownership, errors).
 */
int varlen_attn_fwd_v3(const void *q, const void *k, const void *v,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int batch, int64_t total_q, int64_t total_k,
                       int max_seqlen_q, int max_seqlen_k,
                       int num_heads, int num_kv_heads, int head_dim,
                       int causal, float scale, int window_left, int window_right,
                       const int32_t *seqused_k, const int32_t *page_table,
                       int page_table_stride, int page_size, const float *sinks,
                       varlen_dtype_t dtype, void *out, float *lse, varlen_stream_t stream);

/*
 * varlen_attn_fwd_v4 — varlen_attn_fwd_v3 plus a split of long key ranges
 * (same operation and results up to rounding; a new symbol under the
 * versioned-entry-point rule of PyTorch pull request #176015).
 *
 * Without a causal rule and without a window, a query row's softmax over the
 * keys of its sequence may be computed in pieces: the key range is cut into
 * at most num_splits ranges of near-equal length, each range gives a partial
 * result (O_i normalised by its own sum, and lse_i), and a second kernel
 * merges them exactly as the softmax over the union of the ranges:
 *   M = max(max_i lse_i, sink),  L = sum_i exp(lse_i - M) + exp(sink - M),
 *   out = sum_i exp(lse_i - M) / L * O_i,  lse = M + ln L
 * (sink terms only with sinks).  Short-query / long-key batches then spread
 * over all SMs instead of leaving a few long work items to a few of them.
 *
 *   num_splits   0: the library chooses (varlen_attn_fwd_num_splits); 1: no
 *                key-range split (with a NULL workspace exactly v3); 2..32: at
 *                most that many pieces per key
 *                range: pieces hold up to S = ceil(ceil(max_seqlen_k / 128) /
 *                num_splits) tiles of 128 keys, and a sequence of at most S
 *                tiles is not cut.  Ignored (no split) with causal or a window.
 *                Outside [0, 32]: VARLEN_ERR_SHAPE.
 *   workspace, workspace_bytes   device buffer (16-byte aligned) of at least
 *                varlen_attn_fwd_workspace_size(total_q, num_heads,
 *                num_kv_heads, head_dim, max_seqlen_q, max_seqlen_k, n)
 *                bytes, n the piece count in force (for num_splits = 0: the
 *                value varlen_attn_fwd_num_splits returns for the same
 *                arguments), or NULL (no split then needs none, and rows are
 *                not replicated).  Contents on entry do not matter and are
 *                scratch afterwards.  Missing, misaligned or too small when
 *                needed: VARLEN_ERR_WORKSPACE, nothing launched.
 *
 * Replicated rows: when a workspace is given, the call is non-causal without
 * a window, H / Hkv is a power of two of at least 2, every sequence's query
 * rows fit in 32 (max_seqlen_q * H / Hkv <= 32: decode-like calls) and
 * max_seqlen_k >= 1024, the library also computes each row as four pieces
 * over interleaved key subsets (a quarter of the exponentials per thread),
 * merged the same way; then at most 8 key-range pieces are used.
 * varlen_attn_fwd_workspace_size accounts for both.
 *
 * With a split or replicated rows, two kernels run on `stream` in order
 * (attention, then the merge); the workspace must stay allocated until both
 * have finished.  Everything else is as in v3.
 */
int varlen_attn_fwd_v4(const void *q, const void *k, const void *v,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int batch, int64_t total_q, int64_t total_k,
                       int max_seqlen_q, int max_seqlen_k,
                       int num_heads, int num_kv_heads, int head_dim,
                       int causal, float scale, int window_left, int window_right,
                       const int32_t *seqused_k, const int32_t *page_table,
                       int page_table_stride, int page_size, const float *sinks,
                       int num_splits, void *workspace, size_t workspace_bytes,
                       varlen_dtype_t dtype, void *out, float *lse, varlen_stream_t stream);

/*
 * Piece count varlen_attn_fwd_v4 uses for num_splits = 0 with these
 * arguments (paged: non-zero when a page table is given; num_sms <= 0: the
 * current device's SM count, which needs a CUDA device).  Host only; returns
 * >= 1, or a negative code for arguments v4 would reject with
 * VARLEN_ERR_SHAPE (or VARLEN_ERR_LAUNCH when the device query fails).
 */
int varlen_attn_fwd_num_splits(int batch, int64_t total_q, int64_t total_k,
                               int max_seqlen_q, int max_seqlen_k, int num_heads,
                               int num_kv_heads, int head_dim, int causal,
                               int window_left, int window_right, int paged, int num_sms);

/*
 * Bytes of workspace varlen_attn_fwd_v4 needs for a non-causal call without a
 * window with these sizes and at most num_splits (>= 1) pieces per key range;
 * 0 when it needs none (no split and no replicated rows, see below) or for
 * invalid sizes.  Host only.  Layout (float32): the pieces' O / l rows
 * [pieces][total_q * num_heads][head_dim], then their lse
 * [pieces][total_q * num_heads].
 */
size_t varlen_attn_fwd_workspace_size(int64_t total_q, int num_heads, int num_kv_heads,
                                      int head_dim, int max_seqlen_q, int max_seqlen_k,
                                      int num_splits);

/* Static, human-readable description of a status code.  Never NULL. */
const char *varlen_attn_strerror(int code);

/*
 * Device-side status word of the current device.  Every wait inside the
 * kernels is bounded (2 s); a wait that runs out ORs a bit into this word,
 * the kernel drains its own in-flight copies and returns instead of hanging.
 * Bits: 1 = pipeline wait timed out; 2 = a page-table entry was outside
 * [0, num_pages) (v3).  A launch that set a bit returned VARLEN_OK (the
 * entry points do not wait for the kernels) and its outputs are not to be
 * trusted: a caller that must detect this reads the word after synchronising
 * with the launch.  A wait can run out without a fault, e.g. when a CTA is
 * descheduled for more than the limit on a shared or time-sliced GPU.
 * Reads the word synchronously into *status (device-wide, shared by all
 * launches of this library on the device); clears it when clear != 0.
 * Returns VARLEN_OK or VARLEN_ERR_LAUNCH / VARLEN_ERR_NULL.
 */
int varlen_attn_device_status(unsigned int *status, int clear);

/*
 * Testing hook: the limit, in nanoseconds, of the kernels' pipeline waits on
 * the current device (0 restores the default of 2 s).  With a limit far below
 * a pipeline's ordinary waits (a microsecond), the kernels of the following
 * launches give up those waits, set bit 1 of the status word, drain their own
 * in-flight copies and tensor-core work and return; their outputs are then
 * incomplete.  This is how the tests exercise that abort path without a
 * fault.  The end-of-kernel drains keep their 2 s limit.  Synchronous with
 * the host; not meant for production use.  Returns VARLEN_OK or
 * VARLEN_ERR_LAUNCH.
 */
int varlen_attn_set_wait_limit(unsigned long long ns);

/*
 * Backward of the packed attention forward (varlen_attn_fwd_v1's operation):
 * the CPU backward loop of boostr 0.2.0, src/ops/cpu/attention/
 * varlen_attention.rs (VarLenAttentionOps::varlen_attention_bwd).  For every
 * sequence b, query head h (kv_h = h / (H / Hkv)) and query qi, with
 * delta = <dO[qi,h], O[qi,h]> and for every key ki visible to qi (causal: not
 * qi < ki, sequence-local):
 *   p  = exp(scale <Q[qi,h], K[ki,kv_h]> - LSE[qi,h])
 *   ds = p (<V[ki,kv_h], dO[qi,h]> - delta)
 *   dQ[qi,h] += scale ds K[ki,kv_h];   dK[ki,kv_h] += scale ds Q[qi,h];
 *   dV[ki,kv_h] += p dO[qi,h]
 * dK and dV of a key/value head sum over its H / Hkv query heads.
 *
 * varlen_attn_bwd_workspace_size — bytes of device workspace the backward
 * needs for total_q query rows and num_heads query heads (0 when either is
 * <= 0).  The workspace holds delta, float32 [total_q, H]; it needs no
 * initialisation and its contents after a call are unspecified.
 */
size_t varlen_attn_bwd_workspace_size(int64_t total_q, int num_heads);

/*
 * varlen_attn_bwd_v1 — gradients of the forward with respect to q, k, v.
 *
 *   dout         [total_q, H, D] dtype: gradient of the loss with respect to out
 *   q, k, v      the forward's inputs (layouts and rules as in varlen_attn_fwd_v1)
 *   out, lse     the forward's outputs for these inputs (out dtype, lse float32)
 *   cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
 *   max_seqlen_k, num_heads, num_kv_heads, causal, scale, dtype
 *                as in varlen_attn_fwd_v1 (head_dim 64, 128 or 256).
 *   dq           [total_q, H, D] dtype, written for rows [0, cu_seqlens_q[batch])
 *   dk, dv       [total_k, Hkv, D] dtype, written for rows [0, cu_seqlens_k[batch]);
 *                a key that no query sees gets zeros.
 *   workspace    device buffer of at least varlen_attn_bwd_workspace_size(total_q,
 *                num_heads) bytes, 16-byte aligned, owned by the caller; it must
 *                not be used by another call running at the same time.
 *   stream       CUDA stream of the two kernel launches.
 *
 * All tensors are device pointers owned by the caller (16-byte aligned;
 * lse and cu_seqlens 4-byte); nothing is allocated.  Returns VARLEN_OK or a
 * negative code (VARLEN_ERR_WORKSPACE when the workspace is missing or too
 * small); every error but VARLEN_ERR_LAUNCH is detected before any launch.
 */
int varlen_attn_bwd_v1(const void *dout, const void *q, const void *k, const void *v,
                       const void *out, const float *lse,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int batch, int64_t total_q, int64_t total_k,
                       int max_seqlen_q, int max_seqlen_k,
                       int num_heads, int num_kv_heads, int head_dim,
                       int causal, float scale, varlen_dtype_t dtype,
                       void *dq, void *dk, void *dv,
                       void *workspace, size_t workspace_bytes, varlen_stream_t stream);

/*
 * varlen_attn_bwd_noalloc — varlen_attn_bwd_v1 without a workspace argument
 * and without any allocation: the scratch (delta, float32 [total_q, H]) lives
 * in a fixed 16 MiB device array of the library (so total_q * H <= 4,194,304;
 * larger problems return VARLEN_ERR_WORKSPACE before anything is launched).
 * The pages have no counterpart: their backward allocates its buffers.
 *
 * The array's device address is looked up (cudaGetSymbolAddress) by the
 * first call on each device, and again by the first call after the device's
 * context has been reset; make that first call before any stream capture.
 * Nothing in the scratch has to start at zero.  Every call on a device uses
 * the same array: calls that overlap in time (other streams or host threads)
 * race on it and give wrong gradients; serialise them.  Arguments, results
 * and errors are otherwise those of varlen_attn_bwd_v1.
 */
int varlen_attn_bwd_noalloc(const void *dout, const void *q, const void *k, const void *v,
                            const void *out, const float *lse,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            int batch, int64_t total_q, int64_t total_k,
                            int max_seqlen_q, int max_seqlen_k,
                            int num_heads, int num_kv_heads, int head_dim,
                            int causal, float scale, varlen_dtype_t dtype,
                            void *dq, void *dk, void *dv, varlen_stream_t stream);

/*
 * varlen_attn_plan_shards — how to split one packed batch over `world` GPUs
 * (one process each) with no exchange between them.  Host only: every
 * pointer is a HOST pointer; nothing is launched or allocated on a device.
 *
 * The forward's units — a sequence and a key/value head with the query heads
 * that map onto it (kv_h = h / (H / Hkv), the GQA head map of the boostr page
 * cited above) — need nothing from one another, so a batch splits with no
 * collective on the data path:
 *
 *   VARLEN_SHARD_KV_HEADS   rank r computes every sequence for key/value
 *                heads [kv_head_lo[r], kv_head_hi[r]) and their query heads
 *                [kv_head_lo[r] * G, kv_head_hi[r] * G) (G = H / Hkv): the
 *                tensor-parallel layout, in which each rank holds contiguous
 *                [T, heads_r, D] slices of q, k, v and out and calls the
 *                forward on them with num_heads = heads_r * G and
 *                num_kv_heads = heads_r.  The first Hkv mod world ranks take
 *                one key/value head more.  Needs world <= num_kv_heads.
 *   VARLEN_SHARD_SEQUENCES  rank r computes all heads of the sequences b with
 *                seq_rank[b] == r (packed on that rank in their original
 *                order): longest processing time first, by unmasked pairs.
 *   VARLEN_SHARD_AUTO  whichever of the two has the smaller largest load
 *                (key/value heads on a tie).
 *
 *   cu_seqlens_q, cu_seqlens_k  [batch + 1] int32 (host), non-decreasing
 *   seqused_k    NULL or [batch] int32 (host): used keys per sequence (v2)
 *   causal, window_left, window_right   the mask of the forward call (v2);
 *                they only weigh the units
 *   seq_rank     [batch] out: the rank of sequence b, -1 in the key/value
 *                head split (every rank computes it)
 *   kv_head_lo, kv_head_hi   [world] out: key/value heads of each rank
 *                ([0, num_kv_heads) for every rank in the sequence split)
 *   rank_pairs   [world] out: unmasked (query, key) pairs summed over the
 *                query heads that rank r computes (the forward's FLOPs are
 *                4 * head_dim * pairs)
 *
 * Returns the split used (VARLEN_SHARD_KV_HEADS or VARLEN_SHARD_SEQUENCES),
 * or VARLEN_ERR_SHAPE (bad sizes, world < 1, mode unknown, a decreasing
 * sequence table, world > num_kv_heads with VARLEN_SHARD_KV_HEADS) or
 * VARLEN_ERR_NULL.
 */
#define VARLEN_SHARD_AUTO 0
#define VARLEN_SHARD_KV_HEADS 1
#define VARLEN_SHARD_SEQUENCES 2
int varlen_attn_plan_shards(const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            const int32_t *seqused_k, int batch, int num_heads, int num_kv_heads,
                            int causal, int window_left, int window_right, int world, int mode,
                            int32_t *seq_rank, int32_t *kv_head_lo, int32_t *kv_head_hi,
                            int64_t *rank_pairs);

/* Library ABI version: 6 for this header (v2, v3, v4, the backward and the
 * shard planner added; v1 unchanged). */
int varlen_attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VARLEN_ATTN_H_ */
