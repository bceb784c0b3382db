/*
 * fwd_pair.cuh — attention forward with two 128-row query tiles per work item
 * that share every K/V tile (D = 64 and 128, H / Hkv even).
 *
 * Two row layouts (KParams::pack_log2):
 *   0      tile A = 128 tokens of query head 2u, tile B = the same tokens of
 *          head 2u+1 (both map to one key/value head because H / Hkv is even:
 *          GQA head map kv_h = h / (H / Hkv));
 *   k > 0  "GQA-packed": a tile holds 128 >> k tokens x the 2^k = H / Hkv query
 *          heads of key/value head u (row r = token r >> k, head r & (2^k - 1));
 *          tile B holds the next 128 >> k tokens.  Short query sequences then
 *          fill the 128 MMA rows, and each K/V tile is read once per key/value
 *          head.
 *
 * One persistent CTA per SM, 384 threads (three warpgroups):
 *   warps 0-3   softmax warpgroup A (thread t = row t of tile A = TMEM lane t)
 *   warps 4-7   softmax warpgroup B
 *   warp 8      scheduler + TMA producer (both Q tiles, K/V ring)
 *   warp 9      TMEM owner and MMA issuer
 *   warps 10-11 idle
 * The kernel is compiled for REG_LAUNCH registers per thread; the third
 * warpgroup gives registers back (REG_LOW) and the softmax warpgroups take
 * them (REG_HIGH): 128 * REG_LOW + 256 * REG_HIGH == 384 * REG_LAUNCH.  The
 * host refuses to launch a build whose register count is not REG_LAUNCH.
 *
 * TMEM: S_A, S_B (128 columns each; P aliases their first 64 columns), O_A,
 * O_B (D columns each).  The MMA warp alternates between the tiles: after
 * S_A(0), S_B(0), for each key tile j it issues PV_A(j), S_A(j+1), PV_B(j),
 * S_B(j+1), so softmax A runs while the tensor cores work for tile B and vice
 * versa.  P_T(j) is handed over in two pieces of 64 keys and PV_T(j) is
 * issued piece by piece.  Because S_T(j) is issued after PV_T(j-1) and its
 * tcgen05.commit tracks every earlier MMA of the issuing thread, the arrival
 * of S_T(j) proves that PV_T(j-1) completed: the softmax may rescale O_T in
 * place, before its first P piece, without a further wait.
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
// P is handed to the MMA warp in NCHUNK pieces of BN / NCHUNK keys.
constexpr int NCHUNK = 2;
constexpr int CHUNK_KEYS = BN / NCHUNK;

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
  uint64_t s_full[2];  // per query tile (A, B)
  uint64_t p_chunk[2][NCHUNK];
  uint64_t o_ready[2], o_free[2];
  uint64_t v_tail;  // an item's last V tile that runs past the used keys has landed
  uint64_t drain;
  ItemRing ring;
  uint32_t tmem_base;
  AbortState abort;
};

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)2 * BM * D * 2 + (size_t)Cfg<D>::NSLOT * BN * D * 2 + sizeof(Barriers) + 1024;
}

// Softmax of one 128-key S tile with fine-grained hand-offs: `chunk_ready(c)`
// once the packed P of keys [CHUNK_KEYS c, CHUNK_KEYS (c + 1)) (columns
// [CHUNK_KEYS c / 2, CHUNK_KEYS (c + 1) / 2)) is in TMEM.  O is rescaled (when
// the running max jumps) before the first chunk is signalled.
template <int D, bool BF16, class ChunkReady>
__device__ __forceinline__ void softmax_tile_chunked(uint32_t tS, uint32_t tO, int j, float sl2,
                                                     bool need_mask, int lo, int hi, float &m,
                                                     float &l, ChunkReady &&chunk_ready) {
  uint32_t sr[BN];
  tmem_ld_wait<BN>(tS, sr);
  float s[BN];
#pragma unroll
  for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(sr[c]);
  if (need_mask) mask_outside(s, lo, hi);
  float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
  for (int c = 4; c + 8 <= BN; c += 8) {
    mx0 = ptx::fmax3(mx0, s[c], s[c + 1]);
    mx1 = ptx::fmax3(mx1, s[c + 2], s[c + 3]);
    mx2 = ptx::fmax3(mx2, s[c + 4], s[c + 5]);
    mx3 = ptx::fmax3(mx3, s[c + 6], s[c + 7]);
  }
  mx0 = ptx::fmax3(mx0, s[BN - 4], s[BN - 3]);
  mx1 = ptx::fmax3(mx1, s[BN - 2], s[BN - 1]);
  const float mx = fmaxf(ptx::fmax3(mx0, mx1, mx2), mx3) * sl2;
  float alpha = 1.f;
  bool need = false;
  update_max(j, mx, m, alpha, need);
  if (__any_sync(0xffffffffu, need)) {
    // 16-column pieces: the whole S row is still live here
    const uint64_t a2 = ptx::f2_pack(alpha, alpha);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 16) {
      uint32_t o[16];
      tmem_ld_wait<16>(tO + c0, o);
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        float o0, o1;
        ptx::f2_unpack(
            ptx::f2_mul(ptx::f2_pack(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), a2), o0,
            o1);
        o[c] = __float_as_uint(o0);
        o[c + 1] = __float_as_uint(o1);
      }
      tmem_st<16>(tO + c0, o);
    }
  }
  const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
  const float negm = exp_offset(m);
  const uint64_t negm_2 = ptx::f2_pack(negm, negm);
  uint64_t sum_ab = ptx::f2_pack(0.f, 0.f), sum_cd = ptx::f2_pack(0.f, 0.f);
#pragma unroll
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = c0 + 2 * i;
      const uint64_t x2 = ptx::f2_fma(ptx::f2_pack(s[c], s[c + 1]), sl2_2, negm_2);
      float x0, x1;
      ptx::f2_unpack(x2, x0, x1);
      const float e0 = ptx::ex2_approx(x0), e1 = ptx::ex2_approx(x1);
      pk[i] = pack2<BF16>(e0, e1);
      // row sum of the unrounded values, two keys per packed add
      uint64_t &acc = (i & 1) ? sum_cd : sum_ab;
      acc = ptx::f2_add(acc, ptx::f2_pack(e0, e1));
    }
    ptx::tmem_st_x16(tS + c0 / 2, pk);
    if ((c0 + 32) % CHUNK_KEYS == 0) {
      ptx::tmem_st_wait();
      chunk_ready(c0 / CHUNK_KEYS);
    }
  }
  float sa, sb, sc, sd;
  ptx::f2_unpack(sum_ab, sa, sb);
  ptx::f2_unpack(sum_cd, sc, sd);
  l = l * alpha + ((sa + sb) + (sc + sd));
}

// Softmax of one S tile in the replicated-rows form (KParams::rep = 4): the
// thread holds row copy `copy` (its warp's TMEM lane quarter) and keeps keys
// [32 copy, 32 copy + 32) of the tile.  It reads those 32 scores, writes their
// P values to packed columns [16 copy, 16 copy + 16) and zeros to the other 48
// packed columns of its row, so that the PV product sums, in this row copy,
// over the copy's keys alone; the running max, sum and O rescale are per copy.
// Both P pieces are signalled once the row is written.
template <int D, bool BF16, class ChunkReady>
__device__ __forceinline__ void softmax_tile_rep(uint32_t tS, uint32_t tO, int copy, int j,
                                                 float sl2, bool need_mask, int lo, int hi,
                                                 float &m, float &l, ChunkReady &&chunk_ready) {
  uint32_t sr[32];
  tmem_ld_wait<32>(tS + 32 * copy, sr);
  float s[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(sr[c]);
  if (need_mask) mask_outside(s, lo, hi, 32 * copy);
  float mx0 = s[0], mx1 = s[1];
#pragma unroll
  for (int c = 2; c < 32; c += 4) {
    mx0 = ptx::fmax3(mx0, s[c], s[c + 1]);
    mx1 = ptx::fmax3(mx1, s[c + 2], s[c + 3]);
  }
  const float mx = fmaxf(mx0, mx1) * sl2;
  float alpha = 1.f;
  bool need = false;
  update_max(j, mx, m, alpha, need);
  if (__any_sync(0xffffffffu, need)) {
    const uint64_t a2 = ptx::f2_pack(alpha, alpha);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 16) {
      uint32_t o[16];
      tmem_ld_wait<16>(tO + c0, o);
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        float o0, o1;
        ptx::f2_unpack(
            ptx::f2_mul(ptx::f2_pack(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), a2), o0,
            o1);
        o[c] = __float_as_uint(o0);
        o[c + 1] = __float_as_uint(o1);
      }
      tmem_st<16>(tO + c0, o);
    }
  }
  const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
  const float negm = exp_offset(m);
  const uint64_t negm_2 = ptx::f2_pack(negm, negm);
  uint64_t sum_ab = ptx::f2_pack(0.f, 0.f), sum_cd = ptx::f2_pack(0.f, 0.f);
  uint32_t pk[16], zr[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint64_t x2 = ptx::f2_fma(ptx::f2_pack(s[2 * i], s[2 * i + 1]), sl2_2, negm_2);
    float x0, x1;
    ptx::f2_unpack(x2, x0, x1);
    const float e0 = ptx::ex2_approx(x0), e1 = ptx::ex2_approx(x1);
    pk[i] = pack2<BF16>(e0, e1);
    uint64_t &acc = (i & 1) ? sum_cd : sum_ab;
    acc = ptx::f2_add(acc, ptx::f2_pack(e0, e1));
    zr[i] = 0u;
  }
  // copy is the same for the whole warp: each branch stores a fixed array
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    if (v == copy)
      ptx::tmem_st_x16(tS + 16 * v, pk);
    else
      ptx::tmem_st_x16(tS + 16 * v, zr);
  }
  ptx::tmem_st_wait();
#pragma unroll
  for (int c = 0; c < NCHUNK; ++c) chunk_ready(c);
  float sa, sb, sc, sd;
  ptx::f2_unpack(sum_ab, sa, sb);
  ptx::f2_unpack(sum_cd, sc, sd);
  l = l * alpha + ((sa + sb) + (sc + sd));
}

template <int D, bool BF16, bool REP>
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
  constexpr uint32_t IDESC_S_FULL = ptx::idesc_f16(BM, BN, BF16, false);
  constexpr uint32_t IDESC_PV = ptx::idesc_f16(BM, D, BF16, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;  // tile A at sQ, tile B at sQ + Q_BYTES
  uint8_t *sKV = smem + 2 * Q_BYTES;
  Barriers *bars = reinterpret_cast<Barriers *>(sKV + NSLOT * KV_BYTES);
  AbortState *abort_flag = &bars->abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int pack = p.pack_log2;
  // replicated rows (compiled separately, so the plain kernel keeps its code)
  constexpr int rep = REP ? 4 : 1;
  constexpr int NT = REP ? 1 : 2;  // query tiles in use

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      ptx::mbar_init(&bars->full[s], 1);
      ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->q_full, 1);
    ptx::mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->s_full[i], 1);
      for (int c = 0; c < NCHUNK; ++c) ptx::mbar_init(&bars->p_chunk[i][c], 4);
      ptx::mbar_init(&bars->o_ready[i], 1);
      ptx::mbar_init(&bars->o_free[i], 4);
    }
    ptx::mbar_init(&bars->v_tail, 1);
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
      // ---------------------------------------------------------- producer
      // The whole warp runs the scheduler and publishes items on the ring;
      // lane 0 issues the TMA copies.
      Scheduler<BN> sched;
      sched.init(p);
      uint32_t rs = 0, rph = 0, q_count = 0;
      bool ok = true;
      KVProducer<BN, D, NSLOT> kv;
      kv.init(sKV, bars->full, bars->empty, &bars->v_tail, abort_flag);
      // Q tiles of an item (lane 0): packed, tile t = the next (BM >> pack)
      // tokens of all query heads of kv_h; otherwise tile t = head 2u + t
      auto load_q = [&](const WorkItem &w) -> bool {
        if (!wait_bar(&bars->q_empty, (q_count & 1u) ^ 1u, abort_flag)) return false;
        if constexpr (REP) {
          // replicated rows: tile A = four copies of the item's 32 rows
          ptx::mbar_arrive_expect_tx(&bars->q_full, Q_BYTES);
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int db = 0; db < DB; ++db)
              ptx::tma_load_3d(sQ + db * (BM * 128) + c * (32 * 128), &tm_q, &bars->q_full,
                               db * 64, w.hu << pack, w.q0);
          ++q_count;
          return true;
        }
        ptx::mbar_arrive_expect_tx(&bars->q_full, 2 * Q_BYTES);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int head = pack ? (w.hu << pack) : (2 * w.hu + t);
          const int tok = pack ? (w.q0 + t * (BM >> pack)) : w.q0;
#pragma unroll
          for (int db = 0; db < DB; ++db)
            ptx::tma_load_3d(sQ + t * Q_BYTES + db * (BM * 128), &tm_q, &bars->q_full, db * 64,
                             head, tok);
        }
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
        if (w.n_kv > 0) {
          const int kv_h = pack ? w.hu : (2 * w.hu) / p.group;
          ok = kv.load_item(p, w, kv_h, &tm_k, &tm_v, [&]() { return load_q(w); });
        } else {
          ok = kv.fix_tail();
        }
        if (!ok) break;
      }
      if (lane == 0) {
        // Drain: every copy this warp issued has landed before the CTA exits.
        kv.drain();
        if (q_count > 0) drain_wait(&bars->q_full, (q_count - 1) & 1u);
      }
    } else if (warp == MMA_WARP && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
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
      // S_t columns [row0, row0 + N) = Q_t K^T for key rows [row0, row0 + N)
      // of the K tile, over D in steps of 16 (K-major, 128-byte swizzle).
      auto issue_s = [&](int t, uint32_t kslot, uint32_t row0, uint32_t idesc) {
        const uint32_t qbase = sQ_addr + t * Q_BYTES;
        const uint32_t kbase = sKV_addr + kslot * KV_BYTES + row0 * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk % 4) * 32u;
          uint64_t a = ptx::sdesc_sw128(qbase + (kk / 4) * (BM * 128) + off, 16, 1024);
          uint64_t bdesc = ptx::sdesc_sw128(kbase + (kk / 4) * (BN * 128) + off, 16, 1024);
          ptx::mma_ss(tmem + t * BN + row0, a, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V for keys [c * CHUNK_KEYS, (c + 1) * CHUNK_KEYS) (P from
      // TMEM, V MN-major), in steps of 16 keys
      auto issue_pv_chunk = [&](int t, uint32_t vslot, int c, bool acc) {
        const uint32_t vbase = sKV_addr + vslot * KV_BYTES;
        constexpr int KS = CHUNK_KEYS / 16;
#pragma unroll
        for (int kk = KS * c; kk < KS * c + KS; ++kk) {
          uint64_t bdesc = ptx::sdesc_sw128(vbase + kk * (16 * 128), BN * 128, 1024);
          ptx::mma_ts(tmem + O_COL0 + t * D, tmem + t * BN + kk * 8, bdesc, IDESC_PV,
                      (acc || kk > KS * c) ? 1u : 0u);
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
        if (!(ok = wait_bar(&bars->q_full, items & 1u, abort_flag))) break;
        ptx::tc_fence_after();
        uint32_t ks;
        if (!(ok = take_slot(ks))) break;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          issue_s(t, ks, 0, IDESC_S_FULL);
          ptx::mma_commit(&bars->s_full[t]);
        }
        ptx::mma_commit(&bars->empty[ks]);
        if (n == 1) ptx::mma_commit(&bars->q_empty);
        for (int j = 0; ok && j < n; ++j) {
          const uint32_t par = (g + j) & 1u;
          const bool more = j + 1 < n;
          uint32_t ks_next = 0, vs = 0;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            if (more && t == 0 && !(ok = take_slot(ks_next))) break;
            if (t == 0 && !(ok = take_slot(vs))) break;
            if (j == 0 && items > 0) {
              if (!(ok = wait_bar(&bars->o_free[t], (items - 1) & 1u, abort_flag))) break;
              ptx::tc_fence_after();
            }
#pragma unroll
            for (int c = 0; c < NCHUNK; ++c) {
              if (!(ok = wait_bar(&bars->p_chunk[t][c], par, abort_flag))) break;
              ptx::tc_fence_after();
              issue_pv_chunk(t, vs, c, j > 0 || c > 0);
            }
            if (!ok) break;
            if (j == n - 1) ptx::mma_commit(&bars->o_ready[t]);
            if (t == NT - 1) ptx::mma_commit(&bars->empty[vs]);
            if (more) {
              issue_s(t, ks_next, 0, IDESC_S_FULL);
              ptx::mma_commit(&bars->s_full[t]);
              if (t == NT - 1) {
                ptx::mma_commit(&bars->empty[ks_next]);
                if (j + 1 == n - 1) ptx::mma_commit(&bars->q_empty);
              }
            }
          }
        }
        g += n;
        ++items;
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      ptx::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
    end_of_kernel();
    if (warp == MMA_WARP) {
      __syncwarp();
      ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
  } else {
    ptx::setmaxnreg_inc<REG_HIGH>();
    // ------------------------------------------------------------ softmax WGs
    const int t = warp / 4;               // query tile A (0) or B (1)
    const int r = threadIdx.x - t * 128;  // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * BN;
    const uint32_t tO = tmem + lane_base + O_COL0 + t * D;
    const float sl2 = p.scale_log2;
    // replicated rows: copy = lane quarter, the copy's row = the lane
    const int copy = warp % 4;
    const int rr = rep > 1 ? lane : r;
    // row -> (token offset in the item, query head offset)
    const int tok_off = pack ? (rep > 1 ? 0 : t * (BM >> pack)) + (rr >> pack) : r;
    const int head_off = pack ? (rr & ((1 << pack) - 1)) : t;
    uint32_t rs = 0, rph = 0;
    uint32_t g = 0, items = 0;
    bool ok = true;
    auto arrive = [&](uint64_t *bar) {
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar);
    };
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
      if (t >= NT) continue;  // tile B is idle with replicated rows
      const int n = w.n_kv;
      const int h = (pack ? (w.hu << pack) : 2 * w.hu) + head_off;
      const int qi = w.qi0 + tok_off;
      const bool row_valid = tok_off < w.q_rows;
      const size_t orow = (size_t)(w.q0 + tok_off) * p.H + h;
      uint16_t *orow_ptr = reinterpret_cast<uint16_t *>(p.out) + orow * D;
      if (n == 0) {
        if (row_valid && (rep == 1 || copy == 0))
          empty_row<D>(orow_ptr, p.lse + orow, sink_log2(p, h));
        continue;
      }
      // visible keys of this row, relative to the first visited key tile
      const int lo = key_lo(p, qi) - w.kofs;
      const int hi = key_hi(p, qi, w.Lk) - w.kofs;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const uint32_t par = (g + j) & 1u;
        bool got = wait_bar(&bars->s_full[t], par, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const bool need_mask = j * BN < w.max_lo || (j + 1) * BN > w.min_hi;
        if constexpr (REP)
          softmax_tile_rep<D, BF16>(tS, tO, copy, j, sl2, need_mask, lo - j * BN, hi - j * BN, m,
                                    l, [&](int c) { arrive(&bars->p_chunk[t][c]); });
        else
          softmax_tile_chunked<D, BF16>(tS, tO, j, sl2, need_mask, lo - j * BN, hi - j * BN, m,
                                        l, [&](int c) { arrive(&bars->p_chunk[t][c]); });
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
      if (w.part < 0 && rep == 1) {
        epilogue_row<D, BF16>(tO, m, l, sink_log2(p, h), row_valid, orow_ptr, p.lse + orow,
                              &bars->o_free[t], lane, p.out_v8 != 0);
      } else {
        // a piece of the row: the key-range piece, and with replicated rows
        // the copy within it
        const size_t piece = (size_t)(w.part < 0 ? 0 : w.part) * rep + (rep > 1 ? copy : 0);
        epilogue_part<D>(tO, m, l, row_valid, p.part_o + (piece * p.part_rows + orow) * D,
                         p.part_lse + piece * p.part_rows + orow, &bars->o_free[t], lane,
                         p.part_v8 != 0);
      }
    }
    end_of_kernel();
  }
}

}  // namespace pair
}  // namespace vattn
