/*
 * bwd_common.cuh — parameters shared by the two backward kernels.
 *
 * What the backward computes is the CPU backward loop of boostr 0.2.0,
 * src/ops/cpu/attention/varlen_attention.rs (varlen_attention_bwd): for every
 * sequence b, query head h (kv_h = h / (H / Hkv)) and query qi,
 *   delta = <dO[qi, h], O[qi, h]>
 * and for every key ki visible to qi (causal: not qi < ki)
 *   p  = exp(scale <Q[qi, h], K[ki, kv_h]> - LSE[qi, h])
 *   ds = p (<V[ki, kv_h], dO[qi, h]> - delta)
 *   dQ[qi, h] += scale ds K[ki, kv_h];  dK[ki, kv_h] += scale ds Q[qi, h];
 *   dV[ki, kv_h] += p dO[qi, h].
 * The page accumulates all three in one loop; here the dQ pass (one query
 * tile per item, looping over key tiles) and the dK/dV pass (one key tile per
 * item, looping over the group's query heads and query tiles) each own their
 * outputs, so no accumulation crosses CTAs.  The dQ pass also writes delta
 * for the dK/dV pass.
 */
#pragma once
#include "fwd_common.cuh"

namespace vattn {

struct BwdParams {
  KParams kp;              // sequence table and head layout (kp.out / kp.lse unused)
  const uint16_t *dout;    // [Tq, H, D]
  const uint16_t *o;       // [Tq, H, D] forward output
  const float *lse;        // [Tq, H] forward LSE (natural log)
  float *delta;            // [Tq, H] workspace: written by the dQ pass, read by the dK/dV pass
  uint16_t *dq;            // [Tq, H, D]
  uint16_t *dk, *dv;       // [Tk, Hkv, D]
  float scale;             // softmax scale (dQ and dK carry it)
  int v8;                  // dq, dk and dv start on 32-byte boundaries: 32-byte row stores
};

constexpr float LOG2E = 1.4426950408889634f;

// Packs a 16-byte vector of bf16 / fp16 values into 8 floats.
template <bool BF16>
__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (BF16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    } else {
      __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
      float2 x = __half22float2(h);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
}

// delta = <dO row, O row> for one (token, head) row of D elements.
template <int D, bool BF16>
__device__ __forceinline__ float row_delta(const uint16_t *dout_row, const uint16_t *o_row) {
  const uint4 *a = reinterpret_cast<const uint4 *>(dout_row);
  const uint4 *b = reinterpret_cast<const uint4 *>(o_row);
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    float x[8], y[8];
    unpack8<BF16>(__ldg(a + c), x);
    unpack8<BF16>(__ldg(b + c), y);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      acc0 = fmaf(x[i], y[i], acc0);
      acc1 = fmaf(x[i + 1], y[i + 1], acc1);
    }
  }
  return acc0 + acc1;
}

// Writes D fp32 values read from TMEM (32-column chunks starting at taddr),
// times `mul`, to a bf16 / fp16 row (32-byte stores when v8, else 16-byte);
// when `valid` is false the values are read (the TMEM load is collective) but
// not stored.
template <int D, bool BF16>
__device__ __forceinline__ void store_tmem_row(uint32_t taddr, float mul, bool valid,
                                               uint16_t *row, bool v8) {
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t v[32];
    tmem_ld_wait<32>(taddr + c0, v);
    if (valid) {
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2)
        pk[c / 2] = pack2<BF16>(__uint_as_float(v[c]) * mul, __uint_as_float(v[c + 1]) * mul);
      store16w(row + c0, pk, v8);
    }
  }
}

template <int D>
__device__ __forceinline__ void zero_row(uint16_t *row) {
  uint4 *dst = reinterpret_cast<uint4 *>(row);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
}

}  // namespace vattn
