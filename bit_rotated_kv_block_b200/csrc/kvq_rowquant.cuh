// One K or V row (one token, one KV head) rotated, quantized and packed by a
// group of LPR consecutive lanes, each owning CPL = max(4, d/32) consecutive
// channels (LPR = d / CPL: 32 lanes, or 16 at d = 64).
//
// Arithmetic and order are those of the tiled append kernel and of the
// method's definition (see kvq.h): butterfly stages h = 1, 2, 4, ... in
// ascending order, each one binary32 add or subtract (stages below CPL in
// registers; wider stages across lanes, the lower-channel lane adding and
// the upper one taking (lower - upper)), the binary32 scale nearest 1/sqrt(b),
// min and max with -0 normalised to +0, m16 rounded down, the scale from the
// upward-rounded binary32 subtraction and division by 15 rounded up to
// binary16, and each code the nearest integer (ties to even) of the exact
// product RN(x - m16) * RN(1/s16) from one fused multiply-add.
#pragma once

#include <cuda_fp16.h>

#include "kvq.h"
#include "kvq_device.cuh"
#include "kvq_rotate.cuh"

namespace kvq {

template <int D>
struct RowQuantShape {
  static constexpr int CPL = D / 32 < 4 ? 4 : D / 32;  // channels per lane
  static constexpr int LPR = D / CPL;                  // lanes per row
};

// x: this lane's CPL channels (binary16 values widened to binary32); rl: the
// lane's index inside its row; quat: the quaternion table (QUAT kinds), the
// sign table (HADAMARD with signs) or NULL. Every lane of the warp must call it (the
// shuffles span the warp; rows never mix because lane distances stay below
// LPR). Returns the lane's codes, channel i of the lane in bits 4i..4i+3.
// The rotation alone (the first step of row_quantize and row_quantize_mx).
template <int D, int ROT, int LGB>
__device__ __forceinline__ void row_rotate(float (&x)[RowQuantShape<D>::CPL], int rl,
                                           const float* quat) {
  constexpr int CPL = RowQuantShape<D>::CPL;
  constexpr int B = 1 << LGB;
  if (ROT == KVQ_ROT_HADAMARD) {
    // randomised-sign Hadamard: `quat` is then the sign table (else NULL)
    if (quat != nullptr) sign_regs<CPL>(x, quat + rl * CPL);
#pragma unroll
    for (int dd = 1; dd < CPL && dd < B; dd <<= 1) {
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        if ((i & dd) == 0) {
          const float p = x[i], q = x[i + dd];
          x[i] = __fadd_rn(p, q);
          x[i + dd] = __fsub_rn(p, q);
        }
      }
    }
#pragma unroll
    for (int m = 1; m * CPL < B; m <<= 1) {
      const bool lower = (rl & m) == 0;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, x[i], m);
        x[i] = lower ? __fadd_rn(x[i], o) : __fsub_rn(o, x[i]);
      }
    }
    const float cb = hadamard_scale(LGB);
#pragma unroll
    for (int i = 0; i < CPL; ++i) x[i] = __fmul_rn(x[i], cb);
  } else if (ROT == KVQ_ROT_QUAT) {
    quat_regs<CPL>(x, quat, rl * CPL);
  } else if (ROT == KVQ_ROT_QUAT_FAST) {
    quat_fast_regs<CPL>(x, quat, rl * CPL);
  } else if (ROT == KVQ_ROT_QUAT_MAT) {
    quat_mat_fly_regs<CPL>(x, quat, rl * CPL);
  }
}

template <int D, int ROT, int LGB>
__device__ __forceinline__ uint32_t row_quantize(float (&x)[RowQuantShape<D>::CPL], int rl,
                                                 const float* quat, __half& s16, __half& m16) {
  constexpr int CPL = RowQuantShape<D>::CPL;
  constexpr int LPR = RowQuantShape<D>::LPR;
  row_rotate<D, ROT, LGB>(x, rl, quat);

  float mn = x[0], mx = x[0];
#pragma unroll
  for (int i = 1; i < CPL; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
  }
#pragma unroll
  for (int m = 1; m < LPR; m <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  }
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  m16 = __float2half_rd(mn);
  const float m = __half2float(m16);
  const float s32 = __fdiv_ru(__fsub_ru(mx, m), 15.0f);
  s16 = __float2half_ru(s32);
  const float s = __half2float(s16);
  uint32_t packed = 0;
  if (s != 0.0f) {
    const float inv = __frcp_rn(s);
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      // nearest integer (ties to even) of the exact product: one fused
      // multiply-add with 1.5 * 2^23 leaves it in the low mantissa bits
      const uint32_t c = __float_as_uint(__fmaf_rn(__fsub_rn(x[i], m), inv, 12582912.0f)) & 0xFu;
      packed |= c << (4 * i);
    }
  }
  return packed;
}

// The microscaled FP4 form of the same rotated row (kvq.h, KVQ_FMT_MXFP4):
// per block of 32 channels (32 / CPL lanes) the maximum magnitude, the
// shared exponent X = floor(log2 amax) - 2 clamped at -127 (its byte
// X + 127 read off the binary32 exponent field), then each x * 2^-X (exact)
// converted to E2M1. Returns the lane's codes as row_quantize does; `pword`
// gets the row's params word (byte g = block g), valid in lane rl = 0.
template <int D, int ROT, int LGB>
__device__ __forceinline__ uint32_t row_quantize_mx(float (&x)[RowQuantShape<D>::CPL], int rl,
                                                    const float* quat, uint32_t& pword) {
  constexpr int CPL = RowQuantShape<D>::CPL;
  constexpr int LPB = 32 / CPL;  // lanes per 32-channel block
  static_assert(LPB >= 1 && 32 % CPL == 0, "a block spans whole lanes");
  row_rotate<D, ROT, LGB>(x, rl, quat);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < CPL; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int m = 1; m < LPB; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
  const int eb = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
  const uint32_t xb = eb > 2 ? (uint32_t)(eb - 2) : 0u;  // X + 127
  const float inv = __uint_as_float((254u - xb) << 23);   // 2^-X
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < CPL; i += 2)
    packed |= e2m1x2(__fmul_rn(x[i], inv), __fmul_rn(x[i + 1], inv)) << (4 * i);
  // gather the blocks' bytes into the row's first lane
  uint32_t w = xb;
  constexpr int NB = D / 32;
#pragma unroll
  for (int g = 1; g < (NB < 4 ? NB : 4); ++g)
    w |= __shfl_down_sync(0xffffffffu, xb, g * LPB) << (8 * g);
  pword = w;
  return packed;
}

// Index of the table level nearest to the exact product t0 * inv (ties to
// the lower index), given the 15 sorted level midpoints: a four-step binary
// search, each step decided exactly by the sign of one fused multiply-add
// (t0 * inv - mid); the same count of midpoints below t0 * inv as a linear
// scan. The next midpoint is picked with selects, so `mid` stays in registers.
__device__ __forceinline__ uint32_t lut_code(float t0, float inv, const float (&mid)[15]) {
  const bool b3 = __fmaf_rn(t0, inv, -mid[7]) > 0.f;
  const float m2 = b3 ? mid[11] : mid[3];
  const bool b2 = __fmaf_rn(t0, inv, -m2) > 0.f;
  const float m1 = b3 ? (b2 ? mid[13] : mid[9]) : (b2 ? mid[5] : mid[1]);
  const bool b1 = __fmaf_rn(t0, inv, -m1) > 0.f;
  const float m0 = b3 ? (b2 ? (b1 ? mid[14] : mid[12]) : (b1 ? mid[10] : mid[8]))
                      : (b2 ? (b1 ? mid[6] : mid[4]) : (b1 ? mid[2] : mid[0]));
  const bool b0 = __fmaf_rn(t0, inv, -m0) > 0.f;
  return (b3 ? 8u : 0u) | (b2 ? 4u : 0u) | (b1 ? 2u : 0u) | (b0 ? 1u : 0u);
}

// The 2-bit, 3-bit and level-table forms of the same rotated row (kvq.h,
// KVQ_FMT_INT2 / INT3 / LUT4): the INT4 statistics with Q = 3, 7 or 15, each
// code the nearest integer of the exact product RN(x - m16) * RN(1/s16) (one
// fused multiply-add with 1.5 * 2^23) or the index of the nearest table level
// (the count of level midpoints below the exact product, each decided by the
// sign of one fused multiply-add). Returns the lane's codes, channel i of the
// lane at bits [i*bits, (i+1)*bits).
template <int D, int ROT, int LGB>
__device__ __forceinline__ uint32_t row_quantize_gen(float (&x)[RowQuantShape<D>::CPL], int rl,
                                                     const float* quat, int fmt,
                                                     const float* levels, __half& s16,
                                                     __half& m16) {
  constexpr int CPL = RowQuantShape<D>::CPL;
  constexpr int LPR = RowQuantShape<D>::LPR;
  row_rotate<D, ROT, LGB>(x, rl, quat);
  const int bits = fmt == KVQ_FMT_INT2 ? 2 : (fmt == KVQ_FMT_INT3 ? 3 : 4);
  const float Q = fmt == KVQ_FMT_INT2 ? 3.f : (fmt == KVQ_FMT_INT3 ? 7.f : 15.f);
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int i = 1; i < CPL; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
  }
#pragma unroll
  for (int m = 1; m < LPR; m <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  }
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  m16 = __float2half_rd(mn);
  const float m = __half2float(m16);
  s16 = __float2half_ru(__fdiv_ru(__fsub_ru(mx, m), Q));
  const float s = __half2float(s16);
  uint32_t packed = 0;
  if (s != 0.0f) {
    const float inv = __frcp_rn(s);
    if (fmt == KVQ_FMT_LUT4) {
      float mid[15];
#pragma unroll
      for (int k = 0; k < 15; ++k) mid[k] = 0.5f * (__ldg(levels + k) + __ldg(levels + k + 1));
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const float t0 = __fsub_rn(x[i], m);
        packed |= lut_code(t0, inv, mid) << (4 * i);
      }
    } else {
      const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const uint32_t c =
            __float_as_uint(__fmaf_rn(__fsub_rn(x[i], m), inv, 12582912.0f)) & mask;
        packed |= c << (bits * i);
      }
    }
  }
  return packed;
}

// Stores the lane's packed codes of a row of `bits`-bit codes (row_bytes =
// D * bits / 8 at `row`). With 12 bits per lane (3-bit codes, 4 channels per
// lane) the even lane of each pair writes both lanes' 24 bits; every lane of
// the warp must call it (nothing is written where `store` is false).
template <int D>
__device__ __forceinline__ void row_store_bits(uint8_t* row, uint32_t packed, int bits, int rl,
                                               bool store) {
  constexpr int CPL = RowQuantShape<D>::CPL;
  const int lb = CPL * bits;  // bits per lane
  if (lb % 8 == 0) {
    uint8_t* p = row + rl * (lb / 8);
    if (store)
      for (int k = 0; k < lb / 8; ++k) p[k] = (uint8_t)(packed >> (8 * k));
  } else {  // 12 bits per lane: lane pairs
    const uint32_t other = __shfl_xor_sync(0xffffffffu, packed, 1);
    if (store && (rl & 1) == 0) {
      const uint32_t v = packed | (other << lb);
      uint8_t* p = row + (rl / 2) * (2 * lb / 8);
      for (int k = 0; k < 2 * lb / 8; ++k) p[k] = (uint8_t)(v >> (8 * k));
    }
  }
}

// Loads this lane's CPL channels of a binary16 row (zeros when !active).
template <int D>
__device__ __forceinline__ void row_load(float (&x)[RowQuantShape<D>::CPL], const __half* src,
                                         bool active) {
  constexpr int CPL = RowQuantShape<D>::CPL;
  if (CPL == 4) {
    const uint2 u = active ? *reinterpret_cast<const uint2*>(src) : make_uint2(0u, 0u);
    const float2 f0 = __half22float2(u32_as_h2(u.x)), f1 = __half22float2(u32_as_h2(u.y));
    x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
  } else {
#pragma unroll
    for (int c = 0; c < CPL / 8; ++c) {
      const uint4 u = active ? reinterpret_cast<const uint4*>(src)[c] : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(u32_as_h2(w4[e]));
        x[8 * c + 2 * e] = f.x;
        x[8 * c + 2 * e + 1] = f.y;
      }
    }
  }
}

// Stores this lane's codes (CPL/2 bytes) at `codes` (the lane's slice).
template <int D>
__device__ __forceinline__ void row_store_codes(uint8_t* codes, uint32_t packed) {
  if (RowQuantShape<D>::CPL == 4)
    *reinterpret_cast<uint16_t*>(codes) = (uint16_t)packed;
  else
    *reinterpret_cast<uint32_t*>(codes) = packed;
}

}  // namespace kvq
