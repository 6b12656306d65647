// Rotation helpers shared by the append, export and attention kernels.
//
// Block-diagonal Walsh-Hadamard rotation ("SAW-INT4: System-Aware 4-Bit
// KV-Cache Quantization for Real-World LLM Serving", Summary/Method;
// "UltraQuant: 4-bit KV caching for long agents", method section) and the
// quaternion block rotation qL v conj(qR) ("IsoQuant: Hardware-Aligned SO(4)
// Isoclinic Rotations for LLM KV Cache Compression", Abstract), both on
// values held in registers: a thread owns E consecutive channels of a row.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

// In-thread Walsh-Hadamard butterflies on blocks of B = 2^LGB channels
// (B <= E), stages h = 1, 2, ..., B/2 in ascending order.
template <int E, int LGB, bool SKIP1 = false>
__device__ __forceinline__ void fwht_regs(float (&x)[E]) {
  constexpr int B = 1 << LGB;
  static_assert(B <= E, "block wider than a thread");
  if (B >= 2 && !SKIP1) {
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      const float a = x[i], c = x[i + 1];
      x[i] = __fadd_rn(a, c);
      x[i + 1] = __fsub_rn(a, c);
    }
  }
#pragma unroll
  for (int h = 2; h < B; h <<= 1) {
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      if ((i & h) == 0) {
        const uint64_t a = pk(x[i], x[i + 1]);
        const uint64_t c = pk(x[i + h], x[i + h + 1]);
        const float2 s = upk(add2(a, c));
        const float2 d = upk(sub2(a, c));
        x[i] = s.x;
        x[i + 1] = s.y;
        x[i + h] = d.x;
        x[i + h + 1] = d.y;
      }
    }
  }
}

// Multiplies by the Hadamard scale. For b a power of 4 the scale is a power
// of two, the product is exact, and a later fusion of it into a
// multiply-add could not change any rounding, so the packed multiply is
// used; otherwise each product is rounded by __fmul_rn, which is never
// contracted into a fused multiply-add.
template <int E, int LGB>
__device__ __forceinline__ void scale_regs(float (&x)[E], float cb) {
  if ((LGB & 1) == 0) {
    const uint64_t c2 = pk(cb, cb);
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      const float2 r = upk(mul2(pk(x[i], x[i + 1]), c2));
      x[i] = r.x;
      x[i + 1] = r.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = __fmul_rn(x[i], cb);
  }
}

// One Hamilton product a (x) b, each component as
// fma(t3, fma(t2, fma(t1, t0))) with the term order of the definition.
__device__ __forceinline__ void hamilton(const float a[4], const float b[4], float o[4]) {
  o[0] = __fmaf_rn(-a[3], b[3], __fmaf_rn(-a[2], b[2], __fmaf_rn(-a[1], b[1], __fmul_rn(a[0], b[0]))));
  o[1] = __fmaf_rn(-a[3], b[2], __fmaf_rn(a[2], b[3], __fmaf_rn(a[1], b[0], __fmul_rn(a[0], b[1]))));
  o[2] = __fmaf_rn(a[3], b[1], __fmaf_rn(a[2], b[0], __fmaf_rn(-a[1], b[3], __fmul_rn(a[0], b[2]))));
  o[3] = __fmaf_rn(a[3], b[0], __fmaf_rn(-a[2], b[1], __fmaf_rn(a[1], b[2], __fmul_rn(a[0], b[3]))));
}

template <int E>
__device__ __forceinline__ void quat_regs(float (&x)[E], const float* tbl, int ch0) {
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    const float* q = tbl + (ch0 / 4 + k) * 8;
    const float qL[4] = {q[0], q[1], q[2], q[3]};
    const float qRc[4] = {q[4], -q[5], -q[6], -q[7]};
    const float v[4] = {x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]};
    float t[4], y[4];
    hamilton(qL, v, t);
    hamilton(t, qRc, y);
    x[4 * k] = y[0];
    x[4 * k + 1] = y[1];
    x[4 * k + 2] = y[2];
    x[4 * k + 3] = y[3];
  }
}

// Full Hadamard rotation of a thread's E channels, block 2^LGB. Blocks wider
// than E (b = 256 with E = 128) finish with one stage across the lane pair
// (2i, 2i+1) given by pair_mask; part 0 holds the lower channels. With
// STAGE1_DONE the first butterfly stage (h = 1) has already been applied;
// without SCALE the 1/sqrt(b) factor is left to the caller.
template <int E, int LGB, bool STAGE1_DONE = false, bool SCALE = true>
__device__ __forceinline__ void hadamard_regs(float (&x)[E], int part, unsigned pair_mask) {
  constexpr int B = 1 << LGB;
  constexpr int LGIN = (B <= E) ? LGB : (E == 128 ? 7 : 6);
  fwht_regs<E, LGIN, STAGE1_DONE>(x);
  if (B > E) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(pair_mask, x[i], 1);
      x[i] = part == 0 ? __fadd_rn(x[i], o) : __fsub_rn(o, x[i]);
    }
  }
  if (SCALE) scale_regs<E, LGB>(x, hadamard_scale(LGB));
}

// Inverse quaternion rotation w -> conj(qL) w qR (the inverse of
// v -> qL v conj(qR) for unit quaternions), plain binary32 arithmetic.
template <int E>
__device__ __forceinline__ void quat_inv_regs(float (&x)[E], const float* tbl, int ch0) {
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    const float* q = tbl + (ch0 / 4 + k) * 8;
    const float qLc[4] = {q[0], -q[1], -q[2], -q[3]};
    const float qR[4] = {q[4], q[5], q[6], q[7]};
    const float w[4] = {x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]};
    float t[4], y[4];
    hamilton(qLc, w, t);
    hamilton(t, qR, y);
    x[4 * k] = y[0];
    x[4 * k + 1] = y[1];
    x[4 * k + 2] = y[2];
    x[4 * k + 3] = y[3];
  }
}

// IsoQuant-Fast: per 4-channel block v -> qL v (one Hamilton product, the
// same fused multiply-add order as the full map); qL[j] from the table of
// the full map (qR unused). Exact inverse for a unit qL: w -> conj(qL) w.
template <int E>
__device__ __forceinline__ void quat_fast_regs(float (&x)[E], const float* tbl, int ch0) {
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    const float* q = tbl + (ch0 / 4 + k) * 8;
    const float qL[4] = {q[0], q[1], q[2], q[3]};
    const float v[4] = {x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]};
    float y[4];
    hamilton(qL, v, y);
    x[4 * k] = y[0];
    x[4 * k + 1] = y[1];
    x[4 * k + 2] = y[2];
    x[4 * k + 3] = y[3];
  }
}
template <int E>
__device__ __forceinline__ void quat_fast_inv_regs(float (&x)[E], const float* tbl, int ch0) {
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    const float* q = tbl + (ch0 / 4 + k) * 8;
    const float qLc[4] = {q[0], -q[1], -q[2], -q[3]};
    const float w[4] = {x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]};
    float y[4];
    hamilton(qLc, w, y);
    x[4 * k] = y[0];
    x[4 * k + 1] = y[1];
    x[4 * k + 2] = y[2];
    x[4 * k + 3] = y[3];
  }
}

// IsoQuant-Full folded into one binary32 4x4 matrix per block: the map
// v -> qL v conj(qR) is linear in v, M = Rm(conj qR) Lm(qL) with Lm(a) the
// matrix of v -> a v and Rm(b) that of t -> t b. Entry (r, c) is the sum over
// k of Rm[r][k] Lm[k][c], k ascending, as a chain of fused multiply-adds
// from the plain first product; q = (qL, qR) as in the quaternion table.
__device__ __forceinline__ void quat_matrix(const float* q, float (&M)[16]) {
  const float aw = q[0], ax = q[1], ay = q[2], az = q[3];
  const float bw = q[4], bx = -q[5], by = -q[6], bz = -q[7];  // conj(qR)
  const float Lm[4][4] = {{aw, -ax, -ay, -az}, {ax, aw, -az, ay}, {ay, az, aw, -ax},
                          {az, -ay, ax, aw}};
  const float Rm[4][4] = {{bw, -bx, -by, -bz}, {bx, bw, bz, -by}, {by, -bz, bw, bx},
                          {bz, by, -bx, bw}};
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float m = __fmul_rn(Rm[r][0], Lm[0][c]);
#pragma unroll
      for (int k = 1; k < 4; ++k) m = __fmaf_rn(Rm[r][k], Lm[k][c], m);
      M[4 * r + c] = m;
    }
}

// y = M v per block (row r: fma(M[r][3] v3, fma(M[r][2] v2, fma(M[r][1] v1,
// M[r][0] v0)))), the matrices read from mats [d/4][16] (ch0 the thread's
// first channel, a multiple of 4).
template <int E>
__device__ __forceinline__ void quat_mat_regs(float (&x)[E], const float* mats, int ch0) {
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    const float4* m4 = reinterpret_cast<const float4*>(mats + (ch0 / 4 + k) * 16);
    const float v0 = x[4 * k], v1 = x[4 * k + 1], v2 = x[4 * k + 2], v3 = x[4 * k + 3];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 m = m4[r];
      x[4 * k + r] = __fmaf_rn(m.w, v3, __fmaf_rn(m.z, v2, __fmaf_rn(m.y, v1, __fmul_rn(m.x, v0))));
    }
  }
}

// The same map with each block's matrix built from the quaternion table on
// the spot (paths that rotate few rows); INV applies the transpose instead
// (the inverse of the orthogonal map), in plain binary32 arithmetic.
template <int E, bool INV = false>
__device__ __forceinline__ void quat_mat_fly_regs(float (&x)[E], const float* tbl, int ch0) {
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    float M[16];
    quat_matrix(tbl + (ch0 / 4 + k) * 8, M);
    const float v[4] = {x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i0 = INV ? r : 4 * r, st = INV ? 4 : 1;
      x[4 * k + r] = __fmaf_rn(M[i0 + 3 * st], v[3],
                               __fmaf_rn(M[i0 + 2 * st], v[2],
                                         __fmaf_rn(M[i0 + st], v[1], __fmul_rn(M[i0], v[0]))));
    }
  }
}

// Randomised-sign Hadamard: each channel times its fixed sign (+1 or -1,
// exact); `signs` offset to the thread's first channel.
template <int E>
__device__ __forceinline__ void sign_regs(float (&x)[E], const float* signs) {
#pragma unroll
  for (int i = 0; i < E; ++i) x[i] = __fmul_rn(x[i], signs[i]);
}

// Rotary position embedding in front of the rotation: channel pairs
// (2i, 2i+1) of a thread's E consecutive channels (starting at an even
// channel) turned by (cos, sin) read from cs (the table row of the position,
// offset to the thread's first channel; 8-byte aligned). Binary32, each
// product and the difference / sum rounded on its own:
//   x'_2i = RN(RN(x_2i c) - RN(x_2i+1 s)), x'_2i+1 = RN(RN(x_2i s) + RN(x_2i+1 c)).
template <int E>
__device__ __forceinline__ void rope_regs(float (&x)[E], const float* cs) {
#pragma unroll
  for (int i = 0; i < E; i += 2) {
    const float2 t = *reinterpret_cast<const float2*>(cs + i);
    const float a = x[i], b = x[i + 1];
    x[i] = __fsub_rn(__fmul_rn(a, t.x), __fmul_rn(b, t.y));
    x[i + 1] = __fadd_rn(__fmul_rn(a, t.y), __fmul_rn(b, t.x));
  }
}

// Rotation of a query row held as quarters: lane j of a group of four
// consecutive lanes owns channels [j*QW, (j+1)*QW). Butterfly stages with
// distance < QW run in registers, wider ones across the lanes (distance QW:
// lane ^ 1, 2*QW: lane ^ 2); the lower-channel lane adds and the upper one
// subtracts. All 32 lanes must call it. Binary32, not part of the bit-exact
// quantize path. `tbl` is the rotation's table (quaternions or signs).
template <int QW>
__device__ __forceinline__ void rotate_quarter(float (&x)[QW], int j, int rot_kind, int lgb,
                                               const float* tbl) {
  if (rot_kind == KVQ_ROT_HADAMARD || rot_kind == KVQ_ROT_HADAMARD_SIGNED) {
    if (rot_kind == KVQ_ROT_HADAMARD_SIGNED) sign_regs<QW>(x, tbl + j * QW);
    constexpr int LQ = QW == 32 ? 5 : 6;
    const int lin = lgb < LQ ? lgb : LQ;
    switch (lin) {
      case 4: fwht_regs<QW, 4>(x); break;
      case 5: fwht_regs<QW, 5>(x); break;
      default: fwht_regs<QW, (LQ > 5 ? 6 : 5)>(x); break;
    }
    for (int hs = QW; hs < (1 << lgb); hs <<= 1) {
      const int m = hs / QW;  // 1 or 2: lane distance
      const bool lower = (j & m) == 0;
#pragma unroll
      for (int i = 0; i < QW; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, x[i], m);
        x[i] = lower ? x[i] + o : o - x[i];
      }
    }
    const float cb = hadamard_scale(lgb);
#pragma unroll
    for (int i = 0; i < QW; ++i) x[i] *= cb;
  } else if (rot_kind == KVQ_ROT_QUAT) {
    quat_regs<QW>(x, tbl, j * QW);
  } else if (rot_kind == KVQ_ROT_QUAT_FAST) {
    quat_fast_regs<QW>(x, tbl, j * QW);
  } else if (rot_kind == KVQ_ROT_QUAT_MAT) {
    quat_mat_fly_regs<QW>(x, tbl, j * QW);
  }
}

}  // namespace kvq
