// Dense export of cached rows: x = c * s16 + m16 (the integer formats),
// t[c] * s16 + m16 (the level table) or e2m1(c) * 2^X (microscaled FP4),
// optionally rotated back.
//
// The dequantization rule is the one of the token-wise asymmetric INT4 format
// ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving", Summary); the inverse rotation is R (Hadamard, R R = I; with the
// sign diagonal S in front, S R), conj(qL) w qR (quaternion, "IsoQuant ...",
// Abstract) or conj(qL) w (its one-factor variant).
//
// One thread owns E = min(d, 128) channels of one (sequence, position, head)
// row; c * s16 is exact in binary32 (4-bit times 11-bit), so the rotated-basis
// value is a single rounding of the exact dequantized value.

#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_launch.h"
#include "kvq_rotate.cuh"

namespace kvq {

struct DequantArgs {
  int S, L, H, P, NP, bt_stride;
  const int32_t* seq_lens;
  const int32_t* block_table;
  const uint8_t* codes;
  const uint32_t* params;
  const float* quat;   // quaternion table (QUAT kinds)
  const float* signs;  // sign table of the randomised-sign Hadamard, or NULL
  int fmt;             // kvq_format
  const float* levels; // the level table (KVQ_FMT_LUT4)
  void* out;
  int32_t* err;
};

template <int D, int ROT, int LGB, bool F32>
__global__ void __launch_bounds__(128) dequant_kernel(const DequantArgs a, int unrotate) {
  constexpr int E = D < 128 ? D : 128;
  constexpr int TPR = D / E;
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gt / TPR;
  const int part = (int)(gt % TPR);
  if (row >= (int64_t)a.S * a.L * a.H) return;
  const int h = (int)(row % a.H);
  const int j = (int)((row / a.H) % a.L);
  const int s = (int)(row / ((int64_t)a.H * a.L));
  const int len = a.seq_lens[s];
  if (len < 0 || len > a.L || (len + a.P - 1) / a.P > a.bt_stride) {
    if (j == 0 && h == 0 && part == 0) raise_flag(a.err, KVQ_ERRF_LEN);
    return;
  }
  if (j >= len) return;
  const int page = a.block_table[(int64_t)s * a.bt_stride + j / a.P];
  if (page < 0 || page >= a.NP) {
    if (h == 0 && part == 0 && (j % a.P == 0 || j == 0)) raise_flag(a.err, KVQ_ERRF_PAGE);
    return;
  }
  const int64_t prow = ((int64_t)page * a.H + h) * a.P + j % a.P;
  const uint32_t pr = a.params[prow];
  const float sc = __half2float(__ushort_as_half((unsigned short)(pr & 0xffffu)));
  const float mn = __half2float(__ushort_as_half((unsigned short)(pr >> 16)));
  float x[E];
  const uint4* src = reinterpret_cast<const uint4*>(a.codes + prow * (D / 2) + part * (E / 2));
  if (a.fmt == KVQ_FMT_INT2 || a.fmt == KVQ_FMT_INT3 || a.fmt == KVQ_FMT_LUT4) {
    // c (or the table's level t[c]) times s16 plus m16, one rounding; the
    // codes of this thread's E channels as a little-endian bit stream
    const int bits = a.fmt == KVQ_FMT_INT2 ? 2 : (a.fmt == KVQ_FMT_INT3 ? 3 : 4);
    const uint8_t* cb = a.codes + prow * (D * bits / 8) + part * (E * bits / 8);
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int bit = i * bits;
      uint32_t v = cb[bit >> 3];
      if ((bit & 7) + bits > 8) v |= (uint32_t)cb[(bit >> 3) + 1] << 8;
      const uint32_t c = (v >> (bit & 7)) & ((1u << bits) - 1u);
      const float lv = a.fmt == KVQ_FMT_LUT4 ? __ldg(a.levels + c) : (float)c;
      x[i] = __fmaf_rn(lv, sc, mn);
    }
  } else if (a.fmt == KVQ_FMT_MXFP4) {
    // E2M1 value (exact in binary16) times 2^X of its 32-channel block:
    // exact in binary32, subnormal results included (X = -127: 2^-127 is the
    // binary32 bit pattern 0x00400000)
#pragma unroll
    for (int c = 0; c < E / 32; ++c) {
      const uint32_t xb = (pr >> (8 * ((part * E) / 32 + c))) & 0xFFu;
      const float sx = __uint_as_float(xb ? xb << 23 : 0x00400000u);
      const uint4 u = src[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          const float2 f = __half22float2(u32_as_h2(e2m1x2_to_h2((w[q] >> (8 * n)) & 0xFFu)));
          x[32 * c + 8 * q + 2 * n] = __fmul_rn(f.x, sx);
          x[32 * c + 8 * q + 2 * n + 1] = __fmul_rn(f.y, sx);
        }
    }
  } else {
#pragma unroll
    for (int c = 0; c < E / 32; ++c) {
      const uint4 u = src[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int n = 0; n < 8; ++n)
          x[32 * c + 8 * q + n] = __fmaf_rn((float)((w[q] >> (4 * n)) & 0xfu), sc, mn);
    }
  }
  if (unrotate) {
    const unsigned pair_mask = 3u << ((threadIdx.x % kWarp) & ~1);
    if (ROT == KVQ_ROT_HADAMARD) {
      hadamard_regs<E, LGB>(x, part, pair_mask);
      if (a.signs != nullptr) sign_regs<E>(x, a.signs + part * E);  // R^-1 = S H
    }
    if (ROT == KVQ_ROT_QUAT) quat_inv_regs<E>(x, a.quat, part * E);
    if (ROT == KVQ_ROT_QUAT_FAST) quat_fast_inv_regs<E>(x, a.quat, part * E);
    if (ROT == KVQ_ROT_QUAT_MAT) quat_mat_fly_regs<E, true>(x, a.quat, part * E);
  }
  const int64_t o = (((int64_t)s * a.L + j) * a.H + h) * D + part * E;
  if (F32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + o);
#pragma unroll
    for (int c = 0; c < E / 4; ++c) dst[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(a.out) + o);
#pragma unroll
    for (int c = 0; c < E / 8; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = h2_as_u32(__floats2half2_rn(x[8 * c + 2 * q], x[8 * c + 2 * q + 1]));
      dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <int D, int ROT, int LGB>
static cudaError_t launch_dq(const DequantArgs& a, int unrotate, int f32, cudaStream_t st) {
  constexpr int TPR = D <= 128 ? 1 : D / 128;
  const int64_t threads = (int64_t)a.S * a.L * a.H * TPR;
  const int64_t grid = (threads + 127) / 128;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  if (f32)
    dequant_kernel<D, ROT, LGB, true><<<(unsigned)grid, 128, 0, st>>>(a, unrotate);
  else
    dequant_kernel<D, ROT, LGB, false><<<(unsigned)grid, 128, 0, st>>>(a, unrotate);
  return cudaGetLastError();
}

template <int D>
static cudaError_t dq_rot(const DequantArgs& a, int rot, int lgb, int unrotate, int f32,
                          cudaStream_t st) {
  if (rot == KVQ_ROT_NONE || !unrotate) return launch_dq<D, KVQ_ROT_NONE, 0>(a, 0, f32, st);
  if (rot == KVQ_ROT_QUAT) return launch_dq<D, KVQ_ROT_QUAT, 0>(a, 1, f32, st);
  if (rot == KVQ_ROT_QUAT_FAST) return launch_dq<D, KVQ_ROT_QUAT_FAST, 0>(a, 1, f32, st);
  if (rot == KVQ_ROT_QUAT_MAT) return launch_dq<D, KVQ_ROT_QUAT_MAT, 0>(a, 1, f32, st);
  switch (lgb) {
    case 4: return launch_dq<D, KVQ_ROT_HADAMARD, 4>(a, 1, f32, st);
    case 5: return launch_dq<D, KVQ_ROT_HADAMARD, 5>(a, 1, f32, st);
    case 6: return launch_dq<D, KVQ_ROT_HADAMARD, 6>(a, 1, f32, st);
    case 7: if (D >= 128) return launch_dq<D, KVQ_ROT_HADAMARD, (D >= 128 ? 7 : 6)>(a, 1, f32, st); break;
    case 8: if (D >= 256) return launch_dq<D, KVQ_ROT_HADAMARD, (D >= 256 ? 8 : 6)>(a, 1, f32, st); break;
  }
  return cudaErrorInvalidValue;
}

int dequant_launch(const kvq_cache_desc& d, int32_t S, const int32_t* seq_lens,
                   int32_t max_seq_len, const int32_t* block_table, int32_t bt_stride,
                   const uint8_t* codes, const void* params, int32_t unrotate, int32_t out_fp32,
                   void* out, int32_t* err, cudaStream_t st) {
  DequantArgs a;
  a.S = S; a.L = max_seq_len; a.H = d.num_kv_heads; a.P = d.page_size; a.NP = d.num_pages;
  a.bt_stride = bt_stride; a.seq_lens = seq_lens; a.block_table = block_table;
  a.codes = codes; a.params = static_cast<const uint32_t*>(params); a.quat = d.quat;
  a.signs = d.rot_kind == KVQ_ROT_HADAMARD_SIGNED ? d.quat : nullptr;
  a.fmt = d.format;
  a.levels = d.levels;
  a.out = out; a.err = err;
  int lgb = 0;
  while ((1 << lgb) < d.rot_block) ++lgb;
  cudaError_t e;
  switch (d.head_dim) {
    case 64: e = dq_rot<64>(a, d.rot_kind, lgb, unrotate, out_fp32, st); break;
    case 128: e = dq_rot<128>(a, d.rot_kind, lgb, unrotate, out_fp32, st); break;
    case 256: e = dq_rot<256>(a, d.rot_kind, lgb, unrotate, out_fp32, st); break;
    default: return KVQ_ERR_UNSUPPORTED;
  }
  if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
