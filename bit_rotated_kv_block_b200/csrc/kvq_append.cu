// Fused rotate -> token-wise INT4 quantize -> pack -> page scatter.
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
// LLM Serving", Summary and Method (token-wise INT4 behind a block-diagonal
// Hadamard rotation, written by one fused kernel into paged KV layouts);
// "UltraQuant: 4-bit KV caching for long agents", method section
// (Walsh-Hadamard rotation); "IsoQuant: Hardware-Aligned SO(4) Isoclinic
// Rotations for LLM KV Cache Compression", Abstract (qL v conj(qR)).
//
// B200 design:
//  * A thread owns E consecutive channels of one (token, head) row of K or V,
//    E = 64 or 128 by configuration (append_e): 128 for Hadamard blocks of
//    16 and 128 and for d = 256, 64 otherwise (two threads per d = 128 row,
//    more warps per SM; one thread per row at d = 64). Every butterfly stage of a block that fits the
//    thread runs in registers; only b = 256 at d = 256 crosses the thread
//    pair, with one xor-1 shuffle stage.
//  * A CTA (384 threads at E = 128, one per SM; 256 threads at E = 64, two
//    per SM) owns a tile of TOK tokens x {K, V} x H heads. One elected thread
//    fills the tile's shared-memory buffer with TMA tensor copies
//    (cp.async.bulk.tensor.3d, boxes of 64 channels x H heads x TOK tokens,
//    128-byte swizzle, so the 128-bit reads of consecutive rows spread over
//    the banks) that complete on the buffer's mbarrier, while the previous
//    tile is computed (two buffers). The grid is persistent and walks the
//    tiles. Waits on the mbarriers are bounded and end in KVQ_ERRF_TIMEOUT,
//    never in a hang.
//  * Batches of at most 8192 rows (a decode step's one token per sequence)
//    go to append_rows_kernel instead: a warp per row, the same arithmetic.
//  * Threads are ordered token-major, head-minor, so a warp's rows are
//    consecutive lines of the swizzled boxes, and the destination of each
//    row (token -> sequence, position -> block table) is resolved one tile
//    ahead of its use.
//  * An optional RoPE table turns every key row before the rotation
//    (binary32, products and sums rounded separately).
//  * Arithmetic is bit-exact with the published definition (see kvq.h):
//    binary32 butterflies in ascending stage order (packed f32x2 lanes for
//    stages >= 2), directed roundings through __fsub_ru / __fdiv_ru /
//    __float2half_rd / __float2half_ru, RN(1/s) by __frcp_rn, and the code
//    as one fused multiply-add (y - m16) * inv + 1.5 * 2^23, which rounds the
//    exact product to the nearest integer, ties to even; the [0, 15] clamp of
//    the definition never acts because every value lies in
//    [m16, m16 + 15 s16], so the low nibble is the code.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_launch.h"
#include "kvq_rotate.cuh"
#include "kvq_rowquant.cuh"

namespace kvq {

// Channels per thread: 64 (two threads per d = 128 row, 256-thread CTAs, two
// CTAs per SM), or 128 (384-thread CTAs, one per SM) where a Hadamard block of
// 128 would need a cross-thread butterfly stage, for d = 256, and for Hadamard
// blocks of 2..16, which measured faster with the wider thread.
__host__ __device__ constexpr int append_e(int D, int rot, int lgb) {
  return D <= 64 ? D
                 : (D == 256 || (rot == KVQ_ROT_HADAMARD && (lgb >= 7 || lgb <= 4))) ? 128 : 64;
}
__host__ __device__ constexpr int append_threads(int E) { return E == 64 ? 256 : 384; }
// bytes of the rotation table in shared memory: quaternion pairs (2 d
// floats), signs (d), or the matrix form's 4x4 matrices (4 d floats)
__host__ __device__ constexpr int append_table_bytes(int D, int rot) {
  return rot == KVQ_ROT_QUAT_MAT ? D * 16 : D * 8;
}
__host__ __device__ constexpr int append_ctas_per_sm(int E) { return E == 64 ? 2 : 1; }

// Row-part encodings of the tile kernel (template argument FMT).
constexpr int kAppInt4 = 0, kAppMx = 1, kAppGen = 2;

// The 2-bit, 3-bit and level-table formats of one thread's E channels: the
// row statistics of INT4 with Q = 3, 7 or 15 levels above zero (the two
// threads of a row combine theirs), then each code from the exact product
// RN(x - m16) * RN(1/s16): the nearest integer (one fused multiply-add with
// 1.5 * 2^23, as for INT4) or the index of the nearest table level (the count
// of level midpoints below it, each decided exactly by the sign of one fused
// multiply-add); codes packed as a little-endian bit stream.
// Codes of one thread's E channels as a little-endian bit stream of BITS
// bits per code (LUT: the level-table rule), into w[E * BITS / 32].
template <int E, int BITS, bool LUT>
__device__ __forceinline__ void gen_codes(const float (&x)[E], float m, float inv,
                                          const float* levels, uint32_t (&w)[E / 8]) {
  float mid[15];
  if (LUT) {
#pragma unroll
    for (int k = 0; k < 15; ++k) mid[k] = 0.5f * (__ldg(levels + k) + __ldg(levels + k + 1));
  }
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const float t0 = __fsub_rn(x[i], m);
    uint32_t c;
    if (LUT) {
      c = lut_code(t0, inv, mid);
    } else {
      c = __float_as_uint(__fmaf_rn(t0, inv, 12582912.0f)) & ((1u << BITS) - 1u);
    }
    const int bit = i * BITS;
    w[bit >> 5] |= c << (bit & 31);
    if ((bit & 31) + BITS > 32) w[(bit >> 5) + 1] |= c >> (32 - (bit & 31));
  }
}

// The 2-bit, 3-bit and level-table formats of one thread's E channels: the
// row statistics of INT4 with Q = 3, 7 or 15 levels above zero (the two
// threads of a row combine theirs), then each code from the exact product
// RN(x - m16) * RN(1/s16): the nearest integer (one fused multiply-add with
// 1.5 * 2^23, as for INT4) or the index of the nearest table level (the count
// of level midpoints below it, each decided exactly by the sign of one fused
// multiply-add); codes packed as a little-endian bit stream.
template <int D, int E, int TPR>
__device__ __forceinline__ void gen_encode_store(float (&x)[E], int fmt, const float* levels,
                                                 int my_part, unsigned pair_mask,
                                                 int64_t dst_cur, uint8_t* codes,
                                                 uint32_t* params) {
  const int bits = fmt == KVQ_FMT_INT2 ? 2 : (fmt == KVQ_FMT_INT3 ? 3 : 4);
  const float Q = fmt == KVQ_FMT_INT2 ? 3.f : (fmt == KVQ_FMT_INT3 ? 7.f : 15.f);
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int i = 1; i < E; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
  }
  if (TPR == 2) {
    mn = fminf(mn, __shfl_xor_sync(pair_mask, mn, 1));
    mx = fmaxf(mx, __shfl_xor_sync(pair_mask, mx, 1));
  }
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  const __half m16 = __float2half_rd(mn);
  const float m = __half2float(m16);
  const __half s16 = __float2half_ru(__fdiv_ru(__fsub_ru(mx, m), Q));
  const float s = __half2float(s16);
  uint32_t w[E / 8];  // E * bits / 32 words used
#pragma unroll
  for (int i = 0; i < E / 8; ++i) w[i] = 0u;
  if (s != 0.0f) {
    const float inv = __frcp_rn(s);
    if (fmt == KVQ_FMT_INT2)
      gen_codes<E, 2, false>(x, m, inv, levels, w);
    else if (fmt == KVQ_FMT_INT3)
      gen_codes<E, 3, false>(x, m, inv, levels, w);
    else
      gen_codes<E, 4, true>(x, m, inv, levels, w);
  }
  if (dst_cur >= 0) {
    const int rb = D * bits / 8;  // code bytes of the row
    const int pb = E * bits / 8;  // this thread's code bytes (a multiple of 8)
    uint2* dst = reinterpret_cast<uint2*>(codes + dst_cur * rb + my_part * pb);
#pragma unroll
    for (int j = 0; j < E / 16; ++j)
      if (8 * j < pb) dst[j] = make_uint2(w[2 * j], w[2 * j + 1]);
    if (my_part == 0)
      params[dst_cur] = (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
  }
}

// One thread's part of one row: E channels of a (token, head) row of K or
// V, read from the row's line of the 128-byte swizzled TMA boxes (channel
// block c of the row sits in box my_part * E/64 + c/8, 16-byte chunk c % 8 at
// position (c % 8) ^ (line & 7)); rotated, quantized and stored at row
// dst_cur of the pools (no store when dst_cur < 0). The two threads of a row
// with E < D are lanes 2i, 2i+1 of one warp.
// With a RoPE table row cs (key rows; NULL otherwise) the row's channel
// pairs are turned before the rotation.
// For ROT == KVQ_ROT_HADAMARD a non-NULL qtbl is the sign table of the
// randomised-sign Hadamard (channels flipped before the butterflies).
// PRE: the kernel turns rows (RoPE) or flips signs before the rotation; without
// it the first butterfly stage is taken straight from binary16.
// FMT: kAppInt4 (INT4), kAppMx (microscaled FP4, KVQ_FMT_MXFP4) or kAppGen
// (the 2-bit, 3-bit and level-table formats, chosen by `fmt` at run time,
// `levels` the table).
template <int D, int ROT, int LGB, bool PRE, int FMT>
__device__ __forceinline__ void quantize_row_part(const uint8_t* boxes, int box_stride,
                                                  int my_line, int my_part, const float* qtbl,
                                                  const float* cs, int64_t dst_cur,
                                                  uint8_t* codes, uint32_t* params, int fmt,
                                                  const float* levels) {
  constexpr bool MX = FMT == kAppMx;
  constexpr bool fused1 = ROT == KVQ_ROT_HADAMARD && !PRE;
  constexpr int E = append_e(D, ROT, LGB);  // channels per thread
  constexpr int TPR = D / E;                // threads per row
  float x[E];
#pragma unroll
  for (int c = 0; c < E / 8; ++c) {
    // channel block c of this thread: box (part*E/64 + c/8), 16-byte
    // chunk c%8 of line my_line, at its 128B-swizzled position
    const uint8_t* box = boxes + (my_part * (E / 64) + c / 8) * box_stride;
    const uint4 u = *reinterpret_cast<const uint4*>(
        box + my_line * 128 + (((c % 8) ^ (my_line & 7)) << 4));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __half2 h2 = u32_as_h2(w[q]);
      if (fused1) {
        // first butterfly stage straight from binary16: widening is
        // exact, so (x_i + x_{i+1}, x_i - x_{i+1}) round as in binary32
        const float b = __high2float(h2);
        x[8 * c + 2 * q] = add_h_f(__low2half(h2), b);
        x[8 * c + 2 * q + 1] = sub_h_f(__low2half(h2), b);
      } else {
        const float2 f = __half22float2(h2);
        x[8 * c + 2 * q] = f.x;
        x[8 * c + 2 * q + 1] = f.y;
      }
    }
  }

  // the two threads of a d = 256 row are lanes 2i, 2i+1 of one warp
  const unsigned pair_mask = 3u << ((threadIdx.x % kWarp) & ~1);
  // For b a power of 4 the Hadamard scale 2^-(lg b)/2 is exact, and for the
  // INT4 codes it is folded into the row's scalars instead of the E values:
  // min and max of the scaled row are the scaled min and max, and with x the
  // unscaled value, RN(x cb - m) * inv = RN(x - m / cb) * (inv cb) exactly
  // (every operand a multiple of 2^-24 far above the subnormal range), so
  // statistics, parameters and codes come out bit for bit the same.
  constexpr bool FOLD = ROT == KVQ_ROT_HADAMARD && (LGB % 2) == 0 && FMT == kAppInt4;
  if (PRE && cs != nullptr) rope_regs<E>(x, cs + my_part * E);
  if (ROT == KVQ_ROT_HADAMARD) {
    if (fused1) {
      hadamard_regs<E, LGB, true, !FOLD>(x, my_part, pair_mask);  // first stage done on load
    } else {
      if (PRE && qtbl != nullptr) sign_regs<E>(x, qtbl + my_part * E);
      hadamard_regs<E, LGB, false, !FOLD>(x, my_part, pair_mask);
    }
  } else if (ROT == KVQ_ROT_QUAT_FAST) {
    quat_fast_regs<E>(x, qtbl, my_part * E);
  } else if (ROT == KVQ_ROT_QUAT) {
    quat_regs<E>(x, qtbl, my_part * E);
  } else if (ROT == KVQ_ROT_QUAT_MAT) {
    quat_mat_regs<E>(x, qtbl, my_part * E);  // the CTA's matrices
  }

  if constexpr (FMT == kAppGen) {
    gen_encode_store<D, E, TPR>(x, fmt, levels, my_part, pair_mask, dst_cur, codes, params);
    return;
  }

  if constexpr (MX) {
    // per block of 32 channels (all inside this thread): the shared
    // exponent from the largest magnitude's exponent field, then E2M1 codes
    // of x * 2^-X (exact scaling)
    uint32_t packed[E / 8];
    uint32_t sbytes = 0;
#pragma unroll
    for (int g = 0; g < E / 32; ++g) {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[32 * g + i]));
      const int eb = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
      const uint32_t xb = eb > 2 ? (uint32_t)(eb - 2) : 0u;  // X + 127
      const float inv = __uint_as_float((254u - xb) << 23);   // 2^-X
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = 32 * g + 8 * c + 2 * q;
          w |= e2m1x2(__fmul_rn(x[i], inv), __fmul_rn(x[i + 1], inv)) << (8 * q);
        }
        packed[4 * g + c] = w;
      }
      sbytes |= xb << (8 * g);
    }
    if constexpr (TPR == 2) {  // the row's second thread holds blocks E/32 .. 2E/32 - 1
      const uint32_t other = __shfl_xor_sync(pair_mask, sbytes, 1);
      if (my_part == 0) sbytes |= other << (8 * (E / 32));
    }
    if (dst_cur >= 0) {
      uint4* dst = reinterpret_cast<uint4*>(codes + dst_cur * (D / 2) + my_part * (E / 2));
#pragma unroll
      for (int c = 0; c < E / 32; ++c)
        dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      if (my_part == 0) params[dst_cur] = sbytes;
    }
    return;
  }

  // row statistics
  float mn0 = fminf(x[0], x[1]), mx0 = fmaxf(x[0], x[1]);
  float mn1 = fminf(x[2], x[3]), mx1 = fmaxf(x[2], x[3]);
#pragma unroll
  for (int i = 4; i < E; i += 4) {
    mn0 = min3(mn0, x[i], x[i + 1]);
    mn1 = min3(mn1, x[i + 2], x[i + 3]);
    mx0 = max3(mx0, x[i], x[i + 1]);
    mx1 = max3(mx1, x[i + 2], x[i + 3]);
  }
  float mn = fminf(mn0, mn1);
  float mx = fmaxf(mx0, mx1);
  if (TPR == 2) {
    mn = fminf(mn, __shfl_xor_sync(pair_mask, mn, 1));
    mx = fmaxf(mx, __shfl_xor_sync(pair_mask, mx, 1));
  }
  // the folded scale cb = 2^-(LGB/2) and its inverse, both exact
  const float cb = FOLD ? __int_as_float((127 - LGB / 2) << 23) : 1.0f;
  const float rcb = FOLD ? __int_as_float((127 + LGB / 2) << 23) : 1.0f;
  if (FOLD) {
    mn = __fmul_rn(mn, cb);
    mx = __fmul_rn(mx, cb);
  }
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  const __half m16 = __float2half_rd(mn);
  const float m = __half2float(m16);
  const float s32 = __fdiv_ru(__fsub_ru(mx, m), 15.0f);
  const __half s16 = __float2half_ru(s32);
  const float s = __half2float(s16);

  uint32_t packed[E / 8];
  if (s != 0.0f) {
    const float inv = __fmul_rn(__frcp_rn(s), cb);  // times cb: exact
    const float mq = __fmul_rn(m, rcb);              // exact
    const uint64_t m2 = pk(mq, mq), inv2 = pk(inv, inv);
    const uint64_t magic2 = pk(12582912.0f, 12582912.0f);  // 1.5 * 2^23
#pragma unroll
    for (int c = 0; c < E / 8; ++c) {
      uint32_t b[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        // code = nearest integer (ties to even) of the exact product
        // t * inv: one fused multiply-add with 1.5 * 2^23 rounds it
        // once, leaving the integer in the low mantissa bits
        const uint64_t t = sub2(pk(x[8 * c + 2 * q], x[8 * c + 2 * q + 1]), m2);
        const float2 r = upk(fma2(t, inv2, magic2));
        b[2 * q] = __float_as_uint(r.x);
        b[2 * q + 1] = __float_as_uint(r.y);
      }
      // low byte of each pair = c_even | c_odd << 4 (no carry: both <= 15)
      const uint32_t p0 = b[0] + (b[1] << 4), p1 = b[2] + (b[3] << 4);
      const uint32_t p2 = b[4] + (b[5] << 4), p3 = b[6] + (b[7] << 4);
      packed[c] = __byte_perm(__byte_perm(p0, p1, 0x0040), __byte_perm(p2, p3, 0x0040),
                              0x5410);
    }
  } else {
#pragma unroll
    for (int c = 0; c < E / 8; ++c) packed[c] = 0u;
  }

  if (dst_cur >= 0) {
    uint4* dst = reinterpret_cast<uint4*>(codes + dst_cur * (D / 2) + my_part * (E / 2));
#pragma unroll
    for (int c = 0; c < E / 32; ++c)
      dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    if (my_part == 0) {
      params[dst_cur] =
          (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
    }
  }
}

struct AppendArgs {
  int T, H, P, lg_page, NP, num_seqs, bt_stride, tok_per_tile, num_tiles;
  int fmt;  // kvq_format
  const float* levels;  // the level table (KVQ_FMT_LUT4)
  int box_stride;  // bytes between TMA boxes in a tile buffer (multiple of 1024)
  const int32_t* token_seq;
  const int32_t* token_pos;
  const int32_t* block_table;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint32_t* k_params;
  uint32_t* v_params;
  const float* quat;
  const float* rope;  // RoPE table [rope_max_pos][D] or NULL
  int rope_max_pos;
  int32_t* err;
};

// D: head_dim, ROT: rotation kind, LGB: log2 of the Hadamard block, PRE: a
// RoPE table or a sign table acts before the rotation, FMT: the row-part
// encoding (kAppInt4, kAppMx, kAppGen).
template <int D, int ROT, int LGB, bool PRE, int FMT>
__global__ void __launch_bounds__(append_threads(append_e(D, ROT, LGB)),
                                  append_ctas_per_sm(append_e(D, ROT, LGB)))
    append_kernel(const AppendArgs a, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv) {
  pdl_wait();     // K/V and the metadata may come from the previous kernel
  pdl_trigger();
  constexpr int E = append_e(D, ROT, LGB);    // channels per thread
  constexpr int kAppendThreads = append_threads(E);
  constexpr int TPR = D / E;             // threads per row
  constexpr int NH = D / 64;             // 64-channel boxes per row

  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled TMA boxes need 1024-byte aligned destinations
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int H = a.H, TOK = a.tok_per_tile;
  const int bufb = 2 * NH * a.box_stride;  // bytes of one tile buffer
  uint8_t* const buf0 = smem;
  uint8_t* const buf1 = smem + bufb;
  float* qtbl = reinterpret_cast<float*>(smem + 2 * bufb);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * bufb + append_table_bytes(D, ROT));

  const int tid = threadIdx.x;
  const int rows_per_tile = 2 * H * TOK * TPR;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_fence_init();
  }
  // the rotation's table in shared memory: quaternions (2 D floats) or signs (D)
  // or, for the matrix form, the 4x4 matrices built from the quaternions
  if (ROT == KVQ_ROT_QUAT_MAT) {
    for (int j = tid; j < D / 4; j += kAppendThreads) {
      float M[16];
      quat_matrix(a.quat + 8 * j, M);
#pragma unroll
      for (int i = 0; i < 16; ++i) qtbl[16 * j + i] = M[i];
    }
  } else if (ROT == KVQ_ROT_QUAT || ROT == KVQ_ROT_QUAT_FAST) {
    for (int i = tid; i < D * 2; i += kAppendThreads) qtbl[i] = a.quat[i];
  } else if (ROT == KVQ_ROT_HADAMARD && a.quat != nullptr) {
    for (int i = tid; i < D; i += kAppendThreads) qtbl[i] = a.quat[i];
  }
  const float* const rtbl =
      (ROT == KVQ_ROT_HADAMARD && a.quat == nullptr) || ROT == KVQ_ROT_NONE ? nullptr : qtbl;

  // this thread's role, fixed for all tiles (token-major):
  // thread row = ((kv*TOK + t)*H + h)*TPR + part
  const bool active = tid < rows_per_tile;
  int my_part = 0, my_t = 0, my_h = 0, my_kv = 0;
  if (active) {
    my_part = tid % TPR;
    const int r = tid / TPR;
    my_h = r % H;
    my_t = (r / H) % TOK;
    my_kv = r / (H * TOK);
  }
  const int my_line = my_t * H + my_h;  // 128-byte line of this row inside each box

  // One elected thread fills a tile buffer: for K and V, NH boxes of
  // (64 channels x H heads x TOK tokens), each landing densely (swizzled) at
  // (kv * NH + box) * box_stride. Tokens past the batch end are zero-filled by
  // the TMA unit and counted in the transaction bytes.
  auto issue_tile = [&](int tile, int bi) {
    if (tile >= a.num_tiles || tid != 0) return;
    uint8_t* buf = bi ? buf1 : buf0;
    mbar_arrive_expect_tx(&bars[bi], (uint32_t)(2 * NH * TOK * H * 128));
#pragma unroll
    for (int kv = 0; kv < 2; ++kv)
#pragma unroll
      for (int hb = 0; hb < NH; ++hb)
        tma_load_3d(buf + (kv * NH + hb) * a.box_stride, kv ? &tmv : &tmk, hb * 64, 0,
                    tile * TOK, &bars[bi]);
  };

  // Destination of this thread's row, resolved one tile ahead so the
  // dependent metadata loads (token -> sequence/position -> block table) are
  // in flight while the previous tile computes. A result < 0: no store.
  const bool lead = my_kv == 0 && my_h == 0 && my_part == 0;  // raises the token's flags
  const int lgP = a.lg_page, Pm = (1 << lgP) - 1;
  auto meta_load = [&](int tile, int& seq, int& pos) {
    const int tok = tile * TOK + my_t;
    seq = -1;
    pos = 0;
    if (active && tile < a.num_tiles && tok < a.T) {
      seq = a.token_seq[tok];
      pos = a.token_pos[tok];
    }
  };
  auto resolve = [&](int seq, int pos) -> int64_t {
    if (seq < 0) return -1;
    if (seq >= a.num_seqs) {
      if (lead) raise_flag(a.err, KVQ_ERRF_SEQ);
      return -1;
    }
    if (pos < 0 || (pos >> lgP) >= a.bt_stride || (a.rope != nullptr && pos >= a.rope_max_pos)) {
      if (lead) raise_flag(a.err, KVQ_ERRF_POS);
      return -1;
    }
    const int page = a.block_table[(int64_t)seq * a.bt_stride + (pos >> lgP)];
    if (page < 0 || page >= a.NP) {
      if (lead) raise_flag(a.err, KVQ_ERRF_PAGE);
      return -1;
    }
    return (((int64_t)page * H + my_h) << lgP) + (pos & Pm);
  };

  __syncthreads();  // barriers initialised, quaternion table visible
  int tile = blockIdx.x;
  issue_tile(tile, 0);
  int seq_n, pos_n;
  meta_load(tile, seq_n, pos_n);
  int64_t dst_cur = resolve(seq_n, pos_n);
  int pos_cur = pos_n;
  uint32_t parity = 0;  // bit b: phase parity to wait for on buffer b

  for (int it = 0; tile < a.num_tiles; ++it, tile += gridDim.x) {
    const int b = it & 1;
    uint8_t* cur = b ? buf1 : buf0;
    const int next = tile + gridDim.x;
    issue_tile(next, b ^ 1);
    meta_load(next, seq_n, pos_n);  // consumed after this tile's compute
    const bool ok = mbar_wait(&bars[b], (parity >> b) & 1u);
    parity ^= 1u << b;
    if (!__syncthreads_and(ok)) {
      // a copy never completed: report, let the other buffer's copies land
      // (bounded), and leave without touching the pools
      if (tid == 0) raise_flag(a.err, KVQ_ERRF_TIMEOUT);
      if (next < a.num_tiles) mbar_wait(&bars[b ^ 1], (parity >> (b ^ 1)) & 1u);
      return;
    }

    const int tok = tile * TOK + my_t;
    // rows of tokens past the batch end do nothing; every other active row
    // computes (the two threads of a d = 256 row always agree) and stores
    // only if its destination resolved
    if (active && tok < a.T) {
      const float* cs = (PRE && a.rope != nullptr && my_kv == 0 && dst_cur >= 0)
                            ? a.rope + (int64_t)pos_cur * D : nullptr;
      quantize_row_part<D, ROT, LGB, PRE, FMT>(cur + my_kv * NH * a.box_stride, a.box_stride,
                                               my_line, my_part, rtbl, cs, dst_cur,
                                               my_kv ? a.v_codes : a.k_codes,
                                               my_kv ? a.v_params : a.k_params, a.fmt, a.levels);
    }
    dst_cur = resolve(seq_n, pos_n);  // next tile's destination (its loads were in flight)
    pos_cur = pos_n;
    __syncthreads();  // buffer `cur` is refilled by the next iteration's issue
  }
}

// ---------------------------------------------------------------------------
// Small batches (a decode step appends one token per sequence): one row of
// K or V per 32 lanes (16 for d = 64), each lane owning CPL = max(4, d/32)
// consecutive channels. The same arithmetic as append_kernel in the same
// order: butterfly stages below CPL in registers, the wider ones across
// lanes (the lower-channel lane adds, the upper one subtracts the lower
// element minus its own), then the scale, the statistics, the parameters
// and the codes. Latency rather than bandwidth decides these launches: the
// work of a row is spread over a warp instead of one thread.
// ---------------------------------------------------------------------------

struct AppendRowsArgs {
  int T, H, P, lg_page, NP, num_seqs, bt_stride;
  int fmt;  // kvq_format
  const float* levels;  // the level table (KVQ_FMT_LUT4)
  int64_t tok_stride;
  const __half* k;
  const __half* v;
  const int32_t* token_seq;
  const int32_t* token_pos;
  const int32_t* block_table;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint32_t* k_params;
  uint32_t* v_params;
  const float* quat;
  const float* rope;  // RoPE table [rope_max_pos][D] or NULL
  int rope_max_pos;
  int32_t* err;
};

constexpr int kRowsWarps = 4;

template <int D, int ROT, int LGB>
__global__ void __launch_bounds__(kRowsWarps * kWarp) append_rows_kernel(const AppendRowsArgs a) {
  pdl_wait();     // K/V and the metadata may come from the previous kernel
  pdl_trigger();
  constexpr int CPL = RowQuantShape<D>::CPL;  // channels per lane
  constexpr int LPR = RowQuantShape<D>::LPR;  // lanes per row (16 or 32)
  constexpr int RPW = kWarp / LPR;            // rows per warp
  const int lane = threadIdx.x % kWarp;
  const int rl = lane % LPR;
  const int row = (blockIdx.x * kRowsWarps + threadIdx.x / kWarp) * RPW + lane / LPR;
  const int nrows = a.T * a.H * 2;
  const bool active = row < nrows;
  // row = ((t * H) + h) * 2 + kv
  const int kv = row & 1;
  const int h = (row >> 1) % a.H;
  const int t = active ? (row >> 1) / a.H : 0;

  // destination first: its dependent loads (token -> sequence and position
  // -> block-table entry) overlap the arithmetic below
  const int seq = active ? a.token_seq[t] : -1;
  const int pos = active ? a.token_pos[t] : 0;
  const bool seq_ok = seq >= 0 && seq < a.num_seqs;
  const bool pos_ok = pos >= 0 && (pos >> a.lg_page) < a.bt_stride &&
                      (a.rope == nullptr || pos < a.rope_max_pos);
  const int page = (seq_ok && pos_ok) ? a.block_table[(int64_t)seq * a.bt_stride + (pos >> a.lg_page)] : -1;

  float x[CPL];
  row_load<D>(x, (kv ? a.v : a.k) + (int64_t)t * a.tok_stride + (int64_t)h * D + rl * CPL, active);
  if (a.rope != nullptr && kv == 0 && pos_ok) rope_regs<CPL>(x, a.rope + (int64_t)pos * D + rl * CPL);
  __half s16, m16;
  uint32_t pword = 0;
  uint32_t packed;
  if (a.fmt == KVQ_FMT_MXFP4) {
    packed = row_quantize_mx<D, ROT, LGB>(x, rl, a.quat, pword);
  } else {
    packed = a.fmt == KVQ_FMT_INT4
                 ? row_quantize<D, ROT, LGB>(x, rl, a.quat, s16, m16)
                 : row_quantize_gen<D, ROT, LGB>(x, rl, a.quat, a.fmt, a.levels, s16, m16);
    pword = (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
  }
  const int bits = a.fmt == KVQ_FMT_INT2 ? 2 : (a.fmt == KVQ_FMT_INT3 ? 3 : 4);
  // 3-bit codes pair lanes for their stores: every lane of a row stays until then
  const bool ok_row = active && seq >= 0;
  const bool lead = kv == 0 && h == 0 && rl == 0;
  bool store = ok_row;
  if (ok_row && !seq_ok) {
    if (lead) raise_flag(a.err, KVQ_ERRF_SEQ);
    store = false;
  } else if (ok_row && !pos_ok) {
    if (lead) raise_flag(a.err, KVQ_ERRF_POS);
    store = false;
  } else if (ok_row && (page < 0 || page >= a.NP)) {
    if (lead) raise_flag(a.err, KVQ_ERRF_PAGE);
    store = false;
  }
  const int64_t dst =
      store ? (((int64_t)page * a.H + h) << a.lg_page) + (pos & ((1 << a.lg_page) - 1)) : 0;
  if (bits == 4) {
    if (store)
      row_store_codes<D>((kv ? a.v_codes : a.k_codes) + dst * (D / 2) + rl * (CPL / 2), packed);
  } else {
    // the pairing shuffle inside involves every lane of the row (a row's
    // lanes share `store`)
    row_store_bits<D>((kv ? a.v_codes : a.k_codes) + dst * (D * bits / 8), packed, bits, rl,
                      store);
  }
  if (store && rl == 0) (kv ? a.v_params : a.k_params)[dst] = pword;
}

template <int D, int ROT, int LGB>
static cudaError_t launch_rows(const AppendRowsArgs& a, cudaStream_t st) {
  constexpr int CPL = D / 32 < 4 ? 4 : D / 32;
  constexpr int RPW = kWarp / (D / CPL);
  const int warps = (a.T * a.H * 2 + RPW - 1) / RPW;
  const cudaError_t e = launch_pdl(append_rows_kernel<D, ROT, LGB>, (warps + kRowsWarps - 1) / kRowsWarps,
                                   kRowsWarps * kWarp, 0, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_rows(const AppendRowsArgs& a, int rot, int lgb, cudaStream_t st) {
  if (rot == KVQ_ROT_NONE) return launch_rows<D, KVQ_ROT_NONE, 0>(a, st);
  if (rot == KVQ_ROT_QUAT) return launch_rows<D, KVQ_ROT_QUAT, 0>(a, st);
  if (rot == KVQ_ROT_QUAT_FAST) return launch_rows<D, KVQ_ROT_QUAT_FAST, 0>(a, st);
  if (rot == KVQ_ROT_QUAT_MAT) return launch_rows<D, KVQ_ROT_QUAT_MAT, 0>(a, st);
  switch (lgb) {
    case 4: return launch_rows<D, KVQ_ROT_HADAMARD, 4>(a, st);
    case 5: return launch_rows<D, KVQ_ROT_HADAMARD, 5>(a, st);
    case 6: return launch_rows<D, KVQ_ROT_HADAMARD, 6>(a, st);
    case 7:
      if (D >= 128) return launch_rows<D, KVQ_ROT_HADAMARD, (D >= 128 ? 7 : 6)>(a, st);
      break;
    case 8:
      if (D >= 256) return launch_rows<D, KVQ_ROT_HADAMARD, (D >= 256 ? 8 : 6)>(a, st);
      break;
  }
  return cudaErrorInvalidValue;
}

// Driver entry point for tensor-map encoding (no link-time libcuda needed).
static PFN_cuTensorMapEncodeTiled encode_fn() {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
  }
  return fn;
}

// [T][H][D] binary16 rows with token stride tok_stride (elements) as a 3-D
// tensor (D innermost); box (64 channels, HB heads, TOK tokens), 128B swizzle.
static bool encode_rows(CUtensorMap* m, const void* base, int D, int H, int T,
                        int64_t tok_stride, int HB, int TOK) {
  PFN_cuTensorMapEncodeTiled fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)tok_stride * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)HB, (cuuint32_t)TOK};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

static size_t append_smem(int D, int rot, int box_stride) {
  return 1024 + 2 * (size_t)(2 * (D / 64)) * box_stride + append_table_bytes(D, rot) +
         2 * sizeof(uint64_t);
}

template <int D, int ROT, int LGB>
static cudaError_t launch_append(const AppendArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                                 int grid, cudaStream_t st) {
  const size_t smem = append_smem(D, ROT, a.box_stride);
  const bool pre = a.rope != nullptr || (ROT == KVQ_ROT_HADAMARD && a.quat != nullptr);
  auto kern = pre ? append_kernel<D, ROT, LGB, true, kAppInt4>
                  : append_kernel<D, ROT, LGB, false, kAppInt4>;
  if (a.fmt != KVQ_FMT_INT4) {  // the other formats: head_dim 128 only
    if constexpr (D == 128) {
      if (a.fmt == KVQ_FMT_MXFP4)
        kern = pre ? append_kernel<D, ROT, LGB, true, kAppMx>
                   : append_kernel<D, ROT, LGB, false, kAppMx>;
      else
        kern = pre ? append_kernel<D, ROT, LGB, true, kAppGen>
                   : append_kernel<D, ROT, LGB, false, kAppGen>;
    } else {
      return cudaErrorInvalidValue;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, grid, append_threads(append_e(D, ROT, LGB)), smem, st, a, tk, tv);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_rot(const AppendArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                                int rot, int lgb, int grid, cudaStream_t st) {
  if (rot == KVQ_ROT_NONE) return launch_append<D, KVQ_ROT_NONE, 0>(a, tk, tv, grid, st);
  if (rot == KVQ_ROT_QUAT) return launch_append<D, KVQ_ROT_QUAT, 0>(a, tk, tv, grid, st);
  if (rot == KVQ_ROT_QUAT_FAST) return launch_append<D, KVQ_ROT_QUAT_FAST, 0>(a, tk, tv, grid, st);
  if (rot == KVQ_ROT_QUAT_MAT) return launch_append<D, KVQ_ROT_QUAT_MAT, 0>(a, tk, tv, grid, st);
  switch (lgb) {
    case 4: return launch_append<D, KVQ_ROT_HADAMARD, 4>(a, tk, tv, grid, st);
    case 5: return launch_append<D, KVQ_ROT_HADAMARD, 5>(a, tk, tv, grid, st);
    case 6: return launch_append<D, KVQ_ROT_HADAMARD, 6>(a, tk, tv, grid, st);
    case 7:
      if (D >= 128) return launch_append<D, KVQ_ROT_HADAMARD, (D >= 128 ? 7 : 6)>(a, tk, tv, grid, st);
      break;
    case 8:
      if (D >= 256) return launch_append<D, KVQ_ROT_HADAMARD, (D >= 256 ? 8 : 6)>(a, tk, tv, grid, st);
      break;
  }
  return cudaErrorInvalidValue;
}

// The kernels' rotation template: the randomised-sign Hadamard runs as the
// Hadamard kernels given its sign table; the table a kernel receives (NULL
// for the plain Hadamard and for no rotation).
static int rot_template(const kvq_cache_desc& d) {
  return d.rot_kind == KVQ_ROT_HADAMARD_SIGNED ? KVQ_ROT_HADAMARD : d.rot_kind;
}
static const float* rot_table(const kvq_cache_desc& d) {
  return (d.rot_kind == KVQ_ROT_NONE || d.rot_kind == KVQ_ROT_HADAMARD) ? nullptr : d.quat;
}

int append_launch(const kvq_cache_desc& d, int32_t T, const void* k, const void* v,
                  int64_t tok_stride, const int32_t* token_seq, const int32_t* token_pos,
                  int32_t num_seqs, const int32_t* block_table, int32_t bt_stride,
                  uint8_t* k_codes, void* k_params, uint8_t* v_codes, void* v_params,
                  int32_t* err, cudaStream_t st) {
  const int D = d.head_dim;
  int lgb0 = 0;
  while ((1 << lgb0) < d.rot_block) ++lgb0;
  const int E = append_e(D, rot_template(d), lgb0);
  const int TPR = D / E;
  const int per_sm = append_ctas_per_sm(E);
  const int tok_max = append_threads(E) / (2 * d.num_kv_heads * TPR);
  if (tok_max < 1 || d.num_kv_heads > 256) return KVQ_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  if (sms <= 0) return KVQ_ERR_CUDA;
  int lgb = 0;
  while ((1 << lgb) < d.rot_block) ++lgb;
  // small batches (up to 8192 rows of K and V): a warp per row
  if ((int64_t)T * d.num_kv_heads * 2 <= 8192) {
    AppendRowsArgs r;
    r.T = T; r.H = d.num_kv_heads; r.P = d.page_size;
    r.lg_page = 0;
    while ((1 << r.lg_page) < d.page_size) ++r.lg_page;
    r.NP = d.num_pages; r.num_seqs = num_seqs; r.bt_stride = bt_stride;
    r.tok_stride = tok_stride;
    r.k = static_cast<const __half*>(k); r.v = static_cast<const __half*>(v);
    r.token_seq = token_seq; r.token_pos = token_pos; r.block_table = block_table;
    r.k_codes = k_codes; r.v_codes = v_codes;
    r.k_params = static_cast<uint32_t*>(k_params); r.v_params = static_cast<uint32_t*>(v_params);
    r.quat = rot_table(d); r.rope = d.rope; r.rope_max_pos = d.rope_max_pos; r.err = err;
    r.fmt = d.format;
    r.levels = d.levels;
    cudaError_t e;
    switch (D) {
      case 64: e = dispatch_rows<64>(r, rot_template(d), lgb, st); break;
      case 128: e = dispatch_rows<128>(r, rot_template(d), lgb, st); break;
      case 256: e = dispatch_rows<256>(r, rot_template(d), lgb, st); break;
      default: return KVQ_ERR_UNSUPPORTED;
    }
    if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
  }
  // small batches: fewer tokens per tile so more SMs share the work
  int tok = (T + per_sm * sms - 1) / (per_sm * sms);
  if (tok > tok_max) tok = tok_max;
  if (tok < 1) tok = 1;
  AppendArgs a;
  a.T = T;
  a.H = d.num_kv_heads;
  a.P = d.page_size;
  a.lg_page = 0;
  while ((1 << a.lg_page) < d.page_size) ++a.lg_page;
  a.NP = d.num_pages;
  a.num_seqs = num_seqs;
  a.bt_stride = bt_stride;
  a.tok_per_tile = tok;
  a.num_tiles = (T + tok - 1) / tok;
  a.box_stride = (tok * d.num_kv_heads * 128 + 1023) / 1024 * 1024;
  a.token_seq = token_seq;
  a.token_pos = token_pos;
  a.block_table = block_table;
  a.k_codes = k_codes;
  a.v_codes = v_codes;
  a.k_params = static_cast<uint32_t*>(k_params);
  a.v_params = static_cast<uint32_t*>(v_params);
  a.quat = rot_table(d);
  a.rope = d.rope;
  a.rope_max_pos = d.rope_max_pos;
  a.err = err;
  a.fmt = d.format;
  a.levels = d.levels;
  CUtensorMap tk, tv;
  if (!encode_rows(&tk, k, D, a.H, T, tok_stride, a.H, tok) ||
      !encode_rows(&tv, v, D, a.H, T, tok_stride, a.H, tok))
    return KVQ_ERR_CUDA;
  const int grid = a.num_tiles < per_sm * sms ? a.num_tiles : per_sm * sms;
  cudaError_t e;
  switch (D) {
    case 64: e = dispatch_rot<64>(a, tk, tv, rot_template(d), lgb, grid, st); break;
    case 128: e = dispatch_rot<128>(a, tk, tv, rot_template(d), lgb, grid, st); break;
    case 256: e = dispatch_rot<256>(a, tk, tv, rot_template(d), lgb, grid, st); break;
    default: return KVQ_ERR_UNSUPPORTED;
  }
  if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
