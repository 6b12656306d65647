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
//  * One thread owns E = min(d, 128) consecutive channels of one (token, head)
//    row of K or V, so every butterfly stage of a block of up to 128 channels
//    runs in registers without shuffles; d = 256 uses two threads per row and
//    one xor-1 shuffle stage for b = 256.
//  * A CTA of 256 threads owns a tile of TOK tokens x {K, V} x H heads. The
//    tile's fp16 rows are copied global -> shared with coalesced 16-byte
//    cp.async (row pitch 2E + 16 bytes, so each thread then reads its own row
//    with conflict-free 128-bit loads) while the previous tile is computed
//    (two buffers). The grid is persistent: one CTA per SM walks the tiles.
//  * Threads are ordered head-major, token-minor, so a warp writes the codes
//    of up to 32 consecutive slots of one (page, head) chunk.
//  * Arithmetic is bit-exact with the published definition (see kvq.h):
//    binary32 butterflies in ascending stage order (packed f32x2 lanes for
//    stages >= 2), directed roundings through __fsub_ru / __fdiv_ru /
//    __float2half_rd / __float2half_ru, RN(1/s) by __frcp_rn, and code
//    rounding by adding 1.5 * 2^23 (exact round-half-even for values in
//    [0, 2^22)); the [0, 15] clamp of the definition never acts because
//    every value lies in [m16, m16 + 15 s16], so the low nibble is the code.

#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_launch.h"
#include "kvq_rotate.cuh"

namespace kvq {

constexpr int kAppendThreads = 256;

struct AppendArgs {
  int T, H, P, NP, num_seqs, bt_stride, tok_per_tile, num_tiles;
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
  int32_t* err;
};

// D: head_dim, ROT: rotation kind, LGB: log2 of the Hadamard block.
template <int D, int ROT, int LGB>
__global__ void __launch_bounds__(kAppendThreads, 1) append_kernel(const AppendArgs a) {
  constexpr int E = D < 128 ? D : 128;   // channels per thread
  constexpr int TPR = D / E;             // threads per row
  constexpr int ROWB = 2 * E + 16;       // shared-memory pitch of a thread row
  constexpr int CHUNKS = D / 8;          // 16-byte chunks per (token, head) row

  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* buf0 = smem;
  uint8_t* buf1 = smem + kAppendThreads * ROWB;
  float* qtbl = reinterpret_cast<float*>(smem + 2 * kAppendThreads * ROWB);

  const int tid = threadIdx.x;
  const int H = a.H, TOK = a.tok_per_tile;
  const int rows_per_tile = 2 * H * TOK * TPR;

  if (ROT == KVQ_ROT_QUAT) {
    for (int i = tid; i < D * 2; i += kAppendThreads) qtbl[i] = a.quat[i];
  }

  // this thread's role, fixed for all tiles: thread row = ((kv*H + h)*TOK + t)*TPR + part
  const bool active = tid < rows_per_tile;
  int my_part = 0, my_t = 0, my_h = 0, my_kv = 0;
  if (active) {
    my_part = tid % TPR;
    const int r = tid / TPR;
    my_t = r % TOK;
    my_h = (r / TOK) % H;
    my_kv = r / (TOK * H);
  }

  auto issue_tile = [&](int tile, uint8_t* buf) {
    const int t0 = tile * TOK;
    const int warp = tid / kWarp, lane = tid % kWarp;
    // one (kv, token) row of H*D halves per warp iteration
    for (int r = warp; r < 2 * TOK; r += kAppendThreads / kWarp) {
      const int kv = r / TOK, t = r % TOK;
      if (t0 + t >= a.T) continue;
      const __half* src = (kv ? a.v : a.k) + (int64_t)(t0 + t) * a.tok_stride;
      for (int c = lane; c < H * CHUNKS; c += kWarp) {
        const int h = c / CHUNKS, w = c % CHUNKS;
        const int ch = w * 8;
        const int tr = ((kv * H + h) * TOK + t) * TPR + ch / E;
        cp_async16(buf + tr * ROWB + (ch % E) * 2, src + h * D + ch);
      }
    }
  };

  // Destination of this thread's row, resolved one tile ahead so the
  // dependent metadata loads (token -> sequence/position -> block table) are
  // in flight while the previous tile computes. row_dst < 0: no store.
  const bool lead = my_kv == 0 && my_h == 0 && my_part == 0;  // raises the token's flags
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
    if (pos < 0 || pos / a.P >= a.bt_stride) {
      if (lead) raise_flag(a.err, KVQ_ERRF_POS);
      return -1;
    }
    const int page = a.block_table[(int64_t)seq * a.bt_stride + pos / a.P];
    if (page < 0 || page >= a.NP) {
      if (lead) raise_flag(a.err, KVQ_ERRF_PAGE);
      return -1;
    }
    return ((int64_t)page * H + my_h) * a.P + pos % a.P;
  };

  int tile = blockIdx.x;
  if (tile < a.num_tiles) issue_tile(tile, buf0);
  cp_async_commit();
  int seq_n, pos_n;
  meta_load(tile, seq_n, pos_n);
  int64_t dst_cur = resolve(seq_n, pos_n);
  __syncthreads();  // quaternion table visible

  for (int it = 0; tile < a.num_tiles; ++it, tile += gridDim.x) {
    uint8_t* cur = (it & 1) ? buf1 : buf0;
    uint8_t* nxt = (it & 1) ? buf0 : buf1;
    const int next = tile + gridDim.x;
    if (next < a.num_tiles) issue_tile(next, nxt);
    cp_async_commit();
    meta_load(next, seq_n, pos_n);  // consumed after this tile's compute
    cp_async_wait<1>();
    __syncthreads();

    const int tok = tile * TOK + my_t;
    // rows of tokens past the batch end do nothing; every other active row
    // computes (the two threads of a d = 256 row always agree) and stores
    // only if its destination resolved
    if (active && tok < a.T) {
      {
        float x[E];
        const uint4* row = reinterpret_cast<const uint4*>(cur + tid * ROWB);
#pragma unroll
        for (int c = 0; c < E / 8; ++c) {
          const uint4 u = row[c];
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(u32_as_h2(w[q]));
            x[8 * c + 2 * q] = f.x;
            x[8 * c + 2 * q + 1] = f.y;
          }
        }

        // the two threads of a d = 256 row are lanes 2i, 2i+1 of one warp
        const unsigned pair_mask = 3u << ((tid % kWarp) & ~1);
        if (ROT == KVQ_ROT_HADAMARD) {
          hadamard_regs<E, LGB>(x, my_part, pair_mask);
        } else if (ROT == KVQ_ROT_QUAT) {
          quat_regs<E>(x, qtbl, my_part * E);
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
        mn = __fadd_rn(mn, 0.0f);
        mx = __fadd_rn(mx, 0.0f);
        const __half m16 = __float2half_rd(mn);
        const float m = __half2float(m16);
        const float s32 = __fdiv_ru(__fsub_ru(mx, m), 15.0f);
        const __half s16 = __float2half_ru(s32);
        const float s = __half2float(s16);

        uint32_t packed[E / 8];
        if (s != 0.0f) {
          const float inv = __frcp_rn(s);
          const uint64_t m2 = pk(m, m);
          const uint64_t magic2 = pk(12582912.0f, 12582912.0f);  // 1.5 * 2^23
#pragma unroll
          for (int c = 0; c < E / 8; ++c) {
            uint32_t b[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              // the product must be rounded on its own before the rounding
              // add: __fmul_rn is never contracted into a fused multiply-add
              // (the packed multiply was seen to be, at exact .5 ties)
              const float2 t = upk(sub2(pk(x[8 * c + 2 * q], x[8 * c + 2 * q + 1]), m2));
              const float t1x = __fmul_rn(t.x, inv), t1y = __fmul_rn(t.y, inv);
              const float2 r = upk(add2(pk(t1x, t1y), magic2));
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
          uint8_t* codes = my_kv ? a.v_codes : a.k_codes;
          uint32_t* params = my_kv ? a.v_params : a.k_params;
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
    }
    dst_cur = resolve(seq_n, pos_n);  // next tile's destination (its loads were in flight)
    __syncthreads();  // buffer `cur` is refilled by the next iteration's issue
  }
  cp_async_wait<0>();
}

template <int D, int ROT, int LGB>
static cudaError_t launch_append(const AppendArgs& a, int grid, cudaStream_t st) {
  constexpr int E = D < 128 ? D : 128;
  const size_t smem = 2 * kAppendThreads * (2 * E + 16) + D * 2 * sizeof(float);
  auto kern = append_kernel<D, ROT, LGB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kAppendThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_rot(const AppendArgs& a, int rot, int lgb, int grid, cudaStream_t st) {
  if (rot == KVQ_ROT_NONE) return launch_append<D, KVQ_ROT_NONE, 0>(a, grid, st);
  if (rot == KVQ_ROT_QUAT) return launch_append<D, KVQ_ROT_QUAT, 0>(a, grid, st);
  switch (lgb) {
    case 4: return launch_append<D, KVQ_ROT_HADAMARD, 4>(a, grid, st);
    case 5: return launch_append<D, KVQ_ROT_HADAMARD, 5>(a, grid, st);
    case 6: return launch_append<D, KVQ_ROT_HADAMARD, 6>(a, grid, st);
    case 7: if (D >= 128) return launch_append<D, KVQ_ROT_HADAMARD, (D >= 128 ? 7 : 6)>(a, grid, st); break;
    case 8: if (D >= 256) return launch_append<D, KVQ_ROT_HADAMARD, (D >= 256 ? 8 : 6)>(a, grid, st); break;
  }
  return cudaErrorInvalidValue;
}

int append_launch(const kvq_cache_desc& d, int32_t T, const void* k, const void* v,
                  int64_t tok_stride, const int32_t* token_seq, const int32_t* token_pos,
                  int32_t num_seqs, const int32_t* block_table, int32_t bt_stride,
                  uint8_t* k_codes, void* k_params, uint8_t* v_codes, void* v_params,
                  int32_t* err, cudaStream_t st) {
  const int D = d.head_dim;
  const int E = D < 128 ? D : 128;
  const int TPR = D / E;
  const int tok_max = kAppendThreads / (2 * d.num_kv_heads * TPR);
  if (tok_max < 1) return KVQ_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  if (sms <= 0) return KVQ_ERR_CUDA;
  // small batches: fewer tokens per tile so more SMs share the work
  int tok = (T + sms - 1) / sms;
  if (tok > tok_max) tok = tok_max;
  if (tok < 1) tok = 1;
  AppendArgs a;
  a.T = T;
  a.H = d.num_kv_heads;
  a.P = d.page_size;
  a.NP = d.num_pages;
  a.num_seqs = num_seqs;
  a.bt_stride = bt_stride;
  a.tok_per_tile = tok;
  a.num_tiles = (T + tok - 1) / tok;
  a.tok_stride = tok_stride;
  a.k = static_cast<const __half*>(k);
  a.v = static_cast<const __half*>(v);
  a.token_seq = token_seq;
  a.token_pos = token_pos;
  a.block_table = block_table;
  a.k_codes = k_codes;
  a.v_codes = v_codes;
  a.k_params = static_cast<uint32_t*>(k_params);
  a.v_params = static_cast<uint32_t*>(v_params);
  a.quat = d.quat;
  a.err = err;
  const int grid = a.num_tiles < sms ? a.num_tiles : sms;
  int lgb = 0;
  while ((1 << lgb) < d.rot_block) ++lgb;
  cudaError_t e;
  switch (D) {
    case 64: e = dispatch_rot<64>(a, d.rot_kind, lgb, grid, st); break;
    case 128: e = dispatch_rot<128>(a, d.rot_kind, lgb, grid, st); break;
    case 256: e = dispatch_rot<256>(a, d.rot_kind, lgb, grid, st); break;
    default: return KVQ_ERR_UNSUPPORTED;
  }
  if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
