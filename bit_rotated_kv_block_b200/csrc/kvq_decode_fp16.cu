// Baseline: paged decode attention over an unquantized binary16 cache.
//
// The method's claim is that the rotated INT4 cache keeps the throughput of a
// plain INT4 cache while giving up little accuracy against full precision
// ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving", Summary and Key takeaways). This kernel is the full-precision
// side of that comparison: the same paged layout ([page][kv_head][slot][d]
// binary16 for K and for V, no parameters), no rotation, and the same
// decomposition as the INT4 kernel (one warp per (sequence, KV head, split),
// split merge by the last-arriving warp).
//
//  * Pages are staged into a per-warp ring with 16-byte cp.async copies; each
//    16-byte unit u of token row t lands at unit u ^ (t & 7) of the row, so
//    the 8x8 ldmatrix loads below are free of bank conflicts.
//  * QK: mma.sync m16n8k16 f16 -> f32, A = the query rows of the GP heads
//    (binary16 input, exact), B = K rows loaded with ldmatrix.
//  * PV: A = V^T fragments loaded with ldmatrix.trans, B = the weights p as
//    binary16 hi + lo columns; each 16-token product joins the running sum
//    through an IEEE round-to-nearest add.
//  * Online softmax in base 2 with a binary32 running max.
#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_launch.h"

namespace kvq {

constexpr int kF16Warps = 4;
constexpr int kF16MaxPages = 256;  // page ids of one work item live in shared memory

struct F16Args {
  int S, Hq, H, G, P, NP, bt_stride, max_seq_len, splits, pages_per_split;
  float scale2;          // sm_scale * log2(e)
  const __half* q;       // [S][Hq][D]
  const int32_t* seq_lens;
  const int32_t* block_table;
  const __half* k;       // [NP][H][P][D]
  const __half* v;       // [NP][H][P][D]
  float* out;            // [S][Hq][D]
  float* part;           // [S][Hq][splits][D + 4]: acc[D], max, sum, pad
  int32_t* counter;      // [S][H], zero between calls
  int32_t* err;
};

template <int D, int P, int GP>
struct F16Cfg {
  static constexpr int ROWB = D * 2;          // bytes per token row
  static constexpr int UPR = ROWB / 16;       // 16-byte units per row
  static constexpr int CHUNK = P * ROWB;      // bytes per (page, head) of one pool
  static constexpr int STAGE_B = 2 * CHUNK;   // K rows then V rows
  static constexpr int NST = STAGE_B <= 8192 ? 3 : 2;
  static constexpr int WARP_B = NST * STAGE_B + kF16MaxPages * 4;
  static constexpr int TILES = P / 16;        // 16-token tiles per page
  static constexpr int NKS = D / 16;          // QK k-steps
  static constexpr int NMT = D / 16;          // PV m-tiles (16 channels)
  static constexpr int NPV = GP == 8 ? 2 : 1; // PV n-tiles (hi / lo columns)
  static_assert(UPR >= 8, "rows of at least 128 bytes");
};

// byte offset of 16-byte unit u of token row t inside a stage's K or V rows
template <int D>
__device__ __forceinline__ int f16_unit(int t, int u) {
  return t * (D * 2) + ((u ^ (t & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Lane (g, t) = (lane / 4, lane % 4). QK: row g of the A operand is query
// head g (GP = 4: rows 4..15 are zero), so lane (g, t) ends with the scores of
// head g and tokens 8nt + 2t + {0, 1} of each 16-token tile (nt = 0, 1).
template <int D, int P, int GP>
__global__ void __launch_bounds__(kF16Warps * kWarp)
    decode_fp16_kernel(const F16Args a) {
  using C = F16Cfg<D, P, GP>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int g = lane >> 2, t = lane & 3;
  const int item = blockIdx.x * kF16Warps + warp;
  const int per_seq = a.H * a.splits;
  if (item >= a.S * per_seq) return;
  const int s = item / per_seq;
  const int h = (item / a.splits) % a.H;
  const int split = item % a.splits;
  uint8_t* ring = smem + warp * C::WARP_B;
  int32_t* ids = reinterpret_cast<int32_t*>(ring + C::NST * C::STAGE_B);

  const bool head_ok = g < a.G && g < GP;  // lane's score row is a real query head
  int L = a.seq_lens[s];
  const int pbeg = split * a.pages_per_split;
  {
    int nload = a.bt_stride - pbeg;
    nload = nload < a.pages_per_split ? nload : a.pages_per_split;
    for (int c = lane; c < nload; c += kWarp) ids[c] = a.block_table[(int64_t)s * a.bt_stride + pbeg + c];
  }
  // query A fragments: head g, channels 16kk + 2t + {0, 1} and + 8
  uint32_t qf[C::NKS][2];
  {
    const uint32_t* qrow =
        reinterpret_cast<const uint32_t*>(a.q + ((int64_t)s * a.Hq + h * a.G + (head_ok ? g : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < C::NKS; ++kk) {
      qf[kk][0] = head_ok ? qrow[8 * kk + t] : 0u;
      qf[kk][1] = head_ok ? qrow[8 * kk + 4 + t] : 0u;
    }
  }
  const bool len_ok = L >= 0 && L <= a.max_seq_len && (L + P - 1) / P <= a.bt_stride;
  if (!len_ok) {
    if (lane == 0 && h == 0 && split == 0) raise_flag(a.err, KVQ_ERRF_LEN);
    L = 0;
  }
  const int npages = (L + P - 1) / P;
  int pend = pbeg + a.pages_per_split;
  if (pend > npages) pend = npages;
  const int nmine = pend > pbeg ? pend - pbeg : 0;
  __syncwarp();

  // ---- page ring (cp.async, one commit group per page)
  const int64_t pstride = (int64_t)a.H * P * D;  // elements between pages of one pool
  const __half* kh = a.k + (int64_t)h * P * D;
  const __half* vh = a.v + (int64_t)h * P * D;
  auto issue = [&](int i) {
    if (i < nmine) {
      const int page = ids[i];
      if (page >= 0 && page < a.NP) {
        uint8_t* st = ring + (i % C::NST) * C::STAGE_B;
        const uint8_t* ks = reinterpret_cast<const uint8_t*>(kh + (int64_t)page * pstride);
        const uint8_t* vs = reinterpret_cast<const uint8_t*>(vh + (int64_t)page * pstride);
#pragma unroll
        for (int m = 0; m < P * C::UPR / kWarp; ++m) {
          const int u = lane + kWarp * m;  // unit u of the chunk: token u / UPR, unit u % UPR
          const int off = f16_unit<D>(u / C::UPR, u % C::UPR);
          cp_async16(st + off, ks + u * 16);
          cp_async16(st + C::CHUNK + off, vs + u * 16);
        }
      }
    }
    cp_async_commit();
  };
  for (int i = 0; i < C::NST - 1; ++i) issue(i);

  // ldmatrix row addresses (stage 0, tile 0): QK, lane l -> token 8nt + (l & 7),
  // unit 2kk + (l >> 3) for k-step pair kk; PV, lane l -> token (l & 7) + 8 (l >> 4),
  // unit 2mt + ((l >> 3) & 1)
  const uint32_t ring_s = smem_u32(ring);
  const int qk_tok = lane & 7, qk_u = lane >> 3;
  const int pv_tok = (lane & 7) + 8 * (lane >> 4), pv_u = (lane >> 3) & 1;

  float acc[C::NMT][C::NPV][4];
#pragma unroll
  for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
    for (int n = 0; n < C::NPV; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][n][e] = 0.f;
  float M = -INFINITY, Lp = 0.f;

  for (int i = 0; i < nmine; ++i) {
    issue(i + C::NST - 1);
    cp_async_wait<C::NST - 1>();
    __syncwarp();
    const int page = ids[i];
    const bool page_ok = page >= 0 && page < a.NP;
    if (!page_ok && lane == 0) raise_flag(a.err, KVQ_ERRF_PAGE);
    const uint32_t st = ring_s + (i % C::NST) * C::STAGE_B;
    const int tok0 = (pbeg + i) * P;

    float z[C::TILES][4];  // head g, tokens 16tt + 8(e >> 1) + 2t + (e & 1)
#pragma unroll
    for (int tt = 0; tt < C::TILES; ++tt) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float c4[4] = {0.f, 0.f, 0.f, 0.f};
        const int tok = 16 * tt + 8 * nt + qk_tok;
#pragma unroll
        for (int kp = 0; kp < C::NKS / 2; ++kp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(st + f16_unit<D>(tok, 4 * kp + qk_u), b0, b1, b2, b3);
          const uint32_t a0[4] = {qf[2 * kp][0], 0u, qf[2 * kp][1], 0u};
          const uint32_t a1[4] = {qf[2 * kp + 1][0], 0u, qf[2 * kp + 1][1], 0u};
          mma16816(c4, a0, b0, b1);
          mma16816(c4, a1, b2, b3);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int tk = tok0 + 16 * tt + 8 * nt + 2 * t + c;
          z[tt][2 * nt + c] = (page_ok && tk < L) ? c4[c] * a.scale2 : -INFINITY;
        }
      }
    }

    // ---- online softmax of head g over the four lanes t
    float mloc = -INFINITY;
#pragma unroll
    for (int tt = 0; tt < C::TILES; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) mloc = fmaxf(mloc, z[tt][e]);
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    const float Mn = fmaxf(M, mloc);
    const float alpha = (Mn == M) ? 1.f : fast_exp2(M - Mn);  // M = -inf: 0
    M = Mn;
    Lp *= alpha;
    // accumulator columns of lane (g, t): heads c0, c0 + 1 with
    // c0 = 2t (GP = 8) or 2(t & 1) (GP = 4: t >= 2 hold the lo columns)
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
      const int c0 = (GP == 8) ? 2 * t : 2 * (t & 1);
      const float a0 = __shfl_sync(0xffffffffu, alpha, 4 * c0);
      const float a1 = __shfl_sync(0xffffffffu, alpha, 4 * c0 + 4);
#pragma unroll
      for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
        for (int n = 0; n < C::NPV; ++n) {
          acc[mt][n][0] *= a0; acc[mt][n][1] *= a1;
          acc[mt][n][2] *= a0; acc[mt][n][3] *= a1;
        }
    }

    // ---- PV per tile
#pragma unroll
    for (int tt = 0; tt < C::TILES; ++tt) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = z[tt][e] == -INFINITY ? 0.f : fast_exp2(z[tt][e] - M);
        Lp += p[e];
      }
      // B operand: column n = head (GP = 8: n-tile 0 hi, 1 lo; GP = 4: columns
      // 0-3 hi of heads 0-3, 4-7 lo of heads 0-3, lanes g >= 4 take the lo
      // of head g - 4 from lane g - 4)
      const __half2 h01 = __floats2half2_rn(p[0], p[1]);
      const __half2 h89 = __floats2half2_rn(p[2], p[3]);
      const float2 f01 = __half22float2(h01), f89 = __half22float2(h89);
      const uint32_t lo01 = h2_as_u32(__floats2half2_rn(p[0] - f01.x, p[1] - f01.y));
      const uint32_t lo89 = h2_as_u32(__floats2half2_rn(p[2] - f89.x, p[3] - f89.y));
      uint32_t pb[C::NPV][2];
      if (GP == 8) {
        pb[0][0] = h2_as_u32(h01);
        pb[0][1] = h2_as_u32(h89);
        pb[C::NPV - 1][0] = lo01;
        pb[C::NPV - 1][1] = lo89;
      } else {
        const uint32_t l01 = __shfl_sync(0xffffffffu, lo01, lane & 15);
        const uint32_t l89 = __shfl_sync(0xffffffffu, lo89, lane & 15);
        pb[0][0] = g >= 4 ? l01 : h2_as_u32(h01);
        pb[0][1] = g >= 4 ? l89 : h2_as_u32(h89);
      }
      if (GP == 4 ? (g & 3) >= a.G : g >= a.G) {
#pragma unroll
        for (int n = 0; n < C::NPV; ++n) pb[n][0] = pb[n][1] = 0u;
      }
#pragma unroll
      for (int mt = 0; mt < C::NMT; ++mt) {
        uint32_t av[4];
        ldsm_x4_t(st + C::CHUNK + f16_unit<D>(16 * tt + pv_tok, 2 * mt + pv_u), av[0], av[1], av[2],
                  av[3]);
        // av: [0] channels 16mt + g, tokens 2t..; [1] channels + 8; [2], [3]
        // the same for tokens 2t + 8.. (matrix order: (tokens 0-7, ch 0-7),
        // (tokens 0-7, ch 8-15), (tokens 8-15, ch 0-7), (tokens 8-15, ch 8-15))
        const uint32_t afr[4] = {av[0], av[1], av[2], av[3]};
#pragma unroll
        for (int n = 0; n < C::NPV; ++n) {
          float t4[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(t4, afr, pb[n][0], pb[n][1]);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][n][e] = __fadd_rn(acc[mt][n][e], t4[e]);
        }
      }
    }
    __syncwarp();  // the stage is refilled by the next issue
  }
  cp_async_wait<0>();

  // ---- partial results: acc per channel, max and sum per query head
  Lp += __shfl_xor_sync(0xffffffffu, Lp, 1);
  Lp += __shfl_xor_sync(0xffffffffu, Lp, 2);
  if (GP == 4) {
    // fold the lo columns (lanes t = 2, 3) onto the hi columns (t = 0, 1)
#pragma unroll
    for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][0][e] += __shfl_xor_sync(0xffffffffu, acc[mt][0][e], 2);
  }
  const int c0 = (GP == 8) ? 2 * t : 2 * (t & 1);
  const bool writer = (GP == 8) || (t < 2);
  const int64_t base = ((int64_t)s * a.Hq + (int64_t)h * a.G) * a.splits + split;
#pragma unroll
  for (int hc = 0; hc < 2; ++hc) {
    const int gh = c0 + hc;
    if (!writer || gh >= a.G) continue;
    float* dst = a.part + (base + (int64_t)gh * a.splits) * (D + 4);
#pragma unroll
    for (int mt = 0; mt < C::NMT; ++mt) {
      float v0 = 0.f, v1 = 0.f;
#pragma unroll
      for (int n = 0; n < C::NPV; ++n) {
        v0 += acc[mt][n][hc];
        v1 += acc[mt][n][2 + hc];
      }
      dst[16 * mt + g] = v0;
      dst[16 * mt + 8 + g] = v1;
    }
  }
  if (t == 0 && head_ok) {
    float* dst = a.part + (base + (int64_t)g * a.splits) * (D + 4);
    dst[D] = M;
    dst[D + 1] = Lp;
  }

  // ---- the last warp of this (sequence, KV head) merges the splits
  __syncwarp();
  int last = 0;
  if (lane == 0) {
    int prev;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                 : "=r"(prev)
                 : "l"(a.counter + (int64_t)s * a.H + h)
                 : "memory");
    last = prev == a.splits - 1;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __syncwarp();  // extends lane 0's acquire to the lanes that read the partials
  // lane l: query head l / (32 / GP) of the group, channels of its share
  constexpr int LPH = kWarp / GP;  // lanes per head (8 or 4)
  constexpr int CW = D / LPH;      // channels per lane
  const int hh = lane / LPH, sub = lane % LPH;
  if (hh < a.G) {
    const float* src = a.part + ((int64_t)s * a.Hq + h * a.G + hh) * a.splits * (D + 4);
    float Mx = -INFINITY;
    for (int i = 0; i < a.splits; ++i) Mx = fmaxf(Mx, __ldcg(src + (int64_t)i * (D + 4) + D));
    float x[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) x[c] = 0.f;
    float Ls = 0.f;
    if (Mx != -INFINITY) {
#pragma unroll 2
      for (int i = 0; i < a.splits; ++i) {
        const float* pi = src + (int64_t)i * (D + 4);
        const float Mi = __ldcg(pi + D);
        const float li = __ldcg(pi + D + 1);
        float4 f[CW / 4];
#pragma unroll
        for (int c = 0; c < CW / 4; ++c) f[c] = __ldcg(reinterpret_cast<const float4*>(pi + sub * CW) + c);
        const float wgt = Mi == -INFINITY ? 0.f : fast_exp2(Mi - Mx);
        Ls += wgt * li;
#pragma unroll
        for (int c = 0; c < CW / 4; ++c) {
          x[4 * c] += wgt * f[c].x;
          x[4 * c + 1] += wgt * f[c].y;
          x[4 * c + 2] += wgt * f[c].z;
          x[4 * c + 3] += wgt * f[c].w;
        }
      }
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    float4* dst = reinterpret_cast<float4*>(a.out + ((int64_t)s * a.Hq + h * a.G + hh) * D + sub * CW);
#pragma unroll
    for (int c = 0; c < CW / 4; ++c)
      dst[c] = make_float4(x[4 * c] * inv, x[4 * c + 1] * inv, x[4 * c + 2] * inv, x[4 * c + 3] * inv);
  }
  if (lane == 0) a.counter[(int64_t)s * a.H + h] = 0;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

#define KVQ_F16_CONFIGS(X)                                                                     \
  X(128, 16, 4) X(128, 16, 8) X(128, 32, 4) X(128, 32, 8) X(128, 64, 4) X(128, 64, 8)          \
  X(256, 16, 4) X(256, 32, 4)

template <int D, int P, int GP>
static size_t f16_smem() {
  return (size_t)kF16Warps * F16Cfg<D, P, GP>::WARP_B;
}

template <int D, int P, int GP>
static int f16_resident_warps() {
  static int cached = -1;
  if (cached < 0) {
    auto kern = decode_fp16_kernel<D, P, GP>;
    const size_t smem = f16_smem<D, P, GP>();
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kF16Warps * kWarp, smem) !=
        cudaSuccess)
      blocks = 1;
    const int sms = device_sm_count();
    cached = (blocks < 1 ? 1 : blocks) * kF16Warps * (sms > 0 ? sms : 148);
  }
  return cached;
}

static int f16_target(int D, int P, int GP) {
#define KVQ_F16_RW(d_, p_, g_) \
  if (D == d_ && P == p_ && GP == g_) return f16_resident_warps<d_, p_, g_>();
  KVQ_F16_CONFIGS(KVQ_F16_RW)
#undef KVQ_F16_RW
  return -1;
}

DecodePlan decode_fp16_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len) {
  DecodePlan pl{};
  const int P = d.page_size;
  pl.pages_max = (max_seq_len + P - 1) / P;
  if (pl.pages_max < 1) pl.pages_max = 1;
  const int G = Hq / d.num_kv_heads;
  const int GP = G <= 4 ? 4 : 8;
  int target = f16_target(d.head_dim, P, GP);
  if (target < 1) target = 148 * 8;
  const int pairs = S * d.num_kv_heads;
  int splits = target / (pairs > 0 ? pairs : 1);
  const int min_splits = (pl.pages_max + kF16MaxPages - 1) / kF16MaxPages;
  if (splits < min_splits) splits = min_splits;
  if (splits < 1) splits = 1;
  if (splits > pl.pages_max) splits = pl.pages_max;
  pl.pages_per_split = (pl.pages_max + splits - 1) / splits;
  pl.splits = (pl.pages_max + pl.pages_per_split - 1) / pl.pages_per_split;
  pl.nhi = S * d.num_kv_heads;  // every pair has `splits` splits
  const size_t counters = (size_t)S * d.num_kv_heads * sizeof(int32_t);
  const size_t parts = (size_t)S * Hq * pl.splits * (d.head_dim + 4) * sizeof(float);
  pl.workspace = (counters + 255) / 256 * 256 + parts;
  return pl;
}

template <int D, int P, int GP>
static cudaError_t launch_f16(const F16Args& a, cudaStream_t st) {
  auto kern = decode_fp16_kernel<D, P, GP>;
  const size_t smem = f16_smem<D, P, GP>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int items = a.S * a.H * a.splits;
  kern<<<(items + kF16Warps - 1) / kF16Warps, kF16Warps * kWarp, smem, st>>>(a);
  return cudaGetLastError();
}

int decode_fp16_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                       const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                       int32_t bt_stride, float sm_scale, const void* k_pages,
                       const void* v_pages, float* out, void* workspace, size_t workspace_bytes,
                       int32_t* err, cudaStream_t st) {
  const int D = d.head_dim, P = d.page_size;
  const int G = Hq / d.num_kv_heads;
  const int GP = G <= 4 ? 4 : 8;
  if (f16_target(D, P, GP) < 0) return KVQ_ERR_UNSUPPORTED;
  const DecodePlan pl = decode_fp16_plan(d, S, Hq, max_seq_len);
  if (workspace == nullptr || workspace_bytes < pl.workspace) return KVQ_ERR_WORKSPACE;
  F16Args a;
  a.S = S; a.Hq = Hq; a.H = d.num_kv_heads; a.G = G; a.P = P; a.NP = d.num_pages;
  a.bt_stride = bt_stride; a.max_seq_len = max_seq_len; a.splits = pl.splits;
  a.pages_per_split = pl.pages_per_split;
  a.scale2 = sm_scale * 1.4426950408889634f;
  a.q = static_cast<const __half*>(q);
  a.seq_lens = seq_lens; a.block_table = block_table;
  a.k = static_cast<const __half*>(k_pages); a.v = static_cast<const __half*>(v_pages);
  a.out = out;
  a.counter = static_cast<int32_t*>(workspace);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                    ((size_t)S * d.num_kv_heads * sizeof(int32_t) + 255) / 256 * 256);
  a.err = err;
  cudaError_t e = cudaErrorInvalidValue;
#define KVQ_F16_LS(d_, p_, g_) \
  if (D == d_ && P == p_ && GP == g_) e = launch_f16<d_, p_, g_>(a, st);
  KVQ_F16_CONFIGS(KVQ_F16_LS)
#undef KVQ_F16_LS
  if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
