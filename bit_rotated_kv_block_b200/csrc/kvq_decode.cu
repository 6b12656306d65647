// Paged decode attention over the rotated INT4 cache.
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
// LLM Serving" (Summary, Key takeaway): the INT4 cache is read by attention in
// its paged layout; the query is rotated by the same orthogonal block
// Hadamard (or quaternion) map as the keys, so q . k is unchanged, and the
// output is rotated back once per query head.
//
// One kernel, one warp per (sequence, KV head, split of the page range):
//  1. The warp rotates its query heads in registers: lane (r, j) holds
//     channels [j*d/4, (j+1)*d/4) of query head r (GP = 8) or r % 4 (GP = 4);
//     butterfly stages inside a quarter run in registers, wider ones across
//     lanes j by shuffles.
//  2. It streams its (page, KV head) chunks (codes + params of K and V,
//     contiguous in the pool) into a 2-4 stage shared-memory ring with
//     cp.async and runs both contractions on tensor cores (mma.sync
//     m16n8k16, f16 x f16 -> f32):
//       QK^T: A = [qhat_hi ; qhat_lo] rows of the query heads, B = K codes
//             (c - 8, exact in f16) as columns, so the score fragment of head
//             r for tokens {2j, 2j+1, 2j+8, 2j+9} already sits in lane (r, j)
//             -- exactly the B operand layout of the PV product;
//       PV:   A = V codes transposed (channels x tokens) built from nibbles
//             with prmt/lop3, B = p * s_v split into f16 hi + lo columns.
//     Scale and zero-point are applied algebraically:
//       qhat . khat = s_k * sum (c - 8) qhat + (m_k + 8 s_k) sum qhat,
//       sum p vhat  = sum (p s_v)(c - 8)     + sum p (m_v + 8 s_v).
//     Online softmax in base 2.
//  3. It writes (acc, max, sum) per query head to the workspace, fences, and
//     bumps a per-(sequence, KV head) counter; the warp that brings the
//     counter to the number of splits merges all splits (log-sum-exp),
//     normalises, rotates back in registers, writes the float32 output and
//     resets the counter to zero. No warp ever waits on another.
#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_launch.h"
#include "kvq_rotate.cuh"

namespace kvq {

constexpr int kDecWarps = 4;
constexpr int kMaxPagesPerSplit = 256;  // page ids of one work item live in shared memory
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  int S, Hq, H, G, P, NP, bt_stride, max_seq_len, splits, pages_per_split;
  int rot_kind, lgb;
  double scale2;  // sm_scale * log2(e), in double
  const __half* q;  // [S][Hq][D]
  const float* quat;
  const int32_t* seq_lens;
  const int32_t* block_table;
  const uint8_t* k_codes;
  const uint32_t* k_params;
  const uint8_t* v_codes;
  const uint32_t* v_params;
  float* out;        // [S][Hq][D]
  float* part;       // [S][Hq][splits][D + 4]: acc[D], max (double), sum, pad
  int32_t* counter;  // [S][H], zero between calls
  int32_t* err;
};

// ---------------------------------------------------------------------------
// 2. split kernel
// ---------------------------------------------------------------------------

template <int D, int P, int GP>
struct DecCfg {
  static constexpr int NKS8 = D / 32;          // QK int8 k-steps over channels
  static constexpr int NQT = GP == 8 ? 2 : 1;  // 16-row tiles of query limbs
  static constexpr int NMT = D / 16;           // PV m-tiles over channels
  static constexpr int TILES = P / 16;         // 16-token tiles per page
  static constexpr int NPV = GP == 8 ? 2 : 1;  // PV n-tiles (hi / lo columns)
  static constexpr int QW = D / 4;             // query channels per lane
  static constexpr int ROWB = D / 2;           // code bytes per token
  static constexpr int CODE_B = P * ROWB;      // code bytes per (page, head)
  static constexpr int STAGE_B = 2 * CODE_B + 8 * P;
  // pipeline depth: about 8-13 KB of pages in flight per warp
  static constexpr int NST = STAGE_B <= 2304 ? 4 : (STAGE_B <= 4608 ? 3 : 2);
  static constexpr int IDS_B = kMaxPagesPerSplit * 4;
  static constexpr int WARP_B = NST * STAGE_B + IDS_B;
};

// Swizzled position of the 16-byte unit `u` of token `t` in the V code
// buffer (conflict-free transposing reads; see the PV fragment loads).
template <int D>
__device__ __forceinline__ int v_unit_off(int t, int u) {
  if (D == 128) {  // 64-byte rows: line = t / 2 holds tokens 2l, 2l+1
    const int line = t >> 1, un = ((t & 1) << 2) | u;
    return line * 128 + ((un ^ ((line & 3) << 1)) << 4);
  } else {  // D == 256: 128-byte rows
    return t * 128 + ((u ^ (t & 7)) << 4);
  }
}
// Position of the 16-byte unit `u` of token `t` in the K code buffer.
template <int D>
__device__ __forceinline__ int k_unit_off(int t, int u) {
  if (D == 256) return t * 128 + ((u ^ (t & 1)) << 4);
  return t * (D / 2) + (u << 4);
}

// Rotation of a query (or output) row held as quarters: lane j of a group
// of four consecutive lanes owns channels [j*QW, (j+1)*QW). Butterfly
// stages with distance < QW run in registers, wider ones across the lanes
// (distance QW: lane ^ 1, 2*QW: lane ^ 2); the lower-channel lane adds and
// the upper one subtracts. All 32 lanes must call it. Binary32, not part of
// the bit-exact quantize path.
template <int QW>
__device__ __forceinline__ void rotate_quarter(float (&x)[QW], int j, int rot_kind, int lgb,
                                               const float* quat, bool inverse) {
  if (rot_kind == KVQ_ROT_HADAMARD) {
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
    if (inverse)
      quat_inv_regs<QW>(x, quat, j * QW);
    else
      quat_regs<QW>(x, quat, j * QW);
  }
}

template <int D, int P, int GP>
__global__ void __launch_bounds__(kDecWarps * kWarp) decode_split_kernel(const DecodeArgs a) {
  static_assert(D == 128 || D == 256, "decode attention supports head_dim 128 and 256");
  using C = DecCfg<D, P, GP>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int r = lane >> 2, j = lane & 3;
  const int item = blockIdx.x * kDecWarps + warp;
  const int per_seq = a.H * a.splits;
  if (item >= a.S * per_seq) return;
  const int s = item / per_seq;
  const int h = (item / a.splits) % a.H;
  const int split = item % a.splits;
  uint8_t* ring = smem + warp * C::WARP_B;

  // ---- sequence length and page range of this work item
  int L = a.seq_lens[s];
  bool len_ok = L >= 0 && L <= a.max_seq_len && (L + a.P - 1) / a.P <= a.bt_stride;
  if (!len_ok) {
    if (lane == 0 && h == 0 && split == 0) raise_flag(a.err, KVQ_ERRF_LEN);
    L = 0;
  }
  const int npages = (L + P - 1) / P;
  const int pbeg = split * a.pages_per_split;
  int pend = pbeg + a.pages_per_split;
  if (pend > npages) pend = npages;
  const int nmine = pend > pbeg ? pend - pbeg : 0;

  // block-table entries of the item's pages, loaded once (independent loads)
  int32_t* ids = reinterpret_cast<int32_t*>(ring + C::NST * C::STAGE_B);
  for (int c = lane; c < nmine; c += kWarp) ids[c] = a.block_table[(int64_t)s * a.bt_stride + pbeg + c];
  __syncwarp();

  // ---- query fragments: rows = [hi ; lo] of the GP heads of this KV head
  // lane (r, j) handles query head hr and channels [j*QW, (j+1)*QW)
  const int hr = (GP == 8) ? r : (r & 3);
  const bool lo_row = (GP == 4) && (r >= 4);
  const int g = h * a.G + hr;           // global query head
  const bool head_ok = hr < a.G;
  // The query as a 30-bit fixed point qint = qhat * 2^30 / amax (amax = the
  // head's largest |qhat|), split into four signed 8-bit limbs
  // qint = l3*2^24 + l2*2^16 + l1*2^8 + l0 for the int8 tensor cores.
  long long qsum;  // sum of qint over the head's channels (exact)
  double zk;       // sm_scale * log2(e) * amax / 2^30
  // A fragments per k-step kk: the lane's 8 channels j*QW + 8kk + [0, 8),
  // even ones in a[0]/a[1], odd ones in a[2]/a[3]. Rows:
  //   GP = 4: rows 0-3 l3, 4-7 l2, 8-11 l1, 12-15 l0 of heads 0-3;
  //   GP = 8: tile 0 rows 0-7 l3, 8-15 l2; tile 1 rows 0-7 l1, 8-15 l0.
  uint32_t qa[C::NQT][C::NKS8][4];
  {
    float x[C::QW];
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + ((int64_t)s * a.Hq + g) * D + j * C::QW);
#pragma unroll
      for (int c = 0; c < C::QW / 8; ++c) {
        const uint4 u = head_ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(u32_as_h2(w4[e]));
          x[8 * c + 2 * e] = f.x;
          x[8 * c + 2 * e + 1] = f.y;
        }
      }
    }
    rotate_quarter<C::QW>(x, j, a.rot_kind, a.lgb, a.quat, false);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < C::QW; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const double mul = amax > 0.f ? 1073741824.0 / (double)amax : 0.0;  // 2^30 / amax
    zk = a.scale2 * ((double)amax * (1.0 / 1073741824.0));
    long long qs_l = 0;
#pragma unroll
    for (int kk = 0; kk < C::NKS8; ++kk) {
      int li[2][4][4];  // [even/odd][l3, l2, l1, l0][4 channels]
#pragma unroll
      for (int od = 0; od < 2; ++od)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int q = __double2int_rn((double)x[8 * kk + 2 * i + od] * mul);  // |q| <= 2^30
          qs_l += q;
          const int l0 = (q << 24) >> 24;
          const int r1 = (q - l0) >> 8;
          const int l1 = (r1 << 24) >> 24;
          const int r2 = (r1 - l1) >> 8;
          const int l2 = (r2 << 24) >> 24;
          li[od][0][i] = (r2 - l2) >> 8;
          li[od][1][i] = l2;
          li[od][2][i] = l1;
          li[od][3][i] = l0;
        }
      auto pk4 = [&](int od, int limb) {
        return pack_s8x4(li[od][limb][0], li[od][limb][1], li[od][limb][2], li[od][limb][3]);
      };
      if (GP == 8) {
        qa[0][kk][0] = pk4(0, 0);
        qa[0][kk][1] = pk4(0, 1);
        qa[0][kk][2] = pk4(1, 0);
        qa[0][kk][3] = pk4(1, 1);
        qa[C::NQT - 1][kk][0] = pk4(0, 2);
        qa[C::NQT - 1][kk][1] = pk4(0, 3);
        qa[C::NQT - 1][kk][2] = pk4(1, 2);
        qa[C::NQT - 1][kk][3] = pk4(1, 3);
      } else {
        // row r: l3 (r < 4) or l2 (r >= 4); row r + 8: l1 (r < 4) or l0
        qa[0][kk][0] = lo_row ? pk4(0, 1) : pk4(0, 0);
        qa[0][kk][2] = lo_row ? pk4(1, 1) : pk4(1, 0);
        qa[0][kk][1] = lo_row ? pk4(0, 3) : pk4(0, 2);
        qa[0][kk][3] = lo_row ? pk4(1, 3) : pk4(1, 2);
      }
    }
    qs_l += __shfl_xor_sync(0xffffffffu, qs_l, 1);
    qs_l += __shfl_xor_sync(0xffffffffu, qs_l, 2);
    qsum = qs_l;
  }

  // ---- page ring: each lane copies the same 16-byte units of every page,
  // so their shared-memory destinations are computed once
  constexpr int UNITS = C::CODE_B / 16;        // 16-byte units of codes per pool
  constexpr int UPT = (D / 2) / 16;            // units per token
  constexpr int UPL = (UNITS + kWarp - 1) / kWarp;  // units per lane
  constexpr int PU = P * 4 / 16;               // 16-byte units of params per pool
  int koff[UPL], voff[UPL];
#pragma unroll
  for (int i = 0; i < UPL; ++i) {
    const int c = lane + kWarp * i;
    koff[i] = k_unit_off<D>(c / UPT, c % UPT);
    voff[i] = C::CODE_B + v_unit_off<D>(c / UPT, c % UPT);
  }
  const int par_dst = lane < PU ? 2 * C::CODE_B + lane * 16 : 2 * C::CODE_B + P * 4 + (lane - PU) * 16;
  auto issue = [&](int i) {
    if (i < nmine) {
      const int page = ids[i];
      if (page >= 0 && page < a.NP) {
        uint8_t* st = ring + (i % C::NST) * C::STAGE_B;
        const int64_t row = (int64_t)page * a.H + h;
        const uint8_t* kc = a.k_codes + row * C::CODE_B + lane * 16;
        const uint8_t* vc = a.v_codes + row * C::CODE_B + lane * 16;
#pragma unroll
        for (int u = 0; u < UPL; ++u) {
          if (UNITS % kWarp == 0 || lane + kWarp * u < UNITS) {
            cp_async16(st + koff[u], kc + u * kWarp * 16);
            cp_async16(st + voff[u], vc + u * kWarp * 16);
          }
        }
        if (lane < 2 * PU) {
          const uint32_t* pp = lane < PU ? a.k_params + row * P : a.v_params + row * P;
          cp_async16(st + par_dst, reinterpret_cast<const uint8_t*>(pp) + (lane % PU) * 16);
        }
      }
    }
    cp_async_commit();
  };

  // ---- state
  float acc[C::NMT][C::NPV][4];
#pragma unroll
  for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
    for (int n = 0; n < C::NPV; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][n][e] = 0.f;
  // Scores are formed in double from exact integers: with a dominant (sink)
  // token the base-2 logits reach ~100, where a binary32 rounding would
  // already move the other tokens' weights visibly.
  double M = -INFINITY;  // running max (base-2 scaled scores) of head hr
  float Lp = 0.f;       // this lane's share of sum p
  float Op = 0.f;       // this lane's share of sum p (m_v + 8 s_v)

  for (int i = 0; i < C::NST - 1; ++i) issue(i);

  for (int i = 0; i < nmine; ++i) {
    issue(i + C::NST - 1);
    cp_async_wait<C::NST - 1>();
    __syncwarp();
    const int pidx = pbeg + i;
    const int page = ids[i];
    const bool page_ok = page >= 0 && page < a.NP;
    if (!page_ok && lane == 0) raise_flag(a.err, KVQ_ERRF_PAGE);
    const uint8_t* st = ring + (i % C::NST) * C::STAGE_B;
    const uint8_t* kbuf = st;
    const uint8_t* vbuf = st + C::CODE_B;
    const uint2* kpar = reinterpret_cast<const uint2*>(st + 2 * C::CODE_B);
    const uint2* vpar = reinterpret_cast<const uint2*>(st + 2 * C::CODE_B + P * 4);

    // ---- scores of all tiles of the page: z[tile][0..3] for tokens
    // 16*tile + {2j, 2j+1, 2j+8, 2j+9}
    double z[C::TILES][4];
#pragma unroll
    for (int tt = 0; tt < C::TILES; ++tt) {
      int ci[C::NQT][2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int t = 0; t < C::NQT; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) ci[t][nt][e] = 0;
        const int tok = 16 * tt + 8 * nt + r;
        uint32_t w[D / 32];
#pragma unroll
        for (int u = 0; u < D / 128; ++u) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(kbuf + k_unit_off<D>(tok, (D / 128) * j + u));
          w[4 * u] = v4.x; w[4 * u + 1] = v4.y; w[4 * u + 2] = v4.z; w[4 * u + 3] = v4.w;
        }
#pragma unroll
        for (int kk = 0; kk < C::NKS8; ++kk) {
          const uint32_t b0 = w[kk] & 0x0F0F0F0Fu;         // even channels as bytes
          const uint32_t b1 = (w[kk] >> 4) & 0x0F0F0F0Fu;  // odd channels
#pragma unroll
          for (int t = 0; t < C::NQT; ++t) mma16832_s8u8(ci[t][nt], qa[t][kk], b0, b1);
        }
      }
      // sum_i (c_i - 8) qint_i of head hr with the four tokens
      // {2j, 2j+1, 2j+8, 2j+9}, exact in 64-bit integers (the centring keeps
      // the two score terms small, so their binary32 rounding stays small)
      long long dt[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int nt = e >> 1, c = e & 1;
        int l3, l2, l1, l0;
        if (GP == 8) {
          l3 = ci[0][nt][c];
          l2 = ci[0][nt][2 + c];
          l1 = ci[C::NQT - 1][nt][c];
          l0 = ci[C::NQT - 1][nt][2 + c];
        } else {
          // lanes r < 4 hold the (l3, l1) rows, lanes r + 4 the (l2, l0) rows
          const int o0 = __shfl_xor_sync(0xffffffffu, ci[0][nt][c], 16);
          const int o2 = __shfl_xor_sync(0xffffffffu, ci[0][nt][2 + c], 16);
          l3 = lo_row ? o0 : ci[0][nt][c];
          l2 = lo_row ? ci[0][nt][c] : o0;
          l1 = lo_row ? o2 : ci[0][nt][2 + c];
          l0 = lo_row ? ci[0][nt][2 + c] : o2;
        }
        dt[e] = (((long long)l3 * 256ll + l2) * 256ll + l1) * 256ll + l0 - 8ll * qsum;
      }
      const uint2 kp01 = kpar[8 * tt + j];      // tokens 16tt + 2j, 2j+1
      const uint2 kp89 = kpar[8 * tt + 4 + j];  // tokens 16tt + 2j+8, 2j+9
      const uint32_t kp[4] = {kp01.x, kp01.y, kp89.x, kp89.y};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 sm = __half22float2(u32_as_h2(kp[e]));  // (scale, min)
        const int tok = pidx * P + 16 * tt + 2 * j + (e & 1) + 8 * (e >> 1);
        const double sd = (double)sm.x, md = (double)sm.y;
        const double sc = zk * (sd * (double)dt[e] + (md + 8.0 * sd) * (double)qsum);
        z[tt][e] = (page_ok && tok < L) ? sc : -INFINITY;
      }
    }

    // ---- online softmax update for head hr (max over the 4 lanes j)
    double mloc = -INFINITY;
#pragma unroll
    for (int tt = 0; tt < C::TILES; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) mloc = fmax(mloc, z[tt][e]);
    mloc = fmax(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmax(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    const double Mn = fmax(M, mloc);
    const float alpha = (Mn == -INFINITY) ? 1.f : fast_exp2((float)(M - Mn));
    M = Mn;
    Lp *= alpha;
    Op *= alpha;
    // rescale the output accumulators: lane (r, j) holds columns of heads
    // c0 = 2(j & (GP/2 - 1)), c0 + 1 -> their alpha from lanes r = c0, c0 + 1
    if (__any_sync(0xffffffffu, alpha != 1.f)) {  // warp-uniform: skip when no max moved
      const int c0 = (GP == 8) ? 2 * j : 2 * (j & 1);
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
      const uint2 vp01 = vpar[8 * tt + j];
      const uint2 vp89 = vpar[8 * tt + 4 + j];
      const uint32_t vp[4] = {vp01.x, vp01.y, vp89.x, vp89.y};
      float pv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // masked tokens may sit on stale or never-written shared memory:
        // their terms are forced to exact zeros rather than p * (params)
        const bool live = z[tt][e] != -INFINITY;
        const float2 sm = __half22float2(u32_as_h2(vp[e]));
        const float p = live ? fast_exp2((float)(z[tt][e] - M)) : 0.f;
        Lp += p;
        Op += live ? p * (sm.y + 8.f * sm.x) : 0.f;
        pv[e] = live ? p * sm.x : 0.f;
      }
      // p * s as f16 hi + lo pairs (packed conversions): hi = RN16(x),
      // lo = RN16(x - hi), for tokens (2j, 2j+1) and (2j+8, 2j+9)
      const __half2 h01 = __floats2half2_rn(pv[0], pv[1]);
      const __half2 h89 = __floats2half2_rn(pv[2], pv[3]);
      const float2 f01 = __half22float2(h01), f89 = __half22float2(h89);
      const uint32_t hi01 = h2_as_u32(h01), hi89 = h2_as_u32(h89);
      const uint32_t lo01 = h2_as_u32(__floats2half2_rn(pv[0] - f01.x, pv[1] - f01.y));
      const uint32_t lo89 = h2_as_u32(__floats2half2_rn(pv[2] - f89.x, pv[3] - f89.y));
      // B operand columns: GP = 8: n-tile 0 = hi, 1 = lo (col r = head r);
      // GP = 4: col r < 4 = hi of head r, r >= 4 = lo of head r - 4
      uint32_t pb[C::NPV][2];
      if (GP == 8) {
        pb[0][0] = hi01;
        pb[0][1] = hi89;
        pb[C::NPV - 1][0] = lo01;
        pb[C::NPV - 1][1] = lo89;
      } else {
        pb[0][0] = lo_row ? lo01 : hi01;
        pb[0][1] = lo_row ? lo89 : hi89;
      }
      if (!head_ok) {
#pragma unroll
        for (int n = 0; n < C::NPV; ++n) pb[n][0] = pb[n][1] = 0u;
      }
      // A operand: V codes of tokens {2j, 2j+1} and {2j+8, 2j+9}, channels of
      // lane row r: [r*D/8, (r+1)*D/8)
      constexpr int WPT = D / 64;  // 32-bit words per token per lane
      uint32_t vw[4][WPT];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = 16 * tt + 2 * j + (e & 1) + 8 * (e >> 1);
        if (D == 128) {
          const uint2 v2 = *reinterpret_cast<const uint2*>(vbuf + v_unit_off<D>(tok, r >> 1) + 8 * (r & 1));
          vw[e][0] = v2.x; vw[e][1] = v2.y;
        } else {
          const uint4 v4 = *reinterpret_cast<const uint4*>(vbuf + v_unit_off<D>(tok, r));
          vw[e][0] = v4.x; vw[e][1] = v4.y; vw[e][2] = v4.z; vw[e][3] = v4.w;
        }
      }
      // m-tile mt: group gq = mt / 8 (words 2gq, 2gq+1), nibble e = mt % 8;
      // row slot r <- word 2gq, slot r+8 <- word 2gq+1
#pragma unroll
      for (int gq = 0; gq < WPT / 2; ++gq) {
        uint32_t pr[2][2][2];  // [token pair][word in group][lo/hi bytes]
#pragma unroll
        for (int tp = 0; tp < 2; ++tp)
#pragma unroll
          for (int wi = 0; wi < 2; ++wi) {
            const int wd = 2 * gq + wi;
            const uint32_t X = vw[2 * tp][wd], Y = vw[2 * tp + 1][wd];
            pr[tp][wi][0] = __byte_perm(X, Y, 0x5410);
            pr[tp][wi][1] = __byte_perm(X, Y, 0x7632);
          }
        // nibbles of every (token pair, word, byte half): nb[tp][wi][bsel][k]
        uint32_t nb[2][2][2][4];
#pragma unroll
        for (int tp = 0; tp < 2; ++tp)
#pragma unroll
          for (int wi = 0; wi < 2; ++wi)
#pragma unroll
            for (int bs = 0; bs < 2; ++bs) nib4(pr[tp][wi][bs], nb[tp][wi][bs]);
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) {
          const int mt = gq * 8 + e8;
          const int bsel = e8 >> 2, k = e8 & 3;
          uint32_t av[4];
          av[0] = nb[0][0][bsel][k];  // slot r,   tokens 2j, 2j+1
          av[1] = nb[0][1][bsel][k];  // slot r+8, tokens 2j, 2j+1
          av[2] = nb[1][0][bsel][k];  // slot r,   tokens 2j+8, 2j+9
          av[3] = nb[1][1][bsel][k];  // slot r+8, tokens 2j+8, 2j+9
          // each 16-token product starts from zero and joins the running sum
          // through an IEEE round-to-nearest add: accumulating inside the
          // tensor core would round toward zero against a large running sum
#pragma unroll
          for (int n = 0; n < C::NPV; ++n) {
            float t4[4] = {0.f, 0.f, 0.f, 0.f};
            mma16816(t4, av, pb[n][0], pb[n][1]);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][n][e] = __fadd_rn(acc[mt][n][e], t4[e]);
          }
        }
      }
    }
    __syncwarp();  // stage i % C::NST is refilled by the next issue
  }
  cp_async_wait<0>();

  // ---- partial results: (acc + sum p (m + 8 s)) per channel, M, sum p
  Lp += __shfl_xor_sync(0xffffffffu, Lp, 1);
  Lp += __shfl_xor_sync(0xffffffffu, Lp, 2);
  Op += __shfl_xor_sync(0xffffffffu, Op, 1);
  Op += __shfl_xor_sync(0xffffffffu, Op, 2);
  if (GP == 4) {
    // fold the lo columns (lanes j = 2, 3) onto the hi columns (j = 0, 1)
#pragma unroll
    for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][0][e] += __shfl_xor_sync(0xffffffffu, acc[mt][0][e], 2);
  }
  const int c0 = (GP == 8) ? 2 * j : 2 * (j & 1);  // heads of this lane's columns
  const float o0 = __shfl_sync(0xffffffffu, Op, 4 * c0);
  const float o1 = __shfl_sync(0xffffffffu, Op, 4 * c0 + 4);
  const bool writer = (GP == 8) || (j < 2);
  const int64_t base = ((int64_t)s * a.Hq + (int64_t)h * a.G) * a.splits + split;
#pragma unroll
  for (int hc = 0; hc < 2; ++hc) {
    const int gh = c0 + hc;
    if (!writer || gh >= a.G) continue;
    float* dst = a.part + (base + (int64_t)gh * a.splits) * (D + 4);
    const float ov = hc ? o1 : o0;
#pragma unroll
    for (int mt = 0; mt < C::NMT; ++mt) {
      // m-tile mt, row slot r <- channel r*D/8 + 16*(mt/8) + mt%8,
      // row slot r+8 <- that channel + 8
      const int ch0 = r * (D / 8) + 16 * (mt / 8) + (mt % 8);
      float v0 = 0.f, v1 = 0.f;
#pragma unroll
      for (int n = 0; n < C::NPV; ++n) {
        v0 += acc[mt][n][hc];
        v1 += acc[mt][n][2 + hc];
      }
      dst[ch0] = v0 + ov;
      dst[ch0 + 8] = v1 + ov;
    }
  }
  // the lanes that own head hr's softmax state write it (one lane per head)
  if (j == 0 && !lo_row && head_ok) {
    float* dst = a.part + (base + (int64_t)hr * a.splits) * (D + 4);
    *reinterpret_cast<double*>(dst + D) = M;  // 8-byte aligned: (D + 4) * 4 * k + 4 * D
    dst[D + 2] = Lp;
  }

  // ---- the last warp of this (sequence, KV head) merges the splits
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atomicAdd(a.counter + (int64_t)s * a.H + h, 1) == a.splits - 1;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  const bool owner = head_ok && !lo_row;
  float x[C::QW];
#pragma unroll
  for (int c = 0; c < C::QW; ++c) x[c] = 0.f;
  if (owner) {
    const float* src = a.part + ((int64_t)s * a.Hq + g) * a.splits * (D + 4);
    double Mx = -INFINITY;
    for (int i = 0; i < a.splits; ++i)
      Mx = fmax(Mx, __ldcg(reinterpret_cast<const double*>(src + (int64_t)i * (D + 4) + D)));
    float Ls = 0.f;
    if (Mx != -INFINITY) {
      for (int i = 0; i < a.splits; ++i) {
        const float* pi = src + (int64_t)i * (D + 4);
        const double Mi = __ldcg(reinterpret_cast<const double*>(pi + D));
        if (Mi == -INFINITY) continue;
        const float wgt = fast_exp2((float)(Mi - Mx));
        Ls += wgt * __ldcg(pi + D + 2);
        const float4* v4 = reinterpret_cast<const float4*>(pi + j * C::QW);
#pragma unroll
        for (int c = 0; c < C::QW / 4; ++c) {
          const float4 f = __ldcg(v4 + c);
          x[4 * c] += wgt * f.x;
          x[4 * c + 1] += wgt * f.y;
          x[4 * c + 2] += wgt * f.z;
          x[4 * c + 3] += wgt * f.w;
        }
      }
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll
    for (int c = 0; c < C::QW; ++c) x[c] *= inv;
  }
  rotate_quarter<C::QW>(x, j, a.rot_kind, a.lgb, a.quat, true);  // R^-1 (R^-1 = R for Hadamard)
  if (owner) {
    float4* dst = reinterpret_cast<float4*>(a.out + ((int64_t)s * a.Hq + g) * D + j * C::QW);
#pragma unroll
    for (int c = 0; c < C::QW / 4; ++c) dst[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
  }
  if (lane == 0) a.counter[(int64_t)s * a.H + h] = 0;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int D, int P, int GP>
static size_t split_smem() {
  return (size_t)kDecWarps * DecCfg<D, P, GP>::WARP_B;
}

template <int D, int P, int GP>
static int split_resident_warps() {
  static int cached = -1;
  if (cached < 0) {
    auto kern = decode_split_kernel<D, P, GP>;
    const size_t smem = split_smem<D, P, GP>();
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kDecWarps * kWarp, smem) !=
        cudaSuccess)
      blocks = 1;
    const int sms = device_sm_count();
    cached = (blocks < 1 ? 1 : blocks) * kDecWarps * (sms > 0 ? sms : 148);
  }
  return cached;
}

#define KVQ_DECODE_CONFIGS(X)                                                                  \
  X(128, 16, 4) X(128, 16, 8) X(128, 32, 4) X(128, 32, 8) X(128, 64, 4) X(128, 64, 8)          \
  X(256, 16, 4) X(256, 32, 4) X(256, 64, 4)

static int resident_warps(int D, int P, int GP) {
#define KVQ_RW(d_, p_, g_) \
  if (D == d_ && P == p_ && GP == g_) return split_resident_warps<d_, p_, g_>();
  KVQ_DECODE_CONFIGS(KVQ_RW)
#undef KVQ_RW
  return 148 * 8;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

DecodePlan decode_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len) {
  DecodePlan pl{};
  const int P = d.page_size;
  pl.pages_max = (max_seq_len + P - 1) / P;
  if (pl.pages_max < 1) pl.pages_max = 1;
  const int G = Hq / d.num_kv_heads;
  const int GP = G <= 4 ? 4 : 8;
  const int target = resident_warps(d.head_dim, P, GP);
  const int pairs = S * d.num_kv_heads;
  int splits = target / (pairs > 0 ? pairs : 1);
  const int min_splits = (pl.pages_max + kMaxPagesPerSplit - 1) / kMaxPagesPerSplit;
  if (splits < min_splits) splits = min_splits;
  if (splits < 1) splits = 1;
  if (splits > pl.pages_max) splits = pl.pages_max;
  pl.pages_per_split = (pl.pages_max + splits - 1) / splits;
  pl.splits = (pl.pages_max + pl.pages_per_split - 1) / pl.pages_per_split;
  const size_t counters = (size_t)S * d.num_kv_heads * sizeof(int32_t);
  const size_t parts = (size_t)S * Hq * pl.splits * (d.head_dim + 4) * sizeof(float);
  pl.workspace = align256(counters) + parts;
  return pl;
}

template <int D, int P, int GP>
static cudaError_t launch_split(const DecodeArgs& a, cudaStream_t st) {
  auto kern = decode_split_kernel<D, P, GP>;
  const size_t smem = split_smem<D, P, GP>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int items = a.S * a.H * a.splits;
  const int grid = (items + kDecWarps - 1) / kDecWarps;
  kern<<<grid, kDecWarps * kWarp, smem, st>>>(a);
  return cudaGetLastError();
}

static cudaError_t launch_split_any(const DecodeArgs& a, int D, int GP, cudaStream_t st) {
#define KVQ_LS(d_, p_, g_) \
  if (D == d_ && a.P == p_ && GP == g_) return launch_split<d_, p_, g_>(a, st);
  KVQ_DECODE_CONFIGS(KVQ_LS)
#undef KVQ_LS
  return cudaErrorInvalidValue;
}

int decode_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                  const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                  int32_t bt_stride, float sm_scale, const uint8_t* k_codes,
                  const void* k_params, const uint8_t* v_codes, const void* v_params,
                  float* out, void* workspace, size_t workspace_bytes, int32_t* err,
                  cudaStream_t st) {
  const int D = d.head_dim;
  const int G = Hq / d.num_kv_heads;
  const int GP = G <= 4 ? 4 : 8;
  if ((D != 128 && D != 256) || (D == 256 && GP != 4)) return KVQ_ERR_UNSUPPORTED;
  const DecodePlan pl = decode_plan(d, S, Hq, max_seq_len);
  if (workspace == nullptr || workspace_bytes < pl.workspace) return KVQ_ERR_WORKSPACE;
  int lgb = 0;
  while ((1 << lgb) < d.rot_block) ++lgb;

  DecodeArgs a;
  a.S = S; a.Hq = Hq; a.H = d.num_kv_heads; a.G = G; a.P = d.page_size; a.NP = d.num_pages;
  a.bt_stride = bt_stride; a.max_seq_len = max_seq_len; a.splits = pl.splits;
  a.pages_per_split = pl.pages_per_split;
  a.rot_kind = d.rot_kind; a.lgb = lgb;
  a.scale2 = (double)sm_scale * 1.4426950408889634074;
  a.q = static_cast<const __half*>(q); a.quat = d.quat;
  a.seq_lens = seq_lens; a.block_table = block_table;
  a.k_codes = k_codes; a.k_params = static_cast<const uint32_t*>(k_params);
  a.v_codes = v_codes; a.v_params = static_cast<const uint32_t*>(v_params);
  a.out = out;
  a.counter = static_cast<int32_t*>(workspace);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                    align256((size_t)S * d.num_kv_heads * sizeof(int32_t)));
  a.err = err;
  const cudaError_t e = launch_split_any(a, D, GP, st);
  if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
