// Decode attention over the 2-bit, 3-bit and level-table caches (kvq.h,
// KVQ_FMT_INT2 / INT3 / LUT4) with QK on Blackwell's tcgen05 integer MMA.
//
// One CTA (4 warps) per (sequence, KV head, split) of 128-token tiles, as the
// microscaled FP4 decode. Per tile:
//  * every thread stages its token's packed K and V rows and parameter words
//    (cp.async, 2 stages), then widens its own K row -- once its copies have
//    landed, no barrier needed -- into the MMA's K-major 8-bit operand: one
//    byte per channel, the code c (2- and 3-bit formats) or 16 t[c] (the
//    table's level on its 1/16 grid, an integer in [0, 240]);
//  * one thread issues four tcgen05.mma kind::i8 (M = 128 tokens, N = 4 G
//    query limb rows, K = 32 channels each): the rotated query is a 26-bit
//    fixed point qint = RN(qhat 2^k) split in four signed 8-bit limbs (the
//    INT4 decode's representation), so the int32 results are exact, and
//    dot = sum_l D_l 256^l - c0 qsum is the exact integer sum of the centred
//    codes times qint;
//  * thread t scores its token: z = (s (dot / u) + (m + c0 s / u) qsum) 2^-k
//    sm_scale log2(e) (u = 16 for the table, 1 else; c0 the centre code);
//    each warp runs its own online softmax and accumulates PV on the f16
//    tensor cores (mma.sync) with the V codes centred as binary16 integers
//    (1024 + v read from the mantissa, minus 1024 + c0) and the weights p s
//    as hi + lo binary16 pairs; sum p (m + c0 s) joins at the end.
// The four warps' states merge in shared memory into the partial-result
// layout of the other decodes; the common merge kernel finishes.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_launch.h"
#include "kvq_rotate.cuh"
#include "kvq_rowquant.cuh"
#include "kvq_tcgen05.cuh"

namespace kvq {

namespace {

constexpr int kGD = 128;        // head_dim
constexpr int kGThreads = 128;  // thread t stages, widens and scores token t of a tile
constexpr int kGTile = 128;
constexpr int kGStages = 2;
constexpr uint32_t kGTmemCols = 32;
constexpr float kGSlack = 8.f;

template <int BITS>
struct GenCfg {
  static constexpr int RB = kGD * BITS / 8;          // packed bytes per row
  static constexpr int A_OFF = 0;                    // 8-bit K operand (16 KB)
  static constexpr int A_B = 16 * 1024;
  static constexpr int KR_OFF = A_OFF + A_B;         // packed K rows
  static constexpr int KP_OFF = KR_OFF + kGTile * RB;  // K params words
  static constexpr int VR_OFF = KP_OFF + kGTile * 4;   // packed V rows
  static constexpr int VP_OFF = VR_OFF + kGTile * RB;  // V params words
  static constexpr int STAGE_B = VP_OFF + kGTile * 4;
  static constexpr int B_OFF = kGStages * STAGE_B;   // query limbs: up to 32 rows x 128 B
  static constexpr int B_B = 4096;
  static constexpr int BAR_OFF = B_OFF + B_B;
  static constexpr int SMEM = BAR_OFF + 16;
  static_assert(STAGE_B % 128 == 0 && B_OFF % 128 == 0, "operand alignment");
  static_assert(4 * 8 * kGD * 4 + 2 * 4 * 8 * 4 <= STAGE_B, "merge scratch fits in a stage");
};

}  // namespace

struct GenDecodeArgs {
  int S, Hq, H, G, P, lg_page, NP, bt_stride, max_seq_len, splits;
  int nhi;  // (sequence, KV head) pairs with `splits` splits; the rest have splits - 1
  int rot_kind, lgb;
  float scale2;
  const __half* q;
  const float* quat;
  const float* rope;
  int rope_max_pos;
  const float* levels;
  const int32_t* seq_lens;
  const int32_t* block_table;
  const uint8_t* k_codes;
  const uint32_t* k_params;
  const uint8_t* v_codes;
  const uint32_t* v_params;
  float* part;
  int32_t* err;
};

// Code i of a packed row of BITS-bit codes held in 32-bit words (little-endian
// bit stream).
template <int BITS, int NW>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[NW], int i) {
  const int bit = i * BITS;
  uint32_t v = w[bit >> 5] >> (bit & 31);
  if ((bit & 31) + BITS > 32) v |= w[(bit >> 5) + 1] << (32 - (bit & 31));
  return v & ((1u << BITS) - 1u);
}

// Byte c (0-15) of the 16-byte table held in four registers.
__device__ __forceinline__ uint32_t lut_byte(const uint32_t (&lut)[4], uint32_t c) {
  const uint32_t lo = __byte_perm(lut[0], lut[1], c & 7u);
  const uint32_t hi = __byte_perm(lut[2], lut[3], c & 7u);
  return ((c & 8u) ? hi : lo) & 0xFFu;
}

// Bytes t[c0..c3] of a 16-byte table held in four registers, for the four
// 4-bit codes of `sel` (code k in bits 4k..4k+3 of its low 16 bits), in
// bytes 0-3: two 8-entry lookups (byte permutes of the low and high halves of
// the table) and a byte mask from the codes' top bits (the sign-replicating
// permute of 0x80 bytes gives 0xFF where a code is >= 8 and 0x80 elsewhere;
// m & (m << 1 | 0x01010101) turns that into 0xFF / 0x00).
__device__ __forceinline__ uint32_t lut16x4(const uint32_t (&t)[4], uint32_t sel) {
  const uint32_t s7 = sel & 0x7777u;
  const uint32_t lo = __byte_perm(t[0], t[1], s7);
  const uint32_t hi = __byte_perm(t[2], t[3], s7);
  uint32_t m;  // the PTX permute itself: __byte_perm ignores the selectors' top bits
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m) : "r"(0x80808080u), "r"(0x80808080u), "r"(sel & 0xFFFFu));
  const uint32_t mask = m & ((m << 1) | 0x01010101u);
  return (hi & mask) | (lo & ~mask);
}

// Eight 4-bit codes (code i in bits 4i..4i+3) -> eight bytes in code order.
__device__ __forceinline__ uint2 nibbles_to_bytes(uint32_t w) {
  const uint32_t ev = w & 0x0F0F0F0Fu;         // codes 0, 2, 4, 6
  const uint32_t od = (w >> 4) & 0x0F0F0F0Fu;  // codes 1, 3, 5, 7
  return make_uint2(__byte_perm(ev, od, 0x5140), __byte_perm(ev, od, 0x7362));
}

// Eight 2-bit codes (bits 0-15) -> the same codes in 4-bit fields.
__device__ __forceinline__ uint32_t crumbs_to_nibbles(uint32_t v) {
  v &= 0xFFFFu;
  v = (v | (v << 8)) & 0x00FF00FFu;
  v = (v | (v << 4)) & 0x0F0F0F0Fu;
  return (v | (v << 2)) & 0x33333333u;
}

// The 16 codes of channels [16 k, 16 k + 16) of one row as 16 bytes in
// channel order (the code, or 16 t[code] for the table); `lo`, `hi`: the 64
// bits starting at the block's first code (the low BITS * 16 used).
template <int BITS, bool LUT>
__device__ __forceinline__ void codes16_bytes(uint32_t lo, uint32_t hi, const uint32_t (&lut)[4],
                                              uint32_t (&o)[4]) {
  if (BITS == 4) {
    if (LUT) {
      o[0] = lut16x4(lut, lo);
      o[1] = lut16x4(lut, lo >> 16);
      o[2] = lut16x4(lut, hi);
      o[3] = lut16x4(lut, hi >> 16);
    } else {
      const uint2 a = nibbles_to_bytes(lo), b = nibbles_to_bytes(hi);
      o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    }
  } else if (BITS == 2) {
    const uint2 a = nibbles_to_bytes(crumbs_to_nibbles(lo));
    const uint2 b = nibbles_to_bytes(crumbs_to_nibbles(lo >> 16));
    o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
  } else {  // 3 bits: code i at bits 3 i of the 48-bit field
    const uint32_t w2[2] = {lo, hi};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t v = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) v |= code_at<3, 2>(w2, 4 * q + b) << (8 * b);
      o[q] = v;
    }
  }
}

// Bits [pos, pos + 32) of a little-endian word array (pos a compile-time
// multiple of 16 after unrolling).
template <int NW>
__device__ __forceinline__ uint32_t bits32(const uint32_t (&w)[NW], int pos) {
  const int i = pos >> 5, sh = pos & 31;
  const uint32_t a = w[i];
  const uint32_t b = i + 1 < NW ? w[i + 1] : 0u;
  return sh ? __funnelshift_r(a, b, sh) : a;
}

// NB as in the FP4 decode (1: G <= 4, hi and lo weights in one MMA; 2: G <= 8).
template <int BITS, bool LUT, int NB>
__global__ void __launch_bounds__(kGThreads) decode_gen_kernel(const GenDecodeArgs a) {
  using C = GenCfg<BITS>;
  constexpr int N = NB == 1 ? 16 : 32;  // B rows: limb l of head g at 4 g + l
  constexpr int U = LUT ? 16 : 1;       // operand units per code value
  constexpr int C0 = LUT ? 128 : (1 << (BITS - 1));  // centre, in operand units
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
  // blocks: the first nhi (sequence, KV head) pairs with `splits` splits
  // each, then the others with splits - 1
  const int hi_items = a.nhi * a.splits;
  int sh, split, nspl;
  if ((int)blockIdx.x < hi_items) {
    sh = blockIdx.x / a.splits;
    split = blockIdx.x - sh * a.splits;
    nspl = a.splits;
  } else {
    nspl = a.splits - 1;
    const int r = blockIdx.x - hi_items;
    const int k = nspl > 0 ? r / nspl : 0;
    sh = a.nhi + k;
    split = r - k * nspl;
  }
  const int h = sh % a.H, s = sh / a.H;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + 8);

  pdl_wait();
  pdl_trigger();

  const int L = a.seq_lens[s];
  const bool len_ok = L >= 0 && L <= a.max_seq_len &&
                      ((L + a.P - 1) >> a.lg_page) <= a.bt_stride &&
                      (a.rope == nullptr || L <= a.rope_max_pos);
  const int ntiles = len_ok ? (L + kGTile - 1) / kGTile : 0;
  // the sequence's tiles dealt out evenly over its splits
  const int t0 = (int)(((int64_t)split * ntiles) / nspl);
  const int t1 = (int)(((int64_t)(split + 1) * ntiles) / nspl);
  const int64_t base = ((int64_t)s * a.Hq + (int64_t)h * a.G) * a.splits + split;
  if (t0 >= t1) {
    if (!len_ok && split == 0 && h == 0 && tid == 0) raise_flag(a.err, KVQ_ERRF_LEN);
    for (int g = 0; g < a.G; ++g) {
      float* dst = a.part + (base + (int64_t)g * a.splits) * (kGD + 4);
      dst[tid] = 0.f;
      if (tid == 0) *reinterpret_cast<float2*>(dst + kGD) = make_float2(-INFINITY, 0.f);
    }
    return;
  }

  if (warp == 0) {
    tmem_alloc(tmem_slot, kGTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  for (int i = tid; i < C::B_B / 16; i += kGThreads)
    reinterpret_cast<uint4*>(smem + C::B_OFF)[i] = make_uint4(0u, 0u, 0u, 0u);

  // the table as bytes 16 t[c] (LUT): four words, byte c % 4 of word c / 4
  uint32_t lut[4] = {0u, 0u, 0u, 0u};
  if (LUT) {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      lut[c >> 2] |= ((uint32_t)__float2int_rn(__ldg(a.levels + c) * 16.f) & 0xFFu) << (8 * (c & 3));
  }

  auto issue = [&](int t, int stage) -> bool {
    uint8_t* st = smem + stage * C::STAGE_B;
    const int tok = t * kGTile + tid;
    int page = -1;
    if (tok < L) page = a.block_table[(int64_t)s * a.bt_stride + (tok >> a.lg_page)];
    const bool ok = page >= 0 && page < a.NP && tok < L;
    uint32_t* kp = reinterpret_cast<uint32_t*>(st + C::KP_OFF + tid * 4);
    uint32_t* vp = reinterpret_cast<uint32_t*>(st + C::VP_OFF + tid * 4);
    if (ok) {
      const int64_t row = (((int64_t)page * a.H + h) << a.lg_page) + (tok & (a.P - 1));
#pragma unroll
      for (int c = 0; c < C::RB / 16; ++c) {
        cp_async16(st + C::KR_OFF + tid * C::RB + 16 * c, a.k_codes + row * C::RB + 16 * c);
        cp_async16(st + C::VR_OFF + tid * C::RB + 16 * c, a.v_codes + row * C::RB + 16 * c);
      }
      cp_async4(kp, a.k_params + row);
      cp_async4(vp, a.v_params + row);
    } else {
      // parameters (0, 0): the row's values are exact zeros whatever its
      // stale codes hold, and the scores are masked anyway
      *kp = 0u;
      *vp = 0u;
      if (tok < L && (tok & (a.P - 1)) == 0) raise_flag(a.err, KVQ_ERRF_PAGE);
    }
    return ok;
  };
  uint32_t vbits = 0;
  if (t0 < t1 && issue(t0, 0)) vbits |= 1u;
  cp_async_commit();

  __syncthreads();  // B zeroed, barrier initialised

  // ---- the query (warp 0): RoPE, rotation, 26-bit fixed point, four signed
  // 8-bit limbs per channel; lane (gq, j) owns channels [32 j, 32 j + 32)
  float k2 = 0.f;   // 2^-k of head g, for lane 4 g
  long long qsum_l = 0;
  if (warp == 0) {
    const int gq = lane >> 2, j = lane & 3;
    const bool hq_ok = gq < a.G;
    float x[32];
    const uint4* qsrc = reinterpret_cast<const uint4*>(
        a.q + ((int64_t)s * a.Hq + (int64_t)h * a.G + (hq_ok ? gq : 0)) * kGD + j * 32);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = hq_ok ? qsrc[c] : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(u32_as_h2(w4[e]));
        x[8 * c + 2 * e] = f.x;
        x[8 * c + 2 * e + 1] = f.y;
      }
    }
    if (a.rope != nullptr && L >= 1) rope_regs<32>(x, a.rope + (int64_t)(L - 1) * kGD + j * 32);
    rotate_quarter<32>(x, j, a.rot_kind, a.lgb, a.quat);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int ebits = (__float_as_int(amax) >> 23) & 0xFF;  // amax < 2^(ebits - 126)
    int kk = 26 - (ebits - 126);
    kk = kk > 126 ? 126 : kk;
    const float mulf = amax > 0.f ? __int_as_float((kk + 127) << 23) : 0.f;
    k2 = __int_as_float((127 - kk) << 23);
    uint8_t* brow = smem + C::B_OFF;
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {  // 8 channels at a time
      uint32_t lw[4][2];                // limb l, two words of 4 channels
#pragma unroll
      for (int hw = 0; hw < 2; ++hw) {
        uint32_t u4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qv = __float2int_rn(x[8 * c8 + 4 * hw + e] * mulf);
          qsum_l += qv;
          u4[e] = (uint32_t)(qv + 0x808080) ^ 0x00808080u;  // bytes = signed limbs
        }
#pragma unroll
        for (int l = 0; l < 4; ++l)
          lw[l][hw] = __byte_perm(__byte_perm(u4[0], u4[1], l | ((4 + l) << 4)),
                                  __byte_perm(u4[2], u4[3], l | ((4 + l) << 4)), 0x5410);
      }
      if (hq_ok) {
        // channels 32 j + 8 c8 .. + 7: K chunk 2 j + c8 / 2, bytes 8 (c8 % 2)
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          const int n = 4 * gq + l;
          uint8_t* dst = brow + (n >> 3) * 1024 + (2 * j + (c8 >> 1)) * 128 + (n & 7) * 16 +
                         8 * (c8 & 1);
          *reinterpret_cast<uint2*>(dst) = make_uint2(lw[l][0], lw[l][1]);
        }
      }
    }
    qsum_l += __shfl_xor_sync(0xffffffffu, qsum_l, 1);
    qsum_l += __shfl_xor_sync(0xffffffffu, qsum_l, 2);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // every thread: 2^-k sm_scale log2(e) and the exact limb sum of each head,
  // from warp 0's lanes 4 g
  __shared__ float hq_k2[8];
  __shared__ long long hq_qs[8];
  if (warp == 0 && (lane & 3) == 0) {
    hq_k2[lane >> 2] = k2;
    hq_qs[lane >> 2] = qsum_l;
  }
  __syncthreads();
  float kq[8];
  long long qsl[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    kq[g] = hq_k2[g] * a.scale2;
    qsl[g] = hq_qs[g];
  }
  const uint64_t bdesc = umma_desc_kmajor(smem_u32(smem + C::B_OFF), 128, 1024);

  const int r8 = lane >> 2, q4 = lane & 3;
  float Mh[8], Lh[8], Oh[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    Mh[g] = -INFINITY;
    Lh[g] = 0.f;
    Oh[g] = 0.f;
  }
  float acc[NB][8][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nb][mt][e] = 0.f;
  bool timed_out = false;
  int it_out = 0;

  for (int t = t0, it = 0; t < t1; ++t, ++it) {
    const int stage = it % kGStages;
    uint8_t* st = smem + stage * C::STAGE_B;
    cp_async_wait<0>();  // this thread's copies of tile t have landed
    {
      // widen this thread's K row into the 8-bit operand (row tid)
      constexpr int NW = C::RB / 4;
      uint32_t w[NW];
#pragma unroll
      for (int c = 0; c < C::RB / 16; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(st + C::KR_OFF + tid * C::RB + 16 * c);
        w[4 * c] = u.x; w[4 * c + 1] = u.y; w[4 * c + 2] = u.z; w[4 * c + 3] = u.w;
      }
      uint8_t* arow = st + C::A_OFF + (tid >> 3) * 1024 + (tid & 7) * 16;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {  // 16 channels per 16-byte chunk
        uint32_t o[4];
        codes16_bytes<BITS, LUT>(bits32<NW>(w, 16 * BITS * ch), bits32<NW>(w, 16 * BITS * ch + 32),
                                 lut, o);
        *reinterpret_cast<uint4*>(arow + ch * 128) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // tile t widened; every thread done with tile t - 1
    tc_fence_after();
    {
      const int tn = t + 1, sn = (it + 1) % kGStages;
      vbits &= ~(1u << sn);
      if (tn < t1 && issue(tn, sn)) vbits |= 1u << sn;
      cp_async_commit();
    }
    if (tid == 0) {
      const uint64_t adesc = umma_desc_kmajor(smem_u32(st + C::A_OFF), 128, 1024);
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
        umma_i8(tmem, adesc + (uint64_t)(16 * kb), bdesc + (uint64_t)(16 * kb),
                umma_idesc_i8(kGTile, N), kb > 0 ? 1u : 0u);
      umma_commit(bar);
    }
    const bool ok = mbar_wait(bar, (uint32_t)(it & 1));
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      it_out = it;
      break;
    }
    tc_fence_after();
    int dl[32];
    {
      uint32_t r[32];
      if (N == 16) {
        uint32_t r16[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), r16);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = r16[i];
#pragma unroll
        for (int i = 16; i < 32; ++i) r[i] = 0u;
      } else {
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), r);
        tmem_ld_wait();
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) dl[i] = (int)r[i];
    }

    // ---- scores of token tid
    const bool valid = (vbits >> stage) & 1u;
    const uint32_t kpw = *reinterpret_cast<const uint32_t*>(st + C::KP_OFF + tid * 4);
    const float2 ksm = __half22float2(u32_as_h2(kpw));  // (scale, min)
    float z[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (g < a.G && valid && 4 * g + 3 < N) {
        const long long dot = (long long)dl[4 * g] + ((long long)dl[4 * g + 1] << 8) +
                              ((long long)dl[4 * g + 2] << 16) + ((long long)dl[4 * g + 3] << 24);
        const float dc = (float)(dot - (long long)C0 * qsl[g]);
        // s (dot_c / U) + (m + C0 s / U) qsum, times 2^-k sm_scale log2(e)
        z[g] = fmaf(ksm.x * (1.f / U), dc, fmaf(ksm.x, (float)C0 / U, ksm.y) * (float)qsl[g]) *
               kq[g];
      } else {
        z[g] = -INFINITY;
      }
    }
    bool need = false;
#pragma unroll
    for (int g = 0; g < 8; ++g) need |= z[g] > Mh[g] + kGSlack;
    if (__any_sync(0xffffffffu, need)) {
      float alpha[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float m = z[g];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float Mn = fmaxf(Mh[g], m);
        alpha[g] = (Mn == Mh[g]) ? 1.f : fast_exp2(Mh[g] - Mn);
        Mh[g] = Mn;
        Lh[g] *= alpha[g];
        Oh[g] *= alpha[g];
      }
      const int c0 = NB == 1 ? (2 * q4) & 3 : 2 * q4;
      float a0 = alpha[0], a1 = alpha[1];
#pragma unroll
      for (int g = 2; g < 8; g += 2)
        if (c0 == g) {
          a0 = alpha[g];
          a1 = alpha[g + 1];
        }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[nb][mt][0] *= a0;
          acc[nb][mt][1] *= a1;
          acc[nb][mt][2] *= a0;
          acc[nb][mt][3] *= a1;
        }
    }
    // weights p s_v (the PV operand) and sum p (m_v + C0 s_v / U)
    const uint32_t vpw = *reinterpret_cast<const uint32_t*>(st + C::VP_OFF + tid * 4);
    const float2 vsm = __half22float2(u32_as_h2(vpw));
    float* pw = reinterpret_cast<float*>(st + C::A_OFF) + warp * 8 * 32;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const float p = z[g] == -INFINITY ? 0.f : fast_exp2(z[g] - Mh[g]);
      Lh[g] += p;
      Oh[g] = fmaf(p, fmaf(vsm.x, (float)C0 / U, vsm.y), Oh[g]);
      pw[g * 32 + lane] = p * vsm.x * (1.f / U);
    }
    __syncwarp();

    // ---- PV over the warp's 32 tokens: m-tile mt, row r8 = channel
    // 16 r8 + 2 mt, row r8 + 8 = channel 16 r8 + 2 mt + 1
    const uint8_t* vst = st + C::VR_OFF;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int tb = warp * 32 + ks * 16;
      const float* pr = pw + (NB == 1 ? (r8 & 3) : r8) * 32 + ks * 16 + 2 * q4;
      const __half2 h01 = __floats2half2_rn(pr[0], pr[1]);
      const __half2 h89 = __floats2half2_rn(pr[8], pr[9]);
      const float2 f01 = __half22float2(h01), f89 = __half22float2(h89);
      const uint32_t lo01 = h2_as_u32(__floats2half2_rn(pr[0] - f01.x, pr[1] - f01.y));
      const uint32_t lo89 = h2_as_u32(__floats2half2_rn(pr[8] - f89.x, pr[9] - f89.y));
      uint32_t b0, b1, bl0 = 0u, bl1 = 0u;
      if (NB == 1) {
        b0 = r8 < 4 ? h2_as_u32(h01) : lo01;
        b1 = r8 < 4 ? h2_as_u32(h89) : lo89;
      } else {
        b0 = h2_as_u32(h01);
        b1 = h2_as_u32(h89);
        bl0 = lo01;
        bl1 = lo89;
      }
      // the 16 codes of channels [16 r8, 16 r8 + 16) of four tokens
      constexpr int LB = 16 * BITS / 8;  // bytes: 4, 6 or 8
      const int ta = tb + 2 * q4;
      uint32_t cw[4][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int tk = ta + (k & 1) + 8 * (k >> 1);  // A, B, C, D
        const uint8_t* src = vst + tk * C::RB + LB * r8;
        if (LB == 8) {
          const uint2 u = *reinterpret_cast<const uint2*>(src);
          cw[k][0] = u.x; cw[k][1] = u.y;
        } else if (LB == 4) {
          cw[k][0] = *reinterpret_cast<const uint32_t*>(src);
          cw[k][1] = 0u;
        } else {  // 6 bytes, 2-byte aligned
          const uint16_t* s16 = reinterpret_cast<const uint16_t*>(src);
          cw[k][0] = (uint32_t)s16[0] | ((uint32_t)s16[1] << 16);
          cw[k][1] = s16[2];
        }
      }
      // each token's 16 codes as 16 bytes in channel order (3-bit codes are
      // taken one by one below: spreading them to bytes first costs more)
      uint32_t cb[4][4];
      if (BITS != 3) {
#pragma unroll
        for (int k = 0; k < 4; ++k) codes16_bytes<BITS, LUT>(cw[k][0], cw[k][1], lut, cb[k]);
      }
      const __half2 bias = __half2half2(__ushort_as_half((unsigned short)(0x6400u + C0)));
      float tacc[8][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) tacc[mt][e] = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t av[4];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {      // rows r8 (even channel), r8 + 8 (odd)
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {    // token pairs (A, B), (C, D)
            const int ci = 2 * mt + rr;
            // byte ci of each token of the pair into bytes 0 and 2, then
            // binary16 1024 + v (v < 1024 exact in the mantissa) minus 1024 + C0
            uint32_t hv;
            if (BITS == 3) {
              hv = 0x64006400u | code_at<3, 2>(cw[2 * pp], ci) |
                   (code_at<3, 2>(cw[2 * pp + 1], ci) << 16);
            } else {
              const uint32_t pr =
                  __byte_perm(cb[2 * pp][ci >> 2], cb[2 * pp + 1][ci >> 2],
                              (uint32_t)(ci & 3) | ((uint32_t)(4 + (ci & 3)) << 8));
              asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(hv) : "r"(pr), "r"(0x00FF00FFu),
                  "r"(0x64006400u));
            }
            av[2 * pp + rr] = h2_as_u32(__hsub2(u32_as_h2(hv), bias));
          }
        }
        if (NB == 1) {
          mma16816(tacc[mt], av, b0, b1);
        } else {
          float t4[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(t4, av, b0, b1);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[0][mt][e] += t4[e];
          float u4[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(u4, av, bl0, bl1);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[NB - 1][mt][e] += u4[e];
        }
      }
      if (NB == 1) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[0][mt][e] += tacc[mt][e];
      }
    }
  }
  cp_async_wait<0>();

  if (timed_out) {
    if (tid == 0) raise_flag(a.err, KVQ_ERRF_TIMEOUT);
    mbar_wait(bar, (uint32_t)(it_out & 1));
  } else {
#pragma unroll
    for (int g = 0; g < 8; ++g)
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        Lh[g] += __shfl_xor_sync(0xffffffffu, Lh[g], o);
        Oh[g] += __shfl_xor_sync(0xffffffffu, Oh[g], o);
      }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (NB == 1)
          acc[0][mt][e] += __shfl_xor_sync(0xffffffffu, acc[0][mt][e], 2);
        else
          acc[0][mt][e] += acc[NB - 1][mt][e];
      }
    tc_fence_before();
    __syncthreads();
    float* accs = reinterpret_cast<float*>(smem);  // [4][8][128]
    float* mls = accs + 4 * 8 * kGD;               // [4][8] M, [4][8] L
    const bool writer = NB == 2 || q4 < 2;
    if (writer) {
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int g = 2 * q4 + hc;
        float og = Oh[0];
#pragma unroll
        for (int gg = 1; gg < 8; ++gg)
          if (g == gg) og = Oh[gg];
        float* row = accs + (warp * 8 + g) * kGD + 16 * r8;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          row[2 * mt] = acc[0][mt][hc] + og;
          row[2 * mt + 1] = acc[0][mt][2 + hc] + og;
        }
      }
    }
    if (lane < 8) {
      float mv = Mh[0], lv = Lh[0];
#pragma unroll
      for (int g = 1; g < 8; ++g)
        if (lane == g) {
          mv = Mh[g];
          lv = Lh[g];
        }
      mls[warp * 8 + lane] = mv;
      mls[32 + warp * 8 + lane] = lv;
    }
    __syncthreads();
    for (int g = 0; g < a.G; ++g) {
      float Mt = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) Mt = fmaxf(Mt, mls[w * 8 + g]);
      float o = 0.f, lt = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = mls[w * 8 + g];
        const float f = mw == -INFINITY ? 0.f : fast_exp2(mw - Mt);
        o = fmaf(f, accs[(w * 8 + g) * kGD + tid], o);
        lt = fmaf(f, mls[32 + w * 8 + g], lt);
      }
      float* dst = a.part + (base + (int64_t)g * a.splits) * (kGD + 4);
      dst[tid] = o;
      if (tid == 0) *reinterpret_cast<float2*>(dst + kGD) = make_float2(Mt, lt);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kGTmemCols);
  }
}

// The new token of every sequence (a fused decode step) in these formats:
// one warp per (sequence, KV head, K or V) row, the append kernels'
// arithmetic, written at position seq_len - 1 before the attention.
struct GenStepArgs {
  int S, H, P, lg_page, NP, bt_stride, fmt;
  const __half* k_new;
  const __half* v_new;
  int64_t new_stride;
  const float* quat;
  const float* rope;
  int rope_max_pos;
  const float* levels;
  const int32_t* seq_lens;
  const int32_t* block_table;
  uint8_t* k_codes;
  uint32_t* k_params;
  uint8_t* v_codes;
  uint32_t* v_params;
  int32_t* err;
};

template <int ROT, int LGB>
__global__ void __launch_bounds__(128) gen_step_rows_kernel(const GenStepArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int CPL = RowQuantShape<kGD>::CPL;
  const int lane = threadIdx.x % kWarp;
  const int row = blockIdx.x * 4 + threadIdx.x / kWarp;
  if (row >= a.S * a.H * 2) return;  // whole warps
  const int kv = row & 1, h = (row >> 1) % a.H, s = (row >> 1) / a.H;
  const int L = a.seq_lens[s];
  const int pos = L - 1;
  if (L < 1 || (pos >> a.lg_page) >= a.bt_stride || (a.rope != nullptr && pos >= a.rope_max_pos))
    return;
  const int page = a.block_table[(int64_t)s * a.bt_stride + (pos >> a.lg_page)];
  float x[CPL];
  row_load<kGD>(x, (kv ? a.v_new : a.k_new) + (int64_t)s * a.new_stride + (int64_t)h * kGD +
                       lane * CPL, true);
  if (kv == 0 && a.rope != nullptr) rope_regs<CPL>(x, a.rope + (int64_t)pos * kGD + lane * CPL);
  __half s16, m16;
  const uint32_t packed = row_quantize_gen<kGD, ROT, LGB>(x, lane, a.quat, a.fmt, a.levels, s16, m16);
  const bool store = page >= 0 && page < a.NP;
  if (!store && lane == 0 && kv == 0 && h == 0) raise_flag(a.err, KVQ_ERRF_PAGE);
  const int bits = a.fmt == KVQ_FMT_INT2 ? 2 : (a.fmt == KVQ_FMT_INT3 ? 3 : 4);
  const int64_t dst = store ? (((int64_t)page * a.H + h) << a.lg_page) + (pos & (a.P - 1)) : 0;
  row_store_bits<kGD>((kv ? a.v_codes : a.k_codes) + dst * (kGD * bits / 8), packed, bits, lane,
                      store);
  if (store && lane == 0)
    (kv ? a.v_params : a.k_params)[dst] =
        (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
}

template <int ROT, int LGB>
static cudaError_t launch_gen_step(const GenStepArgs& a, cudaStream_t st) {
  const int rows = a.S * a.H * 2;
  cudaError_t e = launch_pdl(gen_step_rows_kernel<ROT, LGB>, (rows + 3) / 4, 128, 0, st, a);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

static cudaError_t dispatch_gen_step(const GenStepArgs& a, int rot, int lgb, cudaStream_t st) {
  if (rot == KVQ_ROT_NONE) return launch_gen_step<KVQ_ROT_NONE, 0>(a, st);
  if (rot == KVQ_ROT_QUAT) return launch_gen_step<KVQ_ROT_QUAT, 0>(a, st);
  if (rot == KVQ_ROT_QUAT_FAST) return launch_gen_step<KVQ_ROT_QUAT_FAST, 0>(a, st);
  if (rot == KVQ_ROT_QUAT_MAT) return launch_gen_step<KVQ_ROT_QUAT_MAT, 0>(a, st);
  switch (lgb) {
    case 4: return launch_gen_step<KVQ_ROT_HADAMARD, 4>(a, st);
    case 5: return launch_gen_step<KVQ_ROT_HADAMARD, 5>(a, st);
    case 6: return launch_gen_step<KVQ_ROT_HADAMARD, 6>(a, st);
    case 7: return launch_gen_step<KVQ_ROT_HADAMARD, 7>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <int BITS, bool LUT, int NB>
static int gen_resident_ctas() {
  static int cached = -1;
  if (cached < 0) {
    const int blocks = resident_ctas_per_sm(
        reinterpret_cast<const void*>(decode_gen_kernel<BITS, LUT, NB>), kGThreads,
        GenCfg<BITS>::SMEM);
    const int sms = device_sm_count();
    cached = blocks * (sms > 0 ? sms : 148);
  }
  return cached;
}

template <int BITS, bool LUT>
static int gen_resident(int G) {
  return G <= 4 ? gen_resident_ctas<BITS, LUT, 1>() : gen_resident_ctas<BITS, LUT, 2>();
}

DecodePlan decode_gen_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len) {
  DecodePlan pl{};
  int tiles = (max_seq_len + kGTile - 1) / kGTile;
  if (tiles < 1) tiles = 1;
  pl.pages_max = tiles;
  const int G = Hq / (d.num_kv_heads > 0 ? d.num_kv_heads : 1);
  const int resident = d.format == KVQ_FMT_INT2   ? gen_resident<2, false>(G)
                       : d.format == KVQ_FMT_INT3 ? gen_resident<3, false>(G)
                                                  : gen_resident<4, true>(G);
  const int pairs = S * d.num_kv_heads > 0 ? S * d.num_kv_heads : 1;
  int splits = resident / pairs;  // a single wave of CTAs
  const int min_splits = (tiles + 63) / 64;
  // `extra` pairs get one split more, so the CTAs fill the resident slots
  int extra = resident - splits * pairs;
  if (splits < min_splits) {
    splits = min_splits;
    extra = 0;
  }
  if (splits < 1) {
    splits = 1;
    extra = 0;
  }
  if (splits >= tiles) {
    splits = tiles;
    extra = 0;
  }
  if (extra < 0) extra = 0;
  pl.pages_per_split = (tiles + splits - 1) / splits;
  pl.splits = extra > 0 ? splits + 1 : splits;
  pl.nhi = extra > 0 ? extra : S * d.num_kv_heads;
  pl.workspace = (size_t)S * Hq * pl.splits * (d.head_dim + 4) * sizeof(float);
  return pl;
}

template <int BITS, bool LUT>
static cudaError_t launch_gen(const GenDecodeArgs& a, int grid, cudaStream_t st) {
  auto kern = a.G <= 4 ? decode_gen_kernel<BITS, LUT, 1> : decode_gen_kernel<BITS, LUT, 2>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GenCfg<BITS>::SMEM);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, grid, kGThreads, GenCfg<BITS>::SMEM, st, a);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

int decode_gen_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                      const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                      int32_t bt_stride, float sm_scale, const uint8_t* k_codes,
                      const void* k_params, const uint8_t* v_codes, const void* v_params,
                      float* out, void* workspace, size_t workspace_bytes, int32_t* err,
                      cudaStream_t st, const DecodeStepRows* step) {
  const int G = Hq / d.num_kv_heads;
  if (d.head_dim != kGD || G > 8) return KVQ_ERR_UNSUPPORTED;
  const DecodePlan pl = decode_gen_plan(d, S, Hq, max_seq_len);
  if (workspace == nullptr || workspace_bytes < pl.workspace) return KVQ_ERR_WORKSPACE;
  int lgb = 0;
  while ((1 << lgb) < d.rot_block) ++lgb;
  int lg_page = 0;
  while ((1 << lg_page) < d.page_size) ++lg_page;
  const int rot = d.rot_kind == KVQ_ROT_HADAMARD_SIGNED ? KVQ_ROT_HADAMARD : d.rot_kind;
  const float* table =
      (d.rot_kind == KVQ_ROT_NONE || d.rot_kind == KVQ_ROT_HADAMARD) ? nullptr : d.quat;
  cudaError_t e;
  if (step != nullptr) {
    GenStepArgs sa;
    sa.S = S; sa.H = d.num_kv_heads; sa.P = d.page_size; sa.lg_page = lg_page;
    sa.NP = d.num_pages; sa.bt_stride = bt_stride; sa.fmt = d.format;
    sa.k_new = static_cast<const __half*>(step->k_new);
    sa.v_new = static_cast<const __half*>(step->v_new);
    sa.new_stride = step->new_stride;
    sa.quat = table; sa.rope = d.rope; sa.rope_max_pos = d.rope_max_pos; sa.levels = d.levels;
    sa.seq_lens = seq_lens; sa.block_table = block_table;
    sa.k_codes = const_cast<uint8_t*>(k_codes);
    sa.k_params = static_cast<uint32_t*>(const_cast<void*>(k_params));
    sa.v_codes = const_cast<uint8_t*>(v_codes);
    sa.v_params = static_cast<uint32_t*>(const_cast<void*>(v_params));
    sa.err = err;
    e = dispatch_gen_step(sa, rot, lgb, st);
    if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return KVQ_ERR_CUDA;
  }
  GenDecodeArgs a;
  a.S = S; a.Hq = Hq; a.H = d.num_kv_heads; a.G = G; a.P = d.page_size; a.lg_page = lg_page;
  a.NP = d.num_pages; a.bt_stride = bt_stride; a.max_seq_len = max_seq_len;
  a.splits = pl.splits; a.nhi = pl.nhi;
  a.rot_kind = d.rot_kind; a.lgb = lgb;
  a.scale2 = (float)((double)sm_scale * 1.4426950408889634074);
  a.q = static_cast<const __half*>(q); a.quat = d.quat;
  a.rope = d.rope; a.rope_max_pos = d.rope_max_pos; a.levels = d.levels;
  a.seq_lens = seq_lens; a.block_table = block_table;
  a.k_codes = k_codes; a.k_params = static_cast<const uint32_t*>(k_params);
  a.v_codes = v_codes; a.v_params = static_cast<const uint32_t*>(v_params);
  a.part = static_cast<float*>(workspace);
  a.err = err;
  const int grid = pl.nhi * pl.splits + (S * d.num_kv_heads - pl.nhi) * (pl.splits - 1);
  if (d.format == KVQ_FMT_INT2)
    e = launch_gen<2, false>(a, grid, st);
  else if (d.format == KVQ_FMT_INT3)
    e = launch_gen<3, false>(a, grid, st);
  else
    e = launch_gen<4, true>(a, grid, st);
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  return decode_merge_launch(d, S, Hq, pl.splits, pl.nhi, a.part, out, st);
}

}  // namespace kvq
