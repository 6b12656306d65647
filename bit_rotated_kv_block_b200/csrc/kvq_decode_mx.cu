// Decode attention over the microscaled FP4 cache (kvq.h, KVQ_FMT_MXFP4):
// UltraQuant's second path ("UltraQuant: 4-bit KV caching for long agents",
// method section: FP4 KV tensors, UE8M0 group scales and FP8 queries taken by
// the matrix cores' scaled multiply-accumulate), on Blackwell's block-scaled
// tcgen05 MMA.
//
// One CTA (4 warps) per (sequence, KV head, split); a split is a range of
// 128-token tiles (8 pages of 16 or 4 of 32). Per tile:
//  * every thread stages one token: its 64 bytes of K codes into the MMA's
//    K-major operand layout for 4-bit elements (each 16-byte chunk holds 16
//    codes in its low 8 bytes), its 4 K block-scale bytes into the scale-
//    factor copy layout, its V codes and V scale word as plain rows;
//    cp.async, a 2-stage ring (4 CTAs per SM for G <= 4);
//  * one thread copies the K scales into tensor memory and issues four
//    tcgen05.mma kind::mxf8f6f4.block_scale (M = 128 tokens, N = 16 query
//    rows, K = 32 channels each): S = (K e2m1 x 2^Xk)(q e4m3 x 2^Xq)^T, fp32
//    in tensor memory; completion on an mbarrier;
//  * thread t reads its token's G scores (tcgen05.ld), each warp keeps its own
//    online softmax over its 32 tokens (base 2, a reference maximum that moves
//    only by more than 8), and accumulates PV on the f16 tensor cores
//    (mma.sync): V codes become binary16 through the hardware E2M1 converter,
//    times 2^Xv of their block (exact while Xv >= -14), token pairs side by
//    side; the weights p enter as binary16 hi + lo; every 16-token product
//    starts from zero and joins the running sum through a binary32 add.
// The four warps' states merge through shared memory into one partial result
// per (query head, split) in the layout the INT4 decode writes, and the same
// merge kernel combines the splits and rotates the output back.
//
// The query is rotated in binary32 exactly as a key row (same butterflies /
// quaternion products), then quantized to MX E4M3 (one shared exponent per 32
// channels) once per CTA: the oracle repeats that arithmetic, so the query
// codes are the same on both sides and the scores differ only by the tensor
// core's fp32 accumulation order.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_launch.h"
#include "kvq_rotate.cuh"
#include "kvq_rowquant.cuh"
#include "kvq_tcgen05.cuh"

namespace kvq {

namespace {

constexpr int kMxD = 128;        // head_dim
constexpr int kMxThreads = 128;  // 4 warps; thread t stages and scores token t of a tile
constexpr int kMxTile = 128;     // tokens per tile: the MMA's M
constexpr int kMxN = 16;         // the MMA's N: query rows of B (G used, the rest zero)
constexpr int kMxStages = 2;
constexpr uint32_t kMxTmemCols = 32;
constexpr uint32_t kColD = 0, kColSFA = 16, kColSFB = 20;  // tensor-memory columns
constexpr float kMxSlack = 8.f;

// one ring stage (bytes)
constexpr int kA_OFF = 0;                   // K codes: 16 row groups x 8 chunks x (8 rows x 16 B)
constexpr int kA_B = 16 * 1024;
constexpr int kSFA_OFF = kA_OFF + kA_B;     // K block scales, byte (t%32)*16 + (t/32)*4 + block
constexpr int kSF_B = 512;
constexpr int kV_OFF = kSFA_OFF + kSF_B;    // V codes, token t at t * 64
constexpr int kV_B = kMxTile * 64;
constexpr int kVS_OFF = kV_OFF + kV_B;      // V params words
constexpr int kStage_B = kVS_OFF + kMxTile * 4;
// behind the ring
constexpr int kB_OFF = kMxStages * kStage_B;  // query E4M3: 2 row groups x 8 chunks x 128 B
constexpr int kB_B = 2048;
constexpr int kSFB_OFF = kB_OFF + kB_B;       // query block scales (rows 0-15 used)
constexpr int kBar_OFF = kSFB_OFF + kSF_B;    // mbarrier, then the tensor-memory base
// per-warp weights [8 heads][32 tokens] fp32 live in the K region of the
// stage being consumed (free once its MMA has completed, refilled only after
// the next barrier)
constexpr int kP_B = 8 * 32 * 4;
static_assert(4 * kP_B <= kA_B, "weights fit in the consumed K region");
constexpr int kMxSmem = kBar_OFF + 16;
static_assert(kStage_B % 128 == 0 && kB_OFF % 1024 == 0, "operand alignment");
// the four warps' states at the end reuse stage 0: [4][8][128] acc + [4][8] M, L
static_assert(4 * 8 * kMxD * 4 + 2 * 4 * 8 * 4 <= kStage_B, "merge scratch fits in a stage");

}  // namespace

struct MxDecodeArgs {
  int S, Hq, H, G, P, lg_page, NP, bt_stride, max_seq_len, splits;
  int nhi;  // (sequence, KV head) pairs with `splits` splits; the rest have splits - 1
  int rot_kind, lgb;
  float scale2;  // sm_scale * log2(e)
  const __half* q;
  const float* quat;
  const float* rope;
  int rope_max_pos;
  const int32_t* seq_lens;
  const int32_t* block_table;
  const uint8_t* k_codes;
  const uint32_t* k_params;
  const uint8_t* v_codes;
  const uint32_t* v_params;
  float* part;  // [S][Hq][splits][D + 4]
  int32_t* err;
};

// NB = 1: G <= 4, one PV MMA per m-tile (columns 0-3 the weights' hi parts of
// heads 0-3, columns 4-7 their lo parts); NB = 2: G <= 8, hi and lo MMAs.
template <int NB>
__global__ void __launch_bounds__(kMxThreads) decode_mx_kernel(const MxDecodeArgs a) {
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
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kBar_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBar_OFF + 8);

  pdl_wait();  // pools and queries may come from the previous kernel
  pdl_trigger();

  const int L = a.seq_lens[s];
  const bool len_ok = L >= 0 && L <= a.max_seq_len &&
                      ((L + a.P - 1) >> a.lg_page) <= a.bt_stride &&
                      (a.rope == nullptr || L <= a.rope_max_pos);
  const int ntiles = len_ok ? (L + kMxTile - 1) / kMxTile : 0;
  // the sequence's tiles dealt out evenly over its splits
  const int t0 = (int)(((int64_t)split * ntiles) / nspl);
  const int t1 = (int)(((int64_t)(split + 1) * ntiles) / nspl);
  const int64_t base = ((int64_t)s * a.Hq + (int64_t)h * a.G) * a.splits + split;
  if (t0 >= t1) {  // nothing to attend: a zero row with maximum -inf and weight 0
    if (!len_ok && split == 0 && h == 0 && tid == 0) raise_flag(a.err, KVQ_ERRF_LEN);
    for (int g = 0; g < a.G; ++g) {
      float* dst = a.part + (base + (int64_t)g * a.splits) * (kMxD + 4);
      dst[tid] = 0.f;
      if (tid == 0) *reinterpret_cast<float2*>(dst + kMxD) = make_float2(-INFINITY, 0.f);
    }
    return;
  }

  if (warp == 0) {
    tmem_alloc(tmem_slot, kMxTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  for (int i = tid; i < (kB_B + kSF_B) / 16; i += kMxThreads)
    reinterpret_cast<uint4*>(smem + kB_OFF)[i] = make_uint4(0u, 0u, 0u, 0u);

  // staging of tile t into a stage; returns whether token tid is cached
  auto issue = [&](int t, int stage) -> bool {
    uint8_t* st = smem + stage * kStage_B;
    const int tok = t * kMxTile + tid;
    int page = -1;
    if (tok < L) page = a.block_table[(int64_t)s * a.bt_stride + (tok >> a.lg_page)];
    const bool ok = page >= 0 && page < a.NP && tok < L;
    uint32_t* sfa = reinterpret_cast<uint32_t*>(st + kSFA_OFF + (tid & 31) * 16 + (tid >> 5) * 4);
    uint32_t* vsc = reinterpret_cast<uint32_t*>(st + kVS_OFF + tid * 4);
    if (ok) {
      const int64_t row = (((int64_t)page * a.H + h) << a.lg_page) + (tok & (a.P - 1));
      const uint8_t* kr = a.k_codes + row * (kMxD / 2);
      uint8_t* adst = st + kA_OFF + (tid >> 3) * 1024 + (tid & 7) * 16;
#pragma unroll
      for (int c = 0; c < 8; ++c) cp_async8(adst + c * 128, kr + 8 * c);
      cp_async4(sfa, a.k_params + row);
      const uint8_t* vr = a.v_codes + row * (kMxD / 2);
#pragma unroll
      for (int c = 0; c < 4; ++c) cp_async16(st + kV_OFF + tid * 64 + 16 * c, vr + 16 * c);
      cp_async4(vsc, a.v_params + row);
    } else {
      // scale bytes 0 (2^-127): stale codes give tiny finite products, and
      // the V values become binary16 zeros; the scores are masked anyway
      *sfa = 0u;
      *vsc = 0u;
      if (tok < L && (tok & (a.P - 1)) == 0) raise_flag(a.err, KVQ_ERRF_PAGE);
    }
    return ok;
  };
  uint32_t vbits = 0;  // bit k: this thread's token of the tile in stage k is cached
#pragma unroll
  for (int k = 0; k < kMxStages - 1; ++k) {
    if (t0 + k < t1 && issue(t0 + k, k)) vbits |= 1u << k;
    cp_async_commit();
  }

  __syncthreads();  // B zeroed, barrier initialised

  // ---- the query: warp 0, lane (gq, j) owns channels [32 j, 32 j + 32) of
  // query head gq: RoPE at position L - 1, the rotation, then MX E4M3 (the
  // lane's 32 channels are one scale block)
  if (warp == 0) {
    const int gq = lane >> 2, j = lane & 3;
    const bool hq_ok = gq < a.G;
    float x[32];
    const uint4* qsrc = reinterpret_cast<const uint4*>(
        a.q + ((int64_t)s * a.Hq + (int64_t)h * a.G + (hq_ok ? gq : 0)) * kMxD + j * 32);
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
    if (a.rope != nullptr && L >= 1) rope_regs<32>(x, a.rope + (int64_t)(L - 1) * kMxD + j * 32);
    rotate_quarter<32>(x, j, a.rot_kind, a.lgb, a.quat);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const int eb = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
    const uint32_t xb = eb > 8 ? (uint32_t)(eb - 8) : 0u;  // X + 127, X = floor(log2 amax) - 8
    const float inv = __uint_as_float((254u - xb) << 23);  // 2^-X
    if (hq_ok) {
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        w[k] = e4m3x2(__fmul_rn(x[4 * k], inv), __fmul_rn(x[4 * k + 1], inv)) |
               (e4m3x2(__fmul_rn(x[4 * k + 2], inv), __fmul_rn(x[4 * k + 3], inv)) << 16);
      // row gq of B: 16-byte K chunks 2j and 2j + 1 (channels 32 j ..)
      uint8_t* bdst = smem + kB_OFF + (gq >> 3) * 1024 + (gq & 7) * 16;
      *reinterpret_cast<uint4*>(bdst + (2 * j) * 128) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(bdst + (2 * j + 1) * 128) = make_uint4(w[4], w[5], w[6], w[7]);
      smem[kSFB_OFF + gq * 16 + j] = (uint8_t)xb;
    }
  }
  fence_async_smem();  // B, its scales and the zero rows, for the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0)  // the query's scale factors, once
    tmem_cp_32x128_x4(tmem + kColSFB, umma_desc_kmajor(smem_u32(smem + kSFB_OFF), 128, 128));
  const uint64_t bdesc = umma_desc_kmajor(smem_u32(smem + kB_OFF), 128, 1024);

  // ---- per-warp softmax state and PV accumulators
  const int r8 = lane >> 2, q4 = lane & 3;
  float Mh[8], Lh[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    Mh[g] = -INFINITY;
    Lh[g] = 0.f;
  }
  float acc[NB][8][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nb][mt][e] = 0.f;
  bool timed_out = false;
  int it_out = 0;  // the iteration whose wait ran out

  for (int t = t0, it = 0; t < t1; ++t, ++it) {
    const int stage = it % kMxStages;
    cp_async_wait<kMxStages - 2>();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // tile t staged; every thread done with tile t - 1
    tc_fence_after();
    {
      const int tn = t + kMxStages - 1, sn = (it + kMxStages - 1) % kMxStages;
      vbits &= ~(1u << sn);
      if (tn < t1 && issue(tn, sn)) vbits |= 1u << sn;
      cp_async_commit();
    }
    uint8_t* st = smem + stage * kStage_B;
    if (tid == 0) {
      tmem_cp_32x128_x4(tmem + kColSFA, umma_desc_kmajor(smem_u32(st + kSFA_OFF), 128, 128));
      const uint64_t adesc = umma_desc_kmajor(smem_u32(st + kA_OFF), 128, 1024);
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        // K block kb: chunks 2 kb, 2 kb + 1 (the start address advances by
        // 256 bytes, 16 in the descriptor's units)
        umma_mx(tmem + kColD, adesc + (uint64_t)(16 * kb), bdesc + (uint64_t)(16 * kb),
                umma_idesc_mx(5, 0, kMxTile, kMxN, kb), (tmem + kColSFA) | ((uint32_t)kb << 30),
                (tmem + kColSFB) | ((uint32_t)kb << 30), kb > 0 ? 1u : 0u);
      }
      umma_commit(bar);
    }
    const bool ok = mbar_wait(bar, (uint32_t)(it & 1));
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      it_out = it;
      break;
    }
    tc_fence_after();
    uint32_t r[16];
    tmem_ld16(tmem + kColD + ((uint32_t)(warp * 32) << 16), r);
    tmem_ld_wait();

    // ---- scores of token tid for the G heads, the warp's online softmax
    const bool valid = (vbits >> stage) & 1u;
    float* pw = reinterpret_cast<float*>(st + kA_OFF) + warp * 8 * 32;
    float z[8];
#pragma unroll
    for (int g = 0; g < 8; ++g)
      z[g] = (g < a.G && valid) ? __uint_as_float(r[g]) * a.scale2 : -INFINITY;
    bool need = false;
#pragma unroll
    for (int g = 0; g < 8; ++g) need |= z[g] > Mh[g] + kMxSlack;
    if (__any_sync(0xffffffffu, need)) {
      float alpha[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float m = z[g];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float Mn = fmaxf(Mh[g], m);
        alpha[g] = (Mn == Mh[g]) ? 1.f : fast_exp2(Mh[g] - Mn);  // Mh = -inf: 0
        Mh[g] = Mn;
        Lh[g] *= alpha[g];
      }
      // this lane's accumulator columns 2 q4 and 2 q4 + 1 (heads (2 q4) & 3
      // and its successor for NB = 1, 2 q4 and 2 q4 + 1 for NB = 2)
      const int c0 = NB == 1 ? (2 * q4) & 3 : 2 * q4;
      float a0 = alpha[0], a1 = alpha[1];
#pragma unroll
      for (int g = 2; g < 8; g += 2)
        if (c0 == g) {
          a0 = alpha[g];
          a1 = alpha[g + 1];
        }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[nb][mt][0] *= a0;
          acc[nb][mt][1] *= a1;
          acc[nb][mt][2] *= a0;
          acc[nb][mt][3] *= a1;
        }
      }
    }
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const float p = z[g] == -INFINITY ? 0.f : fast_exp2(z[g] - Mh[g]);
      Lh[g] += p;
      pw[g * 32 + lane] = p;
    }
    __syncwarp();

    // ---- PV over the warp's 32 tokens, two k-steps of 16. For NB = 1 the
    // tile's two k-steps accumulate in the MMA from zero and join the running
    // sums once; for NB = 2 (hi and lo products) each k-step does.
    const uint8_t* vst = st + kV_OFF;
    const uint32_t* vsw = reinterpret_cast<const uint32_t*>(st + kVS_OFF);
    float tacc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) tacc[mt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int tb = warp * 32 + ks * 16;  // first token of the k-step in the tile
      // B: column r8, tokens 2 q4, 2 q4 + 1 (b0) and 2 q4 + 8, 2 q4 + 9 (b1)
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
      // A: V codes of tokens tb + 2 q4 (+1) and tb + 2 q4 + 8 (+9), bytes
      // 8 r8 .. 8 r8 + 7 of each row: m-tile mt takes byte mt; row r8 is
      // channel 16 r8 + 2 mt (low nibble), row r8 + 8 channel 16 r8 + 2 mt + 1
      const int ta = tb + 2 * q4;
      const uint2 VA = *reinterpret_cast<const uint2*>(vst + ta * 64 + 8 * r8);
      const uint2 VB = *reinterpret_cast<const uint2*>(vst + (ta + 1) * 64 + 8 * r8);
      const uint2 VC = *reinterpret_cast<const uint2*>(vst + (ta + 8) * 64 + 8 * r8);
      const uint2 VD = *reinterpret_cast<const uint2*>(vst + (ta + 9) * 64 + 8 * r8);
      // 2^Xv of block r8 / 2 for each token, as binary16 pairs
      auto p2 = [&](int tk) {
        const uint32_t xb = (vsw[tk] >> (8 * (r8 >> 1))) & 0xFFu;
        return __uint_as_float(xb << 23);
      };
      const __half2 sAB = __floats2half2_rn(p2(ta), p2(ta + 1));
      const __half2 sCD = __floats2half2_rn(p2(ta + 8), p2(ta + 9));
#pragma unroll
      for (int hw = 0; hw < 2; ++hw) {
        const uint32_t wa = hw ? VA.y : VA.x, wb = hw ? VB.y : VB.x;
        const uint32_t wc = hw ? VC.y : VC.x, wd = hw ? VD.y : VD.x;
        // low nibbles of token pair (A, B) side by side, high nibbles likewise
        const uint32_t e0 = (wa & 0x0F0F0F0Fu) | ((wb << 4) & 0xF0F0F0F0u);
        const uint32_t o0 = ((wa >> 4) & 0x0F0F0F0Fu) | (wb & 0xF0F0F0F0u);
        const uint32_t e1 = (wc & 0x0F0F0F0Fu) | ((wd << 4) & 0xF0F0F0F0u);
        const uint32_t o1 = ((wc >> 4) & 0x0F0F0F0Fu) | (wd & 0xF0F0F0F0u);
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4) {
          const int mt = 4 * hw + m4;
          uint32_t av[4];
          av[0] = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2((e0 >> (8 * m4)) & 0xFFu)), sAB));
          av[1] = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2((o0 >> (8 * m4)) & 0xFFu)), sAB));
          av[2] = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2((e1 >> (8 * m4)) & 0xFFu)), sCD));
          av[3] = h2_as_u32(__hmul2(u32_as_h2(e2m1x2_to_h2((o1 >> (8 * m4)) & 0xFFu)), sCD));
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
      }
    }
    if (NB == 1) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[0][mt][e] += tacc[mt][e];
    }
  }
  cp_async_wait<0>();

  if (timed_out) {
    // the tensor core may still be working on the last tile: give it one more
    // bounded wait before the tensor memory is freed; outputs are undefined
    if (tid == 0) raise_flag(a.err, KVQ_ERRF_TIMEOUT);
    mbar_wait(bar, (uint32_t)(it_out & 1));
  } else {
    // ---- per-warp totals: weights over lanes, lo columns folded onto hi
#pragma unroll
    for (int g = 0; g < 8; ++g)
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) Lh[g] += __shfl_xor_sync(0xffffffffu, Lh[g], o);
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
    __syncthreads();  // every warp is done with the ring: stage 0 becomes scratch
    float* accs = reinterpret_cast<float*>(smem);          // [4][8][128]
    float* mls = accs + 4 * 8 * kMxD;                       // [4][8] M, then [4][8] L
    const bool writer = NB == 2 || q4 < 2;
    if (writer) {
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int g = 2 * q4 + hc;
        float* row = accs + (warp * 8 + g) * kMxD + 16 * r8;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          row[2 * mt] = acc[0][mt][hc];
          row[2 * mt + 1] = acc[0][mt][2 + hc];
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
    // thread tid: channel tid of every head; the four warps' states combined
    for (int g = 0; g < a.G; ++g) {
      float Mt = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) Mt = fmaxf(Mt, mls[w * 8 + g]);
      float o = 0.f, lt = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = mls[w * 8 + g];
        const float f = mw == -INFINITY ? 0.f : fast_exp2(mw - Mt);
        o = fmaf(f, accs[(w * 8 + g) * kMxD + tid], o);
        lt = fmaf(f, mls[32 + w * 8 + g], lt);
      }
      float* dst = a.part + (base + (int64_t)g * a.splits) * (kMxD + 4);
      dst[tid] = o;
      if (tid == 0) *reinterpret_cast<float2*>(dst + kMxD) = make_float2(Mt, lt);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kMxTmemCols);
  }
}

// The new token of every sequence (a fused decode step): one warp per
// (sequence, KV head, K or V) row, quantized with the same arithmetic as the
// append kernels and written at position seq_len - 1 before the attention.
struct MxStepArgs {
  int S, H, P, lg_page, NP, bt_stride, rot_kind, lgb;
  const __half* k_new;
  const __half* v_new;
  int64_t new_stride;
  const float* quat;
  const float* rope;
  int rope_max_pos;
  const int32_t* seq_lens;
  const int32_t* block_table;
  uint8_t* k_codes;
  uint32_t* k_params;
  uint8_t* v_codes;
  uint32_t* v_params;
  int32_t* err;
};

template <int ROT, int LGB>
__global__ void __launch_bounds__(128) mx_step_rows_kernel(const MxStepArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int CPL = RowQuantShape<kMxD>::CPL;
  const int lane = threadIdx.x % kWarp;
  const int row = blockIdx.x * 4 + threadIdx.x / kWarp;  // ((s * H) + h) * 2 + kv
  if (row >= a.S * a.H * 2) return;  // whole warps leave together
  const int kv = row & 1, h = (row >> 1) % a.H, s = (row >> 1) / a.H;
  const int L = a.seq_lens[s];
  const int pos = L - 1;
  if (L < 1 || (pos >> a.lg_page) >= a.bt_stride || (a.rope != nullptr && pos >= a.rope_max_pos))
    return;  // no new token to place (the attention flags a bad length)
  const int page = a.block_table[(int64_t)s * a.bt_stride + (pos >> a.lg_page)];
  float x[CPL];
  row_load<kMxD>(x, (kv ? a.v_new : a.k_new) + (int64_t)s * a.new_stride + (int64_t)h * kMxD +
                        lane * CPL, true);
  if (kv == 0 && a.rope != nullptr) rope_regs<CPL>(x, a.rope + (int64_t)pos * kMxD + lane * CPL);
  uint32_t pword;
  const uint32_t packed = row_quantize_mx<kMxD, ROT, LGB>(x, lane, a.quat, pword);
  if (page < 0 || page >= a.NP) {
    if (lane == 0 && kv == 0 && h == 0) raise_flag(a.err, KVQ_ERRF_PAGE);
    return;
  }
  const int64_t dst = (((int64_t)page * a.H + h) << a.lg_page) + (pos & (a.P - 1));
  row_store_codes<kMxD>((kv ? a.v_codes : a.k_codes) + dst * (kMxD / 2) + lane * (CPL / 2), packed);
  if (lane == 0) (kv ? a.v_params : a.k_params)[dst] = pword;
}

template <int ROT, int LGB>
static cudaError_t launch_mx_step(const MxStepArgs& a, cudaStream_t st) {
  const int rows = a.S * a.H * 2;
  cudaError_t e = launch_pdl(mx_step_rows_kernel<ROT, LGB>, (rows + 3) / 4, 128, 0, st, a);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

static cudaError_t dispatch_mx_step(const MxStepArgs& a, int rot, int lgb, cudaStream_t st) {
  if (rot == KVQ_ROT_NONE) return launch_mx_step<KVQ_ROT_NONE, 0>(a, st);
  if (rot == KVQ_ROT_QUAT) return launch_mx_step<KVQ_ROT_QUAT, 0>(a, st);
  if (rot == KVQ_ROT_QUAT_FAST) return launch_mx_step<KVQ_ROT_QUAT_FAST, 0>(a, st);
  if (rot == KVQ_ROT_QUAT_MAT) return launch_mx_step<KVQ_ROT_QUAT_MAT, 0>(a, st);
  switch (lgb) {  // Hadamard (its randomised-sign form takes the sign table)
    case 4: return launch_mx_step<KVQ_ROT_HADAMARD, 4>(a, st);
    case 5: return launch_mx_step<KVQ_ROT_HADAMARD, 5>(a, st);
    case 6: return launch_mx_step<KVQ_ROT_HADAMARD, 6>(a, st);
    case 7: return launch_mx_step<KVQ_ROT_HADAMARD, 7>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <int NB>
static int mx_resident_ctas() {
  static int cached = -1;
  if (cached < 0) {
    const int blocks =
        resident_ctas_per_sm(reinterpret_cast<const void*>(decode_mx_kernel<NB>), kMxThreads,
                             kMxSmem);
    const int sms = device_sm_count();
    cached = blocks * (sms > 0 ? sms : 148);
  }
  return cached;
}

DecodePlan decode_mx_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len) {
  DecodePlan pl{};
  int tiles = (max_seq_len + kMxTile - 1) / kMxTile;
  if (tiles < 1) tiles = 1;
  pl.pages_max = tiles;
  const int G = Hq / (d.num_kv_heads > 0 ? d.num_kv_heads : 1);
  const int resident = G <= 4 ? mx_resident_ctas<1>() : mx_resident_ctas<2>();
  const int pairs = S * d.num_kv_heads > 0 ? S * d.num_kv_heads : 1;
  // at most one CTA per resident slot (a single wave: a second, partial one
  // would double the time), at least one split per 64 tiles
  int splits = resident / pairs;
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

int decode_mx_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                     const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                     int32_t bt_stride, float sm_scale, const uint8_t* k_codes,
                     const void* k_params, const uint8_t* v_codes, const void* v_params,
                     float* out, void* workspace, size_t workspace_bytes, int32_t* err,
                     cudaStream_t st, const DecodeStepRows* step) {
  const int G = Hq / d.num_kv_heads;
  if (d.head_dim != kMxD || G > 8) return KVQ_ERR_UNSUPPORTED;
  const DecodePlan pl = decode_mx_plan(d, S, Hq, max_seq_len);
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
    MxStepArgs sa;
    sa.S = S; sa.H = d.num_kv_heads; sa.P = d.page_size; sa.lg_page = lg_page;
    sa.NP = d.num_pages; sa.bt_stride = bt_stride; sa.rot_kind = rot; sa.lgb = lgb;
    sa.k_new = static_cast<const __half*>(step->k_new);
    sa.v_new = static_cast<const __half*>(step->v_new);
    sa.new_stride = step->new_stride;
    sa.quat = table; sa.rope = d.rope; sa.rope_max_pos = d.rope_max_pos;
    sa.seq_lens = seq_lens; sa.block_table = block_table;
    sa.k_codes = const_cast<uint8_t*>(k_codes);
    sa.k_params = static_cast<uint32_t*>(const_cast<void*>(k_params));
    sa.v_codes = const_cast<uint8_t*>(v_codes);
    sa.v_params = static_cast<uint32_t*>(const_cast<void*>(v_params));
    sa.err = err;
    e = dispatch_mx_step(sa, rot, lgb, st);
    if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return KVQ_ERR_CUDA;
  }
  MxDecodeArgs a;
  a.S = S; a.Hq = Hq; a.H = d.num_kv_heads; a.G = G; a.P = d.page_size; a.lg_page = lg_page;
  a.NP = d.num_pages; a.bt_stride = bt_stride; a.max_seq_len = max_seq_len;
  a.splits = pl.splits; a.nhi = pl.nhi;
  a.rot_kind = d.rot_kind; a.lgb = lgb;
  a.scale2 = (float)((double)sm_scale * 1.4426950408889634074);
  a.q = static_cast<const __half*>(q); a.quat = d.quat;
  a.rope = d.rope; a.rope_max_pos = d.rope_max_pos;
  a.seq_lens = seq_lens; a.block_table = block_table;
  a.k_codes = k_codes; a.k_params = static_cast<const uint32_t*>(k_params);
  a.v_codes = v_codes; a.v_params = static_cast<const uint32_t*>(v_params);
  a.part = static_cast<float*>(workspace);
  a.err = err;
  auto kern = G <= 4 ? decode_mx_kernel<1> : decode_mx_kernel<2>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMxSmem);
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  const int grid = pl.nhi * pl.splits + (S * d.num_kv_heads - pl.nhi) * (pl.splits - 1);
  e = launch_pdl(kern, grid, kMxThreads, kMxSmem, st, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  return decode_merge_launch(d, S, Hq, pl.splits, pl.nhi, a.part, out, st);
}

}  // namespace kvq
