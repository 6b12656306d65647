// Paged decode attention over the rotated INT4 cache.
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
// LLM Serving" (Summary, Key takeaway): the INT4 cache is read by attention in
// its paged layout; the query is rotated by the same orthogonal block
// Hadamard (or quaternion) map as the keys, so q . k is unchanged, and the
// output is rotated back once per query head.
//
// Two kernels on the caller's stream, the second launched with programmatic
// serialization so that it is resident as the first drains.
// Split kernel, one warp per (sequence, KV head, split of the page range):
//  0. For a fused decode step (kvq_decode_step) the warp whose range holds
//     the page of position seq_len - 1 quantizes that sequence's new K and V
//     rows for its KV head exactly as kvq_quantize_append would, writes them
//     to the pools and patches them into its staged copy of that page (so
//     the attention reads them without a fence or a global round trip).
//  1. The warp rotates its query heads in registers: lane (r, j) holds
//     channels [j*d/4, (j+1)*d/4) of query head r (GP = 8) or r % 4 (GP = 4);
//     butterfly stages inside a quarter run in registers, wider ones across
//     lanes j by shuffles. Each rotated head is then held as a fixed point
//     qint = RN(qhat * 2^k), 2^k the power of two that brings the head's
//     largest |qhat| just below 2^26 (so qhat * 2^k is exact in binary32),
//     split into four signed 8-bit limbs (even channels of a code byte as
//     16 qint_e - qint_o, odd ones as qint_o).
//  2. The sequence's pages are dealt out to its splits as contiguous ranges
//     of near-equal size. The warp streams its (page, KV head) chunks (codes
//     + params of K and V, contiguous in the pool) into a two-stage
//     shared-memory ring of 64-token stages (32 at d = 256) with cp.async
//     and runs both contractions on tensor
//     cores (mma.sync):
//       QK^T: m16n8k32 s8 x u8 -> s32, A = the query limbs (one row per
//             (head, limb)), B = the K codes as bytes (even slots the low
//             nibble c_e of a code byte, one AND per word; odd slots the
//             byte itself, c_e + 16 c_o); the limb dots recombine exactly
//             into 16 sum_i (c_i - 8) qint_i, and the score
//               z = sm_scale log2(e) 2^-k (s_k dot + (m_k + 8 s_k) sum qint)
//             is formed in binary32;
//       PV:   m16n8k16 f16 x f16 -> f32, A = V codes transposed (channels x
//             tokens) as c - 8, exact in binary16 (a logic operation and a
//             half2 subtract per pair of codes after a byte interleave),
//             B = p * s_v split into binary16 hi + lo, summed over a
//             64-token stage in the tensor core and added to the running
//             sum once per stage; sum p (m_v + 8 s_v) is kept aside.
//             Online softmax in base 2 against a per-head reference maximum
//             that moves only when a score exceeds it by more than 8.
//  3. It writes (acc, max, sum) per query head to the workspace.
// Merge kernel, one warp per (sequence, query head): combines the splits
// (log-sum-exp), normalises, rotates back in registers and writes the
// float32 output. No warp ever waits on another.
#include <cuda_runtime.h>

#include <type_traits>

#include "kvq_device.cuh"
#include "kvq_launch.h"
#include "kvq_rotate.cuh"
#include "kvq_rowquant.cuh"

namespace kvq {

constexpr int kDecWarps = 4;

struct DecodeArgs {
  int S, Hq, H, G, P, NP, bt_stride, max_seq_len, splits;
  int nhi;  // (sequence, KV head) pairs with `splits` splits; the rest have splits - 1
  int lead;  // pages the last split gives up to the others
  int rot_kind, lgb;
  float scale2;   // sm_scale * log2(e)
  const __half* q;  // [S][Hq][D]
  const float* quat;
  const float* rope;  // RoPE table [rope_max_pos][D] or NULL
  int rope_max_pos;
  const int32_t* seq_lens;
  const int32_t* block_table;
  const uint8_t* k_codes;
  const uint32_t* k_params;
  const uint8_t* v_codes;
  const uint32_t* v_params;
  float* out;        // [S][Hq][D]
  float* part;       // [S][Hq][splits][D + 4]: acc[D], reference max, sum p, pad
  int32_t* err;
  // fused decode step (kvq_decode_step): the new token of each sequence, K
  // and V rows [S][H][D] binary16 (row (s, h) at s * new_stride + h * D),
  // quantized into the pools at position seq_lens[s] - 1 before attention;
  // nullptr for plain decode attention
  const __half* k_new;
  const __half* v_new;
  int64_t new_stride;
  uint8_t* k_codes_w;
  uint32_t* k_params_w;
  uint8_t* v_codes_w;
  uint32_t* v_params_w;
};

// The new token of one (sequence, KV head) (position L - 1), quantized by
// one warp exactly as kvq_quantize_append would: this lane's code bytes of
// the K and V rows (CPL / 2 of them, little-endian in the word) and the
// (scale, min) words of both rows.
struct StepRow {
  uint32_t kc, vc;
  uint32_t kp, vp;
};

// raw: the new K row then the V row (binary16, staged in shared memory)
template <int D, int ROT, int LGB>
__device__ __forceinline__ StepRow step_rows(const __half* raw, const float* quat,
                                             const float* cs, int lane) {
  constexpr int CPL = RowQuantShape<D>::CPL;
  StepRow o;
#pragma unroll 1
  for (int kv = 0; kv < 2; ++kv) {
    float x[CPL];
    row_load<D>(x, raw + kv * D + lane * CPL, true);
    if (kv == 0 && cs != nullptr) rope_regs<CPL>(x, cs + lane * CPL);
    __half s16, m16;
    const uint32_t packed = row_quantize<D, ROT, LGB>(x, lane, quat, s16, m16);
    const uint32_t word =
        (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
    if (kv) {
      o.vc = packed;
      o.vp = word;
    } else {
      o.kc = packed;
      o.kp = word;
    }
  }
  return o;
}

// cs: the RoPE table row of the token's position (NULL: no RoPE)
template <int D>
__device__ __noinline__ StepRow quantize_step_token(const __half* raw, const float* quat,
                                                    const float* cs, int rot_kind, int lgb,
                                                    int lane) {
  if (rot_kind == KVQ_ROT_NONE) return step_rows<D, KVQ_ROT_NONE, 0>(raw, quat, cs, lane);
  if (rot_kind == KVQ_ROT_QUAT) return step_rows<D, KVQ_ROT_QUAT, 0>(raw, quat, cs, lane);
  if (rot_kind == KVQ_ROT_QUAT_FAST) return step_rows<D, KVQ_ROT_QUAT_FAST, 0>(raw, quat, cs, lane);
  if (rot_kind == KVQ_ROT_QUAT_MAT) return step_rows<D, KVQ_ROT_QUAT_MAT, 0>(raw, quat, cs, lane);
  // the Hadamard rows take the sign table (randomised signs) or NULL
  if (rot_kind == KVQ_ROT_HADAMARD) quat = nullptr;
  switch (lgb) {
    case 4: return step_rows<D, KVQ_ROT_HADAMARD, 4>(raw, quat, cs, lane);
    case 5: return step_rows<D, KVQ_ROT_HADAMARD, 5>(raw, quat, cs, lane);
    case 6: return step_rows<D, KVQ_ROT_HADAMARD, 6>(raw, quat, cs, lane);
    case 7: return step_rows<D, KVQ_ROT_HADAMARD, 7>(raw, quat, cs, lane);
    default: return step_rows<D, KVQ_ROT_HADAMARD, (D >= 256 ? 8 : 7)>(raw, quat, cs, lane);
  }
}

// Stores / loads a lane's CPL / 2 code bytes (shared or global memory).
template <int D>
__device__ __forceinline__ void put_codes(uint8_t* p, uint32_t packed) {
  if (RowQuantShape<D>::CPL == 4)
    *reinterpret_cast<uint16_t*>(p) = (uint16_t)packed;
  else
    *reinterpret_cast<uint32_t*>(p) = packed;
}
template <int D>
__device__ __forceinline__ uint32_t get_codes(const uint8_t* p) {
  if (RowQuantShape<D>::CPL == 4) return *reinterpret_cast<const uint16_t*>(p);
  return *reinterpret_cast<const uint32_t*>(p);
}

// ---------------------------------------------------------------------------
// 2. split kernel
// ---------------------------------------------------------------------------

template <int D, int P, int GP>
struct DecCfg {
  static constexpr int NKS8 = D / 32;          // QK int8 k-steps over channels
  static constexpr int NQT = GP == 8 ? 2 : 1;  // 16-row tiles of query limbs
  static constexpr int NMT = D / 16;           // PV m-tiles over channels
  static constexpr int TILES = P / 16;         // 16-token tiles per page
  static constexpr int NE = GP == 8 ? 4 : 2;   // scores per lane per tile
  static constexpr int QW = D / 4;             // query channels per lane
  static constexpr int ROWB = D / 2;           // code bytes per token
  static constexpr int CODE_B = P * ROWB;      // code bytes per (page, head)
  static constexpr int PAGE_B = 2 * CODE_B + 8 * P;  // K codes, V codes, K and V params
  // pages per pipeline stage: 64 tokens at d = 128 (32 at d = 256), so a
  // stage's fixed costs (copy issue, wait, page checks) spread over 4 (2)
  // tiles whatever the page size
  static constexpr int PG = (D == 128 ? 64 : 32) / P > 1 ? (D == 128 ? 64 : 32) / P : 1;
  static constexpr int TPG = TILES * PG;             // 16-token tiles per stage
  static constexpr int STAGE_B = PG * PAGE_B;
  // pipeline depth: one stage (8.5 KB) in flight while the other computes
  static constexpr int NST = 2;
  // behind the ring, for a fused decode step: the new token's binary16 K and
  // V rows as copied in, then its K and V code rows and parameter words,
  // kept until its page is staged
  static constexpr int RAW_B = 2 * D * 2;
  static constexpr int STEP_B = (RAW_B + 2 * ROWB + 8 + 127) / 128 * 128;
  static constexpr int WARP_B = (NST * STAGE_B + STEP_B + 127) / 128 * 128;
};
// Online-softmax slack in base-2 logit units: a head's reference maximum M
// moves only when a score exceeds it by more than this, so every weight
// 2^(z - M) stays below 2^8 (binary16 weights and binary32 sums have room to
// spare) and most page groups skip the cross-lane maximum and the rescale.
constexpr float kMaxSlack = 8.f;

template <int D, int P, int GP>
__global__ void __launch_bounds__(kDecWarps * kWarp, D == 256 ? 2 : 3)
    decode_split_kernel(const DecodeArgs a) {
  static_assert(D == 128 || D == 256, "decode attention supports head_dim 128 and 256");
  using C = DecCfg<D, P, GP>;
  constexpr int NE = C::NE;
  extern __shared__ __align__(128) uint8_t smem[];
  // inputs may come from the previous kernel of the stream: nothing is read
  // before it has completed; the next launch may be scheduled right away
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int r = lane >> 2, j = lane & 3;
  const int item = blockIdx.x * kDecWarps + warp;
  // items: the first nhi (sequence, KV head) pairs with `splits` splits
  // each, then the others with splits - 1
  const int hi_items = a.nhi * a.splits;
  int pair, split, nspl;
  if (item < hi_items) {
    pair = item / a.splits;
    split = item - pair * a.splits;
    nspl = a.splits;
  } else {
    nspl = a.splits - 1;
    const int r = item - hi_items;
    const int k = nspl > 0 ? r / nspl : 0;
    pair = a.nhi + k;
    split = r - k * nspl;
  }
  if (pair >= a.S * a.H || nspl < 1) return;
  const int s = pair / a.H;
  const int h = pair - s * a.H;
  uint8_t* ring = smem + warp * C::WARP_B;

  // ---- independent loads first: the sequence length and the query rows
  const int hr = (GP == 8) ? r : (r & 3);
  const bool lo_row = (GP == 4) && (r >= 4);
  const int g = h * a.G + hr;           // global query head
  const bool head_ok = hr < a.G;
  int L = a.seq_lens[s];
  uint4 qraw[C::QW / 8];
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.q + ((int64_t)s * a.Hq + g) * D + j * C::QW);
#pragma unroll
    for (int c = 0; c < C::QW / 8; ++c) qraw[c] = head_ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
  }
  bool len_ok = L >= 0 && L <= a.max_seq_len && (L + a.P - 1) / a.P <= a.bt_stride &&
                (a.rope == nullptr || L <= a.rope_max_pos);
  if (!len_ok) {
    if (lane == 0 && h == 0 && split == 0) raise_flag(a.err, KVQ_ERRF_LEN);
    L = 0;
  }
  const int npages = (L + P - 1) / P;
  // this warp's pages: a contiguous range; the sequence's pages are dealt
  // out evenly over its splits (range sizes differ by at most one page)
  // In a fused step the last split also quantizes the new token first: it
  // takes `lead` pages fewer than an even share (as if the sequence had
  // npages + lead pages and its last ones were that work), so it does not
  // finish after the others. Plain decode attention uses the same ranges,
  // so both calls sum in the same order. Sequences with fewer than 4 pages
  // per split keep even shares. Between that and (n - 1) lead + n pages the
  // last split can come out empty: the split before it then holds the last
  // page and quantizes the new token (the owner is whichever split holds
  // that page), and every page is still in exactly one range.
  const int lead = npages >= 4 * nspl ? a.lead : 0;
  const int64_t vpages = (int64_t)npages + lead;
  const int pg_lo = split == 0 ? 0 : (int)min((int64_t)npages, (split * vpages) / nspl);
  const int pg_hi = split + 1 == nspl ? npages : (int)min((int64_t)npages, ((split + 1) * vpages) / nspl);
  const int ngrp = (pg_hi - pg_lo + C::PG - 1) / C::PG;  // stage groups
  const int32_t* const bt_row = a.block_table + (int64_t)s * a.bt_stride;
  // fused step: the warp whose range holds the page of position L - 1
  // quantizes the sequence's new token for this KV head (after its first
  // copies are in flight, below), writes it to the pools and patches it into
  // the staged copy of that page, so no fence or global round trip stands
  // between the write and the attention that reads it
  const int new_pg = L >= 1 ? (L - 1) / P : -1;
  const bool step_owner = a.k_new != nullptr && new_pg >= pg_lo && new_pg < pg_hi;
  int new_grp = -1;  // group of the new token's page (-1: none to patch)
  // its inputs go out before this warp's (and ahead of most warps') page
  // copies, so they do not queue behind the page traffic: the two binary16
  // rows by cp.async into the stash behind the ring (part of the first
  // commit group), the block-table entry into a register
  uint8_t* const stash = ring + C::NST * C::STAGE_B;  // [K, V raw rows][K, V codes][params]
  int step_page = -1;
  if (step_owner) {
    step_page = bt_row[new_pg];
    const int64_t src = (int64_t)s * a.new_stride + (int64_t)h * D;
    constexpr int LB = D / 16;  // raw bytes per lane and row: 8 (d 128) or 16 (d 256)
    if (LB == 16) {
      cp_async16(stash + lane * 16, a.k_new + src + lane * 8);
      cp_async16(stash + 2 * D + lane * 16, a.v_new + src + lane * 8);
    } else {
      cp_async8(stash + lane * 8, a.k_new + src + lane * 4);
      cp_async8(stash + 2 * D + lane * 8, a.v_new + src + lane * 4);
    }
  }
  // The warp's block-table entries sit in lane registers, 32 pages at a
  // time: lane i holds the entry of page pg_lo + 32 c + i of chunk c. An
  // entry outside [0, NP) raises KVQ_ERRF_PAGE when it is loaded and its page
  // is skipped; -1 marks a skipped page or one past the range.
  const int npg = pg_hi - pg_lo;  // pages of this warp
  auto load_ids = [&](int c) {
    const int pi = 32 * c + lane;
    int id = -1;
    if (pi < npg) {
      id = bt_row[pg_lo + pi];
      if (id < 0 || id >= a.NP) {
        raise_flag(a.err, KVQ_ERRF_PAGE);
        id = -1;
      }
    }
    return id;
  };

  // ---- page ring: the warp stages each (page, head) chunk (K codes, V
  // codes, K params, V params, all contiguous in their pools) with 16-byte
  // cp.async copies, linear in shared memory: 16-byte unit u of a page block
  // is copied by lane u % 32. One commit group per stage of PG pages.
  constexpr int KU = C::CODE_B / 16;  // units of codes per pool (a multiple of 32)
  constexpr int PU = P / 4;           // units of params per pool (<= 16)
  static_assert(KU % kWarp == 0 && 2 * PU <= kWarp, "page block does not tile the warp");
  // page strides of the code and parameter pools (H * 8 KB at most: 32-bit
  // products, widened once into the 64-bit address)
  const uint32_t cstride = (uint32_t)a.H * C::CODE_B, pstride = (uint32_t)a.H * P * 4;
  const uint8_t* const kc_l = a.k_codes + (int64_t)h * C::CODE_B + lane * 16;
  const uint8_t* const vc_l = a.v_codes + (int64_t)h * C::CODE_B + lane * 16;
  const uint8_t* const par_l =
      lane < PU ? reinterpret_cast<const uint8_t*>(a.k_params) + (int64_t)h * P * 4 + lane * 16
                : reinterpret_cast<const uint8_t*>(a.v_params) + (int64_t)h * P * 4 + (lane - PU) * 16;
  // ids_a holds chunk cidx of the entries, ids_b the next chunk (loaded 32
  // pages ahead of its use); okbits bit (slot * PG + q): page q of the group
  // in ring slot `slot` was copied
  int cidx = 0;
  int ids_a = load_ids(0), ids_b = load_ids(1);
  uint32_t okbits = 0;
  // copy group gn into ring slot `slot` (one commit group per call)
  auto issue = [&](int gn, int slot) {
    if ((gn * C::PG) >> 5 != cidx) {  // the group starts the next chunk
      ids_a = ids_b;
      ++cidx;
      ids_b = load_ids(cidx + 1);
    }
    // a page past the range or skipped (id < 0) is not read: its copies
    // zero-fill from page 0's address and its okbits bit stays clear (no
    // branch, so no divergence bookkeeping for a warp-uniform condition)
    uint32_t okm = 0;
#pragma unroll
    for (int q = 0; q < C::PG; ++q) {
      const int id = __shfl_sync(0xffffffffu, ids_a, (gn * C::PG + q) & 31);
      const bool ok = id >= 0;
      okm |= (uint32_t)ok << q;
      const uint32_t idc = ok ? (uint32_t)id : 0u;
      const uint32_t nb = ok ? 16u : 0u;
      const uint64_t co = (uint64_t)idc * cstride;
      uint8_t* dst = ring + slot * C::STAGE_B + q * C::PAGE_B + lane * 16;
#pragma unroll
      for (int m = 0; m < KU / kWarp; ++m) cp_async16_zf(dst + m * 512, kc_l + co + m * 512, nb);
#pragma unroll
      for (int m = 0; m < KU / kWarp; ++m)
        cp_async16_zf(dst + C::CODE_B + m * 512, vc_l + co + m * 512, nb);
      if (lane < 2 * PU)
        cp_async16_zf(dst + 2 * C::CODE_B, par_l + (uint64_t)idc * pstride, nb);
    }
    okbits = (okbits & ~(((1u << C::PG) - 1) << (slot * C::PG))) | (okm << (slot * C::PG));
    cp_async_commit();
  };

  // Tokens of a 16-token tile are visited in the order
  //   pi(8h + n) = 8h + (n ^ ((n >> 1) & 1))      (n < 8)
  // in both products: QK column n of half h is token pi(8h + n), and the PV
  // k index 2j + c (+ 8h) is the same token. The swap of the pair members for
  // odd j makes the four lanes j of a V fragment load alternate between the
  // two 64-byte halves of a 128-byte line (no bank conflicts without a
  // swizzle).
  const int tk_r = r ^ ((r >> 1) & 1);        // K row of lane r within a half
  int tk_e[4];                                 // token of score / PV slot e
#pragma unroll
  for (int e = 0; e < 4; ++e) tk_e[e] = 8 * (e >> 1) + 2 * j + ((e & 1) ^ (j & 1));
  constexpr int VB = D == 128 ? 8 : 16;        // V bytes per lane per token
  // byte offsets inside a stage (tile 0; tile tt adds 16 tt rows)
  int k_ld[2], v_ld[4], kp_ld[4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) k_ld[nt] = (8 * nt + tk_r) * C::ROWB + j * 16 * (D / 128);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v_ld[e] = C::CODE_B + tk_e[e] * C::ROWB + r * VB;
    kp_ld[e] = 2 * C::CODE_B + tk_e[e] * 4;
  }
  const int own = lo_row ? 1 : 0;  // GP = 4: token half of this lane
  int kps[NE], tks[NE];            // K-param offset and token of score e
#pragma unroll
  for (int e = 0; e < NE; ++e) {
    kps[e] = GP == 8 ? kp_ld[e] : (own ? kp_ld[2 + e] : kp_ld[e]);
    tks[e] = GP == 8 ? tk_e[e] : (own ? tk_e[2 + e] : tk_e[e]);
  }

  // ---- state: PV accumulators (rows = channels, columns = query heads;
  // GP = 4 keeps the hi and lo weight columns apart until the end), the
  // head's reference maximum and this lane's shares of the sums
  float acc[C::NMT][4];
#pragma unroll
  for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
  float M = -INFINITY;  // reference maximum (base-2 scaled scores) of head hr
  float Lp = 0.f;       // this lane's share of sum p
  float Op = 0.f;       // this lane's share of sum p (m_v + 8 s_v)
  // GP = 8: lane (r, j) scores head r with the tokens of slots e = 0..3;
  // GP = 4: lanes r and r + 4 share head r % 4 and split those slots,
  // {0, 1} for r < 4 and {2, 3} for r >= 4

  // the first NST - 1 groups are copied now
#pragma unroll
  for (int k = 0; k < C::NST - 1; ++k) {
    if (k < ngrp)
      issue(k, k);
    else
      cp_async_commit();
  }
  if (step_owner) {
    // the new token's rows came in the first commit group: wait for that
    // group alone, quantize the rows, write them to the pools and keep the
    // codes for the patch of the staged page
    cp_async_wait<C::NST - 2>();
    __syncwarp();
    if (step_page >= 0 && step_page < a.NP) {
      const StepRow nr = quantize_step_token<D>(
          reinterpret_cast<const __half*>(stash), a.quat,
          a.rope != nullptr ? a.rope + (int64_t)(L - 1) * D : nullptr, a.rot_kind, a.lgb, lane);
      const int64_t row = ((int64_t)step_page * a.H + h) * P + (L - 1) % P;
      constexpr int LB = RowQuantShape<D>::CPL / 2;  // code bytes per lane
      uint8_t* const cst = stash + C::RAW_B;
      put_codes<D>(a.k_codes_w + row * (D / 2) + lane * LB, nr.kc);
      put_codes<D>(a.v_codes_w + row * (D / 2) + lane * LB, nr.vc);
      put_codes<D>(cst + lane * LB, nr.kc);
      put_codes<D>(cst + C::ROWB + lane * LB, nr.vc);
      if (lane == 0) {
        a.k_params_w[row] = nr.kp;
        a.v_params_w[row] = nr.vp;
        *reinterpret_cast<uint2*>(cst + 2 * C::ROWB) = make_uint2(nr.kp, nr.vp);
      }
      new_grp = (new_pg - pg_lo) / C::PG;
      __syncwarp();
    } else if (lane == 0) {
      raise_flag(a.err, KVQ_ERRF_PAGE);
    }
  }

  // ---- the query, while the first pages are in flight: rotated, then held
  // as a 26-bit fixed point qint = RN(qhat * 2^k) (2^k the power of two that
  // brings the head's largest |qhat| just below 2^26, so qhat * 2^k is exact
  // in binary32) and split into four signed 8-bit limbs for the int8 tensor
  // cores. The code byte of channels (e, o) = (2i, 2i + 1) enters twice,
  // masked to c_e against 16 qint_e - qint_o and whole (c_e + 16 c_o, never
  // shifted) against qint_o, so the contraction gives 16 sum_i c_i qint_i
  // exactly with one AND per word of codes.
  // score z = (s_k zs) dot_c + (m_k + 8 s_k) zq in base-2 logit units, with
  // dot_c = 16 sum_i (c_i - 8) qint_i = dot' - 128 qsum: centred codes keep
  // both terms near the score's own size instead of two large ones that
  // cancel. 128 qsum = QA * 2^16 + QB (0 <= QB < 2^16) comes off the limb
  // halves before they are combined.
  float zs, zq, zq8, zA, zB;
  int QA, QB;
  // A fragments per k-step kk: the lane's 8 channels j*QW + 8kk + [0, 8),
  // even ones in a[0]/a[1], odd ones in a[2]/a[3]. Rows:
  //   GP = 4: rows 0-3 l3, 4-7 l1, 8-11 l2, 12-15 l0 of heads 0-3;
  //   GP = 8: tile 0 rows 0-7 l3, 8-15 l2; tile 1 rows 0-7 l1, 8-15 l0.
  uint32_t qa[C::NQT][C::NKS8][4];
  {
    float x[C::QW];
#pragma unroll
    for (int c = 0; c < C::QW / 8; ++c) {
      const uint4 u = qraw[c];
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(u32_as_h2(w4[e]));
        x[8 * c + 2 * e] = f.x;
        x[8 * c + 2 * e + 1] = f.y;
      }
    }
    // the query's RoPE at its own position L - 1, in front of the rotation
    if (a.rope != nullptr && L >= 1) rope_regs<C::QW>(x, a.rope + (int64_t)(L - 1) * D + j * C::QW);
    rotate_quarter<C::QW>(x, j, a.rot_kind, a.lgb, a.quat);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < C::QW; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int ebits = (__float_as_int(amax) >> 23) & 0xFF;  // amax < 2^(ebits - 126)
    int k = 26 - (ebits - 126);
    k = k > 126 ? 126 : k;
    const float mulf = amax > 0.f ? __int_as_float((k + 127) << 23) : 0.f;
    const float zk = a.scale2 * __int_as_float((127 - k) << 23);  // sm_scale log2(e) 2^-k
    long long qs_l = 0;
#pragma unroll
    for (int kk = 0; kk < C::NKS8; ++kk) {
      // limbs of the lane's 8 channels: with t = q + 0x808080 (128 added to
      // each of the three low bytes), q = sum_k (T_k - 128 [k < 3]) 256^k for
      // the bytes T_k of t, so the signed limbs are the bytes of
      // t ^ 0x00808080, byte k = limb k (|q| <= 2^30 keeps the top limb in s8)
      int qi[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        qi[c] = __float2int_rn(x[8 * kk + c] * mulf);
        qs_l += qi[c];
      }
      // the K operand of an even slot is its byte's low nibble c_e, of an odd
      // slot the whole byte c_e + 16 c_o: with 16 q_e - q_o against the first
      // and q_o against the second, c_e q_o cancels and the pair contributes
      // 16 (c_e q_e + c_o q_o) (|16 q_e - q_o| < 17 * 2^26 stays in 4 limbs)
      uint32_t u[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int qe = (c & 1) ? qi[c] : 16 * qi[c] - qi[c + 1];
        u[c] = (uint32_t)(qe + 0x808080) ^ 0x00808080u;
      }
      // limb `lb` (0 = lowest) of channels {o, o+2, o+4, o+6} as one s8x4 word
      auto pk4 = [&](int o, int lb) {
        const uint32_t lo = __byte_perm(u[o], u[o + 2], (lb) | ((4 + lb) << 4));
        const uint32_t hi = __byte_perm(u[o + 4], u[o + 6], (lb) | ((4 + lb) << 4));
        return __byte_perm(lo, hi, 0x5410);
      };
      if (GP == 8) {
        qa[0][kk][0] = pk4(0, 3);
        qa[0][kk][1] = pk4(0, 2);
        qa[0][kk][2] = pk4(1, 3);
        qa[0][kk][3] = pk4(1, 2);
        qa[C::NQT - 1][kk][0] = pk4(0, 1);
        qa[C::NQT - 1][kk][1] = pk4(0, 0);
        qa[C::NQT - 1][kk][2] = pk4(1, 1);
        qa[C::NQT - 1][kk][3] = pk4(1, 0);
      } else {
        // row r: l3 (r < 4) or l1 (r >= 4); row r + 8: l2 (r < 4) or l0
        qa[0][kk][0] = lo_row ? pk4(0, 1) : pk4(0, 3);
        qa[0][kk][2] = lo_row ? pk4(1, 1) : pk4(1, 3);
        qa[0][kk][1] = lo_row ? pk4(0, 0) : pk4(0, 2);
        qa[0][kk][3] = lo_row ? pk4(1, 0) : pk4(1, 2);
      }
    }
    qs_l += __shfl_xor_sync(0xffffffffu, qs_l, 1);
    qs_l += __shfl_xor_sync(0xffffffffu, qs_l, 2);
    zs = zk * 0.0625f;          // exact: the factor 16 of dot'
    zq = zk * (float)qs_l;      // sum of qint over the head's channels
    zq8 = 8.f * zq;             // exact
    // weights of the two halves of dot_c; for GP = 4 a lane's own half is
    // the high one (r < 4) or the low one (r >= 4)
    const float zhi = zs * 65536.f, zlo = zs;
    zA = (GP == 4 && lo_row) ? zlo : zhi;
    zB = (GP == 4 && lo_row) ? zhi : zlo;
    const long long q128 = qs_l * 128;  // |qsum| < 2^26 d: no overflow
    QA = (int)(q128 >> 16);             // floor division
    QB = (int)(q128 - ((long long)QA << 16));
  }

  int slot = 0;               // ring slot of group gi
  int slot_n = C::NST - 1;    // ring slot of group gi + NST - 1
  for (int gi = 0; gi < ngrp; ++gi) {
    if (gi + C::NST - 1 < ngrp)
      issue(gi + C::NST - 1, slot_n);
    else
      cp_async_commit();
    slot_n = slot_n + 1 == C::NST ? 0 : slot_n + 1;
    cp_async_wait<C::NST - 1>();  // this lane's copies of group gi have landed
    __syncwarp();                 // ... and every other lane's
    bool pgok[C::PG];             // page q of the group was copied
    bool all_ok = true;
#pragma unroll
    for (int q = 0; q < C::PG; ++q) {
      pgok[q] = (okbits >> (slot * C::PG + q)) & 1u;
      all_ok = all_ok && pgok[q];
    }
    uint8_t* const st = ring + slot * C::STAGE_B;
    slot = slot + 1 == C::NST ? 0 : slot + 1;
    if (gi == new_grp) {
      // the staged page may predate this launch's write of the new token:
      // its rows and parameters are replaced by the stashed values (each
      // lane copies the bytes it stashed)
      constexpr int LB = RowQuantShape<D>::CPL / 2;
      uint8_t* const pb = st + ((new_pg - pg_lo) % C::PG) * C::PAGE_B;
      const int sl = (L - 1) % P;
      const uint8_t* const cst = stash + C::RAW_B;
      put_codes<D>(pb + sl * C::ROWB + lane * LB, get_codes<D>(cst + lane * LB));
      put_codes<D>(pb + C::CODE_B + sl * C::ROWB + lane * LB, get_codes<D>(cst + C::ROWB + lane * LB));
      if (lane == 0) {
        const uint2 pw = *reinterpret_cast<const uint2*>(cst + 2 * C::ROWB);
        *reinterpret_cast<uint32_t*>(pb + 2 * C::CODE_B + sl * 4) = pw.x;
        *reinterpret_cast<uint32_t*>(pb + 2 * C::CODE_B + P * 4 + sl * 4) = pw.y;
      }
      __syncwarp();
    }
    const int tok0 = (pg_lo + gi * C::PG) * P;  // first token of the group
    // groups whose every token is cached skip all per-token masking
    const bool full = all_ok && tok0 + C::PG * P <= L;

    auto body = [&](auto masked_tag) {
      constexpr bool MASKED = decltype(masked_tag)::value;
      // ---- QK and scores of every tile (tiles of a skipped page: -inf)
      float z[C::TPG][NE];
#pragma unroll
      for (int tt = 0; tt < C::TPG; ++tt) {
        if (MASKED && !pgok[tt / C::TILES]) {
#pragma unroll
          for (int e = 0; e < NE; ++e) z[tt][e] = -INFINITY;
          continue;
        }
        // tile tt of the group: page tt / TILES, 16-token tile tt % TILES
        const int cofs = (tt / C::TILES) * C::PAGE_B + (tt % C::TILES) * 16 * C::ROWB;
        const int pofs = (tt / C::TILES) * C::PAGE_B + (tt % C::TILES) * 64;
        int ci[C::NQT][2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t w[D / 32];
#pragma unroll
          for (int u = 0; u < D / 128; ++u) {
            const uint4 v4 = *reinterpret_cast<const uint4*>(st + k_ld[nt] + cofs + 16 * u);
            w[4 * u] = v4.x; w[4 * u + 1] = v4.y; w[4 * u + 2] = v4.z; w[4 * u + 3] = v4.w;
          }
#pragma unroll
          for (int kk = 0; kk < C::NKS8; ++kk) {
            const uint32_t b0 = w[kk] & 0x0F0F0F0Fu;  // even slots: c_e
#pragma unroll
            for (int t = 0; t < C::NQT; ++t) {
              if (kk == 0)
                mma16832_s8u8_z(ci[t][nt], qa[t][kk], b0, w[kk]);
              else
                mma16832_s8u8(ci[t][nt], qa[t][kk], b0, w[kk]);
            }
          }
        }
        // dot' = 16 sum_i c_i qint_i of head hr with each of the lane's
        // tokens: the limb dots combine as (l3*256 + l2) * 2^16 + (l1*256 + l0)
        // halves of dot_c: hA = l3*256 + l2 - QA and hB = l1*256 + l0 - QB
        // (|.| < 2^31), weighted in binary32 by zA = 2^16 zs and zB = zs
        float fA[NE], fB[NE];
        if (GP == 8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int nt = e >> 1, c = e & 1;
            fA[e] = (float)(ci[0][nt][c] * 256 + (ci[0][nt][2 + c] - QA));
            fB[e] = (float)(ci[C::NQT - 1][nt][c] * 256 + (ci[C::NQT - 1][nt][2 + c] - QB));
          }
        } else {
          // lanes r < 4 hold the (l3, l2) rows and form hA, lanes r + 4 the
          // (l1, l0) rows and form hB, for both token halves; each sends its
          // partner the half that partner scores (zA, zB swap with the role)
          const int Qh = lo_row ? QB : QA;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int loc0 = ci[0][0][c] * 256 + (ci[0][0][2 + c] - Qh);
            const int loc1 = ci[0][1][c] * 256 + (ci[0][1][2 + c] - Qh);
            const int got = __shfl_xor_sync(0xffffffffu, lo_row ? loc0 : loc1, 16);
            fA[c] = (float)(lo_row ? loc1 : loc0);  // this lane's own half
            fB[c] = (float)got;
          }
        }
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          // zs dot_c + 8 zq, then z = s (zs dot_c + 8 zq) + m zq
          const float zd = fmaf(fA[e], zA, fmaf(fB[e], zB, zq8));
          const uint32_t kpw = *reinterpret_cast<const uint32_t*>(st + kps[e] + pofs);
          const float2 sm = __half22float2(u32_as_h2(kpw));  // (scale, min)
          const float sc = fmaf(sm.x, zd, sm.y * zq);
          if (MASKED) {
            const int tok = tok0 + (tt / C::TILES) * P + (tt % C::TILES) * 16 + tks[e];
            z[tt][e] = tok < L ? sc : -INFINITY;
          } else {
            z[tt][e] = sc;
          }
        }
      }

      // ---- online softmax: move head hr's reference maximum only when a
      // score of the group exceeds it by more than kMaxSlack (warp-uniform)
      float mloc = -INFINITY;
#pragma unroll
      for (int tt = 0; tt < C::TPG; ++tt)
#pragma unroll
        for (int e = 0; e < NE; ++e) mloc = fmaxf(mloc, z[tt][e]);
      if (__any_sync(0xffffffffu, mloc > M + kMaxSlack)) {
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
        if (GP == 4) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 16));
        const float Mn = fmaxf(M, mloc);
        const float alpha = (Mn == M) ? 1.f : fast_exp2(M - Mn);  // M = -inf: 0
        M = Mn;
        Lp *= alpha;
        Op *= alpha;
        // lane (r, j) holds columns of heads c0 = 2(j & (GP/2 - 1)), c0 + 1:
        // their factors from lanes r = c0, c0 + 1
        const int c0 = (GP == 8) ? 2 * j : 2 * (j & 1);
        const float a0 = __shfl_sync(0xffffffffu, alpha, 4 * c0);
        const float a1 = __shfl_sync(0xffffffffu, alpha, 4 * c0 + 4);
#pragma unroll
        for (int mt = 0; mt < C::NMT; ++mt) {
          acc[mt][0] *= a0; acc[mt][1] *= a1;
          acc[mt][2] *= a0; acc[mt][3] *= a1;
        }
      }

      // ---- PV per tile, summed over the stage's tiles in the tensor core
      // from zero (the first tile's product writes the stage sum; a masked
      // stage, whose first tile may be skipped, starts from explicit zeros)
      // and then added to the running sum with one round-to-nearest add: the
      // tensor core truncates each product sum against its accumulator, so
      // the bias of a chain grows with its length, and a chain is kept to
      // one stage whatever the length of the split. At d = 256 (no registers
      // for a second set of sums) each tile's product is added on its own.
      constexpr bool SSUM = D == 128;
      float t4[C::NMT][4];
      if (SSUM && MASKED) {
#pragma unroll
        for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) t4[mt][e] = 0.f;
      }
#pragma unroll
      for (int tt = 0; tt < C::TPG; ++tt) {
        if (MASKED && !pgok[tt / C::TILES]) continue;
        const int cofs = (tt / C::TILES) * C::PAGE_B + (tt % C::TILES) * 16 * C::ROWB;
        const int pofs = (tt / C::TILES) * C::PAGE_B + (tt % C::TILES) * 64;
        float wv[NE];
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          const uint32_t vpw = *reinterpret_cast<const uint32_t*>(st + kps[e] + P * 4 + pofs);
          const float2 sm = __half22float2(u32_as_h2(vpw));  // (scale, min)
          // masked tokens may sit on stale or never-written shared memory:
          // their terms are forced to exact zeros rather than p * (params)
          const bool live = !MASKED || z[tt][e] != -INFINITY;
          const float p = live ? fast_exp2(z[tt][e] - M) : 0.f;
          Lp += p;
          Op = live ? fmaf(p, fmaf(8.f, sm.x, sm.y), Op) : Op;  // p (m_v + 8 s_v)
          wv[e] = live ? p * sm.x : 0.f;
        }
        // weights p * s as binary16 hi + lo pairs: hi = RN16(w), lo = RN16(w - hi)
        uint32_t bh[2], bl[2];
        if (GP == 8) {
          const __half2 h01 = __floats2half2_rn(wv[0], wv[1]);
          const __half2 h23 = __floats2half2_rn(wv[NE - 2], wv[NE - 1]);
          const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
          bh[0] = h2_as_u32(h01);
          bh[1] = h2_as_u32(h23);
          bl[0] = h2_as_u32(__floats2half2_rn(wv[0] - f01.x, wv[1] - f01.y));
          bl[1] = h2_as_u32(__floats2half2_rn(wv[NE - 2] - f23.x, wv[NE - 1] - f23.y));
        } else {
          // column r < 4 = hi of head r, r >= 4 = lo of head r - 4: lane r
          // keeps hi (or lo) of its own token half and takes the other
          // half's from its partner r ^ 4
          const __half2 ho = __floats2half2_rn(wv[0], wv[1]);
          const float2 fo = __half22float2(ho);
          const uint32_t hi_own = h2_as_u32(ho);
          const uint32_t lo_own = h2_as_u32(__floats2half2_rn(wv[0] - fo.x, wv[1] - fo.y));
          const uint32_t got = __shfl_xor_sync(0xffffffffu, lo_row ? hi_own : lo_own, 16);
          bh[0] = lo_row ? got : hi_own;  // slots 0, 1
          bh[1] = lo_row ? lo_own : got;  // slots 2, 3
          bl[0] = bl[1] = 0u;
        }
        // (columns of padding heads, hr >= G, carry weights of a zero query;
        // they never mix with other columns and are never written)
        // A operand: V codes of the slots' tokens, channels of lane row r:
        // [r*D/8, (r+1)*D/8)
        constexpr int WPT = D / 64;  // 32-bit words per token per lane
        uint32_t vw[4][WPT];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint8_t* src = st + v_ld[e] + cofs;
          if (D == 128) {
            const uint2 v2 = *reinterpret_cast<const uint2*>(src);
            vw[e][0] = v2.x; vw[e][1] = v2.y;
          } else {
            const uint4 v4 = *reinterpret_cast<const uint4*>(src);
            vw[e][0] = v4.x; vw[e][1] = v4.y; vw[e][2] = v4.z; vw[e][3] = v4.w;
          }
        }
        // Each code enters the f16 tensor core as c - 8, exact in binary16:
        // the nibble is OR-ed into the mantissa of 1024 (one three-input
        // logic operation on a masked word; nibbles in bits 4-7 land at
        // 1024 + 16 c) and the bias comes off with one half2 subtract
        // (1024 + c - 1032) or fused multiply-add ((1024 + 16 c) / 16 - 72).
        // (Subnormal operands without a bias would save that operation, but
        // the tensor core does not keep their products exact.) Token pairs
        // are interleaved first (bytes of tokens 2j and 2j+1 side by side),
        // so one operation yields the half2 of a channel for both tokens of
        // a k pair. m-tile mt: group gq = mt / 8 (words 2gq, 2gq+1), channel
        // e8 = mt % 8 of the word's 8 (byte e8 / 2, nibble e8 % 2); row slot
        // r <- word 2gq, slot r+8 <- word 2gq+1.
#pragma unroll
        for (int gq = 0; gq < WPT / 2; ++gq)
#pragma unroll
          for (int bsel = 0; bsel < 2; ++bsel) {
          // bytes 2 bsel, 2 bsel + 1 of the group's words, token pairs interleaved
          uint32_t pr[2][2][2];  // [slot pair][word in group][shifted]
#pragma unroll
          for (int tp = 0; tp < 2; ++tp)
#pragma unroll
            for (int wi = 0; wi < 2; ++wi) {
              const int wd = 2 * gq + wi;
              const uint32_t X = vw[2 * tp][wd], Y = vw[2 * tp + 1][wd];
              pr[tp][wi][0] = __byte_perm(X, Y, bsel ? 0x7632 : 0x5410);
              pr[tp][wi][1] = pr[tp][wi][0] >> 8;
            }
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const int e8 = 4 * bsel + e4;
            const int mt = gq * 8 + e8;
            const int sh = (e8 >> 1) & 1;
            const uint32_t mask = (e8 & 1) ? 0x00F000F0u : 0x000F000Fu;
            uint32_t av[4];
            av[0] = nib_c8(pr[0][0][sh], mask, e8 & 1);  // row slot r,   k slots 0, 1
            av[1] = nib_c8(pr[0][1][sh], mask, e8 & 1);  // row slot r+8, k slots 0, 1
            av[2] = nib_c8(pr[1][0][sh], mask, e8 & 1);  // row slot r,   k slots 2, 3
            av[3] = nib_c8(pr[1][1][sh], mask, e8 & 1);  // row slot r+8, k slots 2, 3
            if (SSUM) {
              if (!MASKED && tt == 0)
                mma16816_z(t4[mt], av, bh[0], bh[1]);
              else
                mma16816(t4[mt], av, bh[0], bh[1]);
              if (GP == 8) mma16816(t4[mt], av, bl[0], bl[1]);
            } else {
              float u4[4];
              mma16816_z(u4, av, bh[0], bh[1]);
              if (GP == 8) mma16816(u4, av, bl[0], bl[1]);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[mt][e] += u4[e];
            }
          }
        }
      }
      if (SSUM) {
#pragma unroll
        for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][e] += t4[mt][e];
      }
    };
    if (full)
      body(std::false_type{});
    else
      body(std::true_type{});
    __syncwarp();  // every lane is done with the stage before it is refilled
  }
  cp_async_wait<0>();

  // ---- partial results: per channel acc + sum p (m + 8 s), the reference
  // maximum M and sum p
  Lp += __shfl_xor_sync(0xffffffffu, Lp, 1);
  Lp += __shfl_xor_sync(0xffffffffu, Lp, 2);
  Op += __shfl_xor_sync(0xffffffffu, Op, 1);
  Op += __shfl_xor_sync(0xffffffffu, Op, 2);
  if (GP == 4) {  // the two token halves of head hr
    Lp += __shfl_xor_sync(0xffffffffu, Lp, 16);
    Op += __shfl_xor_sync(0xffffffffu, Op, 16);
    // fold the lo columns (lanes j = 2, 3) onto the hi columns (j = 0, 1)
#pragma unroll
    for (int mt = 0; mt < C::NMT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] += __shfl_xor_sync(0xffffffffu, acc[mt][e], 2);
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
    // lane row r holds channels [r*D/8, (r+1)*D/8) of head gh: m-tile mt,
    // row slot r <- channel r*D/8 + 16*(mt/8) + mt%8, row slot r+8 <- that
    // channel + 8
    float4* dst = reinterpret_cast<float4*>(a.part + (base + (int64_t)gh * a.splits) * (D + 4) +
                                            r * (D / 8));
    const float ov = hc ? o1 : o0;
#pragma unroll
    for (int gq = 0; gq < D / 128; ++gq)
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int q4 = 0; q4 < 2; ++q4) {
          const int mt = 8 * gq + 4 * q4;
          const int e = 2 * half + hc;
          dst[4 * gq + 2 * half + q4] = make_float4(acc[mt][e] + ov, acc[mt + 1][e] + ov,
                                                    acc[mt + 2][e] + ov, acc[mt + 3][e] + ov);
        }
  }
  // the lanes that own head hr's softmax state write it (one lane per head)
  if (j == 0 && !lo_row && head_ok) {
    float* dst = a.part + (base + (int64_t)hr * a.splits) * (D + 4);
    *reinterpret_cast<float2*>(dst + D) = make_float2(M, Lp);
  }
}

// ---------------------------------------------------------------------------
// 3. merge kernel: one warp per (sequence, query head), launched after the
// split kernel with programmatic serialization (its blocks wait for every
// split's partial result). Lane l owns channels [l*CPL, (l+1)*CPL). The
// splits' (acc, M, L) are combined in rounds of RB with a running maximum
// (log-sum-exp), normalised by the total weight, rotated back by R^-1 and
// written as the float32 output.
// ---------------------------------------------------------------------------

struct MergeArgs {
  int S, Hq, G, splits, nhi, rot_kind, lgb;
  const float* quat;
  const float* part;  // [S][Hq][splits][D + 4]
  float* out;         // [S][Hq][D]
};

// R^-1 of a row held as CPL consecutive channels per lane over the 32 lanes
// (the inverse of the block Hadamard rotation is the rotation itself, after
// it the sign flip when there is one; the quaternion maps are inverted block
// by block). Binary32, not part of the
// bit-exact quantize path.
template <int CPL>
__device__ __forceinline__ void row_unrotate(float (&x)[CPL], int lane, int rot_kind, int lgb,
                                             const float* quat) {
  if (rot_kind == KVQ_ROT_HADAMARD || rot_kind == KVQ_ROT_HADAMARD_SIGNED) {
    const int b = 1 << lgb;
#pragma unroll
    for (int dd = 1; dd < CPL; dd <<= 1) {
      if (dd >= b) break;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        if ((i & dd) == 0) {
          const float p = x[i], q = x[i + dd];
          x[i] = p + q;
          x[i + dd] = p - q;
        }
      }
    }
    for (int m = 1; m * CPL < b; m <<= 1) {
      const bool lower = (lane & m) == 0;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, x[i], m);
        x[i] = lower ? x[i] + o : o - x[i];
      }
    }
    const float cb = hadamard_scale(lgb);
#pragma unroll
    for (int i = 0; i < CPL; ++i) x[i] *= cb;
    // R = H S with the sign diagonal S: R^-1 = S H
    if (rot_kind == KVQ_ROT_HADAMARD_SIGNED) sign_regs<CPL>(x, quat + lane * CPL);
  } else if (rot_kind == KVQ_ROT_QUAT) {
    quat_inv_regs<CPL>(x, quat, lane * CPL);
  } else if (rot_kind == KVQ_ROT_QUAT_FAST) {
    quat_fast_inv_regs<CPL>(x, quat, lane * CPL);
  } else if (rot_kind == KVQ_ROT_QUAT_MAT) {
    quat_mat_fly_regs<CPL, true>(x, quat, lane * CPL);
  }
}

template <int D>
__global__ void __launch_bounds__(kDecWarps * kWarp) decode_merge_kernel(const MergeArgs m) {
  constexpr int CPL = D / 32;              // channels per lane
  constexpr int RB = CPL == 4 ? 16 : 8;    // splits per round
  pdl_wait();  // every partial result of the split kernel is written
  pdl_trigger();
  const int lane = threadIdx.x % kWarp;
  const int gw = blockIdx.x * kDecWarps + threadIdx.x / kWarp;
  if (gw >= m.S * m.Hq) return;
  const float* src = m.part + (int64_t)gw * m.splits * (D + 4);
  // the query head's (sequence, KV head) pair and its number of splits
  const int nspl = gw / m.G < m.nhi ? m.splits : m.splits - 1;
  float Mr = -INFINITY, Ls = 0.f;
  float x[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) x[c] = 0.f;
  for (int i0 = 0; i0 < nspl; i0 += RB) {
    float4 f[RB][CPL / 4];
    float2 ml[RB];  // (M, L) of each split
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
      const int i = i0 + rb;
      const float* pi = src + (int64_t)i * (D + 4);
      const bool in = i < nspl;
      ml[rb] = in ? __ldcg(reinterpret_cast<const float2*>(pi + D)) : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int c = 0; c < CPL / 4; ++c)
        f[rb][c] = in ? __ldcg(reinterpret_cast<const float4*>(pi + lane * CPL) + c)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float Mc = Mr;
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) Mc = fmaxf(Mc, ml[rb].x);
    if (Mc != Mr) {  // rescale what is summed so far (Mr = -inf: nothing yet)
      const float sc = Mr == -INFINITY ? 0.f : fast_exp2(Mr - Mc);
      Ls *= sc;
#pragma unroll
      for (int c = 0; c < CPL; ++c) x[c] *= sc;
      Mr = Mc;
    }
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
      // an empty split (max -inf) has a zero row and a zero sum: weight 0
      const float wgt = ml[rb].x == -INFINITY ? 0.f : fast_exp2(ml[rb].x - Mr);
      Ls = fmaf(wgt, ml[rb].y, Ls);
#pragma unroll
      for (int c = 0; c < CPL / 4; ++c) {
        x[4 * c] = fmaf(wgt, f[rb][c].x, x[4 * c]);
        x[4 * c + 1] = fmaf(wgt, f[rb][c].y, x[4 * c + 1]);
        x[4 * c + 2] = fmaf(wgt, f[rb][c].z, x[4 * c + 2]);
        x[4 * c + 3] = fmaf(wgt, f[rb][c].w, x[4 * c + 3]);
      }
    }
  }
  const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll
  for (int c = 0; c < CPL; ++c) x[c] *= inv;
  row_unrotate<CPL>(x, lane, m.rot_kind, m.lgb, m.quat);
  float4* dst = reinterpret_cast<float4*>(m.out + (int64_t)gw * D + lane * CPL);
#pragma unroll
  for (int c = 0; c < CPL / 4; ++c)
    dst[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
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

DecodePlan decode_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len) {
  if (d.format == KVQ_FMT_MXFP4) return decode_mx_plan(d, S, Hq, max_seq_len);
  if (d.format != KVQ_FMT_INT4) return decode_gen_plan(d, S, Hq, max_seq_len);
  DecodePlan pl{};
  const int P = d.page_size;
  pl.pages_max = (max_seq_len + P - 1) / P;
  if (pl.pages_max < 1) pl.pages_max = 1;
  const int G = Hq / d.num_kv_heads;
  const int GP = G <= 4 ? 4 : 8;
  const int target = resident_warps(d.head_dim, P, GP);
  const int pairs = S * d.num_kv_heads > 0 ? S * d.num_kv_heads : 1;
  // one wave of the resident warps: `extra` pairs get one split more than
  // the others, so every resident slot holds a warp of near-equal work
  // (whole splits per pair would leave up to pairs - 1 slots empty, and the
  // SMs that hold one CTA more than the rest set the launch time)
  int splits = target / pairs;
  int extra = target - splits * pairs;
  // long contexts get at least one split per 256 pages: with lengths that
  // vary across the batch this puts more warps on the long sequences' pairs
  // (short pairs' warps leave the GPU early and the next CTAs take their place)
  const int min_splits = (pl.pages_max + 255) / 256;
  if (splits < min_splits) {
    splits = min_splits;
    extra = 0;
  }
  if (splits < 1) {
    splits = 1;
    extra = 0;
  }
  if (splits >= pl.pages_max) {
    splits = pl.pages_max;
    extra = 0;
  }
  pl.splits = extra > 0 ? splits + 1 : splits;
  pl.nhi = extra > 0 ? extra : pairs;
  pl.pages_per_split = (pl.pages_max + splits - 1) / splits;
  pl.workspace = (size_t)S * Hq * pl.splits * (d.head_dim + 4) * sizeof(float);
  return pl;
}

template <int D, int P, int GP>
static cudaError_t launch_split(const DecodeArgs& a, cudaStream_t st) {
  auto kern = decode_split_kernel<D, P, GP>;
  const size_t smem = split_smem<D, P, GP>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int items = a.nhi * a.splits + (a.S * a.H - a.nhi) * (a.splits - 1);
  const int grid = (items + kDecWarps - 1) / kDecWarps;
  e = launch_pdl(kern, grid, kDecWarps * kWarp, smem, st, a);
  if (e != cudaSuccess) return e;
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
                  cudaStream_t st, const DecodeStepRows* step) {
  if (d.format == KVQ_FMT_MXFP4)
    return decode_mx_launch(d, S, Hq, q, seq_lens, max_seq_len, block_table, bt_stride, sm_scale,
                            k_codes, k_params, v_codes, v_params, out, workspace,
                            workspace_bytes, err, st, step);
  if (d.format != KVQ_FMT_INT4)
    return decode_gen_launch(d, S, Hq, q, seq_lens, max_seq_len, block_table, bt_stride,
                             sm_scale, k_codes, k_params, v_codes, v_params, out, workspace,
                             workspace_bytes, err, st, step);
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
  a.bt_stride = bt_stride; a.max_seq_len = max_seq_len; a.splits = pl.splits; a.nhi = pl.nhi;
  a.rot_kind = d.rot_kind; a.lgb = lgb;
  a.scale2 = (float)((double)sm_scale * 1.4426950408889634074);
  a.q = static_cast<const __half*>(q); a.quat = d.quat;
  a.rope = d.rope; a.rope_max_pos = d.rope_max_pos;
  a.seq_lens = seq_lens; a.block_table = block_table;
  a.k_codes = k_codes; a.k_params = static_cast<const uint32_t*>(k_params);
  a.v_codes = v_codes; a.v_params = static_cast<const uint32_t*>(v_params);
  a.out = out;
  a.part = static_cast<float*>(workspace);
  a.err = err;
  a.lead = (128 + d.page_size - 1) / d.page_size;  // 128 tokens: measured best of 48-208
  a.k_new = step ? static_cast<const __half*>(step->k_new) : nullptr;
  a.v_new = step ? static_cast<const __half*>(step->v_new) : nullptr;
  a.new_stride = step ? step->new_stride : 0;
  a.k_codes_w = const_cast<uint8_t*>(k_codes);
  a.v_codes_w = const_cast<uint8_t*>(v_codes);
  a.k_params_w = static_cast<uint32_t*>(const_cast<void*>(k_params));
  a.v_params_w = static_cast<uint32_t*>(const_cast<void*>(v_params));
  cudaError_t e = launch_split_any(a, D, GP, st);
  if (e == cudaErrorInvalidValue) return KVQ_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  return decode_merge_launch(d, S, Hq, pl.splits, pl.nhi, a.part, out, st);
}

int decode_merge_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, int splits, int nhi,
                        const float* part, float* out, cudaStream_t st) {
  const int D = d.head_dim;
  int lgb = 0;
  while ((1 << lgb) < d.rot_block) ++lgb;
  MergeArgs mg;
  mg.S = S; mg.Hq = Hq; mg.G = Hq / d.num_kv_heads; mg.splits = splits; mg.nhi = nhi;
  mg.rot_kind = d.rot_kind; mg.lgb = lgb;
  mg.quat = d.quat; mg.part = part; mg.out = out;
  const int mgrid = (S * Hq + kDecWarps - 1) / kDecWarps;
  cudaError_t e = D == 128 ? launch_pdl(decode_merge_kernel<128>, mgrid, kDecWarps * kWarp, 0, st, mg)
                           : launch_pdl(decode_merge_kernel<256>, mgrid, kDecWarps * kWarp, 0, st, mg);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
