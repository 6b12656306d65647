/*
 * kvq.h -- C ABI of libkvq: a rotated, token-wise INT4, paged KV cache for
 * NVIDIA B200 (sm_100a).
 *
 * The method (page "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for
 * Real-World LLM Serving", Summary and Method): every (token, KV head) row of
 * K and of V is rotated by a block-diagonal Hadamard matrix, quantized to
 * 4-bit codes with one scale and one zero-point per row, and written straight
 * into a paged cache through a block table; attention then reads the INT4
 * pages with the query rotated by the same orthogonal matrix, so q . k is
 * unchanged by the rotation. The Walsh-Hadamard rotation spreads outlier
 * channels before quantization (page "UltraQuant: 4-bit KV caching for long
 * agents", method section). An alternative rotation maps each 4-channel block
 * v to qL v conj(qR) with unit quaternions (page "IsoQuant: Hardware-Aligned
 * SO(4) Isoclinic Rotations for LLM KV Cache Compression", Abstract).
 *
 * Conventions for every entry point:
 *  - Every pointer argument except `desc` is a DEVICE pointer (cudaMalloc'd
 *    or a torch CUDA tensor's data pointer) unless its comment says "host".
 *    `desc` itself is a host pointer; `desc->quat` is a device pointer.
 *  - The caller owns every buffer. The library never allocates, frees or
 *    synchronises; all work is enqueued on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream). Calls on one stream run in order.
 *  - The return value (kvq_status) is decided on the host before launch:
 *    argument and shape checks, 16-byte alignment of pointers and strides,
 *    workspace size, and cudaGetLastError() after the launch. A non-OK status
 *    means nothing was launched (except KVQ_ERR_CUDA).
 *  - Device-side problems (a block-table entry outside [0, num_pages), a
 *    position outside the table, a sequence index or length out of range)
 *    never fault or trap: the affected write or page is skipped and a bit is
 *    OR-ed into *err_flags (KVQ_ERRF_*) if err_flags is not NULL. The caller
 *    reads it after its own synchronisation.
 *  - Inputs are never modified; pool bytes not addressed by a call are never
 *    touched.
 *
 * Cache layout (per pool, K and V have separate pools):
 *  codes  : uint8  [num_pages][num_kv_heads][page_size][head_dim/2]
 *           two 4-bit codes per byte, even channel in the low nibble.
 *  params : binary16 pairs [num_pages][num_kv_heads][page_size][2] =
 *           (scale s16, minimum m16) of each row; the row dequantizes to
 *           x_i = c_i * s16 + m16 in the rotated basis.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1, /* a size, index or pointer argument is invalid */
  KVQ_ERR_UNSUPPORTED = 2, /* a valid geometry the library has no kernel for */
  KVQ_ERR_MISALIGNED = 3,  /* a pointer or stride is not 16-byte aligned   */
  KVQ_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required   */
  KVQ_ERR_CUDA = 5         /* the CUDA runtime reported an error at launch  */
} kvq_status;

typedef enum {
  KVQ_ROT_NONE = 0,            /* identity: the rotation-free INT4 baseline      */
  KVQ_ROT_HADAMARD = 1,        /* block-diagonal Walsh-Hadamard, block rot_block  */
  KVQ_ROT_QUAT = 2,            /* per 4-channel block v -> qL v conj(qR)
                                  (IsoQuant-Full)                                */
  KVQ_ROT_QUAT_FAST = 3,       /* per 4-channel block v -> qL v: one isoclinic
                                  factor (IsoQuant-Fast)                         */
  KVQ_ROT_HADAMARD_SIGNED = 4, /* channel i times a fixed sign s_i = +-1, then
                                  the block Walsh-Hadamard rotation              */
  KVQ_ROT_QUAT_MAT = 5         /* IsoQuant-Full folded into one binary32 4x4
                                  matrix per block, M = Rm(conj qR) Lm(qL), built
                                  from the quaternion table (16 multiply-adds per
                                  block instead of 32; another rounding)         */
} kvq_rot_kind;

/* Storage format of a rotated (token, head) row; both pools of a cache
 * share it: codes [NP][H][P][d * bits / 8] bytes (bits 4 except for the
 * 2- and 3-bit formats), one 32-bit params word per row. Every format but
 * INT4 needs head_dim 128.
 *  KVQ_FMT_INT4   token-wise asymmetric INT4 (SAW-INT4, Summary): codes
 *                 c = nearest of (x - m16)/s16 in [0, 15]; params (s16, m16).
 *  KVQ_FMT_MXFP4  microscaled FP4 (UltraQuant page, method section: FP4 KV
 *                 tensors with UE8M0 group scales, FP8 queries, scaled
 *                 matrix-core MMA), read as the OCP MX formats: each block of
 *                 32 channels shares the scale 2^X, X = floor(log2 amax) - 2
 *                 clamped to [-127, 127] (an all-zero block: -127), stored as
 *                 the byte X + 127 (params byte g = block g); codes are E2M1
 *                 (bit 3 sign, magnitude index into {0, 0.5, 1, 1.5, 2, 3, 4,
 *                 6}) of x / 2^X, nearest with ties to even, saturating at 6,
 *                 the sign kept (a negative value rounding to zero is -0).
 *                 Decode quantizes the rotated query to MX E4M3 (X =
 *                 floor(log2 amax) - 8 per 32 channels, nearest-even,
 *                 saturating at 448, sign kept) and takes QK on the tensor
 *                 cores' block-scaled MMA. */
typedef enum {
  KVQ_FMT_INT4 = 0,
  KVQ_FMT_MXFP4 = 1,
  KVQ_FMT_INT2 = 2,  /* the INT4 rule with 2-bit codes (Q = 3 levels above zero;
                        IsoQuant page, Abstract: bit widths {2, 3, 4}); a row's
                        codes are a little-endian bit stream of d/4 bytes      */
  KVQ_FMT_INT3 = 3,  /* 3-bit codes (Q = 7), 3d/8 bytes per row; the codes
                        pool is [NP][H][P][d * bits / 8] for every format      */
  KVQ_FMT_LUT4 = 4   /* a calibrated 16-entry level table in place of the
                        uniform INT4 levels (UltraQuant page, method section:
                        the refitted 16-entry table): the INT4 statistics, the
                        code the index of the level t nearest to the exact
                        RN(x - m16) * RN(1/s16) (ties to the lower index),
                        x^ = t[c] s16 + m16                                    */
} kvq_format;

/* Bits OR-ed into *err_flags by the kernels. */
#define KVQ_ERRF_PAGE 1 /* block-table entry outside [0, num_pages): page skipped */
#define KVQ_ERRF_POS 2  /* position < 0 or position/page_size >= bt_stride       */
#define KVQ_ERRF_SEQ 4  /* token's sequence index >= num_seqs                    */
#define KVQ_ERRF_LEN 8  /* seq_lens[s] < 0, > max_seq_len, or past the table      */
#define KVQ_ERRF_TIMEOUT 16 /* a bounded wait for an asynchronous copy expired (never
                               expected). Copies of that launch may still have been in
                               flight when its blocks returned: every output of the
                               launch is then undefined and the caller should discard
                               the whole batch (pool bytes outside the batch's slots
                               are still untouched).                               */

/* Geometry of one paged cache (both pools share it).
 *  head_dim     d: 64, 128 or 256.
 *  num_kv_heads H: 1 .. 65536 (larger counts return KVQ_ERR_UNSUPPORTED).
 *  page_size    P: tokens per page; 16, 32 or 64.
 *  num_pages    NP: pool capacity in pages (>= 1).
 *  rot_kind     a kvq_rot_kind.
 *  rot_block    b, for KVQ_ROT_HADAMARD and KVQ_ROT_HADAMARD_SIGNED: a power
 *               of two in [16, 256] dividing d (ignored otherwise).
 *  quat         the rotation's table, a device pointer (NULL for
 *               KVQ_ROT_NONE and KVQ_ROT_HADAMARD):
 *               KVQ_ROT_QUAT, KVQ_ROT_QUAT_FAST, KVQ_ROT_QUAT_MAT: float
 *               [d/4][2][4], per block j (qL[j], qR[j]) as (w, x, y, z); unit
 *               quaternions (the fast map uses qL only; the matrix form builds
 *               its matrices from the same table inside each launch).
 *               Channels 4j..4j+3 form block j.
 *               KVQ_ROT_HADAMARD_SIGNED: float [d] of signs, each +1 or -1.
 *               The quaternion maps' Hamilton components are fused
 *               multiply-add chains in the term order of the quantize
 *               definition below; the sign flip is exact.
 *  rope         optional rotary position embedding in front of the rotation
 *               (NULL: none): device float [rope_max_pos][d/2][2], row p
 *               holding (cos, sin) of the angle of each channel pair
 *               (2i, 2i+1) at position p, 16-byte aligned. Every key row is
 *               turned by the row of its token's position before it is
 *               rotated and quantized (values are not), and the query of a
 *               decode by the row of position seq_len - 1:
 *                 x'_2i = RN(RN(x_2i c) - RN(x_2i+1 s)),
 *                 x'_2i+1 = RN(RN(x_2i s) + RN(x_2i+1 c))   (binary32).
 *               The pages describe no RoPE; it is the step in front of the
 *               method's path in a decode step, offered here so that the key
 *               rows need not be turned by a separate kernel.
 *  rope_max_pos rows of the rope table (>= 1 when rope is set); a position at
 *               or past it is invalid (KVQ_ERRF_POS in an append, the row is
 *               skipped; KVQ_ERRF_LEN in a decode, the output is zero).
 *  format       a kvq_format: how a rotated row is stored (0, the token-wise
 *               INT4 of the pages, for a zero-initialised descriptor).
 *  levels       KVQ_FMT_LUT4 only (NULL otherwise): device float [16], the
 *               level table, strictly increasing, each level a multiple of
 *               1/16 in [0, 15] (16 t an integer in [0, 240]); 4-byte aligned.
 *               A table that breaks these rules gives unspecified codes. */
typedef struct {
  int32_t head_dim;
  int32_t num_kv_heads;
  int32_t page_size;
  int32_t num_pages;
  int32_t rot_kind;
  int32_t rot_block;
  const float* quat;
  const float* rope;
  int32_t rope_max_pos;
  int32_t format;
  const float* levels;
} kvq_cache_desc;

/*
 * kvq_quantize_append -- rotate, quantize, pack and scatter new tokens of K
 * and V into the INT4 pools ("SAW-INT4", Summary/Method: the fused
 * rotation-quantization kernel writing into paged KV-cache layouts).
 *
 *  num_tokens  T >= 0 (T = 0 is a no-op returning KVQ_OK).
 *  k, v        binary16 [T][H][d]: token t's row for head h starts at element
 *              t*tok_stride + h*d. Both 16-byte aligned.
 *  tok_stride  elements between consecutive tokens, >= H*d, multiple of 8.
 *  token_seq   int32 [T]: sequence of each token; < 0 skips the token.
 *  token_pos   int32 [T]: position of each token within its sequence.
 *  num_seqs    rows of block_table.
 *  block_table int32 [num_seqs][bt_stride]: page of (seq, pos / P).
 *  k_codes ... v_params: the pools (layout above), 16-byte aligned.
 *
 * Per row (token t, head h), in binary32: x = widen(k[t][h]); y = R x
 * (Hadamard: butterflies h = 1, 2, ..., b/2 on each block, pair (i, i+h)
 * -> (x_i + x_{i+h}, x_i - x_{i+h}), then times the binary32 value nearest
 * 1/sqrt(b); quaternion: (qL (x) v) (x) conj(qR) with the Hamilton
 * components as fused multiply-adds in a fixed term order); mn = min y + 0,
 * mx = max y + 0; m16 = binary16 round-down(mn); s16 = binary16 round-up of
 * round-up32(round-up32(mx - m16) / 15); inv = round-nearest32(1/s16);
 * code_i = nearest integer, ties to even, of the exact product
 * RN(y_i - m16) * inv, in [0, 15] (all 0 when s16 = 0). Codes, scale and
 * minimum are bit-identical to that definition.
 * Domain: inputs finite, and every rotated value as well as the scale within
 * the binary16 range (|y| <= 65504); outside it (e.g. a minimum that rounds
 * to -inf) the row's codes are unspecified, but nothing outside the row's
 * slot is written.
 * Tokens writing the same slot in one call race (caller error).
 */
int kvq_quantize_append(const kvq_cache_desc* desc, int32_t num_tokens, const void* k,
                        const void* v, int64_t tok_stride, const int32_t* token_seq,
                        const int32_t* token_pos, int32_t num_seqs,
                        const int32_t* block_table, int32_t bt_stride, uint8_t* k_codes,
                        void* k_params, uint8_t* v_codes, void* v_params,
                        int32_t* err_flags, void* stream);

/*
 * kvq_decode_workspace_bytes -- bytes of device workspace that
 * kvq_paged_decode_attn needs for these sizes (0 on invalid arguments). The
 * workspace holds the per-split partial results (float32, written and then
 * read by each call); it needs no initialisation, and one workspace serves
 * any number of later calls on the same stream. Calls that share a
 * workspace must not overlap in time.
 */
size_t kvq_decode_workspace_bytes(const kvq_cache_desc* desc, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t max_seq_len);

/*
 * kvq_paged_decode_attn -- one query token per sequence attends over its
 * cached INT4 tokens ("SAW-INT4", Key takeaway: serving-compatible attention
 * over the rotated INT4 cache).
 *
 *  num_seqs     S >= 1; num_q_heads Hq: a multiple of H with Hq/H <= 8.
 *  q            binary16 [S][Hq][d], not rotated (the kernel rotates it).
 *  seq_lens     int32 [S]: cached tokens of each sequence (0 gives out = 0).
 *  max_seq_len  upper bound of seq_lens (sizes the split-K work).
 *  sm_scale     softmax scale (typically 1/sqrt(d)).
 *  out          float32 [S][Hq][d], in the original (un-rotated) basis.
 *  workspace    >= kvq_decode_workspace_bytes(...) bytes, 16-byte aligned
 *               (see above).
 *
 * For query head g (KV head h = g / (Hq/H)): qhat = R q_g;
 * z_j = sm_scale * qhat . khat_j; p = softmax(z); out = R^-1 sum_j p_j vhat_j,
 * with khat_j, vhat_j the dequantized rows. Results match a double-precision
 * evaluation of that definition to about 1e-4 absolute for unit-scale data
 * (the contractions run on tensor cores with split binary16 operands).
 */
int kvq_paged_decode_attn(const kvq_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                          const void* q, const int32_t* seq_lens, int32_t max_seq_len,
                          const int32_t* block_table, int32_t bt_stride, float sm_scale,
                          const uint8_t* k_codes, const void* k_params,
                          const uint8_t* v_codes, const void* v_params, float* out,
                          void* workspace, size_t workspace_bytes, int32_t* err_flags,
                          void* stream);

/*
 * kvq_dequantize_pages -- dense export of the cached rows of one pool:
 * out[s][j][h][:] = c * s16 + m16 (optionally rotated back by R^-1) for
 * j < seq_lens[s]; rows j >= seq_lens[s] are not written.
 *
 *  out       float32 (out_fp32 != 0) or binary16 [S][max_seq_len][H][d].
 *  unrotate  0: values in the rotated basis (exact in float32);
 *            1: R^-1 applied in binary32 arithmetic.
 */
int kvq_dequantize_pages(const kvq_cache_desc* desc, int32_t num_seqs,
                         const int32_t* seq_lens, int32_t max_seq_len,
                         const int32_t* block_table, int32_t bt_stride, const uint8_t* codes,
                         const void* params, int32_t unrotate, int32_t out_fp32, void* out,
                         int32_t* err_flags, void* stream);

/*
 * kvq_decode_step -- one decode step in one call: for every sequence s with
 * seq_lens[s] >= 1, the new token's K and V rows are rotated, quantized and
 * written at position seq_lens[s] - 1 exactly as kvq_quantize_append writes
 * them (token_seq = s, token_pos = seq_lens[s] - 1), and decode attention then
 * runs over positions [0, seq_lens[s]) as kvq_paged_decode_attn. The pools
 * and the output equal those of the two calls in that order. The quantized
 * write inside the paged cache follows the method (page "SAW-INT4:
 * System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving",
 * Summary and Method); doing it inside the attention kernel, by the warp
 * that reads that page, is this library's own step (the write needs no
 * launch of its own and overlaps the attention's start-up latency).
 *
 *  k_new, v_new  device binary16 rows of the new tokens: row (s, h) starts at
 *                element s * new_stride + h * head_dim; 16-byte aligned,
 *                new_stride a multiple of 8 elements and >= H * head_dim.
 *  seq_lens      device int32 [S], lengths INCLUDING the new token.
 *  k_codes, k_params, v_codes, v_params
 *                the pools, written at the new tokens' slots and read.
 *  all other arguments, the workspace, the return codes and the flags as for
 *  kvq_paged_decode_attn; a block-table entry outside [0, num_pages) for a
 *  new token's page skips that write and sets KVQ_ERRF_PAGE.
 */
int kvq_decode_step(const kvq_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                    const void* q, const void* k_new, const void* v_new, int64_t new_stride,
                    const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                    int32_t bt_stride, float sm_scale, uint8_t* k_codes, void* k_params,
                    uint8_t* v_codes, void* v_params, float* out, void* workspace,
                    size_t workspace_bytes, int32_t* err_flags, void* stream);

/*
 * Full-precision baseline: decode attention over an UNQUANTIZED binary16
 * paged cache, without rotation. The INT4 cache is measured against it (page
 * "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
 * Serving", Summary and Key takeaways: INT4 against full-precision KV caches).
 *
 *  k_pages, v_pages  device binary16 [num_pages][num_kv_heads][page_size]
 *                    [head_dim], 16-byte aligned, filled by the caller with the
 *                    plain K and V rows of each cached token.
 *  desc              geometry as for the INT4 cache; rot_kind, rot_block and
 *                    quat are ignored (nothing is rotated).
 *  q, seq_lens, max_seq_len, block_table, bt_stride, sm_scale, out
 *                    as for kvq_paged_decode_attn; out is float32 [S][Hq][d]
 *                    = softmax(sm_scale q K^T) V per query head.
 *  workspace         >= kvq_decode_fp16_workspace_bytes(...) bytes, 16-byte
 *                    aligned, zero-filled before its first use (the counters
 *                    are left at zero by every call).
 * Supported: head_dim 128 with page_size 16, 32 or 64 and GQA group <= 8;
 * head_dim 256 with page_size 16 or 32 and group <= 4 (else
 * KVQ_ERR_UNSUPPORTED). Errors and flags as for kvq_paged_decode_attn.
 */
size_t kvq_decode_fp16_workspace_bytes(const kvq_cache_desc* desc, int32_t num_seqs,
                                       int32_t num_q_heads, int32_t max_seq_len);
int kvq_paged_decode_attn_fp16(const kvq_cache_desc* desc, int32_t num_seqs,
                               int32_t num_q_heads, const void* q, const int32_t* seq_lens,
                               int32_t max_seq_len, const int32_t* block_table,
                               int32_t bt_stride, float sm_scale, const void* k_pages,
                               const void* v_pages, float* out, void* workspace,
                               size_t workspace_bytes, int32_t* err_flags, void* stream);

/* Size of the fixed scratch array behind kvq_paged_decode_attn_noalloc. */
#define KVQ_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * kvq_paged_decode_attn_noalloc -- kvq_paged_decode_attn for callers that
 * cannot allocate device memory (no counterpart in the method's pages; it is
 * a deployment convenience). Some callers have no way to hand over a
 * workspace: an engine whose device memory is planned once at start-up and
 * whose allocator refuses later requests, a plug-in living inside a host
 * framework that owns every device allocation, or a serving path that must
 * not call cudaMalloc/cudaFree because those calls synchronise the device.
 *
 * Arguments and results are those of kvq_paged_decode_attn without
 * `workspace` / `workspace_bytes`. The scratch is a 16 MiB array compiled
 * into the library (KVQ_NOALLOC_SCRATCH_BYTES): every GPU that loads libkvq
 * holds it until the process exits. The call allocates and frees nothing;
 * it enqueues the decode kernels on `stream`. Nothing in the scratch needs
 * clearing between calls: each call writes every byte it reads there.
 *  - Sizes whose workspace (kvq_decode_workspace_bytes) exceeds
 *    KVQ_NOALLOC_SCRATCH_BYTES are rejected with KVQ_ERR_WORKSPACE before
 *    anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it for that
 *    device's current CUDA context; a call in a context not seen before
 *    (after a device reset, or from a non-primary context) looks it up
 *    again. Make the first call on each device and context before any
 *    stream capture there.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents: calls that overlap on the GPU (different streams, or
 *    different host threads without ordering) race and give wrong results.
 */
int kvq_paged_decode_attn_noalloc(const kvq_cache_desc* desc, int32_t num_seqs,
                                  int32_t num_q_heads, const void* q, const int32_t* seq_lens,
                                  int32_t max_seq_len, const int32_t* block_table,
                                  int32_t bt_stride, float sm_scale, const uint8_t* k_codes,
                                  const void* k_params, const uint8_t* v_codes,
                                  const void* v_params, float* out, int32_t* err_flags,
                                  void* stream);

/* Human-readable name of a kvq_status value (static storage). */
const char* kvq_status_string(int status);

/* Library build string (static storage). */
const char* kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
