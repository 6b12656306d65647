// C ABI of libkvq (declared in include/kvq.h): host-side argument checks,
// then one launcher per entry point. No entry point allocates, frees or
// synchronises; all work goes to the caller's stream.

#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include "kvq.h"
#include "kvq_launch.h"

namespace kvq {

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev < 64) cache[dev] = n;
  return n;
}

// CTAs of `kern` that fit on one SM at once, from its registers and shared
// memory and the device's limits (the occupancy query reports one CTA for
// the tensor-memory kernels although several run side by side).
int resident_ctas_per_sm(const void* kern, int threads, size_t dyn_smem) {
  cudaFuncAttributes fa;
  int dev = 0, smem_sm = 0, res_blk = 0, regs_sm = 0, max_blk = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&res_blk, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&max_blk, cudaDevAttrMaxBlocksPerMultiprocessor, dev) != cudaSuccess)
    return 1;
  const size_t per_blk = dyn_smem + fa.sharedSizeBytes + (size_t)res_blk;
  int n = per_blk > 0 ? (int)((size_t)smem_sm / per_blk) : max_blk;
  const int warps = (threads + 31) / 32;
  const int regs_blk = warps * ((fa.numRegs * 32 + 255) / 256 * 256);
  if (regs_blk > 0 && regs_sm / regs_blk < n) n = regs_sm / regs_blk;
  if (n > max_blk) n = max_blk;
  return n < 1 ? 1 : n;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
static bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Geometry checks shared by every entry point.
static int check_desc(const kvq_cache_desc* d) {
  if (d == nullptr) return KVQ_ERR_INVALID_ARG;
  if (d->head_dim <= 0 || d->num_kv_heads <= 0 || d->page_size <= 0 || d->num_pages <= 0)
    return KVQ_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256) return KVQ_ERR_UNSUPPORTED;
  // page strides of a pool (heads x page bytes) stay 32-bit products
  if (d->num_kv_heads > 65536) return KVQ_ERR_UNSUPPORTED;
  if (d->page_size != 16 && d->page_size != 32 && d->page_size != 64) return KVQ_ERR_UNSUPPORTED;
  if (d->format < KVQ_FMT_INT4 || d->format > KVQ_FMT_LUT4) return KVQ_ERR_INVALID_ARG;
  if (d->format != KVQ_FMT_INT4 && d->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if ((d->format == KVQ_FMT_LUT4) != (d->levels != nullptr)) return KVQ_ERR_INVALID_ARG;
  if (d->levels != nullptr && !aligned4(d->levels)) return KVQ_ERR_MISALIGNED;
  switch (d->rot_kind) {
    case KVQ_ROT_NONE:
      break;
    case KVQ_ROT_HADAMARD:
    case KVQ_ROT_HADAMARD_SIGNED:
      if (!pow2(d->rot_block) || d->rot_block > d->head_dim) return KVQ_ERR_INVALID_ARG;
      if (d->rot_block < 16 || d->rot_block > 256) return KVQ_ERR_UNSUPPORTED;
      if (d->rot_kind == KVQ_ROT_HADAMARD_SIGNED) {
        if (d->quat == nullptr) return KVQ_ERR_INVALID_ARG;
        if (!aligned16(d->quat)) return KVQ_ERR_MISALIGNED;
      }
      break;
    case KVQ_ROT_QUAT:
    case KVQ_ROT_QUAT_FAST:
    case KVQ_ROT_QUAT_MAT:
      if (d->quat == nullptr) return KVQ_ERR_INVALID_ARG;
      if (!aligned16(d->quat)) return KVQ_ERR_MISALIGNED;
      break;
    default:
      return KVQ_ERR_INVALID_ARG;
  }
  if (d->rope != nullptr) {
    if (d->rope_max_pos < 1) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(d->rope)) return KVQ_ERR_MISALIGNED;
  }
  return KVQ_OK;
}

}  // namespace kvq

using namespace kvq;

extern "C" {

int kvq_quantize_append(const kvq_cache_desc* desc, int32_t num_tokens, const void* k,
                        const void* v, int64_t tok_stride, const int32_t* token_seq,
                        const int32_t* token_pos, int32_t num_seqs,
                        const int32_t* block_table, int32_t bt_stride, uint8_t* k_codes,
                        void* k_params, uint8_t* v_codes, void* v_params,
                        int32_t* err_flags, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (num_tokens < 0 || num_seqs < 0 || bt_stride < 1) return KVQ_ERR_INVALID_ARG;
  if (num_tokens == 0) return KVQ_OK;
  if (!k || !v || !token_seq || !token_pos || !k_codes || !k_params || !v_codes || !v_params)
    return KVQ_ERR_INVALID_ARG;
  if (num_seqs > 0 && !block_table) return KVQ_ERR_INVALID_ARG;
  if (tok_stride < (int64_t)desc->num_kv_heads * desc->head_dim) return KVQ_ERR_INVALID_ARG;
  if (tok_stride % 8 != 0) return KVQ_ERR_MISALIGNED;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_codes) || !aligned16(v_codes) ||
      !aligned16(k_params) || !aligned16(v_params) || !aligned4(token_seq) ||
      !aligned4(token_pos) || (block_table && !aligned4(block_table)) ||
      (err_flags && !aligned4(err_flags)))
    return KVQ_ERR_MISALIGNED;
  return append_launch(*desc, num_tokens, k, v, tok_stride, token_seq, token_pos, num_seqs,
                       block_table, bt_stride, k_codes, k_params, v_codes, v_params, err_flags,
                       static_cast<cudaStream_t>(stream));
}

size_t kvq_decode_workspace_bytes(const kvq_cache_desc* desc, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t max_seq_len) {
  if (check_desc(desc) != KVQ_OK || num_seqs < 1 || num_q_heads < 1 || max_seq_len < 0 ||
      num_q_heads % desc->num_kv_heads != 0)
    return 0;
  return decode_plan(*desc, num_seqs, num_q_heads, max_seq_len).workspace;
}

int kvq_paged_decode_attn(const kvq_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                          const void* q, const int32_t* seq_lens, int32_t max_seq_len,
                          const int32_t* block_table, int32_t bt_stride, float sm_scale,
                          const uint8_t* k_codes, const void* k_params,
                          const uint8_t* v_codes, const void* v_params, float* out,
                          void* workspace, size_t workspace_bytes, int32_t* err_flags,
                          void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (num_seqs < 1 || num_q_heads < 1 || max_seq_len < 0 || bt_stride < 1 ||
      !std::isfinite(sm_scale))
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % desc->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  const int G = num_q_heads / desc->num_kv_heads;
  if (desc->head_dim == 64 || G > 8 || (desc->head_dim == 256 && G > 4))
    return KVQ_ERR_UNSUPPORTED;
  if (!q || !seq_lens || !block_table || !k_codes || !k_params || !v_codes || !v_params || !out)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_codes) || !aligned16(v_codes) ||
      !aligned16(k_params) || !aligned16(v_params) || !aligned4(seq_lens) ||
      !aligned4(block_table) || (err_flags && !aligned4(err_flags)))
    return KVQ_ERR_MISALIGNED;
  if (workspace && !aligned16(workspace)) return KVQ_ERR_MISALIGNED;
  return decode_launch(*desc, num_seqs, num_q_heads, q, seq_lens, max_seq_len, block_table,
                       bt_stride, sm_scale, k_codes, k_params, v_codes, v_params, out, workspace,
                       workspace_bytes, err_flags, static_cast<cudaStream_t>(stream));
}

int kvq_decode_step(const kvq_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                    const void* q, const void* k_new, const void* v_new, int64_t new_stride,
                    const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                    int32_t bt_stride, float sm_scale, uint8_t* k_codes, void* k_params,
                    uint8_t* v_codes, void* v_params, float* out, void* workspace,
                    size_t workspace_bytes, int32_t* err_flags, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (num_seqs < 1 || num_q_heads < 1 || max_seq_len < 0 || bt_stride < 1 ||
      !std::isfinite(sm_scale))
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % desc->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  const int G = num_q_heads / desc->num_kv_heads;
  if (desc->head_dim == 64 || G > 8 || (desc->head_dim == 256 && G > 4)) return KVQ_ERR_UNSUPPORTED;
  if (!q || !k_new || !v_new || !seq_lens || !block_table || !k_codes || !k_params || !v_codes ||
      !v_params || !out)
    return KVQ_ERR_INVALID_ARG;
  if (new_stride < (int64_t)desc->num_kv_heads * desc->head_dim) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_new) || !aligned16(v_new) ||
      new_stride % 8 != 0 || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(k_params) ||
      !aligned16(v_params) || !aligned4(seq_lens) || !aligned4(block_table) ||
      (err_flags && !aligned4(err_flags)))
    return KVQ_ERR_MISALIGNED;
  if (workspace && !aligned16(workspace)) return KVQ_ERR_MISALIGNED;
  const DecodeStepRows rows{k_new, v_new, new_stride};
  return decode_launch(*desc, num_seqs, num_q_heads, q, seq_lens, max_seq_len, block_table,
                       bt_stride, sm_scale, k_codes, k_params, v_codes, v_params, out, workspace,
                       workspace_bytes, err_flags, static_cast<cudaStream_t>(stream), &rows);
}

size_t kvq_decode_fp16_workspace_bytes(const kvq_cache_desc* desc, int32_t num_seqs,
                                       int32_t num_q_heads, int32_t max_seq_len) {
  if (check_desc(desc) != KVQ_OK || num_seqs < 1 || num_q_heads < 1 || max_seq_len < 0 ||
      num_q_heads % desc->num_kv_heads != 0)
    return 0;
  return decode_fp16_plan(*desc, num_seqs, num_q_heads, max_seq_len).workspace;
}

int kvq_paged_decode_attn_fp16(const kvq_cache_desc* desc, int32_t num_seqs,
                               int32_t num_q_heads, const void* q, const int32_t* seq_lens,
                               int32_t max_seq_len, const int32_t* block_table,
                               int32_t bt_stride, float sm_scale, const void* k_pages,
                               const void* v_pages, float* out, void* workspace,
                               size_t workspace_bytes, int32_t* err_flags, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (num_seqs < 1 || num_q_heads < 1 || max_seq_len < 0 || bt_stride < 1 ||
      !std::isfinite(sm_scale))
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % desc->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  const int G = num_q_heads / desc->num_kv_heads;
  if (desc->head_dim == 64 || G > 8 || (desc->head_dim == 256 && G > 4)) return KVQ_ERR_UNSUPPORTED;
  if (!q || !seq_lens || !block_table || !k_pages || !v_pages || !out) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_pages) || !aligned16(v_pages) ||
      !aligned4(seq_lens) || !aligned4(block_table) || (err_flags && !aligned4(err_flags)))
    return KVQ_ERR_MISALIGNED;
  if (workspace && !aligned16(workspace)) return KVQ_ERR_MISALIGNED;
  return decode_fp16_launch(*desc, num_seqs, num_q_heads, q, seq_lens, max_seq_len, block_table,
                            bt_stride, sm_scale, k_pages, v_pages, out, workspace,
                            workspace_bytes, err_flags, static_cast<cudaStream_t>(stream));
}

int kvq_dequantize_pages(const kvq_cache_desc* desc, int32_t num_seqs,
                         const int32_t* seq_lens, int32_t max_seq_len,
                         const int32_t* block_table, int32_t bt_stride, const uint8_t* codes,
                         const void* params, int32_t unrotate, int32_t out_fp32, void* out,
                         int32_t* err_flags, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (num_seqs < 0 || max_seq_len < 0 || bt_stride < 1) return KVQ_ERR_INVALID_ARG;
  if (num_seqs == 0 || max_seq_len == 0) return KVQ_OK;
  if (!seq_lens || !block_table || !codes || !params || !out) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(params) || !aligned16(out) || !aligned4(seq_lens) ||
      !aligned4(block_table) || (err_flags && !aligned4(err_flags)))
    return KVQ_ERR_MISALIGNED;
  return dequant_launch(*desc, num_seqs, seq_lens, max_seq_len, block_table, bt_stride, codes,
                        params, unrotate ? 1 : 0, out_fp32 ? 1 : 0, out, err_flags,
                        static_cast<cudaStream_t>(stream));
}

const char* kvq_status_string(int status) {
  switch (status) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_MISALIGNED: return "KVQ_ERR_MISALIGNED";
    case KVQ_ERR_WORKSPACE: return "KVQ_ERR_WORKSPACE";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
  }
  return "KVQ_UNKNOWN_STATUS";
}

const char* kvq_version(void) { return "libkvq 0.1 sm_100a"; }

}  // extern "C"
