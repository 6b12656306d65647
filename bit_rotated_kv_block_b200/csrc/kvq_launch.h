// Host-side launchers of the libkvq kernels (internal; the public ABI is
// include/kvq.h). Each returns a kvq_status and enqueues work on `st` only.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();
// CTAs of `kern` (threads per CTA, dynamic shared memory) resident per SM.
int resident_ctas_per_sm(const void* kern, int threads, size_t dyn_smem);

int append_launch(const kvq_cache_desc& d, int32_t T, const void* k, const void* v,
                  int64_t tok_stride, const int32_t* token_seq, const int32_t* token_pos,
                  int32_t num_seqs, const int32_t* block_table, int32_t bt_stride,
                  uint8_t* k_codes, void* k_params, uint8_t* v_codes, void* v_params,
                  int32_t* err, cudaStream_t st);

int dequant_launch(const kvq_cache_desc& d, int32_t S, const int32_t* seq_lens,
                   int32_t max_seq_len, const int32_t* block_table, int32_t bt_stride,
                   const uint8_t* codes, const void* params, int32_t unrotate, int32_t out_fp32,
                   void* out, int32_t* err, cudaStream_t st);

// Split-K plan of the decode attention for these sizes.
// Launches `kern` with programmatic stream serialization (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int threads, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

struct DecodePlan {
  int pages_max;        // ceil(max_seq_len / P)
  int splits;           // work items per (sequence, KV head): the first `nhi`
                        // (sequence, KV head) pairs have `splits`, the others
                        // splits - 1 (so the total can match the resident warps)
  int nhi;
  int pages_per_split;  // pages per split (contiguous ranges; an even share for interleaved groups)
  size_t workspace;     // bytes of partial results
};
DecodePlan decode_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len);

// New-token rows of a fused decode step (kvq_decode_step).
struct DecodeStepRows {
  const void* k_new;   // binary16 [S][H][d] rows, row (s, h) at s * new_stride + h * d
  const void* v_new;
  int64_t new_stride;  // elements between consecutive sequences' rows
};

// step == nullptr: decode attention only; otherwise the new token of every
// sequence is quantized into the pools (which the kernel then writes) first.
int decode_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                  const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                  int32_t bt_stride, float sm_scale, const uint8_t* k_codes,
                  const void* k_params, const uint8_t* v_codes, const void* v_params,
                  float* out, void* workspace, size_t workspace_bytes, int32_t* err,
                  cudaStream_t st, const DecodeStepRows* step = nullptr);

// The merge kernel over split partial results [S][Hq][splits][d + 4] (the
// running sums, then the base-2 maximum and total weight), rotated back.
// Query heads of the first `nhi` (sequence, KV head) pairs combine `splits`
// partials, the others splits - 1.
int decode_merge_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, int splits, int nhi,
                        const float* part, float* out, cudaStream_t st);

// Decode attention over the microscaled FP4 cache (QK on the block-scaled
// tensor-core MMA); plan (pages_per_split counts 128-token tiles) and launch.
DecodePlan decode_mx_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len);
int decode_mx_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                     const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                     int32_t bt_stride, float sm_scale, const uint8_t* k_codes,
                     const void* k_params, const uint8_t* v_codes, const void* v_params,
                     float* out, void* workspace, size_t workspace_bytes, int32_t* err,
                     cudaStream_t st, const DecodeStepRows* step);

// Decode attention over the 2-bit, 3-bit and level-table caches (QK on the
// tensor cores' integer MMA); plan (pages_per_split counts 128-token tiles)
// and launch.
DecodePlan decode_gen_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len);
int decode_gen_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                      const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                      int32_t bt_stride, float sm_scale, const uint8_t* k_codes,
                      const void* k_params, const uint8_t* v_codes, const void* v_params,
                      float* out, void* workspace, size_t workspace_bytes, int32_t* err,
                      cudaStream_t st, const DecodeStepRows* step);

// Baseline decode attention over a binary16 paged cache.
DecodePlan decode_fp16_plan(const kvq_cache_desc& d, int32_t S, int32_t Hq, int32_t max_seq_len);
int decode_fp16_launch(const kvq_cache_desc& d, int32_t S, int32_t Hq, const void* q,
                       const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table,
                       int32_t bt_stride, float sm_scale, const void* k_pages,
                       const void* v_pages, float* out, void* workspace, size_t workspace_bytes,
                       int32_t* err, cudaStream_t st);

}  // namespace kvq
