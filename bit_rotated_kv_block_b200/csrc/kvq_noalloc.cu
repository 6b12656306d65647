// Decode attention for callers that cannot allocate device memory.
//
// kvq_paged_decode_attn needs a caller-provided workspace. Some callers have
// no way to provide one: an engine whose device memory is planned once at
// start-up and whose allocator refuses requests afterwards, a plug-in that
// runs inside a host framework that owns every device allocation, or code
// that must not call cudaMalloc/cudaFree on its serving path because those
// calls synchronise the device. This file gives them one more entry point,
// kvq_paged_decode_attn_noalloc, whose scratch is a fixed array compiled
// into the library: every GPU that loads libkvq holds kNoallocScratchBytes of
// it until the process exits, and no call allocates or frees anything.

#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <mutex>

#include "kvq.h"
#include "kvq_launch.h"

namespace kvq {

constexpr size_t kNoallocScratchBytes = KVQ_NOALLOC_SCRATCH_BYTES;
static_assert(kNoallocScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

// The scratch itself: zero at module load, shared by every call on a device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the array per device, looked up once with that device
// current (in host code the array's name is only a host-side stand-in).
static void* g_scratch_addr[64] = {nullptr};
static std::mutex g_scratch_mu;

static int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return KVQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return KVQ_OK;
}

}  // namespace kvq

using namespace kvq;

extern "C" int kvq_paged_decode_attn_noalloc(
    const kvq_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads, const void* q,
    const int32_t* seq_lens, int32_t max_seq_len, const int32_t* block_table, int32_t bt_stride,
    float sm_scale, const uint8_t* k_codes, const void* k_params, const uint8_t* v_codes,
    const void* v_params, float* out, int32_t* err_flags, void* stream) {
  // same host-side checks as kvq_paged_decode_attn, before any CUDA call
  if (desc == nullptr || num_seqs < 1 || num_q_heads < 1 || max_seq_len < 0 || bt_stride < 1 ||
      !std::isfinite(sm_scale) || desc->num_kv_heads < 1 || num_q_heads % desc->num_kv_heads != 0)
    return KVQ_ERR_INVALID_ARG;
  const size_t need =
      kvq_decode_workspace_bytes(desc, num_seqs, num_q_heads, max_seq_len);
  if (need == 0) return KVQ_ERR_INVALID_ARG;
  if (need > kNoallocScratchBytes) return KVQ_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != KVQ_OK) return st;
  // the per-(sequence, KV head) counters at the start of the scratch must be
  // zero when the kernel starts; the previous call normally leaves them so,
  // but a call that failed part-way might not: clear them on the stream
  const size_t counters = (size_t)num_seqs * desc->num_kv_heads * sizeof(int32_t);
  if (cudaMemsetAsync(scratch, 0, counters, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return kvq_paged_decode_attn(desc, num_seqs, num_q_heads, q, seq_lens, max_seq_len,
                               block_table, bt_stride, sm_scale, k_codes, k_params, v_codes,
                               v_params, out, scratch, kNoallocScratchBytes, err_flags, stream);
}
