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

#include <cuda.h>
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

// In host code the array's name is only a host-side stand-in: its device
// address is looked up (cudaGetSymbolAddress) with the device current and
// remembered per device together with the unique id of the CUDA context it
// belongs to. A device reset, or a caller running in another context of the
// same device, gives a new id, and the address is looked up again instead of
// reusing one from a context that no longer holds the array.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

static void* driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// Unique id of the calling thread's current context; false if there is none
// yet (the runtime creates it on its first use) or the driver lacks the call.
static bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_ctx = reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent"));
  static CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_entry("cuCtxGetId"));
  if (get_ctx == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  unsigned long long ctx_id;  // context the address belongs to
  bool known;                 // ctx_id is valid
  void* addr;
};
static ScratchSlot g_scratch[kMaxDevices] = {};
static std::mutex g_scratch_mu;

static int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& sl = g_scratch[dev];
  if (sl.addr == nullptr || !have_id || !sl.known || sl.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return KVQ_ERR_CUDA;
    sl.addr = p;
    // the lookup made the runtime's context current if there was none
    sl.known = current_context_id(&sl.ctx_id);
  }
  *out = sl.addr;
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
  // every byte the decode kernels read from the scratch is written by the
  // same call first (the partial result of each split), so nothing left by
  // an earlier call needs clearing
  return kvq_paged_decode_attn(desc, num_seqs, num_q_heads, q, seq_lens, max_seq_len,
                               block_table, bt_stride, sm_scale, k_codes, k_params, v_codes,
                               v_params, out, scratch, kNoallocScratchBytes, err_flags, stream);
}
