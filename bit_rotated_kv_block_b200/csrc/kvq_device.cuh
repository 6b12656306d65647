// Device helpers shared by the libkvq kernels (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libkvq is written for sm_100a (B200) only"
#endif

namespace kvq {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// Packed binary32 pairs: each lane rounds as IEEE binary32 with
// round-to-nearest-even. A packed multiply may be fused with a following add
// by the code generator, so mul2 is only used where the product is exact
// (a power-of-two factor); products that must round on their own use
// __fmul_rn, which is never contracted.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint64_t pk(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 upk(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Packed fused multiply-add: one rounding of a*b + c per lane.
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// Mixed-precision add / subtract: widen the binary16 operand exactly, then
// one binary32 rounding (a + c, a - c).
__device__ __forceinline__ float add_h_f(__half a, float c) {
  float d;
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(__half_as_ushort(a)), "f"(c));
  return d;
}
__device__ __forceinline__ float sub_h_f(__half a, float c) {
  float d;
  asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(__half_as_ushort(a)), "f"(c));
  return d;
}

// Three-input minimum / maximum (exact, order-free).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Binary32 value nearest 1/sqrt(b) for b = 2^lg: 2^(-lg/2) for even lg,
// sqrt(2) * 2^(-(lg+1)/2) for odd lg (sqrt(2) rounded to binary32 is
// 0x3FB504F3; scaling by a power of two is exact).
__host__ __device__ __forceinline__ float hadamard_scale(int lg) {
  const float r2 = 1.41421353816986083984375f;  // binary32 nearest sqrt(2)
  float s = (lg & 1) ? r2 : 1.0f;
  int e = (lg & 1) ? (lg + 1) / 2 : lg / 2;
  for (int i = 0; i < e; ++i) s *= 0.5f;
  return s;
}

// ---------------------------------------------------------------------------
// Error flags
// ---------------------------------------------------------------------------

__device__ __forceinline__ void raise_flag(int32_t* flags, int32_t bit) {
  if (flags) atomicOr(flags, bit);
}

// ---------------------------------------------------------------------------
// Asynchronous global -> shared copies (16 bytes per thread, no staging
// through registers). The hardware tracks completion per commit group; no
// software spin-wait is involved.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
// 16 bytes of which the first `src_bytes` (0 or 16) are read from global
// memory and the rest zero-filled: a copy switched off without a branch
// (gmem_src must still be a valid address).
__device__ __forceinline__ void cp_async16_zf(void* smem_dst, const void* gmem_src,
                                              uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch. A kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream finishes;
// pdl_wait() then blocks until that kernel has completed and its writes are
// visible, so it must precede every read of memory another kernel may have
// written (it is a no-op for an ordinary launch). pdl_trigger() lets the next
// such launch be scheduled as soon as every CTA of this grid has started.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Bulk (TMA) copies global -> shared completing on an mbarrier. No multicast.
// Waits are bounded: after kMbarSpinLimit polls the caller gets `false` and
// must raise KVQ_ERRF_TIMEOUT instead of hanging.
// ---------------------------------------------------------------------------

constexpr uint32_t kMbarSpinLimit = 1u << 22;

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// true once the phase with the given parity has completed; false on timeout
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t it = 0; it < kMbarSpinLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
// Tiled TMA load of one 3-D box (coordinates in elements, innermost first)
// into shared memory, completing on an mbarrier. No multicast.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core MMA: D[16x8] (f32) += A[16x16] (f16) * B[16x8] (f16).
// Fragment ownership (lane = 4*r + j):
//   A: a[0] = (row r,   k 2j..2j+1)   a[1] = (row r+8, k 2j..2j+1)
//      a[2] = (row r,   k 2j+8..+9)   a[3] = (row r+8, k 2j+8..+9)
//   B: b[0] = (k 2j..2j+1, col r)     b[1] = (k 2j+8..+9, col r)
//   C: c[0..1] = (row r, cols 2j, 2j+1)  c[2..3] = (row r+8, cols 2j, 2j+1)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same product with a zero accumulator.
__device__ __forceinline__ void mma16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// Warp-level integer MMA: D[16x8] (s32) += A[16x32] (s8) * B[32x8] (u8).
// Fragment ownership (lane = 4*r + j), four 8-bit values per register:
//   A: a[0] = (row r,   k 4j..4j+3)     a[1] = (row r+8, k 4j..4j+3)
//      a[2] = (row r,   k 4j+16..+19)   a[3] = (row r+8, k 4j+16..+19)
//   B: b0 = (k 4j..4j+3, col r)         b1 = (k 4j+16..+19, col r)
//   C: c[0..1] = (row r, cols 2j, 2j+1)  c[2..3] = (row r+8, cols 2j, 2j+1)
// Integer accumulation is exact.
__device__ __forceinline__ void mma16832_s8u8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same product with a zero accumulator (the first k-step of a sum).
__device__ __forceinline__ void mma16832_s8u8_z(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

// INT4 -> binary16 by the exponent-bias ("magic number") method published for
// weight-only INT4 GEMM kernels (Kim et al., "Who Says Elephants Can't Run:
// Bringing Large Scale MoE Models into Cloud Scale Production", 2022): OR-ing
// a nibble into the mantissa of the binary16 value 1024 (0x6400) with one
// three-input logic operation gives 1024 + c exactly, and one subtraction or
// fused multiply-add removes the bias. The constants follow from the binary16
// format.
// Two codes (one channel of a token pair, selected by `mask` at bits 0-3 and
// 16-19, or at bits 4-7 and 20-23 when `high`) as the half2 (c - 8): they
// read 1024 + c (or 1024 + 16 c), and one subtraction of 1032 (or a multiply
// by 1/16 and an add of -72) leaves c - 8. Exact: every intermediate is an
// integer below 2048 or a multiple of 1/16 below 128 in binary16.
__device__ __forceinline__ uint32_t nib_c8(uint32_t z, uint32_t mask, int high) {
  uint32_t t;
  asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(t) : "r"(z), "r"(mask), "r"(0x64006400u));
  return high ? h2_as_u32(__hfma2(u32_as_h2(t), u32_as_h2(0x2C002C00u), u32_as_h2(0xD480D480u)))
              : h2_as_u32(__hsub2(u32_as_h2(t), u32_as_h2(0x64086408u)));
}

// ---------------------------------------------------------------------------
// Microscaling (MX) element conversions with the hardware's converters:
// round to nearest, ties to even, saturating at the largest finite value.
// The sign of each input is OR-ed into its code so that a negative value
// that rounds to zero is -0 whatever the converter does with it.
// ---------------------------------------------------------------------------

// Two binary32 values -> one byte of E2M1 codes, `lo` in bits 0-3.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return (r & 0xFFu) | ((__float_as_uint(lo) >> 31) << 3) | ((__float_as_uint(hi) >> 31) << 7);
}

// Two binary32 values -> two E4M3 bytes, `lo` in bits 0-7.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r | ((__float_as_uint(lo) >> 31) << 7) | ((__float_as_uint(hi) >> 31) << 15);
}

// One byte of two E2M1 codes (bits 0-3 and 4-7) -> the half2 of their values
// (bits 0-3 in the low half); exact.
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(byte));
  return r;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

}  // namespace kvq
