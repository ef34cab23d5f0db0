// Shared device helpers for the CSA / HCA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

constexpr int kDQK = CSA_D_QK;     // 192
constexpr int kDNope = CSA_D_NOPE; // 128
constexpr int kDRope = CSA_D_ROPE; // 64
constexpr int kDV = CSA_D_V;       // 128
constexpr int kHI = CSA_H_I;       // 4
constexpr int kDI = CSA_D_I;       // 64
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy (L2 only); src_bytes = 0 zero-fills.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes = 16) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                        const void* smem) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(smem)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                          const void* smem) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(smem)));
}

// D += A(16x16, bf16, row) * B(16x8, bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// bf16 pair in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two E4M3 codes (low byte first) -> two bf16 in one word (exact: every E4M3
// value is representable in bf16).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t codes) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes), __NV_E4M3);
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  float2 f = __half22float2(hh);
  return pack_bf16x2(f.x, f.y);
}

// Four E4M3 codes (bytes 0..3) -> fp16 pairs (bytes 0,1) and (bytes 2,3),
// exactly (every E4M3 value, subnormals included, is an fp16 value).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t codes, uint32_t& lo, uint32_t& hi) {
  asm("{\n.reg .b16 l, h;\nmov.b32 {l, h}, %2;\ncvt.rn.f16x2.e4m3x2 %0, l;\ncvt.rn.f16x2.e4m3x2 %1, h;\n}\n"
      : "=r"(lo), "=r"(hi)
      : "r"(codes));
}

// One byte of E2M1 codes (OCP MX FP4: sign, 2 exponent bits with bias 1,
// 1 mantissa bit), the low nibble first -> an fp16 pair, the low nibble's
// value in the low half (every E2M1 value is an fp16 value: exact).  The byte
// is passed in the low 8 bits of a 16-bit register and narrowed to the 8-bit
// operand the conversion takes.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint16_t byte) {
  uint32_t r;
  asm("{\n.reg .b8 t;\ncvt.u8.u16 t, %1;\ncvt.rn.f16x2.e2m1x2 %0, t;\n}\n" : "=r"(r) : "h"(byte));
  return r;
}
// Two bytes of E2M1 codes -> fp16 pairs (byte 0's two values) and (byte 1's).
__device__ __forceinline__ void e2m1x4_to_f16x2x2(uint16_t two_bytes, uint32_t& lo, uint32_t& hi) {
  lo = e2m1x2_to_f16x2(static_cast<uint16_t>(two_bytes & 0xffu));
  hi = e2m1x2_to_f16x2(static_cast<uint16_t>(two_bytes >> 8));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void mma_f16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Programmatic dependent launch.  Every kernel of the library starts with
// pdl_wait() (returns once the previous kernel on the stream has completed and
// its memory is visible; a no-op when the launch carries no programmatic
// dependency), and each CTA calls pdl_trigger() once the rest of its work is
// short (at its start for small or multi-wave kernels, before the epilogue
// for the long single-wave ones), letting the next kernel's CTAs be scheduled
// and wait while this one finishes.  No global memory is touched before
// pdl_wait(), so the overlap never changes a result.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Order-preserving map float -> uint32 (larger float -> larger key).  -0 is
// folded onto +0 by the callers (s + 0.0f) so equal scores get equal keys.
__device__ __forceinline__ uint32_t f2key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Packed sequences: the largest s in [0, n) with cu[s] <= v (cu ascending,
// cu[0] <= v), i.e. the sequence that owns packed row v of offsets cu.  Empty
// sequences (equal consecutive offsets) are skipped over.
__device__ __forceinline__ int seq_of(const int32_t* cu, int n, int64_t v) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

namespace tc {
// Error word of the translation unit that includes this header: set when a
// bounded wait gives up (the kernel then finishes without trusting its data
// instead of hanging), or when a checked build finds an access out of bounds.
// Read back by the unit's device_error reader (CSA_DEFINE_DEVICE_ERROR_READER)
// and reported by csa_check_device_error.
static __device__ int g_device_error;
constexpr int kErrWaitTimeout = 1;
constexpr int kErrBounds = 4;
}  // namespace tc

// Checked builds (compiled with -DCSA_CHECKED): CSA_INBOUNDS(cond) records
// kErrBounds in the unit's error word when `cond` is false, and the access it
// guards is skipped.  In the normal build it is `true` and costs nothing.
__device__ __forceinline__ bool checked_ok(bool cond) {
  if (!cond) atomicOr(&tc::g_device_error, tc::kErrBounds);
  return cond;
}
#ifdef CSA_CHECKED
#define CSA_INBOUNDS(cond) (::csa::checked_ok(cond))
#else
#define CSA_INBOUNDS(cond) (true)
#endif

// Host reader of this unit's error word (defined once per .cu file).
#define CSA_DEFINE_DEVICE_ERROR_READER(fn)                                              \
  int fn(bool clear) {                                                                  \
    int word = 0;                                                                       \
    if (cudaMemcpyFromSymbol(&word, tc::g_device_error, sizeof(int)) != cudaSuccess)    \
      return -1;                                                                        \
    if (word && clear) {                                                                \
      const int zero = 0;                                                               \
      cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(int));                       \
    }                                                                                   \
    return word;                                                                        \
  }

__device__ __forceinline__ uint4 ldg_nc16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

}  // namespace csa
