// common.cuh -- device helpers shared by the libnvfp4 kernels (sm_100a).
//
// Format conversions use the documented PTX cvt forms for E2M1 / E4M3 /
// bf16 (round to nearest even, saturating to the largest finite value).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <utility>
#include <stdint.h>

#include "../../include/nvfp4.h"

namespace nvfp4 {

// ---------------------------------------------------------------- workspace
// Byte offsets of the scratch words inside the caller's workspace.  The amax
// and counter words return to zero at the end of every call that uses them.
constexpr int kWsAmax0 = 0;    // u32: bits of max|x| (plain tensor, or K)
constexpr int kWsAmax1 = 4;    // u32: bits of max|x| of V
constexpr int kWsCount0 = 8;   // u32: CTAs done with plane 0
constexpr int kWsCount1 = 12;  // u32: CTAs done with plane 1
constexpr int kWsStatus = 16;  // u32: first device-side error (nvfp4_status)
constexpr size_t kWsBytes = 256;

__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code) {
  atomicCAS(status, 0u, code);
}

// Tensor scales the recipe accepts: 0, or [2^-108, 2^100].  Keeps every
// intermediate of the scale arithmetic (6*s_t, s_b*s_t, 1/s_t, 1/(s_b*s_t))
// a normal binary32 number.
__host__ __device__ __forceinline__ bool tensor_scale_in_domain(float s_t) {
  return s_t == 0.0f || (s_t >= 0x1p-108f && s_t <= 0x1p100f);
}

// ---------------------------------------------------------------- division
// Unsigned 32-bit division by an invariant divisor d >= 1 (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994,
// section 4): with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
// n / d = (mulhi(m, n) + n) >> l for every 32-bit n (33-bit sum kept).
struct FastDiv {
  uint32_t d, m, l;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t l = 0;
  while ((uint64_t(1) << l) < d) ++l;
  f.l = l;
  f.m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1);
  return f;
}

__device__ __forceinline__ uint32_t fast_div(const FastDiv& f, uint32_t n) {
  uint32_t hi = __umulhi(n, f.m);
  return uint32_t((uint64_t(hi) + n) >> f.l);
}

// ---------------------------------------------------------------- formats
// Eight binary32 values -> eight E2M1 codes (sign bit 3) packed little-endian
// (value i in nibble i).  cvt.e2m1x2 puts its first source in the high nibble.
__device__ __forceinline__ uint32_t e2m1x8(float y0, float y1, float y2, float y3, float y4,
                                           float y5, float y6, float y7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "f"(y4), "f"(y5), "f"(y6), "f"(y7));
  return out;
}

// Two binary32 values -> E4M3 bytes (RNE, saturating): lo in bits 0..7, hi in 8..15.
__device__ __forceinline__ uint32_t e4m3x2(float hi, float lo) {
  unsigned short h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
  return h;
}

// E4M3 byte (finite) -> binary32, exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  unsigned short h = (unsigned short)(byte & 0xFF);
  uint32_t f16x2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(f16x2) : "h"(h));
  return __half2float(__ushort_as_half((unsigned short)(f16x2 & 0xFFFF)));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// ---------------------------------------------------------------- loads
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Read-only 16-byte load that may allocate in L1 (for a thread reading a
// 32-byte block in two halves: the second half then hits L1).
__device__ __forceinline__ uint4 ld_nc_v4_l1(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------- launches
// Programmatic dependent launch: every kernel of this library is launched so
// that it may start while the previous kernel on the stream finishes; it
// runs only its on-chip prologue before pdl_wait(), which returns once every
// earlier grid on the stream has completed and its memory is visible.  Then
// pdl_trigger() lets the next launch start the same way.  Without the launch
// attribute both instructions do nothing.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// 32-byte store (sm_100 256-bit access); p must be 32-byte aligned.
__device__ __forceinline__ void st_v8(void* p, uint4 a, uint4 b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x),
               "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// 32-byte read-only load (sm_100 256-bit access); p must be 32-byte aligned.
__device__ __forceinline__ void ld_nc_v8(const void* p, uint4& a, uint4& b) {
  asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z),
                 "=r"(b.w)
               : "l"(p));
}

}  // namespace nvfp4
