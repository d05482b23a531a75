// quant.cu -- NVFP4 quantizers: tensor amax pass and the encode pass, for
// dense tensors (nvfp4_quantize) and for KV-cache chunks (nvfp4_kv_quant_chunk).
//
// Recipe (one IEEE binary32 operation per step, round to nearest even):
//   s_t = amax / 2688;  s_b = E4M3(amax_b / (6 s_t));  q = E2M1(x / (s_b s_t)).
// Format: E2M1 elements with an FP8 scale per 16-element block and an FP32
// tensor scale (neurohive.io LongLive-2.0 article, section "Ключевые
// компоненты LongLive-2.0"; tailorednewshub.com LongLive-2.0 article, section
// "Entrenamiento NVFP4").  KV chunks of up to 8 frames share one tensor scale
// (hyper.ai LongLive-2.0 summary, section "方法").
//
// Exact quotients without a division per element.  Every quotient of the
// recipe is x / d with d fixed for a tensor (d = RN(6 s_t)) or a block
// (d = RN(s_b s_t)); the kernels hold, per d, y = RN(1/d), y_rd = RD(1/d) and
// y_lo = RN((1 - d y_rd) y_rd), form q0 = RN(x y_rd + RN(x y_lo)), within one
// ulp of x / d, and correct it once with the exact remainder:
// q = RN(q0 + (x - d q0) y) = RN(x / d) (Markstein's theorem: a faithful
// quotient corrected with the correctly rounded reciprocal gives the correctly
// rounded quotient).  Quotients below 2^-10 may lose their last bits (the
// theorem assumes no underflow) but keep their sign and code to zero either
// way.  Exact ties on E2M1 or E4M3 rounding boundaries, frequent when the
// tensor scale has a short significand (an amax whose significand is a
// multiple of 21 makes s_t = amax / 2688 exact), need no special path.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

constexpr int kQuantThreads = 256;
constexpr int kAmaxUnroll = 4;  // blocks a thread of the amax pass loads at once

// Where the 8-element units of an input plane live.
struct InMap {
  const void* x;
  uint32_t units;   // elements / 8
  FastDiv upr;      // units per row   (cols / 8)
  FastDiv rpg;      // rows per group  (1 for a dense tensor, heads for KV)
  int64_t gstride;  // elements between groups (row stride / token stride)
  int64_t rstride;  // elements between rows of a group (0 / head_dim)
};

template <typename InT, bool kContig>
__device__ __forceinline__ const InT* unit_ptr(const InMap& m, uint32_t u) {
  if (kContig) return reinterpret_cast<const InT*>(m.x) + 8 * size_t(u);
  uint32_t row = fast_div(m.upr, u);
  uint32_t cu = u - row * m.upr.d;
  uint32_t g = fast_div(m.rpg, row);
  uint32_t r = row - g * m.rpg.d;
  return reinterpret_cast<const InT*>(m.x) + int64_t(g) * m.gstride + int64_t(r) * m.rstride +
         8 * int64_t(cu);
}

// 8 elements of one unit, as raw bits: bf16 -> 4 words, fp32 -> 8 words.
template <typename InT>
struct Raw;
template <>
struct Raw<__nv_bfloat16> {
  uint32_t w[4];
};
template <>
struct Raw<float> {
  uint32_t w[8];
};

// Loads are unconditional: a thread past the end loads the last block again
// (always a valid address) and discards it, which costs less than a branch
// around each load.
template <typename InT>
__device__ __forceinline__ void load_unit(const InT* p, Raw<InT>& r);
template <>
__device__ __forceinline__ void load_unit<__nv_bfloat16>(const __nv_bfloat16* p,
                                                         Raw<__nv_bfloat16>& r) {
  uint4 v = ld_nc_v4_l1(p);
  r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
}
template <>
__device__ __forceinline__ void load_unit<float>(const float* p, Raw<float>& r) {
  uint4 a = ld_nc_v4_l1(p);
  uint4 b = ld_nc_v4_l1(p + 4);
  r.w[0] = a.x; r.w[1] = a.y; r.w[2] = a.z; r.w[3] = a.w;
  r.w[4] = b.x; r.w[5] = b.y; r.w[6] = b.z; r.w[7] = b.w;
}

// max |x| of the 8 elements of a unit, as binary32 bits (NaN and Inf inputs
// give bits >= 0x7F800000, so they dominate the max).
template <typename InT>
__device__ __forceinline__ uint32_t unit_absmax(const Raw<InT>& r);
template <>
__device__ __forceinline__ uint32_t unit_absmax<__nv_bfloat16>(const Raw<__nv_bfloat16>& r) {
  const uint32_t m = __vmaxu2(__vmaxu2(r.w[0] & 0x7FFF7FFFu, r.w[1] & 0x7FFF7FFFu),
                              __vmaxu2(r.w[2] & 0x7FFF7FFFu, r.w[3] & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16) << 16;
}
template <>
__device__ __forceinline__ uint32_t unit_absmax<float>(const Raw<float>& r) {
  uint32_t mx = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) mx = max(mx, r.w[i] & 0x7FFFFFFFu);
  return mx;
}

// The 8 elements of a unit as binary32, sign included (bf16 -> binary32 is
// exact: the bf16 bits are the high half).
template <typename InT>
__device__ __forceinline__ void unit_values(const Raw<InT>& r, float a[8]);
template <>
__device__ __forceinline__ void unit_values<__nv_bfloat16>(const Raw<__nv_bfloat16>& r,
                                                           float a[8]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    a[2 * j] = __uint_as_float(r.w[j] << 16);
    a[2 * j + 1] = __uint_as_float(r.w[j] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void unit_values<float>(const Raw<float>& r, float a[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = __uint_as_float(r.w[i]);
}

// ---------------------------------------------------------------- block access
// A thread handles one 16-element block: two 8-element units.
template <typename InT, bool kContig>
__device__ __forceinline__ const InT* block_ptr(const InMap& m, uint32_t b) {
  if (kContig) return reinterpret_cast<const InT*>(m.x) + 16 * size_t(b);
  return unit_ptr<InT, kContig>(m, 2 * b);
}

template <typename InT>
struct RawBlock {
  Raw<InT> h[2];
};

template <typename InT>
__device__ __forceinline__ void load_block(const InT* p, RawBlock<InT>& r) {
  load_unit<InT>(p, r.h[0]);
  load_unit<InT>(p + 8, r.h[1]);
}

// ---------------------------------------------------------------- amax pass
struct AmaxArgs {
  InMap in[2];
  uint32_t* ws;  // workspace words
};

template <typename InT, bool kContig>
__global__ void __launch_bounds__(kQuantThreads) amax_kernel(AmaxArgs args) {
  pdl_wait();
  pdl_trigger();
  const int plane = blockIdx.y;
  const InMap m = plane == 0 ? args.in[0] : args.in[1];
  const uint32_t blocks = m.units >> 1;
  uint32_t mx = 0;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x; b0 < blocks;
       b0 += kAmaxUnroll * stride) {
    RawBlock<InT> raw[kAmaxUnroll];
#pragma unroll
    for (int i = 0; i < kAmaxUnroll; ++i) {
      const uint32_t b = b0 + i * stride;
      load_block<InT>(block_ptr<InT, kContig>(m, min(b, blocks - 1)), raw[i]);
    }
#pragma unroll
    for (int i = 0; i < kAmaxUnroll; ++i)
      mx = max(mx, max(unit_absmax<InT>(raw[i].h[0]), unit_absmax<InT>(raw[i].h[1])));
  }
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  __shared__ uint32_t warp_max[kQuantThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < kQuantThreads / 32 ? warp_max[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    if (threadIdx.x == 0 && v != 0) atomicMax(args.ws + (kWsAmax0 / 4) + plane, v);
  }
}

// ---------------------------------------------------------------- encode pass
// Division entry of a divisor d (see the file header).  The reciprocals are
// stored negated and the kernels divide -x: with the operands in this order a
// zero quotient keeps the dividend's sign, as IEEE division does (round to
// nearest adds opposite zeros to +0; here only zeros of one sign meet).
// y_lo >= 0 because y_rd <= 1/d.
struct DivEnt {
  float d, ny_rd, ny_lo, ny_rn;
};

__device__ __forceinline__ DivEnt div_entry(float d) {
  const float y_rd = __frcp_rd(d);
  const float rho = __fmaf_rn(-d, y_rd, 1.0f);  // 1 - d y_rd, exact
  DivEnt e;
  e.d = d;
  e.ny_rd = -y_rd;
  e.ny_lo = -__fmul_rn(rho, y_rd);
  e.ny_rn = -__frcp_rn(d);
  return e;
}

// RN(x / d), given nx = -x.
__device__ __forceinline__ float div_rn(const DivEnt& e, float nx) {
  const float q0 = __fmaf_rn(nx, e.ny_rd, __fmul_rn(nx, e.ny_lo));
  const float r = __fmaf_rn(e.d, q0, nx);  // d q0 - x, exact
  return __fmaf_rn(r, e.ny_rn, q0);
}

// The same for two dividends on the packed fp32 pipe.
__device__ __forceinline__ float2 div_rn2(const DivEnt& e, float2 nx) {
  const float2 q0 = __ffma2_rn(nx, make_float2(e.ny_rd, e.ny_rd),
                               __fmul2_rn(nx, make_float2(e.ny_lo, e.ny_lo)));
  const float2 r = __ffma2_rn(make_float2(e.d, e.d), q0, nx);
  return __ffma2_rn(r, make_float2(e.ny_rn, e.ny_rn), q0);
}

struct ScaleConsts {
  DivEnt c;  // divisor of the block scale: RN(top * s_t)
  float s_t;
  bool zero;
};

// Constants of the block-scale quotient amax_b / (top * s_t); top = 6 is the
// recipe, 4 the Four Over Six alternative.
__device__ __forceinline__ ScaleConsts make_consts(float s_t, float top = 6.0f) {
  ScaleConsts k;
  k.s_t = s_t;
  k.zero = (s_t == 0.0f);
  k.c = div_entry(__fmul_rn(top, s_t));
  return k;
}

// Division entries of d = RN(s_b s_t) for every scale byte (entry 0 and the
// NaN byte 0x7F are never used for codes), one CTA's copy in shared memory.
__device__ __forceinline__ void fill_div_table(DivEnt* tab, float s_t, uint32_t tid,
                                               uint32_t nthreads) {
  for (uint32_t b = tid; b < 128; b += nthreads)
    tab[b] = div_entry(__fmul_rn(e4m3_to_f32(b), s_t));
}

// The 8 elements of a unit negated, as binary32 (flipping the sign bits
// first; bf16 -> binary32 is exact).
template <typename InT>
__device__ __forceinline__ void unit_neg_values(const Raw<InT>& r, float a[8]);
template <>
__device__ __forceinline__ void unit_neg_values<__nv_bfloat16>(const Raw<__nv_bfloat16>& r,
                                                               float a[8]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w = r.w[j] ^ 0x80008000u;
    a[2 * j] = __uint_as_float(w << 16);
    a[2 * j + 1] = __uint_as_float(w & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void unit_neg_values<float>(const Raw<float>& r, float a[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = __uint_as_float(r.w[i] ^ 0x80000000u);
}

// The plane's tensor scale: s_t_in if given, else amax / 2688 with the amax
// the producer accumulated (amax_in) or the one this call's amax pass left in
// the workspace.  Every thread reads the word itself, so no thread waits for
// another before it starts encoding.
__device__ __forceinline__ float read_scale(const float* s_t_in, const float* amax_in,
                                            const uint32_t* ws, int plane) {
  if (s_t_in) return *s_t_in;
  const uint32_t* const word =
      amax_in ? reinterpret_cast<const uint32_t*>(amax_in) : ws + kWsAmax0 / 4 + plane;
  uint32_t bits;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(bits) : "l"(word) : "memory");
  return __fdiv_rn(__uint_as_float(bits), 2688.0f);
}

// Every CTA calls this once, after all of its threads have read the amax word
// (a CTA barrier first).  Thread 0 checks the CTA in on the plane's counter
// (release: the CTA's reads are ordered before the check-in); the CTA that
// checks in last (acquire: every other CTA's reads happened before) zeroes the
// amax word and the counter for the next call.  Nothing to do when the scale
// was handed in as s_t_in.
__device__ __forceinline__ void check_in(const float* s_t_in, float* amax_in, uint32_t* ws,
                                         int plane) {
  if (s_t_in) return;
  __syncthreads();
  if (threadIdx.x != 0) return;
  uint32_t* const word = amax_in ? reinterpret_cast<uint32_t*>(amax_in) : ws + kWsAmax0 / 4 + plane;
  uint32_t* const counter = ws + kWsCount0 / 4 + plane;
  uint32_t done;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
               : "=r"(done)
               : "l"(counter)
               : "memory");
  if (done == gridDim.x - 1) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(word) : "memory");
    asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(counter) : "memory");
  }
}

// Input blocks a thread keeps in flight while it encodes the ones it holds.
template <typename InT>
struct Prefetch {
  static constexpr int kDepth = 1;
};

// ---- dense tensors
struct QuantArgs {
  InMap in;
  uint8_t* codes;
  uint8_t* sf;
  float* s_t_out;
  const float* s_t_in;
  float* amax_in;
  uint32_t* ws;
  uint32_t nkb;          // blocks per row
  FastDiv nkb_div;
  uint32_t ktiles;       // ceil(nkb / 4)   (MMA layout)
  uint32_t rows;
  uint32_t rows_pad;     // rows rounded up to 128 (MMA layout)
};

__device__ __forceinline__ uint32_t sf_mma_offset(uint32_t row, uint32_t kb, uint32_t ktiles) {
  return ((row >> 7) * ktiles + (kb >> 2)) * 512u + (row & 31u) * 16u + ((row >> 5) & 3u) * 4u +
         (kb & 3u);
}

// Quantize one block held in `raw`: returns its scale byte and writes its two
// code words (all +0 when the scale is 0).  E2M1 is sign-magnitude and round
// to nearest even is symmetric, so the sign of x carries into the code, and a
// negative value that rounds to zero gives -0.
template <typename InT>
__device__ __forceinline__ uint32_t quantize_block(const RawBlock<InT>& raw, const DivEnt* tab,
                                                   const ScaleConsts& k, uint2& codes) {
  const uint32_t mx = max(unit_absmax<InT>(raw.h[0]), unit_absmax<InT>(raw.h[1]));
  const uint32_t sb =
      k.zero ? 0u : (e4m3x2(0.0f, div_rn(k.c, -__uint_as_float(mx))) & 0xFFu);
  const DivEnt e = tab[sb & 0x7Fu];
  float na[16], q[16];
  unit_neg_values<InT>(raw.h[0], na);
  unit_neg_values<InT>(raw.h[1], na + 8);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 v = div_rn2(e, make_float2(na[i], na[i + 1]));
    q[i] = v.x;
    q[i + 1] = v.y;
  }
  codes = sb ? make_uint2(e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]),
                          e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]))
             : make_uint2(0u, 0u);
  return sb;
}

// ---- Four Over Six (KV chunks)
// Magnitude of E2M1 code q (0..7): 0, .5, 1, 1.5, 2, 3, 4, 6, built from its
// bits (code 1 = 0.5; codes 2..7 = (1 + (q & 1) / 2) * 2^(q / 2 - 1)).
__device__ __forceinline__ float e2m1_magnitude(uint32_t q) {
  const uint32_t bits = q < 2 ? (q ? 0x3F000000u : 0u)
                              : ((126u + (q >> 1)) << 23) | ((q & 1u) << 22);
  return __uint_as_float(bits);
}

// The same squared error in binary32 (v(q) * s_b exact, then one rounding per
// operation).  Against the exact sum it is off by less than 2^-15.5 M^2 with
// M = 2 amax_b (each |x| and each decoded value is below M): per element the
// difference carries at most 2^-23 M, its square 2^-22 M^2 + 2^-24 M^2, and the
// 16 additions 16 * 2^-24 * 16 M^2.
__device__ __forceinline__ float block_sq_error_f32(const float a[16], uint2 codes, uint32_t sb,
                                                    float s_t) {
  const float sbv = e4m3_to_f32(sb & 0x7Fu);
  float e = 0.0f;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    const uint32_t q = ((t < 8 ? codes.x : codes.y) >> (4 * (t & 7))) & 7u;
    const float recon = __fmul_rn(__fmul_rn(e2m1_magnitude(q), sbv), s_t);
    const float diff = __fsub_rn(fabsf(a[t]), recon);
    e = __fadd_rn(e, __fmul_rn(diff, diff));
  }
  return e;
}

// Squared error of a block coded as (sb, codes) against the exactly decoded
// values: sum over the 16 elements, in order, of (|x| - v(|q|) * s_b * s_t)^2,
// each operation one binary64 rounding (explicit intrinsics: no contraction).
template <typename InT>
__device__ __forceinline__ double block_sq_error(const RawBlock<InT>& raw, uint2 codes,
                                                 uint32_t sb, float s_t) {
  float a[16];
  unit_values<InT>(raw.h[0], a);
  unit_values<InT>(raw.h[1], a + 8);
  const double sbv = double(e4m3_to_f32(sb & 0x7Fu));
  double e = 0.0;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    const uint32_t q = ((t < 8 ? codes.x : codes.y) >> (4 * (t & 7))) & 7u;
    double recon = __dmul_rn(double(e2m1_magnitude(q)), sbv);
    recon = __dmul_rn(recon, double(s_t));
    const double diff = __dsub_rn(double(fabsf(a[t])), recon);
    e = __dadd_rn(e, __dmul_rn(diff, diff));
  }
  return e;
}

// Out of line: the binary64 decision, for the rare blocks whose two binary32
// errors are too close to order safely.
template <typename InT>
__device__ __noinline__ bool four_beats_six_exact(const RawBlock<InT> raw, uint2 c4, uint32_t sb4,
                                                  uint2 c6, uint32_t sb6, float s_t) {
  return block_sq_error<InT>(raw, c4, sb4, s_t) < block_sq_error<InT>(raw, c6, sb6, s_t);
}

// A block under Four Over Six: coded both ways (maximum onto 6 with k6, onto
// 4 with k4), the one with the smaller squared error kept, 6 on a tie.  The
// errors are compared in binary32 when they differ by more than twice the
// binary32 error bound (2^-12 amax_b^2 > 2 * 2^-15.5 (2 amax_b)^2), where the
// order is certainly the binary64 one; otherwise in binary64.
template <typename InT>
__device__ __forceinline__ uint32_t quantize_block_4over6(const RawBlock<InT>& raw,
                                                          const DivEnt* tab,
                                                          const ScaleConsts& k6,
                                                          const ScaleConsts& k4, uint2& codes) {
  uint2 c6, c4;
  const uint32_t sb6 = quantize_block<InT>(raw, tab, k6, c6);
  const uint32_t sb4 = quantize_block<InT>(raw, tab, k4, c4);
  codes = c6;
  if (sb4 == sb6) return sb6;
  float a[16];
  unit_values<InT>(raw.h[0], a);
  unit_values<InT>(raw.h[1], a + 8);
  const float amax_b =
      __uint_as_float(max(unit_absmax<InT>(raw.h[0]), unit_absmax<InT>(raw.h[1])));
  const float e6 = block_sq_error_f32(a, c6, sb6, k6.s_t);
  const float e4 = block_sq_error_f32(a, c4, sb4, k6.s_t);
  const float margin = __fmul_rn(__fmul_rn(amax_b, amax_b), 0x1p-12f);
  const bool four = fabsf(__fsub_rn(e4, e6)) > margin
                        ? e4 < e6
                        : four_beats_six_exact<InT>(raw, c4, sb4, c6, sb6, k6.s_t);
  if (four) {
    codes = c4;
    return sb4;
  }
  return sb6;
}

// The dense quantizer.  Each thread encodes whole blocks (grid-stride over
// the tensor's blocks), loading the blocks of its next pass before it encodes
// the ones it holds; the first loads go out before the tensor scale is known.
template <typename InT, bool kContig, int kSfLayout>
__global__ void __launch_bounds__(kQuantThreads, 4) quant_kernel(QuantArgs args) {
  constexpr int D = Prefetch<InT>::kDepth;
  __shared__ DivEnt div_tab[128];
  pdl_wait();
  pdl_trigger();
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint32_t blocks = args.in.units >> 1;
  uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x;
  RawBlock<InT> cur[D];
#pragma unroll
  for (int i = 0; i < D; ++i) {
    const uint32_t b = b0 + i * stride;
    load_block<InT>(block_ptr<InT, kContig>(args.in, min(b, blocks - 1)), cur[i]);
  }
  const float s_t = read_scale(args.s_t_in, args.amax_in, args.ws, 0);
  const bool in_domain = tensor_scale_in_domain(s_t);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *args.s_t_out = s_t;
    if (!in_domain) record_status(args.ws + kWsStatus / 4, NVFP4_ERR_DOMAIN);
  }
  fill_div_table(div_tab, s_t, threadIdx.x, blockDim.x);
  __syncthreads();
  if (in_domain) {
    const ScaleConsts k = make_consts(s_t);
    for (; b0 < blocks; b0 += D * stride) {
      RawBlock<InT> nxt[D];
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const uint32_t b = b0 + (D + i) * stride;
        load_block<InT>(block_ptr<InT, kContig>(args.in, min(b, blocks - 1)), nxt[i]);
      }
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const uint32_t b = b0 + i * stride;
        if (b < blocks) {
          uint2 codes;
          const uint32_t sb = quantize_block<InT>(cur[i], div_tab, k, codes);
          reinterpret_cast<uint2*>(args.codes)[b] = codes;
          if (kSfLayout == NVFP4_SF_ROWMAJOR) {
            args.sf[b] = uint8_t(sb);
          } else {
            const uint32_t row = fast_div(args.nkb_div, b);
            args.sf[sf_mma_offset(row, b - row * args.nkb, args.ktiles)] = uint8_t(sb);
          }
        }
        cur[i] = nxt[i];
      }
    }
  }
  if (kSfLayout == NVFP4_SF_MMA128x4) {
    // zero the padding of the tensor-core scale layout: rows [rows, rows_pad)
    // and blocks [nkb, 4*ktiles) of real rows
    const uint32_t nkb4 = args.ktiles * 4u;
    const uint32_t pad_rows = (args.rows_pad - args.rows) * nkb4;
    const uint32_t pad_cols = args.rows * (nkb4 - args.nkb);
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < pad_rows + pad_cols;
         i += gridDim.x * blockDim.x) {
      uint32_t row, kb;
      if (i < pad_rows) {
        row = args.rows + i / nkb4;
        kb = i % nkb4;
      } else {
        uint32_t j = i - pad_rows, extra = nkb4 - args.nkb;
        row = j / extra;
        kb = args.nkb + j % extra;
      }
      args.sf[sf_mma_offset(row, kb, args.ktiles)] = 0;
    }
  }
  check_in(args.s_t_in, args.amax_in, args.ws, 0);
}

// ---- dense tensors with contiguous rows, staged through shared memory
// A resident grid of CTAs, each streaming one contiguous range of the tensor's
// blocks: warp 8 (one lane) fills a 4-stage shared-memory ring with 1-D bulk
// copies (16 KB a stage, completion counted on the stage's mbarrier), and
// warps 0..7 encode each stage's blocks out of shared memory while the next
// stages are in flight, so the load latency is hidden by the ring rather than
// by per-thread prefetch registers.  Each CTA's range is cut into equal parts
// so that every SM finishes at the same time.
constexpr int kTqConsumers = 256;                  // warps 0..7
constexpr int kTqThreads = kTqConsumers + 32;      // + the copy warp
constexpr int kTqStageBytes = 16384;
constexpr int kTqStages = 4;
constexpr int kTqSmem = kTqStages * kTqStageBytes + 2 * kTqStages * 8 + 128;

struct TmaQuantArgs {
  QuantArgs q;
  uint32_t per_cta;       // blocks per CTA (the last one may hold fewer)
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20000)
      : "memory");
  return ok != 0;
}

// Bounded wait on phase `parity` of `bar`: false (and NVFP4_ERR_TIMEOUT in the
// status word, and the CTA's abort flag raised) once limit_ns has passed, or
// at once when another thread of the CTA already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  while (true) {
    if (*abort) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (gtimer() - t0 > limit_ns) {
      record_status(status, NVFP4_ERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

template <typename InT, int kSfLayout>
__global__ void __launch_bounds__(kTqThreads) quant_tma_kernel(const TmaQuantArgs ta) {
  constexpr uint32_t kBlockBytes = 16 * sizeof(InT);
  constexpr uint32_t kStageBlocks = kTqStageBytes / kBlockBytes;
  const QuantArgs& args = ta.q;
  extern __shared__ __align__(128) uint8_t tq_smem[];
  __shared__ DivEnt div_tab[128];
  __shared__ int abort_flag;
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(tq_smem));
  const uint32_t bar_full = sbase + kTqStages * kTqStageBytes;
  const uint32_t bar_empty = bar_full + 8 * kTqStages;
  uint32_t* const status = args.ws + kWsStatus / 4;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTqStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_full + 8 * s) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_empty + 8 * s),
                   "r"(kTqConsumers / 32)
                   : "memory");
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const uint32_t blocks = args.in.units >> 1;
  const uint32_t b_lo = blockIdx.x * ta.per_cta;
  const uint32_t b_hi = min(blocks, b_lo + ta.per_cta);
  const uint32_t n_stages = b_hi > b_lo ? (b_hi - b_lo + kStageBlocks - 1) / kStageBlocks : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &abort_flag;

  if (warp == kTqConsumers / 32) {
    // ------------------------------------------------------------ copy warp
    if (lane == 0) {
      const uint8_t* src = static_cast<const uint8_t*>(args.in.x) + size_t(b_lo) * kBlockBytes;
      uint32_t k = 0;
      for (; k < n_stages; ++k) {
        const uint32_t s = k % kTqStages;
        if (!mbar_wait(bar_empty + 8 * s, ((k / kTqStages) & 1) ^ 1, ta.wait_limit_ns, abort,
                       status))
          break;
        const uint32_t n = min(kStageBlocks, b_hi - b_lo - k * kStageBlocks);
        const uint32_t bytes = n * kBlockBytes;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_full + 8 * s),
                     "r"(bytes)
                     : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
                "r"(sbase + s * kTqStageBytes),
            "l"(src + size_t(k) * kTqStageBytes), "r"(bytes), "r"(bar_full + 8 * s)
            : "memory");
      }
      // drain: every copy issued has landed before the CTA may leave
      for (uint32_t d = (k > kTqStages ? k - kTqStages : 0); d < k; ++d) {
        const uint32_t s = d % kTqStages;
        const uint64_t t0 = gtimer();
        while (!mbar_try_wait(bar_full + 8 * s, (d / kTqStages) & 1)) {
          if (gtimer() - t0 > 2000000000ull) {
            record_status(status, NVFP4_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ encoders
    const float s_t = read_scale(args.s_t_in, args.amax_in, args.ws, 0);
    const bool in_domain = tensor_scale_in_domain(s_t);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      *args.s_t_out = s_t;
      if (!in_domain) record_status(status, NVFP4_ERR_DOMAIN);
    }
    fill_div_table(div_tab, s_t, threadIdx.x, kTqConsumers);
    asm volatile("bar.sync 1, %0;" ::"n"(kTqConsumers) : "memory");  // encoders only
    const ScaleConsts kc = make_consts(s_t);
    for (uint32_t k = 0; k < n_stages; ++k) {
      const uint32_t s = k % kTqStages;
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar_full + 8 * s, (k / kTqStages) & 1,
                                                        ta.wait_limit_ns, abort, status));
      if (!ok) break;
      const uint32_t base = b_lo + k * kStageBlocks;
      const uint32_t n = min(kStageBlocks, b_hi - base);
      if (in_domain) {
#pragma unroll
        for (uint32_t r = 0; r < kStageBlocks / kTqConsumers; ++r) {
          const uint32_t i = threadIdx.x + r * kTqConsumers;
          if (i < n) {
            RawBlock<InT> raw;
            const uint32_t a = sbase + s * kTqStageBytes + i * kBlockBytes;
#pragma unroll
            for (uint32_t v = 0; v < kBlockBytes / 16; ++v) {
              uint32_t* w = reinterpret_cast<uint32_t*>(&raw) + 4 * v;
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                           : "r"(a + 16 * v));
            }
            uint2 codes;
            const uint32_t sb = quantize_block<InT>(raw, div_tab, kc, codes);
            const uint32_t b = base + i;
            reinterpret_cast<uint2*>(args.codes)[b] = codes;
            if (kSfLayout == NVFP4_SF_ROWMAJOR) {
              args.sf[b] = uint8_t(sb);
            } else {
              const uint32_t row = fast_div(args.nkb_div, b);
              args.sf[sf_mma_offset(row, b - row * args.nkb, args.ktiles)] = uint8_t(sb);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_empty + 8 * s)
                                  : "memory");
    }
    if (kSfLayout == NVFP4_SF_MMA128x4) {
      // zero the padding of the tensor-core scale layout: rows [rows, rows_pad)
      // and blocks [nkb, 4*ktiles) of real rows
      const uint32_t nkb4 = args.ktiles * 4u;
      const uint32_t pad_rows = (args.rows_pad - args.rows) * nkb4;
      const uint32_t pad_cols = args.rows * (nkb4 - args.nkb);
      for (uint32_t i = blockIdx.x * kTqConsumers + threadIdx.x; i < pad_rows + pad_cols;
           i += gridDim.x * kTqConsumers) {
        uint32_t row, kb;
        if (i < pad_rows) {
          row = args.rows + i / nkb4;
          kb = i % nkb4;
        } else {
          uint32_t j = i - pad_rows, extra = nkb4 - args.nkb;
          row = j / extra;
          kb = args.nkb + j % extra;
        }
        args.sf[sf_mma_offset(row, kb, args.ktiles)] = 0;
      }
    }
  }
  check_in(args.s_t_in, args.amax_in, args.ws, 0);
}

// ---- bf16 tensors whose rows are a multiple of 64 elements, tile by tile
// The tensor is cut into tiles of 128 rows x 64 columns: 16 KB of bf16, whose
// 128 x 4 scale bytes are exactly one 512-byte tile of the tensor-core scale
// layout.  A resident grid of CTAs takes equal runs of tiles (row-major tile
// order).  Warp 8 (one lane) loads each tile with one 2-D TMA copy (128-byte
// swizzle) into a 4-stage ring; warps 0..7 encode it.  Thread t takes row
// t / 2 and blocks 2 (t % 2), 2 (t % 2) + 1 of the tile (64 bytes of its row):
// its four 16-byte chunks sit at swizzled positions that differ across the 8
// threads of a quarter warp, so the shared-memory reads have no bank
// conflicts; the warp releases the stage once the chunks are in registers.
// The thread stores its 16 bytes of codes (the two threads of a row fill a
// 32-byte sector together) and its two scale bytes.  Rows past the end of the
// tensor arrive as zeros from the TMA copy: their scale bytes are the zero
// padding the tensor-core layout needs, and their codes are not stored.
constexpr int kTtConsumers = 256;
constexpr int kTtThreads = kTtConsumers + 32;
constexpr int kTtRows = 128;
constexpr int kTtStageBytes = kTtRows * 128;
constexpr int kTtStages = 4;
// ring (1024-byte aligned: the swizzle pattern repeats every 8 rows of 128 B),
// the barriers, and the alignment slack
constexpr int kTtSmem = kTtStages * kTtStageBytes + 2 * kTtStages * 8 + 1024;

struct TileQuantArgs {
  QuantArgs q;
  uint32_t n_ct;      // column tiles: cols / 64
  uint32_t n_tiles;   // row tiles * column tiles
  uint32_t per_cta;   // tiles per CTA (the first `extra` CTAs take one more)
  uint32_t extra;
  uint64_t wait_limit_ns;
};

// Division entry of a divisor with each value twice, for the packed fp32 pipe.
struct DivEnt2 {
  float2 d, ny_rd, ny_lo, ny_rn;
};

__device__ __forceinline__ float2 div_rn2(const DivEnt2& e, float2 nx) {
  const float2 q0 = __ffma2_rn(nx, e.ny_rd, __fmul2_rn(nx, e.ny_lo));
  const float2 r = __ffma2_rn(e.d, q0, nx);
  return __ffma2_rn(r, e.ny_rn, q0);
}

__device__ __forceinline__ DivEnt2 div_entry2(float d) {
  const DivEnt e = div_entry(d);
  DivEnt2 e2;
  e2.d = make_float2(e.d, e.d);
  e2.ny_rd = make_float2(e.ny_rd, e.ny_rd);
  e2.ny_lo = make_float2(e.ny_lo, e.ny_lo);
  e2.ny_rn = make_float2(e.ny_rn, e.ny_rn);
  return e2;
}

// max |x| over the 16 bf16 of a block (8 words), as binary32 bits: a tree of
// packed magnitude maxima (their signs are the xor of the operands' and are
// dropped at the end), then the larger half.
__device__ __forceinline__ uint32_t bf16_block_absmax(const uint32_t w[8]) {
  uint32_t m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[i]) : "r"(w[2 * i]), "r"(w[2 * i + 1]));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[0]) : "r"(m[0]), "r"(m[1]));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[2]) : "r"(m[2]), "r"(m[3]));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[0]) : "r"(m[0]), "r"(m[2]));
  const uint32_t a = m[0] & 0x7FFF7FFFu;
  uint32_t b;
  asm("max.u16x2 %0, %1, %2;" : "=r"(b) : "r"(a), "r"(prmt(a, 0u, 0x1032u)));
  return b << 16;
}

// Codes of one bf16 block (8 words) for a block with division entry e.
__device__ __forceinline__ uint2 bf16_block_codes(const uint32_t w[8], const DivEnt2& e) {
  float q[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // -x of both halves: the low half moved up with its sign bit flipped
    // (adding 2^31 flips bit 31), the high half masked and flipped
    const float2 nx = make_float2(__uint_as_float(w[j] * 0x10000u + 0x80000000u),
                                  __uint_as_float((w[j] & 0xFFFF0000u) ^ 0x80000000u));
    const float2 v = div_rn2(e, nx);
    q[2 * j] = v.x;
    q[2 * j + 1] = v.y;
  }
  return make_uint2(e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]),
                    e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]));
}

template <int kSfLayout>
__global__ void __launch_bounds__(kTtThreads) quant_tile_kernel(
    const __grid_constant__ CUtensorMap map_x, const TileQuantArgs ta) {
  const QuantArgs& args = ta.q;
  extern __shared__ uint8_t tt_smem[];
  __shared__ DivEnt2 div_tab[128];
  __shared__ int abort_flag;
  const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(tt_smem));
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint32_t bar_full = sbase + kTtStages * kTtStageBytes;
  const uint32_t bar_empty = bar_full + 8 * kTtStages;
  uint32_t* const status = args.ws + kWsStatus / 4;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTtStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_full + 8 * s) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_empty + 8 * s),
                   "r"(kTtConsumers / 32)
                   : "memory");
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x == kTtConsumers)
    asm volatile("prefetch.tensormap [%0];" ::"l"(&map_x) : "memory");
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const uint32_t t_lo = blockIdx.x * ta.per_cta + min(blockIdx.x, ta.extra);
  const uint32_t n_local = ta.per_cta + (blockIdx.x < ta.extra ? 1u : 0u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &abort_flag;

  if (warp == kTtConsumers / 32) {
    // ------------------------------------------------------------ TMA warp
    if (lane == 0) {
      uint32_t k = 0;
      for (; k < n_local; ++k) {
        const uint32_t s = k % kTtStages;
        if (!mbar_wait(bar_empty + 8 * s, ((k / kTtStages) & 1) ^ 1, ta.wait_limit_ns, abort,
                       status))
          break;
        const uint32_t tile = t_lo + k;
        const uint32_t rt = tile / ta.n_ct, ct = tile - rt * ta.n_ct;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_full + 8 * s),
                     "r"(kTtStageBytes)
                     : "memory");
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
            "[%0], [%1, {%2, %3}], [%4];" ::"r"(sbase + s * kTtStageBytes),
            "l"(&map_x), "r"(int32_t(ct * 64)), "r"(int32_t(rt * kTtRows)), "r"(bar_full + 8 * s)
            : "memory");
      }
      // drain: every copy issued has landed before the CTA may leave
      for (uint32_t d = (k > kTtStages ? k - kTtStages : 0); d < k; ++d) {
        const uint32_t s = d % kTtStages;
        const uint64_t t0 = gtimer();
        while (!mbar_try_wait(bar_full + 8 * s, (d / kTtStages) & 1)) {
          if (gtimer() - t0 > 2000000000ull) {
            record_status(status, NVFP4_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ encoders
    const uint32_t tid = threadIdx.x;
    const float s_t = read_scale(args.s_t_in, args.amax_in, args.ws, 0);
    const bool in_domain = tensor_scale_in_domain(s_t);
    if (blockIdx.x == 0 && tid == 0) {
      *args.s_t_out = s_t;
      if (!in_domain) record_status(status, NVFP4_ERR_DOMAIN);
    }
    if (tid < 128) div_tab[tid] = div_entry2(__fmul_rn(e4m3_to_f32(tid), s_t));
    asm volatile("bar.sync 1, %0;" ::"n"(kTtConsumers) : "memory");  // encoders only
    const DivEnt2 kc = div_entry2(__fmul_rn(6.0f, s_t));
    const bool zero = s_t == 0.0f;
    constexpr bool mma = kSfLayout == NVFP4_SF_MMA128x4;
    const uint32_t r = tid >> 1, h = tid & 1;
    // this thread's chunks (logical 4h .. 4h+3 of row r) in a stage
    uint32_t off[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) off[j] = r * 128u + (((4u * h + j) ^ (r & 7u)) << 4);
    const uint32_t sf_off = (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + 2u * h;
    const size_t row_bytes = size_t(args.nkb) * 8u;
    // the tile's row and column tile, advanced one tile per iteration
    uint32_t rt = t_lo / ta.n_ct, ct = t_lo - rt * ta.n_ct;
    for (uint32_t k = 0; k < n_local; ++k, ++ct) {
      if (ct == ta.n_ct) {
        ct = 0;
        ++rt;
      }
      const uint32_t s = k % kTtStages;
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar_full + 8 * s, (k / kTtStages) & 1,
                                                        ta.wait_limit_ns, abort, status));
      if (!ok) break;
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[4 * j]), "=r"(w[4 * j + 1]), "=r"(w[4 * j + 2]), "=r"(w[4 * j + 3])
                     : "r"(sbase + s * kTtStageBytes + off[j]));
      // The stage is released after the stores below: a store cannot issue
      // before the values it writes, and so the loads behind them, are
      // complete.  Released straight after the loads, the next TMA copy into
      // the stage could land before slow loads had read it (seen on B200 as
      // a few corrupted blocks in large tensors).
      auto release = [&]() {
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_empty + 8 * s)
                       : "memory");
      };
      if (!in_domain) {  // nothing is read from the stage
        release();
        continue;
      }
      const uint32_t am0 = bf16_block_absmax(w), am1 = bf16_block_absmax(w + 8);
      // both block scales at once: amax_b / RN(6 s_t), then E4M3 (block 0 in
      // the low byte)
      const float2 qs = div_rn2(kc, make_float2(-__uint_as_float(am0), -__uint_as_float(am1)));
      const uint32_t sb2 = zero ? 0u : e4m3x2(qs.y, qs.x);
      const uint32_t sb0 = sb2 & 0xFFu, sb1 = sb2 >> 8;
      uint2 c0 = bf16_block_codes(w, div_tab[sb0 & 0x7Fu]);
      uint2 c1 = bf16_block_codes(w + 8, div_tab[sb1 & 0x7Fu]);
      if (sb0 == 0) c0 = make_uint2(0u, 0u);
      if (sb1 == 0) c1 = make_uint2(0u, 0u);
      const uint32_t grow = rt * kTtRows + r;
      if (grow < args.rows) {
        st_v4(args.codes + size_t(grow) * row_bytes + ct * 32u + h * 16u,
              make_uint4(c0.x, c0.y, c1.x, c1.y));
        if (!mma)
          *reinterpret_cast<uint16_t*>(args.sf + size_t(grow) * args.nkb + ct * 4u + 2u * h) =
              uint16_t(sb2);
      }
      // tensor-core layout: tile (rt, ct) is scale tile rt * ktiles + ct =
      // t_lo + k (ktiles == n_ct), padding rows included
      if (mma)
        *reinterpret_cast<uint16_t*>(args.sf + size_t(t_lo + k) * 512u + sf_off) = uint16_t(sb2);
      release();
    }
  }
  check_in(args.s_t_in, args.amax_in, args.ws, 0);
}

// ---- KV-cache chunks (K and V planes in one launch, blockIdx.y)
struct KvQuantArgs {
  InMap in[2];
  uint8_t* codes[2];   // slot pools
  uint8_t* sf[2];
  float* st[2];
  float* amax_in[2];  // producer-accumulated amax per plane, or both null
  uint32_t* ws;
  uint32_t units_per_frame;
  FastDiv bpf_div;  // blocks per frame
  int32_t slots[NVFP4_KV_MAX_CHUNK_FRAMES];
  int32_t n_frames;
};

template <bool kContig, int kRule>
__global__ void __launch_bounds__(kQuantThreads, kRule == NVFP4_SCALE_ONTO_6 ? 4 : 3)
    kv_quant_kernel(KvQuantArgs args) {
  constexpr int D = Prefetch<__nv_bfloat16>::kDepth;
  __shared__ DivEnt div_tab[128];
  pdl_wait();
  pdl_trigger();
  const int plane = blockIdx.y;
  const InMap m = plane == 0 ? args.in[0] : args.in[1];
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint32_t blocks = m.units >> 1;
  uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x;
  RawBlock<__nv_bfloat16> cur[D];
#pragma unroll
  for (int i = 0; i < D; ++i) {
    const uint32_t b = b0 + i * stride;
    load_block<__nv_bfloat16>(block_ptr<__nv_bfloat16, kContig>(m, min(b, blocks - 1)),
                              cur[i]);
  }
  float* const amax_in = plane == 0 ? args.amax_in[0] : args.amax_in[1];
  const float s_t = read_scale(nullptr, amax_in, args.ws, plane);
  const bool in_domain = tensor_scale_in_domain(s_t);
  if (blockIdx.x == 0 && threadIdx.x < args.n_frames)
    args.st[plane][args.slots[threadIdx.x]] = s_t;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !in_domain)
    record_status(args.ws + kWsStatus / 4, NVFP4_ERR_DOMAIN);
  fill_div_table(div_tab, s_t, threadIdx.x, blockDim.x);
  __syncthreads();
  if (in_domain) {
    uint8_t* const codes_pool = plane == 0 ? args.codes[0] : args.codes[1];
    uint8_t* const sf_pool = plane == 0 ? args.sf[0] : args.sf[1];
    const ScaleConsts k = make_consts(s_t);
    const ScaleConsts k4 = make_consts(s_t, 4.0f);
    const uint32_t bpf = args.units_per_frame >> 1;  // blocks per frame
    for (; b0 < blocks; b0 += D * stride) {
      RawBlock<__nv_bfloat16> nxt[D];
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const uint32_t b = b0 + (D + i) * stride;
        load_block<__nv_bfloat16>(block_ptr<__nv_bfloat16, kContig>(m, min(b, blocks - 1)),
                                  nxt[i]);
      }
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const uint32_t b = b0 + i * stride;
        if (b < blocks) {
          uint2 codes;
          const uint32_t sb =
              kRule == NVFP4_SCALE_ONTO_6
                  ? quantize_block<__nv_bfloat16>(cur[i], div_tab, k, codes)
                  : quantize_block_4over6<__nv_bfloat16>(cur[i], div_tab, k, k4, codes);
          const uint32_t f = fast_div(args.bpf_div, b);
          const uint32_t bf = b - f * bpf;
          const size_t slot = size_t(args.slots[f]);
          reinterpret_cast<uint2*>(codes_pool + slot * bpf * 8)[bf] = codes;
          sf_pool[slot * bpf + bf] = uint8_t(sb);
        }
        cur[i] = nxt[i];
      }
    }
  }
  check_in(nullptr, amax_in, args.ws, plane);
}

// ---- KV chunks staged through shared memory (K and V planes: blockIdx.y)
// The chunk's tokens are rows of heads * head_dim contiguous elements at
// token_stride apart (a fused QKV output, or a plain [tokens][heads][dim]
// tensor).  As in quant_tma_kernel, a copy warp streams whole token rows (one
// 1-D bulk copy per row) through a 4-stage ring of 24 KB stages and eight
// warps encode them; each CTA takes an equal run of tokens of one plane.
constexpr int kKvStageBytes = 24576;
constexpr int kKvSmem = kTqStages * kKvStageBytes + 2 * kTqStages * 8 + 128;

struct KvTmaArgs {
  KvQuantArgs kv;
  const uint8_t* src[2];    // K, V: first element of token 0
  uint64_t token_bytes;     // bytes between tokens
  uint32_t row_blocks;      // 16-element blocks per token (heads * head_dim / 16)
  uint32_t rows;            // tokens in the chunk
  uint32_t rows_per_stage;
  uint32_t per_cta;         // tokens per CTA
  uint64_t wait_limit_ns;
};

template <int kRule>
__global__ void __launch_bounds__(kTqThreads) kv_quant_tma_kernel(const KvTmaArgs ta) {
  const KvQuantArgs& args = ta.kv;
  extern __shared__ __align__(128) uint8_t kq_smem[];
  __shared__ DivEnt div_tab[128];
  __shared__ int abort_flag;
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(kq_smem));
  const uint32_t bar_full = sbase + kTqStages * kKvStageBytes;
  const uint32_t bar_empty = bar_full + 8 * kTqStages;
  uint32_t* const status = args.ws + kWsStatus / 4;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTqStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_full + 8 * s) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_empty + 8 * s),
                   "r"(kTqConsumers / 32)
                   : "memory");
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const int plane = blockIdx.y;
  const uint32_t r_lo = blockIdx.x * ta.per_cta;
  const uint32_t r_hi = min(ta.rows, r_lo + ta.per_cta);
  const uint32_t rps = ta.rows_per_stage;
  const uint32_t n_stages = r_hi > r_lo ? (r_hi - r_lo + rps - 1) / rps : 0;
  const uint32_t row_bytes = ta.row_blocks * 32u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &abort_flag;
  float* const amax_in = plane == 0 ? args.amax_in[0] : args.amax_in[1];

  if (warp == kTqConsumers / 32) {
    // ------------------------------------------------------------ copy warp
    if (lane == 0) {
      const uint8_t* src = plane == 0 ? ta.src[0] : ta.src[1];
      uint32_t k = 0;
      for (; k < n_stages; ++k) {
        const uint32_t s = k % kTqStages;
        if (!mbar_wait(bar_empty + 8 * s, ((k / kTqStages) & 1) ^ 1, ta.wait_limit_ns, abort,
                       status))
          break;
        const uint32_t r0 = r_lo + k * rps;
        const uint32_t n = min(rps, r_hi - r0);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_full + 8 * s),
                     "r"(n * row_bytes)
                     : "memory");
        for (uint32_t i = 0; i < n; ++i)
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
              "[%3];" ::"r"(sbase + s * kKvStageBytes + i * row_bytes),
              "l"(src + size_t(r0 + i) * ta.token_bytes), "r"(row_bytes), "r"(bar_full + 8 * s)
              : "memory");
      }
      for (uint32_t d = (k > kTqStages ? k - kTqStages : 0); d < k; ++d) {
        const uint32_t s = d % kTqStages;
        const uint64_t t0 = gtimer();
        while (!mbar_try_wait(bar_full + 8 * s, (d / kTqStages) & 1)) {
          if (gtimer() - t0 > 2000000000ull) {
            record_status(status, NVFP4_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ encoders
    const float s_t = read_scale(nullptr, amax_in, args.ws, plane);
    const bool in_domain = tensor_scale_in_domain(s_t);
    if (blockIdx.x == 0 && threadIdx.x < args.n_frames)
      args.st[plane][args.slots[threadIdx.x]] = s_t;
    if (blockIdx.x == 0 && threadIdx.x == 0 && !in_domain) record_status(status, NVFP4_ERR_DOMAIN);
    fill_div_table(div_tab, s_t, threadIdx.x, kTqConsumers);
    asm volatile("bar.sync 1, %0;" ::"n"(kTqConsumers) : "memory");  // encoders only
    uint8_t* const codes_pool = plane == 0 ? args.codes[0] : args.codes[1];
    uint8_t* const sf_pool = plane == 0 ? args.sf[0] : args.sf[1];
    const ScaleConsts k6 = make_consts(s_t);
    const ScaleConsts k4 = make_consts(s_t, 4.0f);
    const uint32_t bpf = args.units_per_frame >> 1;  // blocks per frame
    for (uint32_t k = 0; k < n_stages; ++k) {
      const uint32_t s = k % kTqStages;
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar_full + 8 * s, (k / kTqStages) & 1,
                                                        ta.wait_limit_ns, abort, status));
      if (!ok) break;
      const uint32_t r0 = r_lo + k * rps;
      const uint32_t nb = min(rps, r_hi - r0) * ta.row_blocks;
      if (in_domain) {
        for (uint32_t i = threadIdx.x; i < nb; i += kTqConsumers) {
          RawBlock<__nv_bfloat16> raw;
          const uint32_t a = sbase + s * kKvStageBytes + i * 32u;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(raw.h[0].w[0]), "=r"(raw.h[0].w[1]), "=r"(raw.h[0].w[2]),
                         "=r"(raw.h[0].w[3])
                       : "r"(a));
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(raw.h[1].w[0]), "=r"(raw.h[1].w[1]), "=r"(raw.h[1].w[2]),
                         "=r"(raw.h[1].w[3])
                       : "r"(a + 16));
          uint2 codes;
          const uint32_t sb =
              kRule == NVFP4_SCALE_ONTO_6
                  ? quantize_block<__nv_bfloat16>(raw, div_tab, k6, codes)
                  : quantize_block_4over6<__nv_bfloat16>(raw, div_tab, k6, k4, codes);
          const uint32_t b = r0 * ta.row_blocks + i;   // block of the chunk
          const uint32_t f = fast_div(args.bpf_div, b);
          const uint32_t bf = b - f * bpf;
          const size_t slot = size_t(args.slots[f]);
          reinterpret_cast<uint2*>(codes_pool + slot * bpf * 8)[bf] = codes;
          sf_pool[slot * bpf + bf] = uint8_t(sb);
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_empty + 8 * s)
                                  : "memory");
    }
  }
  check_in(nullptr, amax_in, args.ws, plane);
}

// ---------------------------------------------------------------- launchers
// CTAs of `kernel` resident on one SM at once.
template <typename Kernel>
static int resident_per_sm(Kernel kernel) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kQuantThreads, 0) != cudaSuccess ||
      n < 1)
    n = 1;
  return n;
}

// CTAs per plane: enough for `per_thread` blocks per thread, at most one
// resident wave of the whole launch (all `planes` planes) so that no CTA
// waits for another to leave.
static int wave_grid(uint32_t units, uint32_t per_thread, int per_sm, int sm_count, int planes) {
  const uint64_t blocks = uint64_t(units) / 2;
  uint64_t want = (blocks + kQuantThreads * per_thread - 1) / (kQuantThreads * per_thread);
  uint64_t cap = uint64_t(per_sm) * uint64_t(sm_count) / uint64_t(planes);
  if (cap < 1) cap = 1;
  if (want < 1) want = 1;
  return int(want < cap ? want : cap);
}

template <typename InT, bool kContig>
static cudaError_t launch_amax(const AmaxArgs& aa, int planes, int sm_count, cudaStream_t st) {
  static const int per_sm = resident_per_sm(amax_kernel<InT, kContig>);
  const int grid = wave_grid(aa.in[0].units, 2, per_sm, sm_count, planes);
  return launch_pdl(amax_kernel<InT, kContig>, dim3(grid, planes), dim3(kQuantThreads), 0, st, aa);
}

template <typename InT, bool kContig, int kSfLayout>
static cudaError_t launch_encode(const QuantArgs& a, int sm_count, cudaStream_t st) {
  static const int per_sm = resident_per_sm(quant_kernel<InT, kContig, kSfLayout>);
  const int grid = wave_grid(a.in.units, 1, per_sm, sm_count, 1);
  return launch_pdl(quant_kernel<InT, kContig, kSfLayout>, dim3(grid), dim3(kQuantThreads), 0, st,
                    a);
}

template <bool kContig, int kRule>
static cudaError_t launch_kv_encode(const KvQuantArgs& a, int sm_count, cudaStream_t st) {
  static const int per_sm = resident_per_sm(kv_quant_kernel<kContig, kRule>);
  const int grid = wave_grid(a.in[0].units, 1, per_sm, sm_count, 2);
  return launch_pdl(kv_quant_kernel<kContig, kRule>, dim3(grid, 2), dim3(kQuantThreads), 0, st,
                    a);
}

static InMap make_inmap(const void* x, int64_t rows_total, int64_t cols, int64_t rows_per_group,
                        int64_t gstride, int64_t rstride) {
  InMap m;
  m.x = x;
  m.units = uint32_t(rows_total * cols / 8);
  m.upr = make_fastdiv(uint32_t(cols / 8));
  m.rpg = make_fastdiv(uint32_t(rows_per_group));
  m.gstride = gstride;
  m.rstride = rstride;
  return m;
}

// The staged quantizer: one resident wave, the blocks split evenly over it.
template <typename InT, int kSfLayout>
static cudaError_t launch_encode_tma(const QuantArgs& a, int sm_count, uint64_t wait_limit_ns,
                                     cudaStream_t st) {
  static std::atomic<int> per_sm_cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int per_sm = per_sm_cache[dev].load(std::memory_order_acquire);
  if (per_sm == 0) {
    cudaError_t e = cudaFuncSetAttribute(quant_tma_kernel<InT, kSfLayout>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kTqSmem);
    if (e != cudaSuccess) return e;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_tma_kernel<InT, kSfLayout>,
                                                      kTqThreads, kTqSmem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    per_sm_cache[dev].store(per_sm, std::memory_order_release);
  }
  constexpr uint32_t kStageBlocks = kTqStageBytes / (16 * sizeof(InT));
  const uint32_t blocks = a.in.units >> 1;
  // enough CTAs for one stage each, at most one resident wave
  uint32_t grid = (blocks + kStageBlocks - 1) / kStageBlocks;
  const uint32_t cap = uint32_t(per_sm) * uint32_t(sm_count);
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  TmaQuantArgs ta;
  ta.q = a;
  ta.per_cta = (blocks + grid - 1) / grid;
  ta.wait_limit_ns = wait_limit_ns;
  return launch_pdl(quant_tma_kernel<InT, kSfLayout>, dim3(grid), dim3(kTqThreads),
                    size_t(kTqSmem), st, ta);
}

// 2-D map over a bf16 tensor [rows][cols] with contiguous rows: box of 64
// columns (128 bytes) x 128 rows, 128-byte swizzle; rows past the end read as
// zeros.
static bool make_bf16_tile_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, uint32_t(kTtRows)};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tile quantizer: one resident wave, the tiles split evenly over it.
template <int kSfLayout>
static cudaError_t launch_encode_tile(const QuantArgs& a, const void* x, uint64_t rows,
                                      uint64_t cols, int sm_count, uint64_t wait_limit_ns,
                                      cudaStream_t st) {
  static std::atomic<int> per_sm_cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int per_sm = per_sm_cache[dev].load(std::memory_order_acquire);
  if (per_sm == 0) {
    cudaError_t e = cudaFuncSetAttribute(quant_tile_kernel<kSfLayout>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kTtSmem);
    if (e != cudaSuccess) return e;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_tile_kernel<kSfLayout>,
                                                      kTtThreads, kTtSmem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    per_sm_cache[dev].store(per_sm, std::memory_order_release);
  }
  CUtensorMap map;
  if (!make_bf16_tile_map(&map, x, rows, cols)) return cudaErrorInvalidValue;
  TileQuantArgs ta;
  ta.q = a;
  ta.n_ct = uint32_t(cols / 64);
  ta.n_tiles = uint32_t((rows + kTtRows - 1) / kTtRows) * ta.n_ct;
  uint32_t grid = uint32_t(per_sm) * uint32_t(sm_count);
  if (grid > ta.n_tiles) grid = ta.n_tiles;
  if (grid < 1) grid = 1;
  ta.per_cta = ta.n_tiles / grid;
  ta.extra = ta.n_tiles % grid;
  ta.wait_limit_ns = wait_limit_ns;
  return launch_pdl(quant_tile_kernel<kSfLayout>, dim3(grid), dim3(kTtThreads), size_t(kTtSmem),
                    st, map, ta);
}

template <int kRule>
static cudaError_t launch_kv_encode_tma(KvTmaArgs ta, int sm_count, cudaStream_t st) {
  static std::atomic<int> per_sm_cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int per_sm = per_sm_cache[dev].load(std::memory_order_acquire);
  if (per_sm == 0) {
    cudaError_t e = cudaFuncSetAttribute(kv_quant_tma_kernel<kRule>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem);
    if (e != cudaSuccess) return e;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kv_quant_tma_kernel<kRule>,
                                                      kTqThreads, kKvSmem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    per_sm_cache[dev].store(per_sm, std::memory_order_release);
  }
  // per plane: enough CTAs for one stage each, at most half a resident wave
  uint32_t grid = (ta.rows + ta.rows_per_stage - 1) / ta.rows_per_stage;
  uint32_t cap = uint32_t(per_sm) * uint32_t(sm_count) / 2;
  if (cap < 1) cap = 1;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  ta.per_cta = (ta.rows + grid - 1) / grid;
  return launch_pdl(kv_quant_tma_kernel<kRule>, dim3(grid, 2), dim3(kTqThreads), size_t(kKvSmem),
                    st, ta);
}

template <typename InT>
static cudaError_t launch_quant_t(const LaunchQuant& q, cudaStream_t st) {
  const bool contig = (q.ld == q.cols);
  InMap m = make_inmap(q.x, q.rows, q.cols, 1, q.ld, 0);
  if (!q.s_t_in && !q.amax_in) {
    AmaxArgs aa;
    aa.in[0] = m;
    aa.in[1] = m;
    aa.ws = static_cast<uint32_t*>(q.ws);
    const cudaError_t e = contig ? launch_amax<InT, true>(aa, 1, q.sm_count, st)
                                 : launch_amax<InT, false>(aa, 1, q.sm_count, st);
    if (e != cudaSuccess) return e;
  }
  QuantArgs a;
  a.in = m;
  a.codes = q.codes;
  a.sf = q.sf;
  a.s_t_out = q.s_t_out;
  a.s_t_in = q.s_t_in;
  a.amax_in = q.amax_in;
  a.ws = static_cast<uint32_t*>(q.ws);
  a.nkb = uint32_t(q.cols / 16);
  a.nkb_div = make_fastdiv(a.nkb);
  a.ktiles = (a.nkb + 3) / 4;
  a.rows = uint32_t(q.rows);
  a.rows_pad = uint32_t((q.rows + 127) / 128 * 128);
  const bool mma = q.sf_layout == NVFP4_SF_MMA128x4;
  // bf16 rows of a multiple of 64 elements at a 16-byte aligned address: the
  // tile kernel (2-D TMA copies)
  if (std::is_same<InT, __nv_bfloat16>::value && contig && q.cols % 64 == 0 &&
      reinterpret_cast<uintptr_t>(q.x) % 16 == 0)
    return mma ? launch_encode_tile<NVFP4_SF_MMA128x4>(a, q.x, uint64_t(q.rows), uint64_t(q.cols),
                                                       q.sm_count, q.wait_limit_ns, st)
               : launch_encode_tile<NVFP4_SF_ROWMAJOR>(a, q.x, uint64_t(q.rows), uint64_t(q.cols),
                                                       q.sm_count, q.wait_limit_ns, st);
  // other contiguous rows: the staged kernel (1-D bulk copies need 16-byte aligned
  // addresses, which the C ABI's checks guarantee)
  if (contig)
    return mma ? launch_encode_tma<InT, NVFP4_SF_MMA128x4>(a, q.sm_count, q.wait_limit_ns, st)
               : launch_encode_tma<InT, NVFP4_SF_ROWMAJOR>(a, q.sm_count, q.wait_limit_ns, st);
  return mma ? launch_encode<InT, false, NVFP4_SF_MMA128x4>(a, q.sm_count, st)
             : launch_encode<InT, false, NVFP4_SF_ROWMAJOR>(a, q.sm_count, st);
}

cudaError_t launch_quantize(const LaunchQuant& q, cudaStream_t st) {
  return q.dtype == NVFP4_BF16 ? launch_quant_t<__nv_bfloat16>(q, st) : launch_quant_t<float>(q, st);
}

cudaError_t launch_kv_quant(const LaunchKvQuant& q, cudaStream_t st) {
  const int64_t tokens = int64_t(q.n_frames) * q.tpf;
  const int64_t row_elems = int64_t(q.heads) * q.head_dim;
  const bool contig = (q.token_stride == row_elems);
  AmaxArgs aa;
  KvQuantArgs ka;
  const void* src[2] = {q.k, q.v};
  for (int p = 0; p < 2; ++p) {
    InMap m = make_inmap(src[p], tokens * q.heads, q.head_dim, q.heads, q.token_stride,
                         q.head_dim);
    aa.in[p] = m;
    ka.in[p] = m;
  }
  aa.ws = static_cast<uint32_t*>(q.ws);
  ka.ws = aa.ws;
  ka.codes[0] = q.k_codes; ka.codes[1] = q.v_codes;
  ka.sf[0] = q.k_sf; ka.sf[1] = q.v_sf;
  ka.st[0] = q.k_st; ka.st[1] = q.v_st;
  ka.amax_in[0] = q.k_amax_in; ka.amax_in[1] = q.v_amax_in;
  ka.units_per_frame = uint32_t(int64_t(q.tpf) * row_elems / 8);
  ka.bpf_div = make_fastdiv(ka.units_per_frame / 2);
  for (int f = 0; f < NVFP4_KV_MAX_CHUNK_FRAMES; ++f) ka.slots[f] = f < q.n_frames ? q.slots[f] : 0;
  ka.n_frames = q.n_frames;
  if (!q.k_amax_in) {
    const cudaError_t e = contig ? launch_amax<__nv_bfloat16, true>(aa, 2, q.sm_count, st)
                                 : launch_amax<__nv_bfloat16, false>(aa, 2, q.sm_count, st);
    if (e != cudaSuccess) return e;
  }
  const uint64_t row_bytes = uint64_t(row_elems) * 2;
  if (row_bytes <= uint64_t(kKvStageBytes)) {
    // token rows fit a stage: the staged kernel
    KvTmaArgs ta;
    ta.kv = ka;
    ta.src[0] = static_cast<const uint8_t*>(q.k);
    ta.src[1] = static_cast<const uint8_t*>(q.v);
    ta.token_bytes = uint64_t(q.token_stride) * 2;
    ta.row_blocks = uint32_t(row_elems / 16);
    ta.rows = uint32_t(tokens);
    ta.rows_per_stage = uint32_t(uint64_t(kKvStageBytes) / row_bytes);
    ta.wait_limit_ns = q.wait_limit_ns;
    return q.scale_rule == NVFP4_SCALE_FOUR_OVER_SIX
               ? launch_kv_encode_tma<NVFP4_SCALE_FOUR_OVER_SIX>(ta, q.sm_count, st)
               : launch_kv_encode_tma<NVFP4_SCALE_ONTO_6>(ta, q.sm_count, st);
  }
  if (q.scale_rule == NVFP4_SCALE_FOUR_OVER_SIX)
    return contig ? launch_kv_encode<true, NVFP4_SCALE_FOUR_OVER_SIX>(ka, q.sm_count, st)
                  : launch_kv_encode<false, NVFP4_SCALE_FOUR_OVER_SIX>(ka, q.sm_count, st);
  return contig ? launch_kv_encode<true, NVFP4_SCALE_ONTO_6>(ka, q.sm_count, st)
                : launch_kv_encode<false, NVFP4_SCALE_ONTO_6>(ka, q.sm_count, st);
}

}  // namespace nvfp4
