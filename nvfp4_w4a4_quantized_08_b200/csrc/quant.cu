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
// Exactness without a division per element.  Both roundings above are
// monotone, so a value's code is pinned once two products that bracket the
// correctly rounded quotient give the same code.  With r = RN(1/c) (c = 6 s_t)
// and p = RN(RN(1/s_t) * RN(1/s_b)), the products RN(a * RN(r (1 -+ 2^-20)))
// and RN(|x| * RN(p (1 -+ 2^-20))) lie below / above RN(a / c) and
// RN(|x| / RN(s_b s_t)): each carries at most six roundings of relative size
// 2^-24, far inside the 2^-20 margin.  Where the two codes differ (the quotient
// sits within ~2^-20 of an E4M3 or E2M1 rounding boundary, a few times in a
// million elements) the kernel takes the IEEE quotient itself.  Denormal
// products only arise for values far below the smallest decision point, where
// both bracket ends already give code 0.
#include <atomic>

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
struct ScaleConsts {
  float s_t, c, rc_lo, rc_hi, inv_st;
  bool zero;
};

// Constants of the block-scale division amax_b / (top * s_t); top = 6 is the
// recipe, 4 the Four Over Six alternative.
__device__ __forceinline__ ScaleConsts make_consts(float s_t, float top = 6.0f) {
  ScaleConsts k;
  k.s_t = s_t;
  k.zero = (s_t == 0.0f);
  k.c = __fmul_rn(top, s_t);
  float rc = k.zero ? 0.0f : __frcp_rn(k.c);
  k.rc_lo = __fmul_rn(rc, 1.0f - 0x1p-20f);
  k.rc_hi = __fmul_rn(rc, 1.0f + 0x1p-20f);
  k.inv_st = k.zero ? 0.0f : __frcp_rn(s_t);
  return k;
}

// The exact fallbacks below are out of line on purpose: inlined, the compiler
// predicates them into the common path, which then issues their divisions for
// every block.  A call is always a real branch.  They are not rare enough to
// ignore: bf16 inputs and a tensor scale derived from a bf16 amax put 0.1 to
// 1 percent of quotients exactly on (or within 2^-20 of) a rounding boundary,
// so a few percent of blocks, and most warps, meet one.
__device__ __noinline__ uint32_t e4m3_of_quotient(float a, float c) {
  return e4m3x2(0.0f, __fdiv_rn(a, c)) & 0xFFu;
}

__device__ __noinline__ uint32_t e2m1_of_quotient(float a, float d) {
  const float y = __fdiv_rn(a, d);
  return e2m1x8(y, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f) & 0xFu;
}

// E4M3 block scale of a block with amax amax_b: E4M3_RNE_sat(amax_b / c).
__device__ __forceinline__ uint32_t block_scale(float amax_b, const ScaleConsts& k) {
  uint32_t two = e4m3x2(__fmul_rn(amax_b, k.rc_hi), __fmul_rn(amax_b, k.rc_lo));
  uint32_t sb = two & 0xFFu;
  if (sb != (two >> 8)) sb = e4m3_of_quotient(amax_b, k.c);
  return k.zero ? 0u : sb;
}

// E2M1 codes of the 16 elements of a block (x in a) for block scale byte sb,
// from the two bracketing products: lo/hi code words of each half.  The codes
// carry the sign (E2M1 is sign-magnitude and rounding to nearest even is
// symmetric, so code(-y) = 8 | code(y); a negative value that rounds to zero
// gives -0).  Nibbles where lo and hi differ need the exact quotient.
__device__ __forceinline__ void bracket_codes(const float a[16], float inv_sb,
                                              const ScaleConsts& k, uint32_t lo[2],
                                              uint32_t hi[2]) {
  const float p = __fmul_rn(k.inv_st, inv_sb);
  const float p_lo = __fmul_rn(p, 1.0f - 0x1p-20f);
  const float p_hi = __fmul_rn(p, 1.0f + 0x1p-20f);
  // products on the packed fp32 pipe, two elements per instruction
  float l[16], h[16];
  const float2 plo2 = make_float2(p_lo, p_lo), phi2 = make_float2(p_hi, p_hi);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 ai = make_float2(a[i], a[i + 1]);
    const float2 vl = __fmul2_rn(ai, plo2), vh = __fmul2_rn(ai, phi2);
    l[i] = vl.x; l[i + 1] = vl.y;
    h[i] = vh.x; h[i + 1] = vh.y;
  }
  lo[0] = e2m1x8(l[0], l[1], l[2], l[3], l[4], l[5], l[6], l[7]);
  lo[1] = e2m1x8(l[8], l[9], l[10], l[11], l[12], l[13], l[14], l[15]);
  hi[0] = e2m1x8(h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7]);
  hi[1] = e2m1x8(h[8], h[9], h[10], h[11], h[12], h[13], h[14], h[15]);
}

// Element i (0..7) of a unit as binary32, selected without indexing the
// register array dynamically (which would move it to local memory).
template <typename InT>
__device__ __forceinline__ float elem_value(const Raw<InT>& r, uint32_t i);
template <>
__device__ __forceinline__ float elem_value<__nv_bfloat16>(const Raw<__nv_bfloat16>& r,
                                                           uint32_t i) {
  const uint32_t j = i >> 1;
  uint32_t w = r.w[0];
  w = j == 1 ? r.w[1] : w;
  w = j == 2 ? r.w[2] : w;
  w = j == 3 ? r.w[3] : w;
  return __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
}
template <>
__device__ __forceinline__ float elem_value<float>(const Raw<float>& r, uint32_t i) {
  uint32_t w = r.w[0];
#pragma unroll
  for (uint32_t j = 1; j < 8; ++j) w = i == j ? r.w[j] : w;
  return __uint_as_float(w);
}

// Replace the codes of a unit whose two bracket codes differ (nonzero nibbles
// of diff) by the codes of the IEEE quotients x / d, d = RN(s_b s_t).
template <typename InT>
__device__ __forceinline__ uint32_t patch_codes(const Raw<InT>& r, uint32_t c, uint32_t diff,
                                                float d) {
  while (diff) {
    const uint32_t sh = (__ffs(diff) - 1) & ~3u;
    c = (c & ~(0xFu << sh)) | (e2m1_of_quotient(elem_value<InT>(r, sh >> 2), d) << sh);
    diff &= ~(0xFu << sh);
  }
  return c;
}

__device__ __forceinline__ void fill_inv_table(float* tab) {
  for (int b = threadIdx.x; b < 128; b += blockDim.x)
    tab[b] = (b == 0 || b == 0x7F) ? 0.0f : __frcp_rn(e4m3_to_f32(b));
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
// code words (all +0 when the scale is 0).
template <typename InT>
__device__ __forceinline__ uint32_t quantize_block(const RawBlock<InT>& raw, const float* inv_tab,
                                                   const ScaleConsts& k, uint2& codes) {
  uint32_t sb, lo[2], hi[2];
  {
    const uint32_t mx = max(unit_absmax<InT>(raw.h[0]), unit_absmax<InT>(raw.h[1]));
    sb = block_scale(__uint_as_float(mx), k);
    float a[16];
    unit_values<InT>(raw.h[0], a);
    unit_values<InT>(raw.h[1], a + 8);
    bracket_codes(a, inv_tab[sb & 0x7Fu], k, lo, hi);
  }
  const uint32_t diff0 = lo[0] ^ hi[0], diff1 = lo[1] ^ hi[1];
  if (diff0 | diff1) {
    const float d = __fmul_rn(e4m3_to_f32(sb), k.s_t);
    lo[0] = patch_codes<InT>(raw.h[0], lo[0], diff0, d);
    lo[1] = patch_codes<InT>(raw.h[1], lo[1], diff1, d);
  }
  codes = sb ? make_uint2(lo[0], lo[1]) : make_uint2(0u, 0u);
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
                                                          const float* inv_tab,
                                                          const ScaleConsts& k6,
                                                          const ScaleConsts& k4, uint2& codes) {
  uint2 c6, c4;
  const uint32_t sb6 = quantize_block<InT>(raw, inv_tab, k6, c6);
  const uint32_t sb4 = quantize_block<InT>(raw, inv_tab, k4, c4);
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
  __shared__ float inv_tab[128];
  fill_inv_table(inv_tab);
  __syncthreads();
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
          const uint32_t sb = quantize_block<InT>(cur[i], inv_tab, k, codes);
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
  __shared__ float inv_tab[128];
  __shared__ int abort_flag;
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(tq_smem));
  const uint32_t bar_full = sbase + kTqStages * kTqStageBytes;
  const uint32_t bar_empty = bar_full + 8 * kTqStages;
  uint32_t* const status = args.ws + kWsStatus / 4;
  fill_inv_table(inv_tab);
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
            const uint32_t sb = quantize_block<InT>(raw, inv_tab, kc, codes);
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
  __shared__ float inv_tab[128];
  fill_inv_table(inv_tab);
  __syncthreads();
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
                  ? quantize_block<__nv_bfloat16>(cur[i], inv_tab, k, codes)
                  : quantize_block_4over6<__nv_bfloat16>(cur[i], inv_tab, k, k4, codes);
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
  __shared__ float inv_tab[128];
  __shared__ int abort_flag;
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(kq_smem));
  const uint32_t bar_full = sbase + kTqStages * kKvStageBytes;
  const uint32_t bar_empty = bar_full + 8 * kTqStages;
  uint32_t* const status = args.ws + kWsStatus / 4;
  fill_inv_table(inv_tab);
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
                  ? quantize_block<__nv_bfloat16>(raw, inv_tab, k6, codes)
                  : quantize_block_4over6<__nv_bfloat16>(raw, inv_tab, k6, k4, codes);
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
  // contiguous rows: the staged kernel (1-D bulk copies need 16-byte aligned
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
