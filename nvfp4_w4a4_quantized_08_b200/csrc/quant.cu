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
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

constexpr int kQuantThreads = 256;
constexpr int kUnroll = 2;

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

template <typename InT>
__device__ __forceinline__ void load_unit(const InT* p, bool valid, Raw<InT>& r);
template <>
__device__ __forceinline__ void load_unit<__nv_bfloat16>(const __nv_bfloat16* p, bool valid,
                                                         Raw<__nv_bfloat16>& r) {
  uint4 v = valid ? ld_nc_v4_l1(p) : make_uint4(0, 0, 0, 0);
  r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
}
template <>
__device__ __forceinline__ void load_unit<float>(const float* p, bool valid, Raw<float>& r) {
  uint4 a = valid ? ld_nc_v4_l1(p) : make_uint4(0, 0, 0, 0);
  uint4 b = valid ? ld_nc_v4_l1(p + 4) : make_uint4(0, 0, 0, 0);
  r.w[0] = a.x; r.w[1] = a.y; r.w[2] = a.z; r.w[3] = a.w;
  r.w[4] = b.x; r.w[5] = b.y; r.w[6] = b.z; r.w[7] = b.w;
}

// |x| of the 8 elements as binary32, their max (as binary32 bits; NaN/Inf
// inputs give bits >= 0x7F800000) and the sign bits placed at bit 3 of each
// output nibble.
template <typename InT>
__device__ __forceinline__ uint32_t unpack_unit(const Raw<InT>& r, float a[8], uint32_t& signs);
template <>
__device__ __forceinline__ uint32_t unpack_unit<__nv_bfloat16>(const Raw<__nv_bfloat16>& r,
                                                               float a[8], uint32_t& signs) {
  uint32_t m[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    m[j] = r.w[j] & 0x7FFF7FFFu;
    a[2 * j] = __uint_as_float(m[j] << 16);
    a[2 * j + 1] = __uint_as_float(m[j] & 0xFFFF0000u);
  }
  uint32_t mx = __vmaxu2(__vmaxu2(m[0], m[1]), __vmaxu2(m[2], m[3]));
  mx = max(mx & 0xFFFFu, mx >> 16) << 16;
  // high bytes of the even elements (low halves) and of the odd elements
  uint32_t p01 = prmt(r.w[0], r.w[1], 0x7351);  // [w0.b1, w1.b1, w0.b3, w1.b3]
  uint32_t p23 = prmt(r.w[2], r.w[3], 0x7351);
  uint32_t even = prmt(p01, p23, 0x5410);  // sign of element 2j at bit 8j+7
  uint32_t odd = prmt(p01, p23, 0x7632);   // sign of element 2j+1 at bit 8j+7
  signs = ((even >> 4) & 0x08080808u) | (odd & 0x80808080u);
  return mx;
}
template <>
__device__ __forceinline__ uint32_t unpack_unit<float>(const Raw<float>& r, float a[8],
                                                       uint32_t& signs) {
  uint32_t mx = 0;
  signs = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t b = r.w[i] & 0x7FFFFFFFu;
    a[i] = __uint_as_float(b);
    mx = max(mx, b);
    signs |= (r.w[i] >> 31) << (4 * i + 3);
  }
  return mx;
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
__device__ __forceinline__ void load_block(const InT* p, bool valid, RawBlock<InT>& r) {
  load_unit<InT>(p, valid, r.h[0]);
  load_unit<InT>(p + 8, valid, r.h[1]);
}

// ---------------------------------------------------------------- amax pass
struct AmaxArgs {
  InMap in[2];
  uint32_t* ws;  // workspace words
};

template <typename InT, bool kContig>
__global__ void __launch_bounds__(kQuantThreads) amax_kernel(AmaxArgs args) {
  const int plane = blockIdx.y;
  const InMap m = plane == 0 ? args.in[0] : args.in[1];
  const uint32_t blocks = m.units >> 1;
  uint32_t mx = 0;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x; b0 < blocks;
       b0 += kUnroll * stride) {
    RawBlock<InT> raw[kUnroll];
#pragma unroll
    for (int i = 0; i < kUnroll; ++i) {
      const uint32_t b = b0 + i * stride;
      const bool valid = b < blocks;
      load_block<InT>(valid ? block_ptr<InT, kContig>(m, b) : nullptr, valid, raw[i]);
    }
#pragma unroll
    for (int i = 0; i < kUnroll; ++i) {
      float a[8];
      uint32_t signs;
      mx = max(mx, unpack_unit<InT>(raw[i].h[0], a, signs));
      mx = max(mx, unpack_unit<InT>(raw[i].h[1], a, signs));
    }
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

__device__ __forceinline__ ScaleConsts make_consts(float s_t) {
  ScaleConsts k;
  k.s_t = s_t;
  k.zero = (s_t == 0.0f);
  k.c = __fmul_rn(6.0f, s_t);
  float rc = k.zero ? 0.0f : __frcp_rn(k.c);
  k.rc_lo = __fmul_rn(rc, 1.0f - 0x1p-20f);
  k.rc_hi = __fmul_rn(rc, 1.0f + 0x1p-20f);
  k.inv_st = k.zero ? 0.0f : __frcp_rn(s_t);
  return k;
}

// E4M3 block scale of a block with amax amax_b: E4M3_RNE_sat(amax_b / c).
__device__ __forceinline__ uint32_t block_scale(float amax_b, const ScaleConsts& k) {
  uint32_t two = e4m3x2(__fmul_rn(amax_b, k.rc_hi), __fmul_rn(amax_b, k.rc_lo));
  uint32_t sb = two & 0xFFu;
  if (sb != (two >> 8)) sb = e4m3x2(0.0f, __fdiv_rn(amax_b, k.c)) & 0xFFu;
  return k.zero ? 0u : sb;
}

// Magnitude codes of the 16 elements of a block (|x| in a) for block scale
// byte sb: two 8-code words.
__device__ __forceinline__ void encode_block(const float a[16], uint32_t sb, float inv_sb,
                                             const ScaleConsts& k, uint32_t& c0, uint32_t& c1) {
  const float p = __fmul_rn(k.inv_st, inv_sb);
  const float p_lo = __fmul_rn(p, 1.0f - 0x1p-20f);
  const float p_hi = __fmul_rn(p, 1.0f + 0x1p-20f);
  float l[16], h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    l[i] = __fmul_rn(a[i], p_lo);
    h[i] = __fmul_rn(a[i], p_hi);
  }
  const uint32_t lo0 = e2m1x8(l[0], l[1], l[2], l[3], l[4], l[5], l[6], l[7]);
  const uint32_t lo1 = e2m1x8(l[8], l[9], l[10], l[11], l[12], l[13], l[14], l[15]);
  const uint32_t hi0 = e2m1x8(h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7]);
  const uint32_t hi1 = e2m1x8(h[8], h[9], h[10], h[11], h[12], h[13], h[14], h[15]);
  c0 = lo0;
  c1 = lo1;
  if ((lo0 != hi0) | (lo1 != hi1)) {
    // a quotient sits within the bracket of a rounding boundary: take it exactly
    const float d = __fmul_rn(e4m3_to_f32(sb), k.s_t);
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fdiv_rn(a[i], d);
    c0 = e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
    c1 = e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
  }
}

__device__ __forceinline__ void fill_inv_table(float* tab) {
  for (int b = threadIdx.x; b < 128; b += blockDim.x)
    tab[b] = (b == 0 || b == 0x7F) ? 0.0f : __frcp_rn(e4m3_to_f32(b));
}

// Resolve the tensor scale of plane `plane`: from s_t_in, or amax / 2688.
__device__ __forceinline__ float plane_scale(const float* s_t_in, const uint32_t* ws, int plane) {
  if (s_t_in) return *s_t_in;
  float amax = __uint_as_float(ws[kWsAmax0 / 4 + plane]);
  return __fdiv_rn(amax, 2688.0f);
}

// The last CTA of a plane to finish clears that plane's amax and counter,
// after every CTA of the plane has read the amax.
__device__ __forceinline__ void self_clean(uint32_t* ws, int plane) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    uint32_t done = atomicAdd(ws + kWsCount0 / 4 + plane, 1u);
    if (done == gridDim.x - 1) {
      atomicExch(ws + kWsAmax0 / 4 + plane, 0u);
      atomicExch(ws + kWsCount0 / 4 + plane, 0u);
    }
  }
}

// ---- dense tensors
struct QuantArgs {
  InMap in;
  uint8_t* codes;
  uint8_t* sf;
  float* s_t_out;
  const float* s_t_in;
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
// code words (sign bits included; all +0 when the scale is 0).
template <typename InT>
__device__ __forceinline__ uint32_t quantize_block(const RawBlock<InT>& raw, const float* inv_tab,
                                                   const ScaleConsts& k, uint2& codes) {
  float a[16];
  uint32_t s0, s1;
  const uint32_t mx = max(unpack_unit<InT>(raw.h[0], a, s0), unpack_unit<InT>(raw.h[1], a + 8, s1));
  const uint32_t sb = block_scale(__uint_as_float(mx), k);
  uint32_t c0, c1;
  encode_block(a, sb, inv_tab[sb & 0x7Fu], k, c0, c1);
  codes = sb ? make_uint2(c0 | s0, c1 | s1) : make_uint2(0u, 0u);
  return sb;
}

template <typename InT, bool kContig, int kSfLayout>
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(QuantArgs args) {
  __shared__ float inv_tab[128];
  fill_inv_table(inv_tab);
  __syncthreads();
  const float s_t = plane_scale(args.s_t_in, args.ws, 0);
  const bool in_domain = tensor_scale_in_domain(s_t);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *args.s_t_out = s_t;
    if (!in_domain) record_status(args.ws + kWsStatus / 4, NVFP4_ERR_DOMAIN);
  }
  if (in_domain) {
    const ScaleConsts k = make_consts(s_t);
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t blocks = args.in.units >> 1;
    for (uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x; b0 < blocks;
         b0 += kUnroll * stride) {
      RawBlock<InT> raw[kUnroll];
#pragma unroll
      for (int i = 0; i < kUnroll; ++i) {
        const uint32_t b = b0 + i * stride;
        const bool valid = b < blocks;
        load_block<InT>(valid ? block_ptr<InT, kContig>(args.in, b) : nullptr, valid, raw[i]);
      }
#pragma unroll
      for (int i = 0; i < kUnroll; ++i) {
        const uint32_t b = b0 + i * stride;
        if (b >= blocks) break;
        uint2 codes;
        const uint32_t sb = quantize_block<InT>(raw[i], inv_tab, k, codes);
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
  if (!args.s_t_in) self_clean(args.ws, 0);
}

// ---- KV-cache chunks (K and V planes in one launch, blockIdx.y)
struct KvQuantArgs {
  InMap in[2];
  uint8_t* codes[2];   // slot pools
  uint8_t* sf[2];
  float* st[2];
  uint32_t* ws;
  uint32_t units_per_frame;
  FastDiv bpf_div;  // blocks per frame
  int32_t slots[NVFP4_KV_MAX_CHUNK_FRAMES];
  int32_t n_frames;
};

template <bool kContig>
__global__ void __launch_bounds__(kQuantThreads) kv_quant_kernel(KvQuantArgs args) {
  __shared__ float inv_tab[128];
  fill_inv_table(inv_tab);
  __syncthreads();
  const int plane = blockIdx.y;
  const float s_t = plane_scale(nullptr, args.ws, plane);
  const bool in_domain = tensor_scale_in_domain(s_t);
  if (blockIdx.x == 0 && threadIdx.x < args.n_frames)
    args.st[plane][args.slots[threadIdx.x]] = s_t;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !in_domain)
    record_status(args.ws + kWsStatus / 4, NVFP4_ERR_DOMAIN);
  if (in_domain) {
    const InMap m = plane == 0 ? args.in[0] : args.in[1];
    uint8_t* const codes_pool = plane == 0 ? args.codes[0] : args.codes[1];
    uint8_t* const sf_pool = plane == 0 ? args.sf[0] : args.sf[1];
    const ScaleConsts k = make_consts(s_t);
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t blocks = m.units >> 1;
    const uint32_t bpf = args.units_per_frame >> 1;  // blocks per frame
    for (uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x; b0 < blocks;
         b0 += kUnroll * stride) {
      RawBlock<__nv_bfloat16> raw[kUnroll];
#pragma unroll
      for (int i = 0; i < kUnroll; ++i) {
        const uint32_t b = b0 + i * stride;
        const bool valid = b < blocks;
        load_block<__nv_bfloat16>(valid ? block_ptr<__nv_bfloat16, kContig>(m, b) : nullptr,
                                  valid, raw[i]);
      }
#pragma unroll
      for (int i = 0; i < kUnroll; ++i) {
        const uint32_t b = b0 + i * stride;
        if (b >= blocks) break;
        uint2 codes;
        const uint32_t sb = quantize_block<__nv_bfloat16>(raw[i], inv_tab, k, codes);
        const uint32_t f = fast_div(args.bpf_div, b);
        const uint32_t bf = b - f * bpf;
        const size_t slot = size_t(args.slots[f]);
        reinterpret_cast<uint2*>(codes_pool + slot * bpf * 8)[bf] = codes;
        sf_pool[slot * bpf + bf] = uint8_t(sb);
      }
    }
  }
  self_clean(args.ws, plane);
}

// ---------------------------------------------------------------- launchers
static int grid_for(uint32_t units, int sm_count) {
  const uint64_t blocks = uint64_t(units) / 2;
  uint64_t want = (blocks + kQuantThreads * kUnroll - 1) / (kQuantThreads * kUnroll);
  uint64_t cap = uint64_t(sm_count) * 8;
  if (want < 1) want = 1;
  return int(want < cap ? want : cap);
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

template <typename InT>
static cudaError_t launch_quant_t(const LaunchQuant& q, cudaStream_t st) {
  const bool contig = (q.ld == q.cols);
  InMap m = make_inmap(q.x, q.rows, q.cols, 1, q.ld, 0);
  const int grid = grid_for(m.units, q.sm_count);
  if (!q.s_t_in) {
    AmaxArgs aa;
    aa.in[0] = m;
    aa.in[1] = m;
    aa.ws = static_cast<uint32_t*>(q.ws);
    if (contig)
      amax_kernel<InT, true><<<dim3(grid, 1), kQuantThreads, 0, st>>>(aa);
    else
      amax_kernel<InT, false><<<dim3(grid, 1), kQuantThreads, 0, st>>>(aa);
  }
  QuantArgs a;
  a.in = m;
  a.codes = q.codes;
  a.sf = q.sf;
  a.s_t_out = q.s_t_out;
  a.s_t_in = q.s_t_in;
  a.ws = static_cast<uint32_t*>(q.ws);
  a.nkb = uint32_t(q.cols / 16);
  a.nkb_div = make_fastdiv(a.nkb);
  a.ktiles = (a.nkb + 3) / 4;
  a.rows = uint32_t(q.rows);
  a.rows_pad = uint32_t((q.rows + 127) / 128 * 128);
  const bool mma = q.sf_layout == NVFP4_SF_MMA128x4;
  if (contig) {
    if (mma) quant_kernel<InT, true, NVFP4_SF_MMA128x4><<<grid, kQuantThreads, 0, st>>>(a);
    else quant_kernel<InT, true, NVFP4_SF_ROWMAJOR><<<grid, kQuantThreads, 0, st>>>(a);
  } else {
    if (mma) quant_kernel<InT, false, NVFP4_SF_MMA128x4><<<grid, kQuantThreads, 0, st>>>(a);
    else quant_kernel<InT, false, NVFP4_SF_ROWMAJOR><<<grid, kQuantThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
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
  ka.units_per_frame = uint32_t(int64_t(q.tpf) * row_elems / 8);
  ka.bpf_div = make_fastdiv(ka.units_per_frame / 2);
  for (int f = 0; f < NVFP4_KV_MAX_CHUNK_FRAMES; ++f) ka.slots[f] = f < q.n_frames ? q.slots[f] : 0;
  ka.n_frames = q.n_frames;
  const int grid = grid_for(aa.in[0].units, q.sm_count);
  if (contig) {
    amax_kernel<__nv_bfloat16, true><<<dim3(grid, 2), kQuantThreads, 0, st>>>(aa);
    kv_quant_kernel<true><<<dim3(grid, 2), kQuantThreads, 0, st>>>(ka);
  } else {
    amax_kernel<__nv_bfloat16, false><<<dim3(grid, 2), kQuantThreads, 0, st>>>(aa);
    kv_quant_kernel<false><<<dim3(grid, 2), kQuantThreads, 0, st>>>(ka);
  }
  return cudaGetLastError();
}

}  // namespace nvfp4
