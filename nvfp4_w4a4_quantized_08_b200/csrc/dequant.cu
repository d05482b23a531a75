// dequant.cu -- NVFP4 -> bf16 for dense tensors (nvfp4_dequantize) and the
// KV-cache window rebuild (nvfp4_kv_dequant_window).
//
// Every element is bf16_RNE((v(q) * s_b) * s_t): v(q) * s_b is exact in
// binary32, the product with s_t one rounding, then one bf16 rounding.  A block
// of 16 elements shares s_b and s_t, so it has only 8 distinct magnitudes: the
// kernel computes those 8 bf16 values once per block and maps the 16 codes
// through them with byte permutes, then ORs in each code's sign bit.
//
// The window rebuild is the "custom parallel CUDA dequantization kernel" of the
// hyper.ai LongLive-2.0 summary (section "方法"): it turns the NVFP4 slots of
// the sink and window frames (171host.com LongLive 2.0 teardown, section 2.2)
// back into contiguous bf16 K and V for attention.
#include "common.cuh"
#include "decode.cuh"
#include "kernels.h"

namespace nvfp4 {

constexpr int kDqThreads = 256;
constexpr int kDqUnroll = 2;

__device__ __forceinline__ uint32_t sf_mma_offset_dq(uint32_t row, uint32_t kb, uint32_t ktiles) {
  return ((row >> 7) * ktiles + (kb >> 2)) * 512u + (row & 31u) * 16u + ((row >> 5) & 3u) * 4u +
         (kb & 3u);
}

struct DequantArgs {
  const uint8_t* codes;
  const uint8_t* sf;
  const float* s_t;
  uint8_t* out;       // bf16
  int64_t ld;         // elements
  uint32_t blocks;    // rows * nkb
  uint32_t nkb;
  FastDiv nkb_div;
  uint32_t ktiles;
};

// Store one decoded block (32 bytes): one 256-bit store when the destination
// is 32-byte aligned (a warp then writes whole sectors), else two 128-bit ones.
template <bool kWide>
__device__ __forceinline__ void store_block(uint8_t* dst, uint4 lo, uint4 hi) {
  if (kWide) {
    st_v8(dst, lo, hi);
  } else {
    st_v4(dst, lo);
    st_v4(dst + 16, hi);
  }
}

// A thread decodes whole blocks (8 code bytes in, 32 bytes out), kDqUnroll
// of them per pass with all their loads issued first.  Threads past the end
// load the last block again and store nothing.
template <int kSfLayout, bool kContig, bool kWide>
__global__ void __launch_bounds__(kDqThreads) dequant_kernel(DequantArgs a) {
  pdl_wait();
  pdl_trigger();
  const float s_t = *a.s_t;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x; b0 < a.blocks;
       b0 += kDqUnroll * stride) {
    uint2 c[kDqUnroll];
    uint32_t sb[kDqUnroll], row[kDqUnroll], kb[kDqUnroll];
#pragma unroll
    for (int i = 0; i < kDqUnroll; ++i) {
      const uint32_t b = min(b0 + i * stride, a.blocks - 1);
      row[i] = fast_div(a.nkb_div, b);
      kb[i] = b - row[i] * a.nkb;
      c[i] = __ldg(reinterpret_cast<const uint2*>(a.codes) + b);
      const uint32_t off =
          kSfLayout == NVFP4_SF_ROWMAJOR ? b : sf_mma_offset_dq(row[i], kb[i], a.ktiles);
      sb[i] = __ldg(a.sf + off);
    }
#pragma unroll
    for (int i = 0; i < kDqUnroll; ++i) {
      const uint32_t b = b0 + i * stride;
      if (b >= a.blocks) break;
      const BlockLut l = make_lut(sb[i], s_t);
      uint8_t* dst = kContig ? a.out + 32 * size_t(b)
                             : a.out + 2 * (int64_t(row[i]) * a.ld + 16 * int64_t(kb[i]));
      store_block<kWide>(dst, decode8(l, c[i].x), decode8(l, c[i].y));
    }
  }
}

struct KvDequantArgs {
  const uint8_t* codes[2];
  const uint8_t* sf[2];
  const float* st[2];
  uint8_t* out[2];
  uint32_t blocks;            // n * blocks_per_frame
  uint32_t blocks_per_frame;
  FastDiv bpf_div;
  int32_t slots[NVFP4_KV_MAX_WINDOW_SLOTS];
};

template <bool kWide>
__global__ void __launch_bounds__(kDqThreads) kv_dequant_kernel(KvDequantArgs a) {
  pdl_wait();
  pdl_trigger();
  const int plane = blockIdx.y;
  const uint8_t* codes = plane == 0 ? a.codes[0] : a.codes[1];
  const uint8_t* sfp = plane == 0 ? a.sf[0] : a.sf[1];
  const float* stp = plane == 0 ? a.st[0] : a.st[1];
  uint8_t* out = plane == 0 ? a.out[0] : a.out[1];
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x; b0 < a.blocks;
       b0 += kDqUnroll * stride) {
    uint2 c[kDqUnroll];
    uint32_t sb[kDqUnroll];
    float st[kDqUnroll];
#pragma unroll
    for (int i = 0; i < kDqUnroll; ++i) {
      const uint32_t b = min(b0 + i * stride, a.blocks - 1);
      const uint32_t j = fast_div(a.bpf_div, b);  // position in the slot list
      const uint32_t bf = b - j * a.blocks_per_frame;
      const size_t s = size_t(a.slots[j]);
      const size_t src = s * a.blocks_per_frame + bf;
      c[i] = __ldg(reinterpret_cast<const uint2*>(codes) + src);
      sb[i] = __ldg(sfp + src);
      st[i] = __ldg(stp + s);
    }
#pragma unroll
    for (int i = 0; i < kDqUnroll; ++i) {
      const uint32_t b = b0 + i * stride;
      if (b >= a.blocks) break;
      const BlockLut l = make_lut(sb[i], st[i]);
      store_block<kWide>(out + 32 * size_t(b), decode8(l, c[i].x), decode8(l, c[i].y));
    }
  }
}

// CTAs per plane: kDqUnroll blocks per thread, at most one resident wave.
template <typename Kernel>
static int dq_grid(Kernel kernel, uint32_t blocks, int sm_count, int planes) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kDqThreads, 0) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  uint64_t want = (uint64_t(blocks) + kDqThreads * kDqUnroll - 1) / (kDqThreads * kDqUnroll);
  uint64_t cap = uint64_t(per_sm) * uint64_t(sm_count) / uint64_t(planes);
  if (cap < 1) cap = 1;
  if (want < 1) want = 1;
  return int(want < cap ? want : cap);
}

cudaError_t launch_dequantize(const LaunchDequant& d, cudaStream_t st) {
  DequantArgs a;
  a.codes = d.codes;
  a.sf = d.sf;
  a.s_t = d.s_t;
  a.out = static_cast<uint8_t*>(d.out);
  a.ld = d.ld;
  a.nkb = uint32_t(d.cols / 16);
  a.blocks = uint32_t(d.rows * a.nkb);
  a.nkb_div = make_fastdiv(a.nkb);
  a.ktiles = (a.nkb + 3) / 4;
  const bool contig = d.ld == d.cols;
  const bool mma = d.sf_layout == NVFP4_SF_MMA128x4;
  const bool wide = reinterpret_cast<uintptr_t>(d.out) % 32 == 0 && (contig || d.ld % 16 == 0);
  auto launch = [&](auto kernel) {
    return launch_pdl(kernel, dim3(dq_grid(kernel, a.blocks, d.sm_count, 1)), dim3(kDqThreads), 0,
                      st, a);
  };
  if (wide) {
    if (mma)
      return contig ? launch(dequant_kernel<NVFP4_SF_MMA128x4, true, true>)
                    : launch(dequant_kernel<NVFP4_SF_MMA128x4, false, true>);
    return contig ? launch(dequant_kernel<NVFP4_SF_ROWMAJOR, true, true>)
                  : launch(dequant_kernel<NVFP4_SF_ROWMAJOR, false, true>);
  }
  if (mma)
    return contig ? launch(dequant_kernel<NVFP4_SF_MMA128x4, true, false>)
                  : launch(dequant_kernel<NVFP4_SF_MMA128x4, false, false>);
  return contig ? launch(dequant_kernel<NVFP4_SF_ROWMAJOR, true, false>)
                : launch(dequant_kernel<NVFP4_SF_ROWMAJOR, false, false>);
}

cudaError_t launch_kv_dequant(const LaunchKvDequant& d, cudaStream_t st) {
  KvDequantArgs a;
  a.codes[0] = d.k_codes; a.codes[1] = d.v_codes;
  a.sf[0] = d.k_sf; a.sf[1] = d.v_sf;
  a.st[0] = d.k_st; a.st[1] = d.v_st;
  a.out[0] = static_cast<uint8_t*>(d.k_out);
  a.out[1] = static_cast<uint8_t*>(d.v_out);
  a.blocks_per_frame = uint32_t(int64_t(d.tpf) * d.heads * d.head_dim / 16);
  a.bpf_div = make_fastdiv(a.blocks_per_frame);
  a.blocks = uint32_t(int64_t(d.n) * a.blocks_per_frame);
  for (int i = 0; i < NVFP4_KV_MAX_WINDOW_SLOTS; ++i) a.slots[i] = i < d.n ? d.slots[i] : 0;
  const bool wide = reinterpret_cast<uintptr_t>(d.k_out) % 32 == 0 &&
                    reinterpret_cast<uintptr_t>(d.v_out) % 32 == 0;
  if (wide) {
    const int grid = dq_grid(kv_dequant_kernel<true>, a.blocks, d.sm_count, 2);
    return launch_pdl(kv_dequant_kernel<true>, dim3(grid, 2), dim3(kDqThreads), 0, st, a);
  }
  const int grid = dq_grid(kv_dequant_kernel<false>, a.blocks, d.sm_count, 2);
  return launch_pdl(kv_dequant_kernel<false>, dim3(grid, 2), dim3(kDqThreads), 0, st, a);
}

}  // namespace nvfp4
