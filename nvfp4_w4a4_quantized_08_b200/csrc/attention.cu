// attention.cu -- windowed attention that reads the NVFP4 KV cache directly.
//
// The new chunk's queries attend to the frames of the attention window (the
// sink frames and the local window: 171host.com LongLive 2.0 teardown, section
// 2.2), whose K and V sit in the cache as NVFP4 frame slots (hyper.ai
// LongLive-2.0 summary, section "方法": KV quantized in frame blocks, rebuilt
// for windowed attention).  Instead of rebuilding the whole window as bf16 in
// HBM and reading it back, each CTA decodes the K and V tiles it is about to
// use into shared memory (the same bf16_RNE((v * s_b) * s_t) values the window
// rebuild writes) and consumes them at once.
//
//   out[t][h] = sum_j softmax_j(scale * q[t][h] . k[j][h]) v[j][h]
//
// over the window's tokens j in slot-list order; no mask inside the window
// (chunk-wise attention: the chunk sees itself and the cached frames whole).
//
// Structure: one CTA per (64 queries, head), 4 warps of 16 query rows each.
// Per 64-token KV tile: all threads decode K into Ks[token][dim] and V
// transposed into Vt[dim][token] (bf16, padded rows); each warp computes its
// 16 x 64 scores with mma.sync m16n8k16 (bf16 in, fp32 accumulate), updates the
// running row max and sum (online softmax in base 2), rounds the probabilities
// to bf16 and accumulates P V with mma.sync into a 16 x 128 fp32 accumulator.
#include "common.cuh"
#include "decode.cuh"
#include "kernels.h"

namespace nvfp4 {

constexpr int kAttD = 128;                 // head_dim
constexpr int kAttBQ = 64;                 // query rows per CTA
constexpr int kAttBK = 64;                 // KV tokens per tile
constexpr int kAttThreads = 128;
constexpr int kLdK = kAttD + 8;            // Ks row: 136 bf16 (272 B, 68 words)
constexpr int kLdV = kAttBK + 8;           // Vt row: 72 bf16 (144 B, 36 words)
constexpr int kDimBlocks = kAttD / 16;     // 16-element blocks per token and head

struct AttnArgs {
  const uint16_t* q;   // bf16 [tq][q_stride], head h at h * 128
  uint16_t* out;       // bf16 [tq][out_stride]
  int64_t q_stride, out_stride;  // elements between tokens
  const uint8_t* codes[2];       // K, V pools
  const uint8_t* sf[2];
  const float* st[2];
  uint32_t tq, heads, tpf, n_kv;  // n_kv = window slots * tpf
  FastDiv tpf_div;
  float scale_log2;               // softmax scale * log2(e)
  int32_t slots[NVFP4_KV_MAX_WINDOW_SLOTS];
};

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(const uint16_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

__global__ void __launch_bounds__(kAttThreads) window_attention_kernel(const AttnArgs a) {
  __shared__ __align__(16) uint16_t Ks[kAttBK * kLdK];
  __shared__ __align__(16) uint16_t Vt[kAttD * kLdV];
  pdl_wait();
  pdl_trigger();
  const uint32_t h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;  // mma fragment row group / column pair
  const uint32_t row_a = blockIdx.x * kAttBQ + warp * 16 + g, row_b = row_a + 8;

  // Q fragments of this warp's 16 rows, 8 K steps of 16 dims (rows past tq: 0)
  uint32_t qa[8][4];
  {
    const uint16_t* qra = a.q + int64_t(row_a) * a.q_stride + h * kAttD + 2 * t;
    const uint16_t* qrb = a.q + int64_t(row_b) * a.q_stride + h * kAttD + 2 * t;
    const bool va = row_a < a.tq, vb = row_b < a.tq;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = va ? __ldg(reinterpret_cast<const uint32_t*>(qra + 16 * ks)) : 0u;
      qa[ks][1] = vb ? __ldg(reinterpret_cast<const uint32_t*>(qrb + 16 * ks)) : 0u;
      qa[ks][2] = va ? __ldg(reinterpret_cast<const uint32_t*>(qra + 16 * ks + 8)) : 0u;
      qa[ks][3] = vb ? __ldg(reinterpret_cast<const uint32_t*>(qrb + 16 * ks + 8)) : 0u;
    }
  }
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;

  const uint32_t n_tiles = (a.n_kv + kAttBK - 1) / kAttBK;
  for (uint32_t kt = 0; kt < n_tiles; ++kt) {
    __syncthreads();  // every warp is done with the previous tile
    // ---- decode the K and V blocks of tokens [64 kt, 64 kt + 64) of head h:
    // 2 planes x 64 tokens x 8 blocks, 8 per thread, every pass's loads issued
    // before any block is decoded.  K passes (it < 4): token threadIdx / 8 +
    // 16 it, dim block threadIdx % 8 (a warp's 16-byte row stores spread over
    // all banks).  V passes: token threadIdx % 64, dim block 2 (it - 4) +
    // threadIdx / 64, so that a warp's transposed 16-bit stores hit 16
    // consecutive words of one Vt row (dim-block-major lanes would put all 8
    // blocks' rows, 16 x 36 words apart, in one bank).
    {
      auto tok_of = [](int it) {
        return it < 4 ? int(threadIdx.x) / kDimBlocks + 16 * it : int(threadIdx.x) % kAttBK;
      };
      auto db_of = [](int it) {
        return it < 4 ? int(threadIdx.x) % kDimBlocks : 2 * (it - 4) + int(threadIdx.x) / kAttBK;
      };
      uint2 c[8];
      uint32_t sb[8];
      float stv[8];
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int plane = it / 4;
        const int tok = tok_of(it), db = db_of(it);
        const uint32_t j = min(kt * kAttBK + tok, a.n_kv - 1);  // past the end: reload, zeroed below
        const uint32_t pos = fast_div(a.tpf_div, j);  // position in the slot list
        const uint32_t local = j - pos * a.tpf;
        const size_t s = size_t(a.slots[pos]);
        const size_t blk = ((s * a.tpf + local) * a.heads + h) * kDimBlocks + db;
        c[it] = __ldg(reinterpret_cast<const uint2*>(a.codes[plane]) + blk);
        sb[it] = __ldg(a.sf[plane] + blk);
        stv[it] = __ldg(a.st[plane] + s);
      }
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int tok = tok_of(it), db = db_of(it);
        uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
        if (kt * kAttBK + tok < a.n_kv) {
          const BlockLut l = make_lut(sb[it], stv[it]);
          lo = decode8(l, c[it].x);
          hi = decode8(l, c[it].y);
        }
        if (it < 4) {
          uint4* dst = reinterpret_cast<uint4*>(Ks + tok * kLdK + 16 * db);
          dst[0] = lo;
          dst[1] = hi;
        } else {
          const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          uint16_t* col = Vt + (16 * db) * kLdV + tok;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            col[(2 * e) * kLdV] = uint16_t(w[e] & 0xFFFFu);
            col[(2 * e + 1) * kLdV] = uint16_t(w[e] >> 16);
          }
        }
      }
    }
    __syncthreads();

    // ---- S = Q K^T for this warp's 16 rows and the tile's 64 tokens
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
      const uint16_t* krow = Ks + (8 * nt + g) * kLdK + 2 * t;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_bf16(s[nt], qa[ks], lds32(krow + 16 * ks), lds32(krow + 16 * ks + 8));
    }
    // ---- online softmax, base 2: tokens past the window get probability 0
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool live = kt * kAttBK + 8 * nt + 2 * t + e < a.n_kv;
        s[nt][e] = live ? __fmul_rn(s[nt][e], a.scale_log2) : -INFINITY;
        s[nt][2 + e] = live ? __fmul_rn(s[nt][2 + e], a.scale_log2) : -INFINITY;
        mx_a = fmaxf(mx_a, s[nt][e]);
        mx_b = fmaxf(mx_b, s[nt][2 + e]);
      }
    }
#pragma unroll
    for (int sh = 1; sh <= 2; sh <<= 1) {
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xFFFFFFFFu, mx_a, sh));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xFFFFFFFFu, mx_b, sh));
    }
    // every tile holds at least one live token, so the new maxima are finite
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float corr_a = exp2f(m_a - mn_a), corr_b = exp2f(m_b - mn_b);
    m_a = mn_a;
    m_b = mn_b;
    float sum_a = 0.0f, sum_b = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[nt][e] = exp2f(s[nt][e] - mn_a);
        s[nt][2 + e] = exp2f(s[nt][2 + e] - mn_b);
        sum_a += s[nt][e];
        sum_b += s[nt][2 + e];
      }
    }
    l_a = l_a * corr_a + sum_a;
    l_b = l_b * corr_b + sum_b;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= corr_a;
      o[nt][1] *= corr_a;
      o[nt][2] *= corr_b;
      o[nt][3] *= corr_b;
    }
    // ---- O += P V: P (bf16) as the A operand, 4 K steps of 16 tokens
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint32_t pa[4] = {bf16x2_rn(s[2 * ks][0], s[2 * ks][1]),
                              bf16x2_rn(s[2 * ks][2], s[2 * ks][3]),
                              bf16x2_rn(s[2 * ks + 1][0], s[2 * ks + 1][1]),
                              bf16x2_rn(s[2 * ks + 1][2], s[2 * ks + 1][3])};
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const uint16_t* vrow = Vt + (8 * nt + g) * kLdV + 16 * ks + 2 * t;
        mma_bf16(o[nt], pa, lds32(vrow), lds32(vrow + 8));
      }
    }
  }

  // ---- normalise and store (rows past tq are not stored)
#pragma unroll
  for (int sh = 1; sh <= 2; sh <<= 1) {
    l_a += __shfl_xor_sync(0xFFFFFFFFu, l_a, sh);
    l_b += __shfl_xor_sync(0xFFFFFFFFu, l_b, sh);
  }
  const float inv_a = 1.0f / l_a, inv_b = 1.0f / l_b;
  if (row_a < a.tq) {
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + int64_t(row_a) * a.out_stride + h * kAttD);
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
      dst[4 * nt + t] = bf16x2_rn(o[nt][0] * inv_a, o[nt][1] * inv_a);
  }
  if (row_b < a.tq) {
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + int64_t(row_b) * a.out_stride + h * kAttD);
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
      dst[4 * nt + t] = bf16x2_rn(o[nt][2] * inv_b, o[nt][3] * inv_b);
  }
}

cudaError_t launch_window_attention(const LaunchAttn& d, cudaStream_t st) {
  AttnArgs a;
  a.q = static_cast<const uint16_t*>(d.q);
  a.out = static_cast<uint16_t*>(d.out);
  a.q_stride = d.q_stride;
  a.out_stride = d.out_stride;
  a.codes[0] = d.k_codes;
  a.codes[1] = d.v_codes;
  a.sf[0] = d.k_sf;
  a.sf[1] = d.v_sf;
  a.st[0] = d.k_st;
  a.st[1] = d.v_st;
  a.tq = uint32_t(d.tq);
  a.heads = uint32_t(d.heads);
  a.tpf = uint32_t(d.tpf);
  a.n_kv = uint32_t(d.n * d.tpf);
  a.tpf_div = make_fastdiv(uint32_t(d.tpf));
  a.scale_log2 = d.scale_log2;
  for (int i = 0; i < d.n; ++i) a.slots[i] = d.slot_ids[i];
  const dim3 grid(uint32_t((d.tq + kAttBQ - 1) / kAttBQ), uint32_t(d.heads));
  return launch_pdl(window_attention_kernel, grid, dim3(kAttThreads), 0, st, a);
}

}  // namespace nvfp4
