// decode.cuh -- NVFP4 block -> bf16 decoding shared by the dequantizers and
// the window attention: bf16_RNE((v(q) * s_b) * s_t) per element, through the
// block's 8 distinct magnitudes.
#pragma once
#include "common.cuh"

namespace nvfp4 {

// The 8 bf16 magnitudes of a block, as byte tables for prmt: lo0/lo1 hold the
// low bytes of values 0..3 / 4..7, hi0/hi1 the high bytes.
struct BlockLut {
  uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Only two products are rounded: f2 = RN(s_b s_t) and f3 = RN((1.5 s_b) s_t).
// The other magnitudes are these times a power of two (0.5 f2, 2 f2, 2 f3,
// 4 f2, 4 f3), and scaling by a power of two commutes with rounding to binary32
// and to bf16 while nothing overflows or leaves the normal range, which the
// tensor-scale domain guarantees (s_b s_t >= 2^-117, 6 s_b s_t < 2^112).  So
// the bf16 words of 2 f and 4 f are those of f with 1 or 2 added to the
// exponent field of each half, and of 0.5 f with 1 taken from it.  A zero
// scale byte gives the all-zero table.
__device__ __forceinline__ BlockLut make_lut(uint32_t sb, float s_t) {
  const float s = e4m3_to_f32(sb);
  const uint32_t t23 = bf16x2_rn(__fmul_rn(s, s_t), __fmul_rn(__fmul_rn(1.5f, s), s_t));
  const uint32_t e1 = t23 ? 0x00800080u : 0u;  // +1 in both exponent fields
  const uint32_t t45 = t23 + e1, t67 = t23 + 2 * e1;
  const uint32_t t01 = (t23 - (e1 & 0xFFFFu)) << 16;  // (0, 0.5 f2)
  BlockLut l;
  l.lo0 = prmt(t01, t23, 0x6420);
  l.hi0 = prmt(t01, t23, 0x7531);
  l.lo1 = prmt(t45, t67, 0x6420);
  l.hi1 = prmt(t45, t67, 0x7531);
  return l;
}

// 8 codes (nibble i of c = element i) -> 8 bf16 in four words.  The low and
// high bytes of the magnitudes come from the block table (byte permutes
// indexed by the 3 magnitude bits), then two permutes interleave them into
// bf16 words.  The sign of element i is bit 4i + 3 of c and belongs at bit 7
// of its high byte: a permute of (c << 4, c) puts the signs of elements
// 0, 1, 2, 3 (bits 3, 7, 11, 15 of c) at bit 7 of bytes 0..3, those of
// elements 4..7 likewise, so one and-or per four high bytes adds them.
__device__ __forceinline__ uint4 decode8(const BlockLut& l, uint32_t c) {
  const uint32_t m = c & 0x77777777u;
  const uint32_t mh = m >> 16;
  const uint32_t c4 = c << 4;
  uint4 o;
  uint32_t lo4 = prmt(l.lo0, l.lo1, m);
  uint32_t hi4 = prmt(l.hi0, l.hi1, m) | (prmt(c4, c, 0x5140) & 0x80808080u);
  o.x = prmt(lo4, hi4, 0x5140);
  o.y = prmt(lo4, hi4, 0x7362);
  lo4 = prmt(l.lo0, l.lo1, mh);
  hi4 = prmt(l.hi0, l.hi1, mh) | (prmt(c4, c, 0x7362) & 0x80808080u);
  o.z = prmt(lo4, hi4, 0x5140);
  o.w = prmt(lo4, hi4, 0x7362);
  return o;
}

}  // namespace nvfp4
