// attention.cu -- windowed attention that reads the NVFP4 KV cache directly,
// on the sm_100a tensor cores.
//
// The new chunk's queries attend to the frames of the attention window (the
// sink frames and the local window: 171host.com LongLive 2.0 teardown, section
// 2.2), whose K and V sit in the cache as NVFP4 frame slots (hyper.ai
// LongLive-2.0 summary, section "方法": KV quantized in frame blocks, rebuilt
// for windowed attention).  Instead of rebuilding the whole window as bf16 in
// HBM and reading it back, each CTA decodes the K and V tiles it is about to
// use into shared memory (the same bf16_RNE((v * s_b) * s_t) values the window
// rebuild writes) and hands them to the tensor core.
//
//   out[t][h] = sum_j softmax_j(scale * q[t][h] . k[j][h]) v[j][h]
//
// over the window's tokens j in slot-list order; no mask inside the window
// (chunk-wise attention: the chunk sees itself and the cached frames whole).
//
// Structure: one CTA per (256 queries, head): two query tiles of 128 rows (Q0,
// Q1) share every decoded K/V tile, so a tile is decoded once per 256 queries;
// 17 warps.
//   warps 0..7  softmax and epilogue: group g = warp / 4 owns query tile g,
//               warp w owns tensor-memory lane quadrant w % 4 (one query row
//               per thread).  They load their Q rows into shared memory once;
//               per KV tile they read their row of S_g = Q_g K^T out of tensor
//               memory, update the running row maximum and sum (base 2), and
//               write the probabilities rounded to bf16 back over S_g, where
//               the P V product reads them as its A operand.
//   warp 8      tensor-memory owner; lane 0 issues the MMAs
//               (tcgen05.mma kind::f16, bf16 in, fp32 accumulate) so that the
//               tensor core works on one query tile while the other's
//               softmax runs: ... PV0_j, S0_{j+1}, PV1_j, S1_{j+1}, PV0_{j+1} ...
//               (each S writes the tensor memory the preceding P V of the same
//               tile read; the tensor core runs one thread's MMAs in order).
//   warps 9..16 decoders: per 128-token tile, the 16-element NVFP4 blocks of
//               K and V of this head -> bf16 (byte-permute table per block),
//               K and V both as [token][dim] in the tensor core's
//               128-byte-swizzled layout (K-major for S = Q K^T; for P V the
//               same bytes are V in the MN-major layout), into a two-stage
//               ring; each decoder loads the next tile's NVFP4
//               bytes into registers before it decodes the current one, so
//               the L2 latency of those loads hides behind the decoding.
// Tensor memory (512 columns): O0, O1, S0, S1 at columns 0, 128, 256, 384.
// The running maximum is raised lazily: while a row's new scores stay within
// 2^16 of the maximum in use, the probabilities are taken against the old one
// (they stay <= 2^16: bf16 P, the fp32 sum and the fp32 O hold that range with
// their relative precision unchanged); only a larger step rescales the row's O
// and sum, which is safe at once: S_g of tile j completes after P V of tile
// j-1 of the same query tile.  Every wait is bounded: one that runs out records
// NVFP4_ERR_TIMEOUT in the workspace status word, and the CTA drains its MMAs,
// frees tensor memory and returns.
#include "common.cuh"
#include "decode.cuh"
#include "kernels.h"

#include <atomic>

namespace nvfp4 {
namespace attn {

constexpr int kD = 128;                   // head_dim
constexpr int kBQ = 128;                  // queries per query tile (tensor-memory lanes)
constexpr int kQTiles = 2;                // query tiles per CTA
constexpr int kBK = 128;                  // keys per tile
constexpr int kDimBlocks = kD / 16;       // 16-element blocks per token and head
constexpr int kSoftWarps = 4 * kQTiles;   // warps 0..7
constexpr int kMmaWarp = kSoftWarps;      // 8
constexpr int kDecWarp0 = kMmaWarp + 1;   // 9
constexpr int kDecWarps = 8;
constexpr int kThreads = (kDecWarp0 + kDecWarps) * 32;  // 544
constexpr int kStages = 2;
constexpr int kChunkBytes = 128 * 128;    // 128 rows x 64 bf16 (one K chunk of an operand)
constexpr int kOpBytes = 2 * kChunkBytes;  // 128 rows x 128 bf16
// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kOffQ = 0;                                 // + g * kOpBytes
constexpr int kOffK = kOffQ + kQTiles * kOpBytes;        // + stage * kOpBytes
constexpr int kOffV = kOffK + kStages * kOpBytes;        // V [token][dim], + stage * kOpBytes
constexpr int kOffBar = kOffV + kStages * kOpBytes;
// q_ready, kv_full[2], kv_empty[2], s_full[2], p_ready[2], pv_done[2], o_full, drain
constexpr int kNumBars = 1 + 2 * kStages + 3 * kQTiles + 2;
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kOffAbort = kOffTmemPtr + 4;
constexpr int kSmemBytes = kOffAbort + 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol0 = 0;            // O_g at kOCol0 + 128 g
constexpr uint32_t kSCol0 = 256;          // S_g (then P_g) at kSCol0 + 128 g
// Instruction descriptor, kind::f16: fp32 D (bit 4), bf16 A and B (bits 7 and
// 10), both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBK >> 3) << 17) |
                            (uint32_t(kBQ >> 4) << 24);
constexpr float kLazyLog2 = 16.0f;         // largest probability kept before a rescale: 2^16

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
  uint32_t* status;
  uint64_t wait_limit_ns;
  int32_t slots[NVFP4_KV_MAX_WINDOW_SLOTS];
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool bar_try_wait(uint32_t bar, uint32_t parity) {
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
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart, descriptor version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// D (+)= A B^T, A and B in shared memory.
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(kIdesc), "r"(acc)
      : "memory");
}
// Shared-memory matrix descriptor of an MN-major operand, 128-byte swizzle:
// 8-row (K) groups 1024 bytes apart (SBO), 64-element MN chunks
// kMnChunkBytes apart (LBO), descriptor version 1.
#ifndef ATTN_V_LBO
#define ATTN_V_LBO (128 * 128)
#endif
#ifndef ATTN_V_SBO
#define ATTN_V_SBO 1024
#endif
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t addr) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(ATTN_V_LBO >> 4) << 16) |
         (uint64_t(ATTN_V_SBO >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// The P V product's descriptor: as kIdesc with B MN-major (bit 16): V is
// stored [key][dim], dims contiguous.
constexpr uint32_t kIdescPV = kIdesc | (1u << 16);
// D (+)= A B^T, A in tensor memory, B MN-major.
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(kIdescPV), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// The same load without its wait (pair with tmem_wait_ld).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Waits for every earlier tensor-memory load of the thread, then ties the
// registers of both loads to the wait so that nothing reading them can be
// scheduled before it.
// max of three (sm_100's three-input form; NaN handling as fmaxf)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void regs_after_wait(uint32_t (&r)[32]) {
  asm volatile(
      ""
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r0)[32], uint32_t (&r1)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  regs_after_wait(r0);
  regs_after_wait(r1);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Byte offset of 16-byte unit u (0..15: elements 8u..8u+7) of row r in a
// 128-row operand tile of 128 bf16 per row, in the tensor core's K-major,
// 128-byte-swizzled layout (two 64-element chunks of 16 KB).
__device__ __forceinline__ uint32_t op_offset(uint32_t r, uint32_t u) {
  return (u >> 3) * kChunkBytes + (r >> 3) * 1024 + (r & 7) * 128 + (((u & 7) ^ (r & 7)) << 4);
}

// 2^x with the hardware approximation (relative error about 2^-22; results
// below 2^-126 flush to zero, which the softmax sums cannot notice).
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Waiter {
  uint64_t limit_ns;
  volatile int* abort;
  uint32_t* status;
  // Wait for phase `parity` of `bar`; false if the CTA aborted or the wait ran out.
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
    if (bar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
      if (*abort) return false;
      if (bar_try_wait(bar, parity)) return true;
      if (globaltimer() - t0 > limit_ns) {
        record_status(status, NVFP4_ERR_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
};

// Decoded bf16 of one 16-element block of K or V: token w of the window
// (position w / tpf in the slot list), dim block db of head h; zeros past the
// window's end.
__device__ __forceinline__ void load_block(const AttnArgs& a, int plane, uint32_t w, uint32_t h,
                                           uint32_t db, uint2& c, uint32_t& sb, float& st) {
  const uint32_t ww = min(w, a.n_kv - 1);
  const uint32_t pos = fast_div(a.tpf_div, ww);
  const uint32_t local = ww - pos * a.tpf;
  const size_t s = size_t(a.slots[pos]);
  const size_t blk = ((s * a.tpf + local) * a.heads + h) * kDimBlocks + db;
  c = __ldg(reinterpret_cast<const uint2*>(a.codes[plane]) + blk);
  sb = __ldg(a.sf[plane] + blk);
  st = __ldg(a.st[plane] + s);
}

__global__ void __launch_bounds__(kThreads, 1) window_attention_kernel(const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_q = sbase + kOffBar;
  const uint32_t bar_kv_full = bar_q + 8;                      // + 8 stage
  const uint32_t bar_kv_empty = bar_kv_full + 8 * kStages;     // + 8 stage
  const uint32_t bar_s_full = bar_kv_empty + 8 * kStages;      // + 8 g
  const uint32_t bar_p_ready = bar_s_full + 8 * kQTiles;       // + 8 g
  const uint32_t bar_pv_done = bar_p_ready + 8 * kQTiles;      // + 8 g
  const uint32_t bar_o_full = bar_pv_done + 8 * kQTiles;
  const uint32_t bar_drain = bar_o_full + 8;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t h = blockIdx.y;
  const uint32_t q_base = blockIdx.x * (kBQ * kQTiles);
  const uint32_t n_tiles = (a.n_kv + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    bar_init(bar_q, kSoftWarps);
    for (int s = 0; s < kStages; ++s) {
      bar_init(bar_kv_full + 8 * s, kDecWarps);
      bar_init(bar_kv_empty + 8 * s, 1);
    }
    for (int g = 0; g < kQTiles; ++g) {
      bar_init(bar_s_full + 8 * g, 1);
      bar_init(bar_p_ready + 8 * g, 4);
      bar_init(bar_pv_done + 8 * g, 1);
    }
    bar_init(bar_o_full, 1);
    bar_init(bar_drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_ptr)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  pdl_wait();
  pdl_trigger();
  const Waiter waiter{a.wait_limit_ns, abort_flag, a.status};

  if (warp < kSoftWarps) {
    // ------------------------------------------------------------ softmax
    const uint32_t g = uint32_t(warp) >> 2;                      // query tile
    const uint32_t quad = uint32_t(warp) & 3;                    // lane quadrant
    const uint32_t row = quad * 32 + uint32_t(lane);             // row within the tile
    const uint32_t q0 = q_base + g * kBQ;
    const uint32_t lane_bits = (quad * 32) << 16;
    const uint32_t o_addr = tmem + lane_bits + kOCol0 + 128 * g;
    const uint32_t s_addr = tmem + lane_bits + kSCol0 + 128 * g;
    // Q row -> shared memory (rows past tq are zero)
    {
      const bool live = q0 + row < a.tq;
      const uint4* src =
          reinterpret_cast<const uint4*>(a.q + int64_t(live ? q0 + row : 0) * a.q_stride + h * kD);
      const uint32_t qs = sbase + kOffQ + g * kOpBytes;
#pragma unroll
      for (uint32_t u = 0; u < 16; ++u) {
        const uint4 v = live ? __ldg(src + u) : make_uint4(0, 0, 0, 0);
        st_shared_v4(qs + op_offset(row, u), v);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) bar_arrive(bar_q);
    }
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (uint32_t j = 0; j < n_tiles && ok; ++j) {
      ok = __all_sync(0xFFFFFFFFu, waiter.wait(bar_s_full + 8 * g, j & 1));
      if (!ok) break;
      tc_fence_after();
      const uint32_t n_valid = min(uint32_t(kBK), a.n_kv - j * kBK);
      // pass 1: the tile's row maximum over the live keys (the scale is
      // positive, so scaling the maximum is the maximum of the scaled scores)
      float mx_raw = -INFINITY;
      const bool tail = n_valid < uint32_t(kBK);
#pragma unroll 1
      for (uint32_t c = 0; c < 4; c += 2) {
        uint32_t r0[32], r1[32];
        tmem_ld32_async(s_addr + 32 * c, r0);
        tmem_ld32_async(s_addr + 32 * c + 32, r1);
        tmem_wait_ld(r0, r1);
        if (!tail) {
#pragma unroll
          for (uint32_t e = 0; e < 32; ++e)
            mx_raw = max3f(mx_raw, __uint_as_float(r0[e]), __uint_as_float(r1[e]));
        } else {
#pragma unroll
          for (uint32_t e = 0; e < 32; ++e) {
            if (32 * c + e < n_valid) mx_raw = fmaxf(mx_raw, __uint_as_float(r0[e]));
            if (32 * c + 32 + e < n_valid) mx_raw = fmaxf(mx_raw, __uint_as_float(r1[e]));
          }
        }
      }
      const float mx = __fmul_rn(mx_raw, a.scale_log2);
      // lazy maximum: keep the one in use while the tile stays within 2^16 of it
      float factor = 1.0f;
      if (mx > m_run + kLazyLog2) {
        factor = exp2_approx(m_run - mx);   // 0 on the first tile
        m_run = mx;
        l_run = l_run * factor;
      }
      // pass 2: probabilities 2^(s scale - m), their sum, bf16 into the score
      // buffer's first 64 columns (chunk c's 16 words go over columns already read)
      const float neg_m = -m_run;
      // both halves of a pair of scores on the packed fp32 pipe (the same
      // roundings as two scalar operations); the sum as fma(p, 1, sum)
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
      const float2 nm2 = make_float2(neg_m, neg_m), one2 = make_float2(1.0f, 1.0f);
      float2 sum2 = make_float2(0.0f, 0.0f);
#pragma unroll 1
      for (uint32_t c = 0; c < 4; c += 2) {
        // two 32-column chunks per tensor-memory round trip
        uint32_t r[2][32];
        tmem_ld32_async(s_addr + 32 * c, r[0]);
        tmem_ld32_async(s_addr + 32 * c + 32, r[1]);
        tmem_wait_ld(r[0], r[1]);
#pragma unroll
        for (uint32_t h2 = 0; h2 < 2; ++h2) {
          uint32_t pk[16];
#pragma unroll
          for (uint32_t e = 0; e < 16; ++e) {
            const uint32_t k0 = 32 * (c + h2) + 2 * e;
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(r[h2][2 * e]), __uint_as_float(r[h2][2 * e + 1])),
                sc2, nm2);
            float p0 = exp2_approx(x.x);
            float p1 = exp2_approx(x.y);
            if (tail) {
              p0 = k0 < n_valid ? p0 : 0.0f;
              p1 = k0 + 1 < n_valid ? p1 : 0.0f;
            }
            sum2 = __ffma2_rn(make_float2(p0, p1), one2, sum2);
            pk[e] = bf16x2_rn(p0, p1);
          }
          // P chunk c + h2 -> columns 16 (c + h2): inside chunks already read
          tmem_st16(s_addr + 16 * (c + h2), pk);
        }
      }
      l_run += sum2.x + sum2.y;
      // a raised maximum rescales this row's O (tile j-1's P V, complete since
      // S_g of tile j is)
      if (__any_sync(0xFFFFFFFFu, factor != 1.0f) && j > 0) {
        ok = __all_sync(0xFFFFFFFFu, waiter.wait(bar_pv_done + 8 * g, (j - 1) & 1));
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (uint32_t c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(o_addr + 32 * c, r);
#pragma unroll
            for (uint32_t e = 0; e < 32; ++e)
              r[e] = __float_as_uint(__fmul_rn(__uint_as_float(r[e]), factor));
            tmem_st32(o_addr + 32 * c, r);
          }
        }
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(bar_p_ready + 8 * g);
    }
    // ---- epilogue: O / l -> bf16 (rows past tq are not stored)
    if (ok) ok = __all_sync(0xFFFFFFFFu, waiter.wait(bar_o_full, 0));
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const bool live = q0 + row < a.tq;
      uint4* dst = reinterpret_cast<uint4*>(a.out + int64_t(live ? q0 + row : 0) * a.out_stride +
                                            h * kD);
#pragma unroll 1
      for (uint32_t c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(o_addr + 32 * c, r);
        if (live) {
#pragma unroll
          for (uint32_t e = 0; e < 4; ++e) {
            uint4 v;
            v.x = bf16x2_rn(__uint_as_float(r[8 * e]) * inv, __uint_as_float(r[8 * e + 1]) * inv);
            v.y = bf16x2_rn(__uint_as_float(r[8 * e + 2]) * inv, __uint_as_float(r[8 * e + 3]) * inv);
            v.z = bf16x2_rn(__uint_as_float(r[8 * e + 4]) * inv, __uint_as_float(r[8 * e + 5]) * inv);
            v.w = bf16x2_rn(__uint_as_float(r[8 * e + 6]) * inv, __uint_as_float(r[8 * e + 7]) * inv);
            dst[4 * c + e] = v;
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = waiter.wait(bar_q, 0);
      // S_g(j) = Q_g K_j^T into S_g
      auto issue_s = [&](uint32_t g, uint32_t j) {
        const uint32_t st = j % kStages;
        const uint64_t qd = desc_sw128(sbase + kOffQ + g * kOpBytes);
        const uint64_t kd = desc_sw128(sbase + kOffK + st * kOpBytes);
#pragma unroll
        for (uint32_t ks = 0; ks < 8; ++ks)  // 16 dims a step: +32 bytes, next chunk after 4
          mma_ss(tmem + kSCol0 + 128 * g, qd + (ks >> 2) * (kChunkBytes >> 4) + 2 * (ks & 3),
                 kd + (ks >> 2) * (kChunkBytes >> 4) + 2 * (ks & 3), ks != 0);
        tc_commit(bar_s_full + 8 * g);
      };
      // O_g += P_g(j) V_j, P from S_g's columns, V from ring stage j % 2
      auto issue_pv = [&](uint32_t g, uint32_t j) {
        if (!waiter.wait(bar_p_ready + 8 * g, j & 1)) return false;
        tc_fence_after();
        const uint64_t vd = desc_mn_sw128(sbase + kOffV + (j % kStages) * kOpBytes);
        const uint32_t p_addr = tmem + kSCol0 + 128 * g;
#pragma unroll
        for (uint32_t ks = 0; ks < 8; ++ks)  // 16 keys a step: 8 columns of P, two 8-key groups of V
          mma_ts(tmem + kOCol0 + 128 * g, p_addr + 8 * ks, vd + ks * (2048 >> 4), (j | ks) != 0);
        tc_commit(bar_pv_done + 8 * g);
        return true;
      };
      auto kv_ready = [&](uint32_t j) {
        if (!waiter.wait(bar_kv_full + 8 * (j % kStages), (j / kStages) & 1)) return false;
        tc_fence_after();
        return true;
      };
      if (ok && n_tiles > 0 && (ok = kv_ready(0))) {
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (uint32_t j = 0; j < n_tiles && ok; ++j) {
        const bool more = j + 1 < n_tiles;
        if (!(ok = issue_pv(0, j))) break;
        if (more) {
          if (!(ok = kv_ready(j + 1))) break;
          issue_s(0, j + 1);
        }
        if (!(ok = issue_pv(1, j))) break;
        tc_commit(bar_kv_empty + 8 * (j % kStages));   // K_j and V_j read by every MMA
        if (more) issue_s(1, j + 1);
      }
      if (ok) tc_commit(bar_o_full);
      // drain: every tcgen05 operation this thread issued has completed
      tc_commit(bar_drain);
      const uint64_t t0 = globaltimer();
      while (!bar_try_wait(bar_drain, 0)) {
        if (globaltimer() - t0 > 2000000000ull) {
          record_status(a.status, NVFP4_ERR_TIMEOUT);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ decoders
    // K and V alike: token t / 8 + 32 i, dim block t % 8 (8 lanes read one
    // token's 64 bytes), stored [token][dim]: K-major for S = Q K^T, and the
    // MN-major layout the P V product reads V in
    const uint32_t t = threadIdx.x - kDecWarp0 * 32;   // 0..255
    struct TileRaw {
      uint2 c[2][4];
      uint32_t sb[2][4];
      float st[2][4];
    };
    auto load_tile = [&](uint32_t j, TileRaw& r) {
      const uint32_t w0 = j * kBK;
#pragma unroll
      for (int pl = 0; pl < 2; ++pl)
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i)
          load_block(a, pl, w0 + t / 8 + 32 * i, h, t % 8, r.c[pl][i], r.sb[pl][i], r.st[pl][i]);
    };
    TileRaw cur, nxt;
    if (n_tiles > 0) load_tile(0, cur);
    bool ok = true;
    for (uint32_t j = 0; j < n_tiles && ok; ++j) {
      if (j + 1 < n_tiles) load_tile(j + 1, nxt);
      const uint32_t b = j % kStages;
      ok = __all_sync(0xFFFFFFFFu, waiter.wait(bar_kv_empty + 8 * b, ((j / kStages) & 1) ^ 1));
      if (!ok) break;
      const uint32_t w0 = j * kBK;
#pragma unroll
      for (int pl = 0; pl < 2; ++pl) {
        const uint32_t base = sbase + (pl == 0 ? kOffK : kOffV) + b * kOpBytes;
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
          const uint32_t tok = t / 8 + 32 * i, db = t % 8;
          uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
          if (w0 + tok < a.n_kv) {
            const BlockLut l = make_lut(cur.sb[pl][i], cur.st[pl][i]);
            lo = decode8(l, cur.c[pl][i].x);
            hi = decode8(l, cur.c[pl][i].y);
          }
          st_shared_v4(base + op_offset(tok, 2 * db), lo);
          st_shared_v4(base + op_offset(tok, 2 * db + 1), hi);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) bar_arrive(bar_kv_full + 8 * b);
      cur = nxt;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace attn

cudaError_t launch_window_attention(const LaunchAttn& d, cudaStream_t st) {
  attn::AttnArgs a;
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
  a.status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(d.ws) + kWsStatus);
  a.wait_limit_ns = d.wait_limit_ns;
  for (int i = 0; i < d.n; ++i) a.slots[i] = d.slot_ids[i];
  static std::atomic<bool> configured[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev].load(std::memory_order_acquire)) {
    const cudaError_t e = cudaFuncSetAttribute(
        attn::window_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
        attn::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev].store(true, std::memory_order_release);
  }
  constexpr int64_t kCtaQ = int64_t(attn::kBQ) * attn::kQTiles;
  const dim3 grid(uint32_t((d.tq + kCtaQ - 1) / kCtaQ), uint32_t(d.heads));
  return launch_pdl(attn::window_attention_kernel, grid, dim3(attn::kThreads),
                    size_t(attn::kSmemBytes), st, a);
}

}  // namespace nvfp4
