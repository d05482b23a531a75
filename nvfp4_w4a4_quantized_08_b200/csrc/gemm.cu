// gemm.cu -- block-scaled NVFP4 x NVFP4 GEMM on the sm_100a tensor cores.
//
// C = A W^T with A: M x K and W: N x K NVFP4 operands (E2M1 codes, E4M3 scale
// per 16 elements along K, FP32 tensor scale): the FP4 GEMM that replaces the
// BF16 linear layers of the DiT (tailorednewshub.com LongLive-2.0 article,
// section "Inferencia W4A4 NVFP4").  Each 16-element block product is scaled
// on the tensor core (tcgen05.mma kind::mxf4nvf4, scale_vec::4X) and
// accumulated in FP32 in tensor memory; the tensor-scale product s_tA * s_tW
// is applied once in the epilogue.
//
// What sets the speed.  The MMAs are issued by one thread, which is held until
// the tensor pipe accepts each one: a stage of four 256 x 256 x 64 pair MMAs
// takes ~800 clocks with the scale hand-off, and a 256 x 192 x 64 MMA takes
// about as long as a 256 x 256 x 64 one, so the tile is as wide as the MMA
// allows.  The operands and their scales must arrive ahead of that pace:
//   * bytes per MAC: in the pair form a cluster of two CTAs on two SMs computes
//     a 256 x 256 tile with one cta_group::2 MMA per K step.  Each CTA stages
//     its own 128 rows of A and its own half of the tile's 256 W rows, and the
//     pair's tensor cores read both halves of W, so a CTA loads 32 KB of codes
//     per 128 x 256 x 256 of work instead of 48 KB (one CTA alone, 128 x 256);
//   * bytes in flight: a stage comes back a load latency after it is
//     requested, so the ring must hold enough stages to cover that latency;
//     the pair form's smaller stages leave room for five.
// The single form (one CTA, 128 x 256 tiles, cta_group::1) serves M <= 128.
//
// Warp roles (every CTA of either form):
//   warp 0      TMA producer: 2-D tensor copies of the A and W code tiles
//               (128-byte K slabs, 128-byte swizzle) and 1-D bulk copies of the
//               matching 512-byte scale tiles into the shared-memory ring.
//   warp 1      tensor-memory owner; lane 0 of the issuing CTA (the pair's
//               leader, or the single CTA) issues one MMA per K = 64 step and
//               one commit per stage.
//   warps 2..9  epilogue: two warps per tensor-memory lane quadrant, each
//               reading half of the accumulator's 256 columns: tcgen05.ld,
//               scale by s_tA * s_tW, activation, round to bf16 / fp32, stage
//               in swizzled shared memory, TMA tensor store (rows past M are
//               clipped by the store).
//   warps 10..13 scale writers: per stage, each writes the scale words its
//               lane quadrant reads into that stage's tensor-memory scale set
//               (tcgen05.st), off the tensor pipe.
// Hand-offs are mbarriers: full[s] (this CTA's TMA bytes landed -> writers),
// sf_ready[s] (the writers of every CTA of the tile -> issuer), empty[s] (the
// stage's MMAs completed -> every producer; a multicast commit in the pair),
// acc_full (the tile's MMAs completed -> every epilogue) and acc_empty (every
// epilogue warp read the accumulator out -> issuer).
// Tensor memory: the 128 x 256 FP32 accumulator in columns [0,256) and one
// 48-column scale set per shared-memory stage after it.
// Every spin-wait is bounded (wait_limit_ns).  A wait that runs out records
// NVFP4_ERR_TIMEOUT, raises the CTA's abort flag, and the CTA drains its own
// copies, MMAs and stores in flight before freeing tensor memory; the CTAs of
// a pair meet at a cluster barrier before either frees its tensor memory, so
// neither leaves while the leader's MMAs may still read its operands.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {
namespace gemm {

constexpr int kBM = 128;          // rows of A per CTA (accumulator lanes)
constexpr int kBN = 256;          // W rows per tile (accumulator columns)
constexpr int kBKBytes = 128;     // K slab per stage: 128 bytes = 256 FP4 values
constexpr int kKSteps = 4;        // MMA K = 64 values = 32 bytes
constexpr int kABytes = kBM * kBKBytes;      // 16 KB
constexpr int kSfaBytes = 4 * 512;           // 4 scale tiles of 128 rows x 4 blocks
constexpr int kSfbBytes = 2 * 4 * 512;       // 2 row tiles of W
constexpr int kEpiWarps = 8;
constexpr int kWriterWarp0 = 2 + kEpiWarps;  // 10
constexpr int kThreads = (kWriterWarp0 + 4) * 32;  // 448
constexpr int kTmemCols = 512;
constexpr int kSfCol = kBN;                  // scale sets after the accumulator
// A stage's scale set: the A scales of K step j at columns 4j (lane quadrant q
// reads column 4j + q), the W scales of K step j at columns 16 + 8j .. 16 + 8j + 7
constexpr int kSfWCol = 4 * kKSteps;         // 16
constexpr int kSfSetCols = kSfWCol + 8 * kKSteps;  // 48
constexpr int kStageBufBytes = 32 * 128;     // epilogue staging: 32 rows x 128 bytes

// Per-form sizes: kPair = 1 (single CTA) or 2 (CTA pair).
template <int kPair>
struct Cfg {
  static constexpr int kStages = kPair == 2 ? 5 : 3;
  static constexpr int kBRows = kBN / kPair;             // W rows staged per CTA
  static constexpr int kBBytes = kBRows * kBKBytes;      // 16 KB / 32 KB
  static constexpr int kTileM = kBM * kPair;             // output rows per tile
  // shared memory map (offsets from a 1024-byte aligned base)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kABytes;
  static constexpr int kOffSfa = kOffB + kStages * kBBytes;
  static constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
  static constexpr int kOffStage = kOffSfb + kStages * kSfbBytes;  // 1024-aligned
  static constexpr int kOffBar = kOffStage + kEpiWarps * kStageBufBytes;
  // full[], empty[], sf_ready[], acc_full, acc_empty, drain
  static constexpr int kNumBars = 3 * kStages + 3;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 4;
  static constexpr int kSmemBytes = kOffAbort + 4 + 1024;  // + alignment slack
  // Instruction descriptor, block-scaled kinds: E2M1 A and B (format 1 at bits
  // 7-9 and 10-12), K-major both, N >> 3 at bits 17-22, E4M3 scales (bit 23 =
  // 0), M >> 4 at bits 24-28 (M of the whole pair for cta_group::2), scale ids 0.
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) |
                                     (uint32_t(kTileM >> 4) << 24);
  static_assert(kOffStage % 1024 == 0, "staging buffers need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kSfCol + kStages * kSfSetCols <= kTmemCols, "tensor memory budget");
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

// Test phase `parity` of `bar`, letting the hardware suspend the thread for up
// to `hint_ns` while the phase is incomplete (it resumes when the phase completes).
__device__ __forceinline__ bool bar_try_wait(uint32_t bar, uint32_t parity,
                                             uint32_t hint_ns = 20000) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of this CTA's shared variable `addr` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier of another CTA of the cluster (default semantics:
// release at CTA scope; a cluster-scope release costs the thread about 1000
// clocks a call).  What an arrival publishes needs no wider release: scale
// words are in tensor memory once tcgen05.wait::st returns, and an epilogue
// warp's tensor-memory reads are complete once tcgen05.wait::ld returns; both
// are ordered for the issuer's tensor-core work by the tcgen05 fences around
// the hand-off.
__device__ __forceinline__ void bar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Every thread of every CTA of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void bar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once the tcgen05 operations issued so far complete: in this
// CTA (single form), or at the same address in both CTAs of the pair.
template <int kPair>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if constexpr (kPair == 1) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
  } else {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar),
        "h"(uint16_t(3))
        : "memory");
  }
}

// Arrive on this CTA's `bar` only (the drain barrier).
template <int kPair>
__device__ __forceinline__ void tc_commit_local(uint32_t bar) {
  if constexpr (kPair == 1) {
    tc_commit<1>(bar);
  } else {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
  }
}

template <int kPair>
__device__ __forceinline__ void tmem_alloc(uint32_t dst) {
  if constexpr (kPair == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  } else {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
}

template <int kPair>
__device__ __forceinline__ void tmem_dealloc(uint32_t tmem) {
  if constexpr (kPair == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  } else {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

template <int kPair>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                       uint32_t accumulate) {
  if constexpr (kPair == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
  }
}

// The load without its wait; tmem_wait_ld32 waits for every earlier load of
// the thread and then ties the registers of `r` to the wait, so that nothing
// reading them can be scheduled before it.
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
__device__ __forceinline__ void tmem_regs_after_wait(uint32_t (&r)[32]) {
  asm volatile(
      ""
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}
__device__ __forceinline__ void tmem_wait_ld2(uint32_t (&r0)[32], uint32_t (&r1)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  tmem_regs_after_wait(r0);
  tmem_regs_after_wait(r1);
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

// 16 and 32 consecutive 32-bit columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// GELU, tanh form: 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), in
// binary32 with the hardware tanh (relative error about 2^-11).
__device__ __forceinline__ float gelu_tanh(float v) {
  const float u = __fmul_rn(v, __fmaf_rn(0.0356774081f, __fmul_rn(v, v), 0.7978845608f));
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
  const float h = __fmul_rn(0.5f, v);
  return __fmaf_rn(h, t, h);
}

// The epilogue's function of y = alpha * acc (fp32 output).
template <bool kGelu>
__device__ __forceinline__ float epi(float acc, float alpha) {
  const float y = __fmul_rn(acc, alpha);
  return kGelu ? gelu_tanh(y) : y;
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// GELU of both bf16 halves of a word, rounded back to bf16.
__device__ __forceinline__ uint32_t gelu_bf16x2(uint32_t w) {
  return bf16x2_rn(gelu_tanh(__uint_as_float(w << 16)),
                   gelu_tanh(__uint_as_float(w & 0xFFFF0000u)));
}

// ---------------------------------------------------------------- bounded waits
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

// Drain wait: ignores the abort flag (it waits for this CTA's own copies and
// MMAs, which complete by themselves); bounded all the same.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint32_t* status) {
  const uint64_t t0 = globaltimer();
  while (!bar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 2000000000ull) {
      record_status(status, NVFP4_ERR_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int32_t x, int32_t y,
                                             uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   map),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until no committed store group still reads shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// One 128-byte segment of each of this warp's 32 output rows (32 words a
// lane) through the warp's 4 KB staging buffer (128-byte swizzle) and a TMA
// tensor store at column x, row y.
__device__ __forceinline__ void store_row_chunk(const uint32_t (&w)[32], uint32_t buf, int lane,
                                                const CUtensorMap* map, int32_t x, int32_t y) {
  // the previous store from this buffer must have finished reading it
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
  const uint32_t row = buf + uint32_t(lane) * 128;
  const uint32_t sw = uint32_t(lane) & 7;  // 128-byte swizzle: 16-byte unit ^ (row % 8)
#pragma unroll
  for (uint32_t u = 0; u < 8; ++u)
    st_shared_v4(row + ((u ^ sw) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, x, y, buf);
    bulk_commit();
  }
}

struct Params {
  const uint8_t* a_sf;
  const uint8_t* w_sf;
  const float* a_st;
  const float* w_st;
  uint32_t M, N;
  uint32_t ktiles;   // ceil(K / 64): MMA K steps, scale tiles along K
  uint32_t kslabs;   // ceil(K / 256)
  uint32_t tiles_m, tiles_n;  // output tiles: tiles_m of 128 * kPair rows, tiles_n of 256 cols
  uint32_t sf_row_tiles;      // 128-row blocks of A that exist (ceil(M / 128))
  uint32_t w_sf_row_tiles;    // 128-row blocks of W that exist (ceil(N / 128))
  uint32_t* status;
  uint32_t* c_amax;  // float bits of max|C| (atomicMax), or null
  uint32_t amax_tiles;  // N tiles per c_amax word (0: one word)
  uint64_t wait_limit_ns;
  int32_t c_dtype;
};

template <int kPair, bool kGelu>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                      const __grid_constant__ CUtensorMap map_w,
                      const __grid_constant__ CUtensorMap map_c, const Params p) {
  using C = Cfg<kPair>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + C::kOffBar;              // + 8 s
  const uint32_t bar_empty = bar_full + 8 * kStages;         // + 8 s
  const uint32_t bar_sf = bar_empty + 8 * kStages;           // + 8 s (issuing CTA)
  const uint32_t bar_acc_full = bar_sf + 8 * kStages;
  const uint32_t bar_acc_empty = bar_acc_full + 8;           // issuing CTA
  const uint32_t bar_drain = bar_acc_empty + 8;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // rank in the pair (0 = leader, the CTA that issues the MMAs)
  const uint32_t rank = kPair == 2 ? cluster_rank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      bar_init(bar_full + 8 * s, 1);
      bar_init(bar_empty + 8 * s, 1);
      bar_init(bar_sf + 8 * s, 4 * kPair);  // every scale-writer warp of the tile
    }
    bar_init(bar_acc_full, 1);
    bar_init(bar_acc_empty, kEpiWarps * kPair);
    bar_init(bar_drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) tmem_alloc<kPair>(smem_u32(tmem_ptr));
  tc_fence_before();
  if constexpr (kPair == 2) {
    cluster_sync();  // the peer's barriers are initialised before any remote arrival
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  // on-chip setup done; from here on global memory is read and written
  pdl_wait();
  pdl_trigger();

  const Waiter waiter{p.wait_limit_ns, abort_flag, p.status};
  const uint32_t num_tiles = p.tiles_m * p.tiles_n;
  // tiles are walked per CTA (single) or per pair, both CTAs of a pair in step
  const uint32_t t0 = blockIdx.x / kPair, t_step = gridDim.x / kPair;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(&map_a) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&map_w) : "memory");
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (uint32_t t = t0; t < num_tiles && ok; t += t_step) {
        const uint32_t tm = t % p.tiles_m, tn = t / p.tiles_m;
        // this CTA's 128-row block of A; past the last one (a pair's follower
        // when the row blocks run out) the code loads read zeros and no scales
        // are loaded
        const uint32_t rt = tm * kPair + rank;
        const bool a_live = rt < p.sf_row_tiles;
        // the tile's second 128 W rows may lie past the last row block of W
        // (N not a multiple of 256): their scales are not loaded, and the
        // output columns they feed are neither stored nor counted in c_amax
        const uint32_t w_halves = 2 * tn + 1 < p.w_sf_row_tiles ? 2u : 1u;
        for (uint32_t kb = 0; kb < p.kslabs; ++kb) {
          if (!waiter.wait(bar_empty + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t nk = min(uint32_t(kKSteps), p.ktiles - kb * kKSteps);
          const uint32_t fb = bar_full + 8 * stage;
          bar_arrive_expect_tx(fb, kABytes + C::kBBytes + ((a_live ? 1u : 0u) + w_halves) * 512u * nk);
          tma_load_2d(sbase + C::kOffA + stage * kABytes, &map_a, int32_t(kb * kBKBytes),
                      int32_t(rt * kBM), fb);
          tma_load_2d(sbase + C::kOffB + stage * C::kBBytes, &map_w, int32_t(kb * kBKBytes),
                      int32_t(tn * kBN + rank * C::kBRows), fb);
          if (a_live)
            bulk_load(sbase + C::kOffSfa + stage * kSfaBytes,
                      p.a_sf + (size_t(rt) * p.ktiles + kb * kKSteps) * 512, 512 * nk, fb);
          // the scales of all 256 W rows of the tile, in either form
          for (uint32_t h = 0; h < w_halves; ++h)
            bulk_load(sbase + C::kOffSfb + stage * kSfbBytes + h * 2048,
                      p.w_sf + (size_t(2 * tn + h) * p.ktiles + kb * kKSteps) * 512, 512 * nk,
                      fb);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      // drain: wait until every copy this thread issued has landed
      for (uint32_t s = 0; s < kStages && s < issued; ++s) {
        const uint32_t last = ((issued - 1 - s) / kStages) * kStages + s;  // last issue on stage s
        drain_wait(bar_full + 8 * s, (last / kStages) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One thread of the issuing CTA.  Per stage: wait until the writers of
    // every CTA of the tile have put the stage's scales in tensor memory (they
    // did so after seeing the stage's operands land), issue the stage's MMAs,
    // commit them to the stage's empty barrier (both CTAs' in a pair).  Per
    // tile: wait until every epilogue warp read the previous accumulator out,
    // and commit the tile's MMAs to acc_full.
    if (leader && lane == 0) {
      uint32_t stage = 0, phase = 0, local = 0;
      bool ok = true;
      for (uint32_t t = t0; t < num_tiles && ok; t += t_step, ++local) {
        if (local > 0 && !waiter.wait(bar_acc_empty, (local - 1) & 1)) break;
        tc_fence_after();
        for (uint32_t kb = 0; kb < p.kslabs; ++kb) {
          if (!waiter.wait(bar_sf + 8 * stage, phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t nk = min(uint32_t(kKSteps), p.ktiles - kb * kKSteps);
          const uint64_t a_d = desc_sw128(sbase + C::kOffA + stage * kABytes);
          const uint64_t b_d = desc_sw128(sbase + C::kOffB + stage * C::kBBytes);
          const uint32_t sf = tmem + kSfCol + kSfSetCols * stage;
          for (uint32_t j = 0; j < nk; ++j)  // K step j: +32 bytes = +2 in the address field
            tc_mma<kPair>(tmem, a_d + 2 * j, b_d + 2 * j, C::kIdesc, sf + 4 * j,
                          sf + kSfWCol + 8 * j, (kb | j) != 0);
          // frees the shared-memory stage and its scale set (of both CTAs of a
          // pair) once these MMAs complete
          tc_commit<kPair>(bar_empty + 8 * stage);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit<kPair>(bar_acc_full);
      }
      // drain: every tcgen05 operation this thread issued has completed
      tc_commit_local<kPair>(bar_drain);
      drain_wait(bar_drain, 0, p.status);
    }
    __syncwarp();
  } else if (warp >= kWriterWarp0) {
    // ------------------------------------------------------------ scale writers
    // Each warp owns one tensor-memory lane quadrant q; lane quadrant q of the
    // tensor core computes output rows 32q..32q+31 of this CTA's 128.  A staged
    // scale tile is 32 chunks of 16 bytes, chunk l holding the four E4M3 scales
    // of rows l, l+32, l+64, l+96 of a 128-row operand tile.  Per K step the
    // MMA reads
    //   A scales of row 32q + l: lane 32q + l, column sfa + q (its own rows);
    //   W scales of row n (any of the 256, every quadrant needs them all):
    //     lane 32q + n % 32, column sfb + n / 32.
    // In a pair each CTA's tensor memory holds the same layout for its own 128
    // rows of A and all 256 W rows of the tile.  So warp q writes A chunk
    // `lane` (of which word q is read) and both W chunks `lane` whole (4 columns
    // each) into its lanes, a stage at a time, into the stage's scale set, then
    // arrives on the issuing CTA's sf_ready barrier of the stage.  A set is free
    // when its stage is full again: the producer refilled the stage after the
    // MMAs that read the set completed.
    const uint32_t q = uint32_t(warp & 3);
    const uint32_t lane_bits = (q * 32) << 16;
    const uint32_t sf_bar0 = kPair == 2 && !leader ? map_to_rank(bar_sf, 0) : bar_sf;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (uint32_t t = t0; t < num_tiles && ok; t += t_step) {
      for (uint32_t kb = 0; kb < p.kslabs; ++kb) {
        ok = __all_sync(0xFFFFFFFFu, waiter.wait(bar_full + 8 * stage, phase));
        if (!ok) break;
        tc_fence_after();
        const uint32_t sfa_s = sbase + C::kOffSfa + stage * kSfaBytes + 16 * uint32_t(lane) + 4 * q;
        const uint32_t sfb_s = sbase + C::kOffSfb + stage * kSfbBytes + 16 * uint32_t(lane);
        const uint32_t col = tmem + lane_bits + kSfCol + kSfSetCols * stage;
        // the whole set in two stores: A word j repeated over columns 4j..4j+3
        // (only column 4j + q of these lanes is read), W chunks j over 16 + 8j..
        // (K steps past nk, in a last partial stage, write values no MMA reads)
        uint32_t av[16], wv[32];
#pragma unroll
        for (int j = 0; j < kKSteps; ++j) {
          const uint32_t a = ld_shared_u32(sfa_s + 512 * j);
          const uint4 lo = ld_shared_v4(sfb_s + 512 * j);
          const uint4 hi = ld_shared_v4(sfb_s + 2048 + 512 * j);
          av[4 * j] = av[4 * j + 1] = av[4 * j + 2] = av[4 * j + 3] = a;
          wv[8 * j] = lo.x, wv[8 * j + 1] = lo.y, wv[8 * j + 2] = lo.z, wv[8 * j + 3] = lo.w;
          wv[8 * j + 4] = hi.x, wv[8 * j + 5] = hi.y, wv[8 * j + 6] = hi.z, wv[8 * j + 7] = hi.w;
        }
        tmem_st16(col, av);
        tmem_st32(col + kSfWCol, wv);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kPair == 2 && !leader) {
            bar_arrive_remote(sf_bar0 + 8 * stage);
          } else {
            bar_arrive(sf_bar0 + 8 * stage);
          }
        }
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w (2..9) reads lane quadrant w % 4 (its 32 output rows) and columns
    // [128 h, 128 h + 128), h = (w - 2) / 4, of the accumulator into registers
    // (bf16: 64 packed words a thread), scales by s_tA * s_tW and releases the
    // accumulator before its stores, so the next tile's MMAs wait only for the
    // reads.  For bf16 output the activation (kGelu) takes the bf16 products
    // after the release; for fp32 output it runs as the values are read.
    const uint32_t ew = uint32_t(warp - 2);
    const uint32_t quad = uint32_t(warp & 3);          // tensor-memory lane quadrant
    const uint32_t half = ew >> 2;                     // column half of the tile
    const float alpha = __fmul_rn(*p.a_st, *p.w_st);
    const bool bf16 = p.c_dtype == NVFP4_BF16;
    const uint32_t buf = sbase + C::kOffStage + ew * kStageBufBytes;
    const uint32_t acc_empty =
        kPair == 2 && !leader ? map_to_rank(bar_acc_empty, 0) : bar_acc_empty;
    auto release = [&]() {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (kPair == 2 && !leader) {
          bar_arrive_remote(acc_empty);
        } else {
          bar_arrive(acc_empty);
        }
      }
    };
    uint32_t local = 0;
    // running max of |stored value| as magnitude bits (two bf16 halves, or
    // fp32) for c_amax word `word`; flushed when the tiles move to another word
    uint32_t vmax = 0, word = 0;
    const bool want_max = p.c_amax != nullptr;
    auto flush_max = [&]() {
      // fold the bf16 halves into fp32 bits (bf16 bits << 16 is the same value)
      const uint32_t bits = bf16 ? (max(vmax & 0xFFFFu, vmax >> 16) << 16) : vmax;
      const uint32_t wmax = __reduce_max_sync(0xFFFFFFFFu, bits);
      if (lane == 0 && wmax != 0) atomicMax(p.c_amax + word, wmax);
      vmax = 0;
    };
    for (uint32_t t = t0; t < num_tiles; t += t_step, ++local) {
      const uint32_t tm = t % p.tiles_m, tn = t / p.tiles_m;
      if (want_max && p.amax_tiles > 0 && tn / p.amax_tiles != word) {
        flush_max();
        word = tn / p.amax_tiles;
      }
      const uint32_t row0 = (tm * kPair + rank) * kBM + quad * 32;  // this warp's first row
      // accumulator lanes past the last row of C hold no output; leave them out
      const bool row_live = want_max && row0 + uint32_t(lane) < p.M;
      const bool store = row0 < p.M;  // warp-uniform: some of the 32 rows exist
      const int32_t y = int32_t(row0);
      const int32_t x0 = int32_t(tn * kBN + half * 128);
      const int32_t n_left = int32_t(p.N) - x0;  // columns of this warp's 128 that exist
      // warp-uniform outcome: tcgen05.ld below is .sync.aligned
      const bool ok = waiter.wait(bar_acc_full, local & 1);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ((quad * 32) << 16) + half * 128;
      if (bf16) {
        uint32_t pk[64];
        auto pack = [&](const uint32_t (&r)[32], int c) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[16 * c + e] = bf16x2_rn(__fmul_rn(__uint_as_float(r[2 * e]), alpha),
                                       __fmul_rn(__uint_as_float(r[2 * e + 1]), alpha));
        };
        // two 32-column loads in flight per wait; chunks 2 and 3 are loaded
        // while chunks 0 and 1 are packed, and the accumulator is released as
        // soon as the last load has landed, before the last packing
        uint32_t r0[32], r1[32], r2[32];
        tmem_ld32_async(taddr, r0);
        tmem_ld32_async(taddr + 32, r1);
        tmem_wait_ld2(r0, r1);
        tmem_ld32_async(taddr + 64, r2);
        pack(r0, 0);
        tmem_ld32_async(taddr + 96, r0);
        pack(r1, 1);
        tmem_wait_ld2(r2, r0);
        release();
        pack(r2, 2);
        pack(r0, 3);
        // the activation runs on the bf16 products once the accumulator is
        // released, overlapping the next tile's MMAs: a bf16 linear layer
        // followed by its activation
        if (kGelu) {
#pragma unroll
          for (int e = 0; e < 64; ++e) pk[e] = gelu_bf16x2(pk[e]);
        }
        if (row_live) {
          if (n_left >= 128) {
#pragma unroll
            for (int e = 0; e < 64; ++e) vmax = __vmaxu2(vmax, pk[e] & 0x7FFF7FFFu);
          } else {  // the tile's last columns lie past N
#pragma unroll
            for (int e = 0; e < 64; ++e)
              vmax = __vmaxu2(vmax, pk[e] & ((2 * e < n_left ? 0x7FFFu : 0u) |
                                             (2 * e + 1 < n_left ? 0x7FFF0000u : 0u)));
          }
        }
        if (store) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
            if (64 * ch < n_left)  // a chunk past N is not stored (a partial one is clipped)
              store_row_chunk(*reinterpret_cast<const uint32_t(*)[32]>(&pk[32 * ch]), buf, lane,
                              &map_c, x0 + 64 * ch, y);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + 32 * c, v);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            v[e] = __float_as_uint(epi<kGelu>(__uint_as_float(v[e]), alpha));
          if (c == 3) release();
          if (row_live) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              vmax = max(vmax, 32 * c + e < n_left ? v[e] & 0x7FFFFFFFu : 0u);
          }
          if (store && 32 * c < n_left) store_row_chunk(v, buf, lane, &map_c, x0 + 32 * c, y);
        }
      }
    }
    if (want_max) flush_max();
    // drain: every store this warp issued has completed
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  if constexpr (kPair == 2) {
    // neither CTA of the pair frees tensor memory or leaves while the leader's
    // MMAs (drained above) or the follower's arrivals may still touch the other
    cluster_sync();
  } else {
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 1) tmem_dealloc<kPair>(tmem);
}

}  // namespace gemm

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D map over uint8 code rows: box of 128 bytes x box_rows, 128-byte swizzle.
static bool make_code_map(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                          uint32_t box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {uint32_t(gemm::kBKBytes), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map over the output C (rows x cols elements, row stride ldc): box of
// 128 bytes x 32 rows, 128-byte swizzle (the epilogue's staging layout).
static bool make_out_map(CUtensorMap* map, void* base, int32_t dtype, uint64_t rows, uint64_t cols,
                         uint64_t ldc) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  const uint64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ldc * esz};
  cuuint32_t box[2] = {uint32_t(128 / esz), 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, dtype == NVFP4_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The pair form whenever A has more than one 128-row block: it computes the
// same tiles with half the W bytes per CTA and half the MMA instructions.
static bool use_pair(int64_t M) { return M > gemm::kBM; }

template <int kPair, bool kGelu>
static cudaError_t launch_form(const CUtensorMap& map_a, const CUtensorMap& map_w,
                               const CUtensorMap& map_c, const gemm::Params& p, int sm_count,
                               cudaStream_t st) {
  using C = gemm::Cfg<kPair>;
  // the shared-memory opt-in is per device; host threads may race here, and
  // setting the attribute twice is harmless, so each device keeps one flag
  // (configured[dev] holds 1 + the number of CTAs -- single -- or pairs that
  // can be resident at once)
  static std::atomic<int> configured[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(gemm::kThreads);
  cfg.dynamicSmemBytes = size_t(C::kSmemBytes);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = kPair;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kPair == 2 ? 2 : 1;
  int slots = configured[dev].load(std::memory_order_acquire) - 1;
  if (slots < 0) {
    cudaError_t e = cudaFuncSetAttribute(gemm::nvfp4_gemm_kernel<kPair, kGelu>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    slots = sm_count / kPair;
    if (kPair == 2) {
      // pairs must sit on two SMs of one GPC: ask how many fit at once
      int n = 0;
      cfg.gridDim = dim3(2 * slots);
      if (cudaOccupancyMaxActiveClusters(&n, gemm::nvfp4_gemm_kernel<kPair, kGelu>, &cfg) ==
              cudaSuccess &&
          n > 0 && n < slots)
        slots = n;
    }
    configured[dev].store(slots + 1, std::memory_order_release);
  }
  const uint32_t tiles = p.tiles_m * p.tiles_n;
  cfg.gridDim = dim3(kPair * int(tiles < uint32_t(slots) ? tiles : uint32_t(slots)));
  return cudaLaunchKernelEx(&cfg, gemm::nvfp4_gemm_kernel<kPair, kGelu>, map_a, map_w, map_c, p);
}

cudaError_t launch_gemm(const LaunchGemm& g, cudaStream_t st) {
  const bool pair = use_pair(g.M);
  const uint32_t w_box_rows = pair ? uint32_t(gemm::Cfg<2>::kBRows) : uint32_t(gemm::kBN);
  CUtensorMap map_a, map_w, map_c;
  if (!make_code_map(&map_a, g.a_codes, uint64_t(g.K / 2), uint64_t(g.M), gemm::kBM) ||
      !make_code_map(&map_w, g.w_codes, uint64_t(g.K / 2), uint64_t(g.N), w_box_rows) ||
      !make_out_map(&map_c, g.c, g.c_dtype, uint64_t(g.M), uint64_t(g.N), uint64_t(g.ldc)))
    return cudaErrorInvalidValue;
  const int64_t tile_m = pair ? 2 * gemm::kBM : gemm::kBM;
  gemm::Params p;
  p.a_sf = g.a_sf;
  p.w_sf = g.w_sf;
  p.a_st = g.a_st;
  p.w_st = g.w_st;
  p.M = uint32_t(g.M);
  p.N = uint32_t(g.N);
  p.ktiles = uint32_t((g.K + 63) / 64);  // a last partial K step reads zero codes and scales
  p.kslabs = uint32_t((g.K + 255) / 256);
  p.tiles_m = uint32_t((g.M + tile_m - 1) / tile_m);
  p.tiles_n = uint32_t((g.N + gemm::kBN - 1) / gemm::kBN);
  p.w_sf_row_tiles = uint32_t((g.N + gemm::kBM - 1) / gemm::kBM);
  p.sf_row_tiles = uint32_t((g.M + gemm::kBM - 1) / gemm::kBM);
  p.status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(g.ws) + kWsStatus);
  p.c_amax = reinterpret_cast<uint32_t*>(g.c_amax);
  p.amax_tiles = uint32_t(g.c_amax_cols / gemm::kBN);
  p.wait_limit_ns = g.wait_limit_ns;
  p.c_dtype = g.c_dtype;
  const bool gelu = g.act == NVFP4_ACT_GELU_TANH;
  if (pair)
    return gelu ? launch_form<2, true>(map_a, map_w, map_c, p, g.sm_count, st)
                : launch_form<2, false>(map_a, map_w, map_c, p, g.sm_count, st);
  return gelu ? launch_form<1, true>(map_a, map_w, map_c, p, g.sm_count, st)
              : launch_form<1, false>(map_a, map_w, map_c, p, g.sm_count, st);
}

}  // namespace nvfp4
