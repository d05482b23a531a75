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
// Structure: one persistent CTA per SM walks 128 x 256 output tiles.
//   warp 0      TMA producer: 2-D tensor copies of the A and W code tiles
//               (128-byte K slabs, 128-byte swizzle) and 1-D bulk copies of the
//               matching 512-byte scale tiles into a 4-stage shared-memory ring.
//   warp 1      tensor-core issuer: copies each stage's scales into tensor
//               memory (tcgen05.cp) and issues 4 MMAs of K = 64 per stage; it
//               also owns the tensor-memory allocation.
//   warps 2..5  epilogue: tensor memory -> registers (tcgen05.ld), scale by
//               s_tA * s_tW, round to bf16 / fp32, store; masked M tail.
// Every spin-wait is bounded (wait_limit_ns).  A wait that runs out records
// NVFP4_ERR_TIMEOUT, raises a CTA-wide abort flag, and the CTA drains its own
// copies and MMAs in flight before freeing tensor memory and returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {
namespace gemm {

constexpr int kBM = 128;          // tile rows (A rows)
constexpr int kBN = 256;          // tile cols (W rows)
constexpr int kBKBytes = 128;     // K slab per stage: 128 bytes = 256 FP4 values
constexpr int kStages = 4;
constexpr int kKSteps = 4;        // MMA K = 64 values = 32 bytes
constexpr int kABytes = kBM * kBKBytes;      // 16 KB
constexpr int kBBytes = kBN * kBKBytes;      // 32 KB
constexpr int kSfaBytes = 4 * 512;           // 4 scale tiles of 128 rows x 4 blocks
constexpr int kSfbBytes = 2 * 4 * 512;       // 2 row tiles of W
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccCols = kBN;                // fp32 accumulator: 128 lanes x 256 cols
constexpr int kSfColsPerStage = 48;          // SFA 4 x 4 + SFB 4 x 8 columns

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStages * kABytes;
constexpr int kOffSfa = kOffB + kStages * kBBytes;
constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
constexpr int kOffBar = kOffSfb + kStages * kSfbBytes;
constexpr int kNumBars = 2 * kStages + 3;    // full[], empty[], acc_full, acc_empty, drain
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kOffAbort = kOffTmemPtr + 4;
constexpr int kSmemBytes = kOffAbort + 4 + 1024;  // + alignment slack

// Instruction descriptor, block-scaled kinds: E2M1 A and B (format 1 at bits
// 7-9 and 10-12), K-major both, N >> 3 at bits 17-22, E4M3 scales (bit 23 = 0),
// M >> 4 at bits 24-28, scale-factor ids 0.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) |
                            (uint32_t(kBM >> 4) << 24);

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
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void bar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Descriptor of a 32-row x 16-byte scale tile (no swizzle; 8-row core
// matrices of 128 bytes, 128 bytes apart), the source of tcgen05.cp 32x128b.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(128 >> 4) << 32) | (uint64_t(1) << 46);
}

__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X"
      " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
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

struct Params {
  const uint8_t* a_sf;
  const uint8_t* w_sf;
  const float* a_st;
  const float* w_st;
  void* c;
  int64_t ldc;
  uint32_t M, N;
  uint32_t ktiles;   // K / 64
  uint32_t kslabs;   // ceil(K / 256)
  uint32_t tiles_m, tiles_n;
  uint32_t* status;
  uint64_t wait_limit_ns;
  int32_t c_dtype;
};

__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                      const __grid_constant__ CUtensorMap map_w, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + kOffBar;                 // + 8 s
  const uint32_t bar_empty = bar_full + 8 * kStages;         // + 8 s
  const uint32_t bar_acc_full = bar_empty + 8 * kStages;
  const uint32_t bar_acc_empty = bar_acc_full + 8;
  const uint32_t bar_drain = bar_acc_empty + 8;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      bar_init(bar_full + 8 * s, 1);
      bar_init(bar_empty + 8 * s, 1);
    }
    bar_init(bar_acc_full, 1);
    bar_init(bar_acc_empty, 4);
    bar_init(bar_drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
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

  const Waiter waiter{p.wait_limit_ns, abort_flag, p.status};
  const uint32_t num_tiles = p.tiles_m * p.tiles_n;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(&map_a) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&map_w) : "memory");
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (uint32_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const uint32_t tm = t % p.tiles_m, tn = t / p.tiles_m;
        for (uint32_t kb = 0; kb < p.kslabs; ++kb) {
          if (!waiter.wait(bar_empty + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t nk = min(uint32_t(kKSteps), p.ktiles - kb * kKSteps);
          const uint32_t fb = bar_full + 8 * stage;
          bar_arrive_expect_tx(fb, kABytes + kBBytes + 3 * 512 * nk);
          tma_load_2d(sbase + kOffA + stage * kABytes, &map_a, int32_t(kb * kBKBytes),
                      int32_t(tm * kBM), fb);
          tma_load_2d(sbase + kOffB + stage * kBBytes, &map_w, int32_t(kb * kBKBytes),
                      int32_t(tn * kBN), fb);
          bulk_load(sbase + kOffSfa + stage * kSfaBytes,
                    p.a_sf + (size_t(tm) * p.ktiles + kb * kKSteps) * 512, 512 * nk, fb);
          for (uint32_t h = 0; h < 2; ++h)
            bulk_load(sbase + kOffSfb + stage * kSfbBytes + h * 2048,
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, local = 0;
      bool ok = true;
      for (uint32_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        if (!waiter.wait(bar_acc_empty, (local & 1) ^ 1)) break;
        tc_fence_after();
        for (uint32_t kb = 0; kb < p.kslabs; ++kb) {
          if (!waiter.wait(bar_full + 8 * stage, phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t nk = min(uint32_t(kKSteps), p.ktiles - kb * kKSteps);
          const uint32_t sf_col = tmem + kAccCols + kSfColsPerStage * stage;
          const uint32_t sfa_s = sbase + kOffSfa + stage * kSfaBytes;
          const uint32_t sfb_s = sbase + kOffSfb + stage * kSfbBytes;
          for (uint32_t j = 0; j < nk; ++j) {
            tc_cp_sf(sf_col + 4 * j, desc_sf(sfa_s + 512 * j));
            tc_cp_sf(sf_col + 16 + 8 * j, desc_sf(sfb_s + 512 * j));
            tc_cp_sf(sf_col + 16 + 8 * j + 4, desc_sf(sfb_s + 2048 + 512 * j));
          }
          const uint32_t a_s = sbase + kOffA + stage * kABytes;
          const uint32_t b_s = sbase + kOffB + stage * kBBytes;
          for (uint32_t j = 0; j < nk; ++j) {
            tc_mma(tmem, desc_sw128(a_s + 32 * j), desc_sw128(b_s + 32 * j), kIdesc,
                   sf_col + 4 * j, sf_col + 16 + 8 * j, (kb | j) != 0);
          }
          tc_commit(bar_empty + 8 * stage);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(bar_acc_full);
      }
      // drain: every tcgen05 operation this thread issued has completed
      tc_commit(bar_drain);
      drain_wait(bar_drain, 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t quad = uint32_t(warp & 3);
    const uint32_t row_in_tile = quad * 32 + lane;
    const float alpha = __fmul_rn(*p.a_st, *p.w_st);
    uint32_t local = 0;
    for (uint32_t t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      const uint32_t tm = t % p.tiles_m, tn = t / p.tiles_m;
      // warp-uniform outcome: tcgen05.ld below is .sync.aligned
      const bool ok = waiter.wait(bar_acc_full, local & 1);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const uint32_t m = tm * kBM + row_in_tile;
      const bool row_ok = m < p.M;
      const uint32_t taddr = tmem + ((quad * 32) << 16);
#pragma unroll 1
      for (uint32_t cb = 0; cb < kBN / 32; ++cb) {
        uint32_t r[32];
        tmem_ld32(taddr + cb * 32, r);
        if (cb == kBN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) bar_arrive(bar_acc_empty);
        }
        if (row_ok) {
          const size_t col = size_t(tn) * kBN + cb * 32;
          if (p.c_dtype == NVFP4_BF16) {
            uint8_t* dst =
                static_cast<uint8_t*>(p.c) + (size_t(m) * size_t(p.ldc) + col) * 2;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              uint32_t* ow = &o.x;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float lo = __fmul_rn(__uint_as_float(r[8 * v + 2 * e]), alpha);
                const float hi = __fmul_rn(__uint_as_float(r[8 * v + 2 * e + 1]), alpha);
                __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
                ow[e] = *reinterpret_cast<uint32_t*>(&b2);
              }
              st_v4(dst + 16 * v, o);
            }
          } else {
            uint8_t* dst =
                static_cast<uint8_t*>(p.c) + (size_t(m) * size_t(p.ldc) + col) * 4;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              uint4 o;
              o.x = __float_as_uint(__fmul_rn(__uint_as_float(r[4 * v + 0]), alpha));
              o.y = __float_as_uint(__fmul_rn(__uint_as_float(r[4 * v + 1]), alpha));
              o.z = __float_as_uint(__fmul_rn(__uint_as_float(r[4 * v + 2]), alpha));
              o.w = __float_as_uint(__fmul_rn(__uint_as_float(r[4 * v + 3]), alpha));
              st_v4(dst + 16 * v, o);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace gemm

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

static bool make_code_map(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                          uint32_t box_rows) {
  auto encode = get_encode();
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

cudaError_t launch_gemm(const LaunchGemm& g, cudaStream_t st) {
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(gemm::nvfp4_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         gemm::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  CUtensorMap map_a, map_w;
  if (!make_code_map(&map_a, g.a_codes, uint64_t(g.K / 2), uint64_t(g.M), gemm::kBM) ||
      !make_code_map(&map_w, g.w_codes, uint64_t(g.K / 2), uint64_t(g.N), gemm::kBN))
    return cudaErrorInvalidValue;
  gemm::Params p;
  p.a_sf = g.a_sf;
  p.w_sf = g.w_sf;
  p.a_st = g.a_st;
  p.w_st = g.w_st;
  p.c = g.c;
  p.ldc = g.ldc;
  p.M = uint32_t(g.M);
  p.N = uint32_t(g.N);
  p.ktiles = uint32_t(g.K / 64);
  p.kslabs = uint32_t((g.K + 255) / 256);
  p.tiles_m = uint32_t((g.M + gemm::kBM - 1) / gemm::kBM);
  p.tiles_n = uint32_t(g.N / gemm::kBN);
  p.status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(g.ws) + kWsStatus);
  p.wait_limit_ns = g.wait_limit_ns;
  p.c_dtype = g.c_dtype;
  const uint32_t tiles = p.tiles_m * p.tiles_n;
  const int grid = int(tiles < uint32_t(g.sm_count) ? tiles : uint32_t(g.sm_count));
  gemm::nvfp4_gemm_kernel<<<grid, gemm::kThreads, gemm::kSmemBytes, st>>>(map_a, map_w, p);
  return cudaGetLastError();
}

}  // namespace nvfp4
