// noalloc.cu -- nvfp4_quantize without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they need to
// quantize: code running inside a fixed memory budget whose allocator is owned
// by someone else (an inference server's arena, an embedded runtime), plugin
// hooks that are handed only input and output buffers, or code paths where a
// cudaMalloc would synchronize the device at the wrong moment.  For them this
// file keeps the quantizer's scratch words (running amax, CTA counter, status
// word) in a fixed array that lives in the library's own device memory: every
// GPU that loads the library holds these 256 bytes until the process exits.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {
namespace {

// The scratch: same word layout as the caller workspace of nvfp4_quantize.
constexpr size_t kNoallocScratchBytes = NVFP4_NOALLOC_SCRATCH_BYTES;
static_assert(kWsBytes <= kNoallocScratchBytes, "scratch layout outgrew the static array");
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.  The cache never expires:
// the address belongs to the device's primary context, so a cudaDeviceReset
// leaves it stale (the header tells callers not to use this entry point on a
// device after resetting it).  The status word at kWsStatus is written by a
// kernel that meets an out-of-domain tensor scale and never read or cleared:
// nothing here reports it.
cudaError_t scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int32_t dtype, int64_t rows,
                                               int64_t cols, int64_t ld, const nvfp4_tensor* out,
                                               const float* s_t_in, void* stream) {
  if (kWsBytes > kNoallocScratchBytes) return NVFP4_ERR_WORKSPACE;
  if (!x || (dtype != NVFP4_BF16 && dtype != NVFP4_FP32)) return NVFP4_ERR_INVALID_ARG;
  if (!out || !out->codes || !out->sf || !out->s_t) return NVFP4_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows != out->rows || cols != out->cols || ld < cols)
    return NVFP4_ERR_INVALID_ARG;
  if (out->sf_layout != NVFP4_SF_ROWMAJOR && out->sf_layout != NVFP4_SF_MMA128x4)
    return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0 || rows * (cols / 8) >= (int64_t(1) << 32))
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  auto al = [](const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; };
  if (!al(x, 16) || (ld * esz) % 16 != 0 || !al(out->codes, 16) || !al(out->sf, 16) ||
      !al(out->s_t, 4) || (s_t_in && !al(s_t_in, 4)))
    return NVFP4_ERR_MISALIGNED;
  int dev = 0, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_ARCH;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || minor != 0) return NVFP4_ERR_ARCH;
  void* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) return NVFP4_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left; the amax and counter
  // words must start at zero.
  if (cudaMemsetAsync(scratch, 0, kWsStatus, st) != cudaSuccess) return NVFP4_ERR_CUDA;
  LaunchQuant q;
  q.x = x;
  q.dtype = dtype;
  q.rows = rows;
  q.cols = cols;
  q.ld = ld;
  q.codes = out->codes;
  q.sf = out->sf;
  q.sf_layout = out->sf_layout;
  q.s_t_out = out->s_t;
  q.s_t_in = s_t_in;
  q.amax_in = nullptr;
  q.ws = scratch;
  q.sm_count = sms;
  q.wait_limit_ns = 2000000000ull;
  return launch_quantize(q, st) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
