// api.cu -- the C ABI of libnvfp4 (declared in include/nvfp4.h): host-side
// argument checks, then one or two kernel launches on the caller's stream.
#include <cmath>
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

using namespace nvfp4;

namespace {

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

struct DeviceInfo {
  bool ok;
  int sm_count;
};

// Compute capability and SM count of the current device, cached per device.
// Host threads may call in concurrently: an entry is published through its
// atomic word (0 = not yet queried, else 1 + sm_count, negated when the
// device is not sm_100), so a reader sees either nothing or a whole entry.
DeviceInfo current_device() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return {false, 0};
  int word = cache[dev].load(std::memory_order_acquire);
  if (word == 0) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    word = (major == 10 && minor == 0) ? 1 + sms : -(1 + sms);
    cache[dev].store(word, std::memory_order_release);
  }
  return {word > 0, (word > 0 ? word : -word) - 1};
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

bool valid_layout(int32_t l) { return l == NVFP4_SF_ROWMAJOR || l == NVFP4_SF_MMA128x4; }

// Checks shared by every NVFP4 tensor argument.
nvfp4_status check_tensor(const nvfp4_tensor* t) {
  if (!t || !t->codes || !t->sf || !t->s_t) return NVFP4_ERR_INVALID_ARG;
  if (t->rows <= 0 || t->cols <= 0 || !valid_layout(t->sf_layout)) return NVFP4_ERR_INVALID_ARG;
  if (t->cols % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (t->rows * (t->cols / 8) >= (int64_t(1) << 32)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(t->codes, 16) || !aligned(t->sf, 16) || !aligned(t->s_t, 4))
    return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

nvfp4_status check_cache(const nvfp4_kv_cache* c) {
  if (!c || !c->k_codes || !c->v_codes || !c->k_sf || !c->v_sf || !c->k_st || !c->v_st)
    return NVFP4_ERR_INVALID_ARG;
  if (c->n_slots <= 0 || c->tokens_per_frame <= 0 || c->heads <= 0 || c->head_dim <= 0)
    return NVFP4_ERR_INVALID_ARG;
  if (c->scale_rule != NVFP4_SCALE_ONTO_6 && c->scale_rule != NVFP4_SCALE_FOUR_OVER_SIX)
    return NVFP4_ERR_INVALID_ARG;
  if (c->head_dim % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const int64_t per_frame = int64_t(c->tokens_per_frame) * c->heads * c->head_dim;
  if (per_frame * c->n_slots / 8 >= (int64_t(1) << 32)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(c->k_codes, 16) || !aligned(c->v_codes, 16) || !aligned(c->k_sf, 16) ||
      !aligned(c->v_sf, 16) || !aligned(c->k_st, 4) || !aligned(c->v_st, 4))
    return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

}  // namespace

extern "C" {

size_t nvfp4_codes_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0 || cols % 16 != 0) return 0;
  return size_t(rows) * size_t(cols / 2);
}

size_t nvfp4_sf_bytes(int64_t rows, int64_t cols, int32_t sf_layout) {
  if (rows < 0 || cols < 0 || cols % 16 != 0 || !valid_layout(sf_layout)) return 0;
  if (sf_layout == NVFP4_SF_ROWMAJOR) return size_t(rows) * size_t(cols / 16);
  const size_t rows_pad = size_t((rows + 127) / 128) * 128;
  const size_t blocks_pad = size_t((cols / 16 + 3) / 4) * 4;
  return rows_pad * blocks_pad;
}

size_t nvfp4_workspace_bytes(void) { return kWsBytes; }

void nvfp4_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or stride";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_ARCH: return "device is not sm_100 (B200)";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    case NVFP4_ERR_DOMAIN: return "tensor scale outside the recipe's domain";
  }
  return "unknown status";
}

nvfp4_status nvfp4_quantize(const void* x, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                            const nvfp4_tensor* out, const float* s_t_in, float* amax_in, void* ws,
                            size_t ws_bytes, void* stream) {
  if (!x || (dtype != NVFP4_BF16 && dtype != NVFP4_FP32)) return NVFP4_ERR_INVALID_ARG;
  if (s_t_in && amax_in) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_tensor(out);
  if (st != NVFP4_OK) return st;
  if (rows != out->rows || cols != out->cols || ld < cols) return NVFP4_ERR_INVALID_ARG;
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  if (!aligned(x, 16) || (ld * esz) % 16 != 0) return NVFP4_ERR_MISALIGNED;
  if ((s_t_in && !aligned(s_t_in, 4)) || (amax_in && !aligned(amax_in, 4)))
    return NVFP4_ERR_MISALIGNED;
  if (!ws || ws_bytes < kWsBytes) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return NVFP4_ERR_MISALIGNED;
  const DeviceInfo dev = current_device();
  if (!dev.ok) return NVFP4_ERR_ARCH;
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
  q.amax_in = amax_in;
  q.ws = ws;
  q.sm_count = dev.sm_count;
  q.wait_limit_ns = g_wait_limit_ns.load();
  return cuda_status(launch_quantize(q, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_dequantize(const nvfp4_tensor* in, void* out, int64_t ld, void* stream) {
  nvfp4_status st = check_tensor(in);
  if (st != NVFP4_OK) return st;
  if (!out || ld < in->cols) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(out, 16) || ld % 8 != 0) return NVFP4_ERR_MISALIGNED;
  const DeviceInfo dev = current_device();
  if (!dev.ok) return NVFP4_ERR_ARCH;
  LaunchDequant d;
  d.codes = in->codes;
  d.sf = in->sf;
  d.s_t = in->s_t;
  d.sf_layout = in->sf_layout;
  d.rows = in->rows;
  d.cols = in->cols;
  d.ld = ld;
  d.out = out;
  d.sm_count = dev.sm_count;
  return cuda_status(launch_dequantize(d, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* W, void* C, int32_t c_dtype,
                        int64_t ldc, int32_t act, float* c_amax, int64_t c_amax_cols, void* ws,
                        size_t ws_bytes, void* stream) {
  nvfp4_status st = check_tensor(A);
  if (st != NVFP4_OK) return st;
  st = check_tensor(W);
  if (st != NVFP4_OK) return st;
  if (!C || (c_dtype != NVFP4_BF16 && c_dtype != NVFP4_FP32)) return NVFP4_ERR_INVALID_ARG;
  if (act != NVFP4_ACT_NONE && act != NVFP4_ACT_GELU_TANH) return NVFP4_ERR_INVALID_ARG;
  if (A->sf_layout != NVFP4_SF_MMA128x4 || W->sf_layout != NVFP4_SF_MMA128x4)
    return NVFP4_ERR_INVALID_ARG;
  if (A->cols != W->cols) return NVFP4_ERR_INVALID_ARG;
  // K: whole 16-byte code rows (TMA); a K step past K reads TMA zero fill and the
  // scale layout's zero padding
  if (A->cols % 32 != 0 || W->rows < 1) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (A->rows >= (int64_t(1) << 31) || W->rows >= (int64_t(1) << 31))
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (ldc < W->rows) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(C, 16) || ldc % 8 != 0) return NVFP4_ERR_MISALIGNED;
  if (c_amax_cols < 0 || (c_amax_cols > 0 && (c_amax_cols % 256 != 0 || W->rows % c_amax_cols != 0)))
    return NVFP4_ERR_INVALID_ARG;
  if (c_amax && !aligned(c_amax, 4)) return NVFP4_ERR_MISALIGNED;
  if (!ws || ws_bytes < kWsBytes) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return NVFP4_ERR_MISALIGNED;
  const DeviceInfo dev = current_device();
  if (!dev.ok) return NVFP4_ERR_ARCH;
  LaunchGemm g;
  g.a_codes = A->codes;
  g.a_sf = A->sf;
  g.a_st = A->s_t;
  g.w_codes = W->codes;
  g.w_sf = W->sf;
  g.w_st = W->s_t;
  g.M = A->rows;
  g.N = W->rows;
  g.K = A->cols;
  g.c = C;
  g.c_dtype = c_dtype;
  g.ldc = ldc;
  g.act = act;
  g.c_amax = c_amax;
  g.c_amax_cols = c_amax_cols;
  g.ws = ws;
  g.wait_limit_ns = g_wait_limit_ns.load();
  g.sm_count = dev.sm_count;
  return cuda_status(launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_kv_quant_chunk(const nvfp4_kv_cache* cache, const void* k, const void* v,
                                  int64_t token_stride, const int32_t* dst_slots, int32_t n_frames,
                                  float* k_amax_in, float* v_amax_in, void* ws, size_t ws_bytes,
                                  void* stream) {
  nvfp4_status st = check_cache(cache);
  if (st != NVFP4_OK) return st;
  if (!k || !v || !dst_slots) return NVFP4_ERR_INVALID_ARG;
  if ((k_amax_in == nullptr) != (v_amax_in == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (n_frames < 1 || n_frames > NVFP4_KV_MAX_CHUNK_FRAMES) return NVFP4_ERR_INVALID_ARG;
  const int64_t row_elems = int64_t(cache->heads) * cache->head_dim;
  if (token_stride < row_elems) return NVFP4_ERR_INVALID_ARG;
  for (int f = 0; f < n_frames; ++f) {
    if (dst_slots[f] < 0 || dst_slots[f] >= cache->n_slots) return NVFP4_ERR_INVALID_ARG;
    for (int g = 0; g < f; ++g)
      if (dst_slots[g] == dst_slots[f]) return NVFP4_ERR_INVALID_ARG;
  }
  if (!aligned(k, 16) || !aligned(v, 16) || token_stride % 8 != 0) return NVFP4_ERR_MISALIGNED;
  if ((k_amax_in && !aligned(k_amax_in, 4)) || (v_amax_in && !aligned(v_amax_in, 4)))
    return NVFP4_ERR_MISALIGNED;
  if (!ws || ws_bytes < kWsBytes) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return NVFP4_ERR_MISALIGNED;
  const DeviceInfo dev = current_device();
  if (!dev.ok) return NVFP4_ERR_ARCH;
  LaunchKvQuant q;
  q.k = k;
  q.v = v;
  q.token_stride = token_stride;
  q.n_frames = n_frames;
  q.tpf = cache->tokens_per_frame;
  q.heads = cache->heads;
  q.head_dim = cache->head_dim;
  q.slots = dst_slots;
  q.k_codes = cache->k_codes;
  q.v_codes = cache->v_codes;
  q.k_sf = cache->k_sf;
  q.v_sf = cache->v_sf;
  q.k_st = cache->k_st;
  q.v_st = cache->v_st;
  q.k_amax_in = k_amax_in;
  q.v_amax_in = v_amax_in;
  q.scale_rule = cache->scale_rule;
  q.ws = ws;
  q.sm_count = dev.sm_count;
  q.wait_limit_ns = g_wait_limit_ns.load();
  return cuda_status(launch_kv_quant(q, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_kv_dequant_window(const nvfp4_kv_cache* cache, const int32_t* slot_ids,
                                     int32_t n, void* k_out, void* v_out, void* stream) {
  nvfp4_status st = check_cache(cache);
  if (st != NVFP4_OK) return st;
  if (!slot_ids || !k_out || !v_out || n < 1 || n > NVFP4_KV_MAX_WINDOW_SLOTS)
    return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (slot_ids[i] < 0 || slot_ids[i] >= cache->n_slots) return NVFP4_ERR_INVALID_ARG;
  const int64_t per_frame = int64_t(cache->tokens_per_frame) * cache->heads * cache->head_dim;
  if (per_frame * n / 8 >= (int64_t(1) << 32)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(k_out, 16) || !aligned(v_out, 16)) return NVFP4_ERR_MISALIGNED;
  const DeviceInfo dev = current_device();
  if (!dev.ok) return NVFP4_ERR_ARCH;
  LaunchKvDequant d;
  d.k_codes = cache->k_codes;
  d.v_codes = cache->v_codes;
  d.k_sf = cache->k_sf;
  d.v_sf = cache->v_sf;
  d.k_st = cache->k_st;
  d.v_st = cache->v_st;
  d.slots = slot_ids;
  d.n = n;
  d.tpf = cache->tokens_per_frame;
  d.heads = cache->heads;
  d.head_dim = cache->head_dim;
  d.k_out = k_out;
  d.v_out = v_out;
  d.sm_count = dev.sm_count;
  return cuda_status(launch_kv_dequant(d, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_window_attention(const nvfp4_kv_cache* cache, const int32_t* slot_ids,
                                    int32_t n, const void* q, int64_t q_token_stride, int64_t tq,
                                    float softmax_scale, void* out, int64_t out_token_stride,
                                    void* ws, size_t ws_bytes, void* stream) {
  nvfp4_status st = check_cache(cache);
  if (st != NVFP4_OK) return st;
  if (!slot_ids || !q || !out || n < 1 || n > NVFP4_KV_MAX_WINDOW_SLOTS)
    return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (slot_ids[i] < 0 || slot_ids[i] >= cache->n_slots) return NVFP4_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return NVFP4_ERR_INVALID_ARG;
  const int64_t row = int64_t(cache->heads) * cache->head_dim;
  if (q_token_stride < row || out_token_stride < row) return NVFP4_ERR_INVALID_ARG;
  if (cache->head_dim != 128 || tq < 1 || tq > (int64_t(1) << 30) || cache->heads > 65535 ||
      int64_t(n) * cache->tokens_per_frame >= (int64_t(1) << 31))
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(q, 16) || !aligned(out, 16) || q_token_stride % 8 != 0 ||
      out_token_stride % 8 != 0)
    return NVFP4_ERR_MISALIGNED;
  if (!ws || ws_bytes < kWsBytes) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return NVFP4_ERR_MISALIGNED;
  const DeviceInfo dev = current_device();
  if (!dev.ok) return NVFP4_ERR_ARCH;
  LaunchAttn d;
  d.k_codes = cache->k_codes;
  d.v_codes = cache->v_codes;
  d.k_sf = cache->k_sf;
  d.v_sf = cache->v_sf;
  d.k_st = cache->k_st;
  d.v_st = cache->v_st;
  d.slot_ids = slot_ids;
  d.n = n;
  d.tpf = cache->tokens_per_frame;
  d.heads = cache->heads;
  d.q = q;
  d.out = out;
  d.q_stride = q_token_stride;
  d.out_stride = out_token_stride;
  d.tq = tq;
  d.scale_log2 = float(double(softmax_scale) * 1.4426950408889634);
  d.ws = ws;
  d.wait_limit_ns = g_wait_limit_ns.load();
  return cuda_status(launch_window_attention(d, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_get_device_status(void* ws, void* stream) {
  if (!ws) return NVFP4_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  uint32_t* dev_word = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + kWsStatus);
  if (cudaMemcpyAsync(&word, dev_word, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (cudaMemsetAsync(dev_word, 0, sizeof(word), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
  return static_cast<nvfp4_status>(word);
}

}  // extern "C"
