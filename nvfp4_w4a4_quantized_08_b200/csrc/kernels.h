// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernel files.  Arguments arrive here already validated.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4.h"

namespace nvfp4 {

// cuTensorMapEncodeTiled from the driver, looked up once per process (null
// when the driver does not provide it).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

struct LaunchQuant {
  const void* x;
  int32_t dtype;
  int64_t rows, cols, ld;
  uint8_t* codes;
  uint8_t* sf;
  int32_t sf_layout;
  float* s_t_out;
  const float* s_t_in;
  float* amax_in;  // producer-accumulated amax (consumed and reset), or NULL
  void* ws;
  int sm_count;
  uint64_t wait_limit_ns;
};
cudaError_t launch_quantize(const LaunchQuant& q, cudaStream_t st);

struct LaunchDequant {
  const uint8_t* codes;
  const uint8_t* sf;
  const float* s_t;
  int32_t sf_layout;
  int64_t rows, cols, ld;
  void* out;
  int sm_count;
};
cudaError_t launch_dequantize(const LaunchDequant& d, cudaStream_t st);

struct LaunchKvQuant {
  const void* k;
  const void* v;
  int64_t token_stride;
  int32_t n_frames, tpf, heads, head_dim;
  const int32_t* slots;  // host, n_frames
  uint8_t *k_codes, *v_codes, *k_sf, *v_sf;
  float *k_st, *v_st;
  float *k_amax_in, *v_amax_in;  // producer-accumulated amax per plane, or both NULL
  int32_t scale_rule;            // nvfp4_scale_rule
  void* ws;
  int sm_count;
  uint64_t wait_limit_ns;
};
cudaError_t launch_kv_quant(const LaunchKvQuant& q, cudaStream_t st);

struct LaunchKvDequant {
  const uint8_t *k_codes, *v_codes, *k_sf, *v_sf;
  const float *k_st, *v_st;
  const int32_t* slots;  // host, n
  int32_t n, tpf, heads, head_dim;
  void* k_out;
  void* v_out;
  int sm_count;
};
cudaError_t launch_kv_dequant(const LaunchKvDequant& d, cudaStream_t st);

struct LaunchAttn {
  const uint8_t *k_codes, *v_codes, *k_sf, *v_sf;
  const float *k_st, *v_st;
  const int32_t* slot_ids;  // host, n
  int32_t n, tpf, heads;
  const void* q;            // bf16
  void* out;                // bf16
  int64_t q_stride, out_stride, tq;
  float scale_log2;         // softmax scale * log2(e)
  void* ws;                 // workspace (status word)
  uint64_t wait_limit_ns;
};
cudaError_t launch_window_attention(const LaunchAttn& d, cudaStream_t st);

struct LaunchGemm {
  const uint8_t* a_codes;
  const uint8_t* a_sf;
  const float* a_st;
  const uint8_t* w_codes;
  const uint8_t* w_sf;
  const float* w_st;
  int64_t M, N, K;
  void* c;
  int32_t c_dtype;
  int64_t ldc;
  int32_t act;    // nvfp4_act applied in the epilogue
  float* c_amax;  // max|C| accumulator(s), or NULL
  int64_t c_amax_cols;  // columns per accumulator word (0: one word)
  void* ws;
  uint64_t wait_limit_ns;
  int sm_count;
};
cudaError_t launch_gemm(const LaunchGemm& g, cudaStream_t st);

}  // namespace nvfp4
