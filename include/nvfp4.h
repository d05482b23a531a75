/*
 * nvfp4.h -- C ABI of libnvfp4, the NVFP4 W4A4 path of a causal video DiT on
 * NVIDIA B200 (sm_100a).
 *
 * The operations are the inference path the LongLive-2.0 pages describe:
 *   - NVFP4 tensors: E2M1 4-bit elements, one FP8 (E4M3) scale per block of 16
 *     elements and one FP32 scale per tensor (neurohive.io LongLive-2.0 article,
 *     section "Ключевые компоненты LongLive-2.0", NVFP4 paragraph;
 *     tailorednewshub.com LongLive-2.0 article, section "Entrenamiento NVFP4").
 *   - W4A4 linear layers: weights and activations both NVFP4, BF16 GEMMs
 *     replaced by FP4 GEMMs on Blackwell tensor cores (tailorednewshub.com,
 *     section "Inferencia W4A4 NVFP4").
 *   - An NVFP4 KV cache quantized in blocks of up to eight latent frames and
 *     rebuilt to bf16 for windowed attention (hyper.ai LongLive-2.0 summary,
 *     section "方法" (Method), second paragraph), over a window of 9 local plus
 *     3 sink frames (171host.com LongLive 2.0 teardown, section 2.2).
 *   - Around them: the FFN's GELU in the GEMM epilogue, windowed attention that
 *     reads the NVFP4 cache directly, and host-side slot planning under the
 *     two-level (global and per-shot) attention sinks of multi-shot generation
 *     (neurohive.io article, inference section; tailorednewshub.com article,
 *     section "Sumidero de Atención Multi-Toma").
 *
 * Quantization recipe (the pages name the format only; this library fixes):
 *   s_t = amax(|x|) / 2688                          (2688 = 6 * 448)
 *   s_b = E4M3_RNE_sat( amax_block(|x|) / (6 * s_t) )   per 16 elements
 *   q   = E2M1_RNE_sat( x / (s_b * s_t) )           code 0 when s_b == 0
 * each step one IEEE binary32 operation rounded to nearest even, in that order.
 * Dequantization: bf16_RNE( (v(q) * s_b) * s_t ).
 *
 * Conventions for every entry point
 *   - Pointers marked "device" are CUDA device pointers on the current device;
 *     "host" pointers are ordinary host memory read before the call returns.
 *   - The caller owns and allocates every buffer; the library allocates no
 *     device memory.  It caches per-device kernel attributes only.
 *   - Every call that takes a `stream` is asynchronous on it (a cudaStream_t;
 *     NULL = the legacy default stream).  Argument checks happen on the host,
 *     before any launch, and a rejected call launches nothing.  The sink-plan
 *     calls are host-only and synchronous.
 *   - A launch failure returns NVFP4_ERR_CUDA.  Errors found on the device (a
 *     bounded wait that ran out, a tensor scale outside the recipe's domain) are
 *     recorded in the workspace status word and returned by
 *     nvfp4_get_device_status().
 *   - Inputs must be finite.  The tensor scale must be 0 or lie in
 *     [2^-108, 2^100] (amax 0 or in about [2^-96.6, 2^111.4]); outside that
 *     the outputs are unspecified and the status word reads NVFP4_ERR_DOMAIN.
 *   - The device must be compute capability 10.0 (B200); anything else returns
 *     NVFP4_ERR_ARCH.  There is no fallback path.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, bad enum */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside what the kernels take */
  NVFP4_ERR_MISALIGNED = 3,        /* a pointer or stride breaks alignment */
  NVFP4_ERR_WORKSPACE = 4,         /* workspace missing or too small */
  NVFP4_ERR_ARCH = 5,              /* current device is not sm_100 */
  NVFP4_ERR_CUDA = 6,              /* a CUDA runtime call or launch failed */
  NVFP4_ERR_TIMEOUT = 7,           /* device: a bounded wait ran out */
  NVFP4_ERR_DOMAIN = 8             /* device: tensor scale outside the domain */
} nvfp4_status;

/* Element type of a dense input or output tensor. */
typedef enum { NVFP4_BF16 = 0, NVFP4_FP32 = 1 } nvfp4_dtype;

/* Layout of the E4M3 block scales of an NVFP4 tensor.
 *   ROWMAJOR: byte [row * (cols/16) + block].
 *   MMA128x4: the tensor-core layout: 512-byte tiles of 128 rows x 4 blocks,
 *     tiles ordered row-tile major then block-tile; inside a tile row r, block
 *     c at (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4.  Rows are padded to a
 *     multiple of 128 and blocks to a multiple of 4; padding bytes are zero.
 *     nvfp4_gemm operands must use this layout. */
typedef enum { NVFP4_SF_ROWMAJOR = 0, NVFP4_SF_MMA128x4 = 1 } nvfp4_sf_layout;

/* How a KV chunk's block scales are chosen.
 *   ONTO_6: s_b = E4M3_RNE_sat(amax_b / (6 s_t)), the recipe of nvfp4_quantize.
 *   FOUR_OVER_SIX: the adaptive choice the pages name for the KV cache
 *     (tailorednewshub.com LongLive-2.0 article, section "Inferencia W4A4
 *     NVFP4"), read as: per block, the scale with the block maximum onto 6 or
 *     onto 4 (E4M3_RNE_sat(amax_b / (4 s_t))), whichever codes the block with
 *     the smaller squared error against the exactly decoded values (binary64,
 *     element order; 6 on a tie).  The stored format is unchanged. */
typedef enum { NVFP4_SCALE_ONTO_6 = 0, NVFP4_SCALE_FOUR_OVER_SIX = 1 } nvfp4_scale_rule;

/* Elementwise function the GEMM epilogue applies to y = (s_tA * s_tW) * acc
 * before rounding to the output type.
 *   NONE: C = y.
 *   GELU_TANH: C = 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))), the GELU of
 *     the DiT's FFN between its up- and down-projection (the transformer blocks
 *     are attention and FFN: 171host.com LongLive-2.0 teardown, usage section
 *     "训练管线", LoRA on Attn/FFN); the pages name no activation form, the
 *     tanh form is the one video DiTs use.  Evaluated in binary32 with the
 *     hardware tanh (tanh.approx.f32, relative error about 2^-11) on y as a
 *     bf16 linear layer hands it to its activation: for bf16 output on y
 *     rounded to bf16, for fp32 output on the fp32 y.  So C is within
 *     2^-11 |y| + 1.13 |y_in - y_exact| of the exact GELU of the exact y, with
 *     y_in the activation's input, plus the output rounding. */
typedef enum { NVFP4_ACT_NONE = 0, NVFP4_ACT_GELU_TANH = 1 } nvfp4_act;

/* An NVFP4 tensor of rows x cols elements (cols a multiple of 16).
 *   codes: device, [rows][cols/2] bytes; element 2j in the low nibble of
 *          byte j, element 2j+1 in the high nibble; sign in bit 3 of a nibble.
 *   sf:    device, nvfp4_sf_bytes(rows, cols, sf_layout) bytes of E4M3 scales.
 *   s_t:   device, one float (the per-tensor scale).
 * codes and sf must be 16-byte aligned, s_t 4-byte aligned. */
typedef struct {
  uint8_t* codes;
  uint8_t* sf;
  float* s_t;
  int64_t rows;
  int64_t cols;
  int32_t sf_layout; /* nvfp4_sf_layout */
} nvfp4_tensor;

/* The NVFP4 KV cache of one layer: a pool of n_slots frame slots for K and for
 * V.  One slot holds one latent frame: tokens_per_frame tokens x heads x
 * head_dim elements, blocks of 16 along head_dim.
 *   k_codes, v_codes: device, [n_slots][tokens_per_frame*heads*head_dim/2]
 *   k_sf, v_sf:       device, [n_slots][tokens_per_frame*heads*head_dim/16],
 *                     row-major ([token][head][head_dim/16]) E4M3 scales
 *   k_st, v_st:       device, [n_slots] floats: the tensor scale of the chunk
 *                     that last wrote the slot
 *   scale_rule:       nvfp4_scale_rule used by nvfp4_kv_quant_chunk
 * Code and scale pools must be 16-byte aligned; head_dim a multiple of 16. */
typedef struct {
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint8_t* k_sf;
  uint8_t* v_sf;
  float* k_st;
  float* v_st;
  int32_t n_slots;
  int32_t tokens_per_frame;
  int32_t heads;
  int32_t head_dim;
  int32_t scale_rule; /* nvfp4_scale_rule */
} nvfp4_kv_cache;

/* Most frames one kv_quant_chunk call writes (the pages' 8-frame block) and
 * most slots one kv_dequant_window call reads. */
#define NVFP4_KV_MAX_CHUNK_FRAMES 8
#define NVFP4_KV_MAX_WINDOW_SLOTS 256

/* Sizes in bytes of the code and scale buffers of a rows x cols tensor
 * (0 for invalid arguments). */
NVFP4_API size_t nvfp4_codes_bytes(int64_t rows, int64_t cols);
NVFP4_API size_t nvfp4_sf_bytes(int64_t rows, int64_t cols, int32_t sf_layout);

/* Size of the device workspace the quantizers and the GEMM take: scratch
 * words for the running amax and CTA counters plus the device status word.
 * The caller zero-fills it once after allocating it; every call leaves the
 * scratch words zero again, so it can be reused without clearing.  Calls that
 * share one workspace must be ordered on the device (one stream, or events):
 * overlapping calls race on the scratch words. */
NVFP4_API size_t nvfp4_workspace_bytes(void);

/* Quantize a dense rows x cols tensor to NVFP4 (the recipe above).
 *   x:      device, bf16 or fp32 (dtype), row stride ld elements (ld >= cols),
 *           16-byte aligned, ld * element size a multiple of 16 bytes.
 *   out:    host struct describing device buffers; out->rows/cols must equal
 *           rows/cols; out->sf_layout picks the scale layout (padding bytes of
 *           the MMA layout are written as zero).
 *   s_t_in: NULL, or a device float holding s_t to use as is (one pass over x;
 *           blocks whose amax exceeds 6 * 448 * s_t saturate).
 *   amax_in: NULL, or a device float into which the producer of x has already
 *           max-accumulated max|x| (nvfp4_gemm's c_amax does this): s_t is
 *           amax_in / 2688 and the amax pass is skipped.  The call sets
 *           *amax_in back to 0 when it is done, ready for the next producer.
 *           With both NULL, s_t comes from an amax pass over x (two passes).
 *           Passing both is INVALID_ARG.
 *   ws:     device workspace of ws_bytes >= nvfp4_workspace_bytes().
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (cols % 16, more than 2^32 / 8
 * elements), MISALIGNED, WORKSPACE, ARCH, CUDA; DOMAIN via the status word. */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x, int32_t dtype, int64_t rows, int64_t cols,
                                      int64_t ld, const nvfp4_tensor* out, const float* s_t_in,
                                      float* amax_in, void* ws, size_t ws_bytes, void* stream);

/* Dequantize an NVFP4 tensor to bf16: out[r * ld + c] = bf16_RNE((v * s_b) * s_t).
 *   in:  host struct of device buffers, either scale layout.
 *   out: device bf16, row stride ld >= cols elements, 16-byte aligned,
 *        ld a multiple of 8.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, ARCH, CUDA. */
NVFP4_API nvfp4_status nvfp4_dequantize(const nvfp4_tensor* in, void* out, int64_t ld, void* stream);

/* Block-scaled FP4 x FP4 GEMM, C = A * W^T:
 *   C[m][n] = (s_tA * s_tW) * sum_k v(qA[m][k]) sA[m][k/16] * v(qW[n][k]) sW[n][k/16]
 * products and sums on the tensor cores with FP32 accumulation, the scale
 * product applied once in the epilogue, then the activation `act`
 * (nvfp4_act), then rounded to c_dtype.
 *   A: M x K activations, W: N x K weights (both K-contiguous), both with
 *      sf_layout == NVFP4_SF_MMA128x4 and the same K.
 *   Shapes: K a multiple of 32, M >= 1 and N >= 1 (any M and N; the tiles'
 *      tail rows and columns are masked, and a last partial 64-wide K step
 *      reads zero codes and the scale layout's zero padding).
 *   C: device, c_dtype (bf16 or fp32), row stride ldc >= N elements, ldc a
 *      multiple of 8, 16-byte aligned.
 *   act: nvfp4_act.
 *   c_amax: NULL, or device floats (4-byte aligned) into which the GEMM
 *      max-accumulates max|C| over the values as stored (after the activation
 *      and the rounding to c_dtype), so that nvfp4_quantize(..., amax_in = c_amax, ...) can
 *      requantize C without an amax pass.  With c_amax_cols == 0 there is one
 *      word for all of C; with c_amax_cols > 0 (a multiple of 256 dividing N)
 *      word g covers columns [g * c_amax_cols, (g + 1) * c_amax_cols), N /
 *      c_amax_cols words in all: one per part of a fused output (for example
 *      the Q, K and V thirds of a QKV projection, whose K and V words feed
 *      nvfp4_kv_quant_chunk).  Every word must hold 0 (or a smaller
 *      non-negative value) before the call: zero-fill them once; a consuming
 *      quantize resets the words it reads.
 *   ws: device workspace (status word for the bounded waits).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, ARCH, CUDA;
 * TIMEOUT via the status word. */
NVFP4_API nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* W, void* C,
                                  int32_t c_dtype, int64_t ldc, int32_t act, float* c_amax,
                                  int64_t c_amax_cols, void* ws, size_t ws_bytes, void* stream);

/* Quantize one chunk of n_frames (1..8) new latent frames of K and V into the
 * cache.  The chunk is one NVFP4 tensor per K and per V: one s_t over the whole
 * chunk, blocks of 16 along head_dim.  Frame f of the chunk goes to slot
 * dst_slots[f], whose s_t entry receives the chunk's s_t.
 *   k, v: device bf16, n_frames * tokens_per_frame tokens, token t at
 *         k + t * token_stride elements, heads x head_dim contiguous within a
 *         token (token_stride >= heads * head_dim, a multiple of 8); this reads
 *         K and V straight out of a fused QKV projection output.
 *   dst_slots: host, n_frames distinct slot ids in [0, n_slots).
 *   k_amax_in, v_amax_in: both NULL (the call runs an amax pass over K and V),
 *         or both device floats (4-byte aligned) holding max|K| and max|V| of
 *         the chunk as accumulated by the producer (nvfp4_gemm's per-column-
 *         group c_amax over the K and V parts of a QKV output); the amax pass
 *         is skipped and both words are reset to 0 when the call is done.
 *   ws: device workspace.
 * Errors: INVALID_ARG (slot ids out of range or repeated, one amax pointer
 * without the other), UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, ARCH, CUDA;
 * DOMAIN via the status word. */
NVFP4_API nvfp4_status nvfp4_kv_quant_chunk(const nvfp4_kv_cache* cache, const void* k, const void* v,
                                  int64_t token_stride, const int32_t* dst_slots, int32_t n_frames,
                                  float* k_amax_in, float* v_amax_in, void* ws, size_t ws_bytes,
                                  void* stream);

/* Rebuild contiguous bf16 K and V for attention from a list of slots, in list
 * order (for example 3 sink frames followed by the 9 window frames).
 *   slot_ids: host, n ids in [0, n_slots), 1 <= n <= NVFP4_KV_MAX_WINDOW_SLOTS;
 *             repeats allowed.
 *   k_out, v_out: device bf16 [n * tokens_per_frame][heads][head_dim],
 *                 16-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, ARCH, CUDA. */
NVFP4_API nvfp4_status nvfp4_kv_dequant_window(const nvfp4_kv_cache* cache, const int32_t* slot_ids,
                                     int32_t n, void* k_out, void* v_out, void* stream);

/* Windowed attention straight from the NVFP4 cache (the consumer of the window
 * rebuild above, without the bf16 round trip through HBM):
 *   out[t][h] = sum_j softmax_j(softmax_scale * q[t][h] . k[j][h]) v[j][h]
 * over the tokens j of the listed slots in list order, k and v the bf16 values
 * nvfp4_kv_dequant_window would write (bf16_RNE((v(q) * s_b) * s_t)); every
 * query sees every window token (the chunk attends to the cached frames and to
 * itself whole).  Scores and sums in fp32 (tensor cores, bf16 inputs), the
 * probabilities rounded to bf16 for the P V product, the output rounded to bf16.
 *   slot_ids: host, n ids in [0, n_slots), 1 <= n <= NVFP4_KV_MAX_WINDOW_SLOTS,
 *             n * tokens_per_frame < 2^31; repeats allowed.
 *   q:   device bf16, tq tokens (1 <= tq <= 2^30), token t at q + t *
 *        q_token_stride elements, heads x head_dim contiguous in a token
 *        (q_token_stride >= heads * head_dim, a multiple of 8), 16-byte aligned;
 *        this reads Q straight out of a fused QKV projection output.
 *   softmax_scale: finite, > 0 (usually 1 / sqrt(head_dim)).
 *   out: device bf16, tq tokens at out_token_stride, same layout as q.
 *   ws:  device workspace of ws_bytes >= nvfp4_workspace_bytes() (its status
 *        word records a bounded wait that ran out: NVFP4_ERR_TIMEOUT, read by
 *        nvfp4_get_device_status; the limit is nvfp4_set_wait_limit_ns's).
 *   head_dim must be 128.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, ARCH, CUDA;
 * TIMEOUT via the status word. */
NVFP4_API nvfp4_status nvfp4_window_attention(const nvfp4_kv_cache* cache, const int32_t* slot_ids,
                                              int32_t n, const void* q, int64_t q_token_stride,
                                              int64_t tq, float softmax_scale, void* out,
                                              int64_t out_token_stride, void* ws, size_t ws_bytes,
                                              void* stream);

/* Slot planning for multi-shot generation (host only: no device work, no
 * stream).  Each chunk of new frames attends to three sets of frames
 * (neurohive.io LongLive-2.0 article, inference section on attention sinks;
 * tailorednewshub.com LongLive-2.0 article, section "Sumidero de Atención
 * Multi-Toma"; 171host.com teardown, section 2.2):
 *   G: the first global_sinks frames of the video, kept for good;
 *   H: the first shot_sinks frames of the current shot, re-bound at each cut;
 *   L: the last `window` frames up to and including the chunk's own.
 * A plan tracks which frame each of the cache's n_slots slots holds.
 *   create:  n_slots >= global_sinks + shot_sinks + window (enough for any
 *            G u H u L), n_slots <= NVFP4_KV_MAX_WINDOW_SLOTS, window >= 1;
 *            NULL on invalid arguments or allocation failure.
 *   next:    plan the next chunk of n_frames frames (1..8, <= window);
 *            new_shot != 0 when the chunk starts a new shot (the first chunk
 *            always does).  Frees every slot whose frame is outside the
 *            chunk's G u H u L (never attended again), writes the lowest free
 *            slots for the chunk's frames to dst_slots[n_frames] (for
 *            nvfp4_kv_quant_chunk), and the slots of G u H u L in frame order
 *            to window_slots (capacity n_slots; count in *n_window) for
 *            nvfp4_kv_dequant_window / nvfp4_window_attention.
 *            Errors: INVALID_ARG (the plan is unchanged).
 *   frame_of_slot: the frame a slot holds, -1 if free or out of range.
 * The caller owns the plan (destroy frees it); a plan is not thread-safe. */
typedef struct nvfp4_sink_plan nvfp4_sink_plan;
NVFP4_API nvfp4_sink_plan* nvfp4_sink_plan_create(int32_t n_slots, int32_t global_sinks,
                                                  int32_t shot_sinks, int32_t window);
NVFP4_API void nvfp4_sink_plan_destroy(nvfp4_sink_plan* plan);
NVFP4_API nvfp4_status nvfp4_sink_plan_next(nvfp4_sink_plan* plan, int32_t n_frames,
                                            int32_t new_shot, int32_t* dst_slots,
                                            int32_t* window_slots, int32_t* n_window);
NVFP4_API int64_t nvfp4_sink_plan_frame_of_slot(const nvfp4_sink_plan* plan, int32_t slot);

/* Size of the library-owned scratch array behind nvfp4_quantize_noalloc. */
#define NVFP4_NOALLOC_SCRATCH_BYTES 256

/* nvfp4_quantize without a workspace argument, for callers that cannot
 * allocate device memory when they quantize: code that runs inside a memory
 * budget whose allocator belongs to someone else (a serving arena, an embedded
 * runtime), hooks that receive only their input and output buffers, or paths
 * where a cudaMalloc would synchronize the device at a bad moment.  (The
 * LongLive-2.0 pages have no counterpart; this is a deployment convenience.)
 *
 * Same arguments, recipe and results as nvfp4_quantize, minus ws / ws_bytes.
 * The scratch words (running amax, CTA counter) live in a fixed array of
 * NVFP4_NOALLOC_SCRATCH_BYTES bytes of the library's own device memory, which
 * every GPU that loads the library keeps until the process exits; the call
 * itself allocates nothing.  The scratch need is constant (20 bytes for any
 * tensor); a layout that would not fit the array is rejected with
 * NVFP4_ERR_WORKSPACE, and tensors of 2^32 / 8 or more elements with
 * NVFP4_ERR_UNSUPPORTED_SHAPE, as in nvfp4_quantize.
 *   - The first call on each device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after a
 *     cudaDeviceReset (or anything else that destroys the device's primary
 *     context) it is stale, so do not call this entry point on that device
 *     again in the same process.
 *   - Each call first clears the scratch words on `stream`.  All calls on a
 *     device share the one array, so calls that may overlap on the GPU (other
 *     streams, other threads) race and must be serialized by the caller.
 *   - A tensor scale outside the recipe's domain is not reported (there is no
 *     workspace status word to read); use nvfp4_quantize where that matters. */
NVFP4_API nvfp4_status nvfp4_quantize_noalloc(const void* x, int32_t dtype, int64_t rows,
                                              int64_t cols, int64_t ld, const nvfp4_tensor* out,
                                              const float* s_t_in, void* stream);

/* Synchronize `stream`, then read and clear the workspace status word: the
 * first device-side error recorded since the last call (NVFP4_OK if none). */
NVFP4_API nvfp4_status nvfp4_get_device_status(void* ws, void* stream);

/* Upper bound, in nanoseconds, on every spin-wait inside the kernels (default
 * 2 s).  A wait that runs out records NVFP4_ERR_TIMEOUT, drains the kernel's own
 * copies and tensor-core work in flight, frees its tensor memory and returns.
 * Applies to launches made after the call (process-wide). */
NVFP4_API void nvfp4_set_wait_limit_ns(uint64_t ns);

/* Human-readable name of a status code. */
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
