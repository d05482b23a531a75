"""libnvfp4: the NVFP4 W4A4 path of a causal video DiT on B200 (sm_100a).

The compute lives in ``libnvfp4.so`` (hand-written CUDA kernels behind the C
ABI declared in ``include/nvfp4.h``); :mod:`.ops` marshals torch tensors'
device pointers and the current CUDA stream into those calls.  There is no CPU
fallback: every call raises if the shared library is missing, and the library
refuses any device that is not sm_100.
"""
from ._native import (ACT_GELU_TANH, ACT_NONE, BF16, FP32, KV_MAX_CHUNK_FRAMES,  # noqa: F401
                      KV_MAX_WINDOW_SLOTS, SCALE_FOUR_OVER_SIX, SCALE_ONTO_6, SF_MMA128x4,
                      SF_ROWMAJOR, NVFP4Error)
from .ops import (KVCache, NVFP4Tensor, SinkPlan, codes_bytes, dequantize,  # noqa: F401
                  device_status, empty, gemm, quantize, set_wait_limit_ns, sf_bytes, workspace)
