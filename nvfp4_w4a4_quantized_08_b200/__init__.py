"""libnvfp4: the NVFP4 W4A4 path of a causal video DiT on B200 (sm_100a).

The compute lives in ``libnvfp4.so`` (hand-written CUDA kernels behind a C ABI
declared in ``include/nvfp4.h``); the functions here marshal torch tensors'
device pointers and the current CUDA stream into those calls.  There is no CPU
fallback: every call raises if the shared library is missing or the device is
not an sm_100 GPU.
"""
