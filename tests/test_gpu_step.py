"""GPU parity of the composed 30-layer denoise step (the launch sequence the
benchmark times), against the oracle.

The step composes what the per-call tests check one call at a time: kernels
launched back to back with programmatic dependent launch inside one CUDA graph,
tensor amax words handed from a GEMM epilogue to the next quantization (within
a layer and from one layer to the next), the GELU epilogue, K and V read out of
the QKV output, and the KV window rebuilt from slots written in the same step.
W4A4 linear layers and the NVFP4 KV cache: tailorednewshub.com LongLive-2.0
article, "Inferencia W4A4 NVFP4"; KV cache in frame blocks rebuilt for windowed
attention: hyper.ai summary, "方法"; 3 sinks + 9 window frames: 171host.com
section 2.2.

1. The step is captured as the benchmark captures it (eager warm-up, one CUDA
   graph of all 30 layers) and replayed; its output and the last layer's
   buffers are kept.
2. A second graph of the same step copies out every intermediate of layers 0
   and 29 right after the launch that writes it.  Its output and last-layer
   buffers must equal those of the first graph bit for bit (the copies change
   nothing), so what is checked below is what the benchmark computes.
3. Per tapped layer, each stage is checked against the oracle with the GPU's
   own input to that stage (GEMM outputs are within a tolerance, not exact, so
   each stage starts from what the GPU actually produced):
   - quantized activations (codes, tensor-core-layout scales, s_t): byte-exact
     against the oracle's quantization of the stage's bf16 input, whether the
     amax came from an amax pass or from the producing GEMM's epilogue;
   - the NVFP4 weights: byte-exact against the oracle's quantization;
   - GEMM outputs (QKV, out-projection, FFN-up with GELU, FFN-down): 64 seeded
     random rows, row 0 and the whole ragged last tile (rows 2560-2639), every
     column, within |y - y_ref| <= 1e-3 sum|a w| (+ half a bf16 ulp; the GELU
     bound for the up-projection);
   - the KV pools (the 12 prefilled frames and the step's 3 new frames read out
     of the QKV output) and the rebuilt 12-frame window: byte-exact.
"""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import workloads as wl
from nvfp4_w4a4_quantized_08_b200.dit_step import D, M, QKV, TPF, WINDOW, DiTStep

from _util import assert_gelu_gemm_close, assert_gemm_close, assert_quant_equal, bits, np_u8

pytestmark = pytest.mark.gpu

LAYERS = wl.LAYERS
TAPPED = (0, LAYERS - 1)
H, HD = wl.HEADS, wl.HEAD_DIM


def _rows(seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=64, replace=False).tolist())
    rows.update(range((M // 128) * 128, M))
    rows.add(0)
    return sorted(rows)


def _graph(step, stream, taps=None):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step.run(taps=taps)
    return g


def _snapshot(step):
    """The buffers the last layer leaves behind, and the step's output."""
    return {"out": step.output().clone(), "qkv": step.qkv_out.clone(),
            "k_win": step.k_win.clone(), "v_win": step.v_win.clone(),
            "o": step.o_out.clone(), "up": step.up_out.clone(),
            "qf_codes": step.qf.codes.clone(), "qf_sf": step.qf.sf.clone(),
            "qa_codes": step.qa.codes.clone()}


@pytest.fixture(scope="module")
def run():
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    step = DiTStep(LAYERS, dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        step.run()
    stream.synchronize()
    plain = _graph(step, stream)
    for _ in range(2):
        plain.replay()
    torch.cuda.synchronize()
    snap = _snapshot(step)
    assert nv.device_status(step.ws) == 0
    taps = step.make_taps(TAPPED)
    tapped = _graph(step, stream, taps)
    tapped.replay()
    torch.cuda.synchronize()
    assert nv.device_status(step.ws) == 0
    yield step, snap, taps
    del plain, tapped
    torch.cuda.synchronize()


def test_taps_change_nothing(run):
    """The tapped graph computes bit for bit what the benchmark's graph does,
    and its layer-29 copies are that graph's last-layer buffers."""
    step, snap, taps = run
    after = _snapshot(step)
    for k in snap:
        assert torch.equal(snap[k], after[k]), k
    t = taps[LAYERS - 1]
    assert torch.equal(t["down"], snap["out"])
    assert torch.equal(t["qkv"], snap["qkv"])
    assert torch.equal(t["up"], snap["up"])
    assert torch.equal(t["o"], snap["o"])
    assert torch.equal(t["k_win"], snap["k_win"])
    assert torch.equal(t["qf"].codes, snap["qf_codes"])
    assert torch.equal(t["qa_o"].codes, snap["qa_codes"])


def _weights(orc, step, l):
    """The oracle's quantization of layer l's seeded weights, checked equal to
    the step's pre-quantized NVFP4 weights."""
    out = []
    for w_bf16, qw in zip(wl.layer_weights_cuda(l, device=step.dev), step.w[l]):
        out.append(assert_quant_equal(orc, qw, bits(w_bf16), nv.SF_MMA128x4))
    return out


def _pools(orc, step, l, qkv_bits):
    """The oracle's KV pools for layer l: the 12 prefilled frames (chunks of 8
    and 4 frames of the seeded prefill, the same tensor as K and V) and the
    step's 3 new frames (K and V thirds of the GPU's QKV output, token stride
    9216), checked equal to the GPU pools byte for byte."""
    per = TPF * H * HD
    n_slots = step.cache[l].n_slots
    pools = {p: [np.zeros((n_slots, per // 2), np.uint8), np.zeros((n_slots, per // 16), np.uint8),
                 np.zeros(n_slots, np.float32)] for p in ("k", "v")}
    pre = bits(wl.kv_tensor_cuda(seed=l, tokens=WINDOW * TPF, device=step.dev)).reshape(-1)
    for f0, nf in ((0, 8), (8, 4)):
        c, s, t = orc.kv_quant_chunk(pre[f0 * per:(f0 + nf) * per], nf, TPF, H, HD)
        for p in ("k", "v"):
            for f in range(nf):
                pools[p][0][f0 + f], pools[p][1][f0 + f], pools[p][2][f0 + f] = c[f], s[f], t[f]
    flat = qkv_bits.reshape(-1)
    for p, col in (("k", D), ("v", 2 * D)):
        c, s, t = orc.kv_quant_chunk(flat[col:], len(step.new_slots), TPF, H, HD,
                                     token_stride=QKV)
        for f, slot in enumerate(step.new_slots):
            pools[p][0][slot], pools[p][1][slot], pools[p][2][slot] = c[f], s[f], t[f]
    cache = step.cache[l]
    for p, (cp, sp, tp) in (("k", (cache.k_codes, cache.k_sf, cache.k_st)),
                            ("v", (cache.v_codes, cache.v_sf, cache.v_st))):
        np.testing.assert_array_equal(np_u8(cp), pools[p][0], err_msg=f"layer {l} {p} codes")
        np.testing.assert_array_equal(np_u8(sp), pools[p][1], err_msg=f"layer {l} {p} scales")
        np.testing.assert_array_equal(tp.cpu().numpy(), pools[p][2], err_msg=f"layer {l} {p} s_t")
    return pools


@pytest.mark.parametrize("layer", TAPPED)
def test_layer_against_oracle(orc, run, layer):
    step, snap, taps = run
    t = taps[layer]
    rows = _rows(layer)
    ow_q, ow_o, ow_u, ow_d = _weights(orc, step, layer)

    x = t["x"]
    if layer == 0:
        assert torch.equal(x, step.x_in)
    # input quantization: amax pass (layer 0) or the previous layer's
    # down-projection epilogue amax (every later layer)
    oa = assert_quant_equal(orc, t["qa_x"], bits(x), nv.SF_MMA128x4)
    y_ref, S = orc.gemm(oa, ow_q, rows=rows)
    assert_gemm_close(t["qkv"][rows].float().cpu().numpy(), y_ref, S, True)

    # K and V of the 3 new frames out of the QKV output (amax from the QKV
    # epilogue's per-third words), the prefilled frames, and the window rebuild
    qkv_bits = bits(t["qkv"])
    pools = _pools(orc, step, layer, qkv_bits)
    for p in ("k", "v"):
        ref = orc.kv_dequant_window(*pools[p], step.window, TPF, H, HD)
        np.testing.assert_array_equal(bits(t[f"{p}_win"]), ref, err_msg=f"{p} window")

    oa = assert_quant_equal(orc, t["qa_attn"], bits(step.attn), nv.SF_MMA128x4)
    y_ref, S = orc.gemm(oa, ow_o, rows=rows)
    assert_gemm_close(t["o"][rows].float().cpu().numpy(), y_ref, S, True)

    # the out-projection's output quantized with the amax its epilogue found
    oa = assert_quant_equal(orc, t["qa_o"], bits(t["o"]), nv.SF_MMA128x4)
    y_ref, S = orc.gemm(oa, ow_u, rows=rows)
    assert_gelu_gemm_close(orc, t["up"][rows].float().cpu().numpy(), y_ref, S, True)

    # the FFN intermediate requantized with the GELU epilogue's amax
    oq = assert_quant_equal(orc, t["qf"], bits(t["up"]), nv.SF_MMA128x4)
    y_ref, S = orc.gemm(oq, ow_d, rows=rows)
    assert_gemm_close(t["down"][rows].float().cpu().numpy(), y_ref, S, True)
    if layer == LAYERS - 1:
        assert torch.equal(t["down"], snap["out"])
