"""GPU: a multi-shot generation driven through the library's slot planner,
the KV chunk quantizer, the window rebuild and the window attention, against
the oracle.

The two-level attention sinks: the first G frames of the video stay for good,
the first H frames of the current shot are re-bound at each cut, and every
chunk also attends the last W frames, its own included (neurohive.io
LongLive-2.0 article, inference section; tailorednewshub.com article,
"Sumidero de Atención Multi-Toma"; G = 3 and W = 9 from 171host.com section
2.2).  The GPU side only ever sees slots: nvfp4_sink_plan hands out each
chunk's destination slots and the slot list it attends.  The oracle side never
sees slots: it keeps every frame's NVFP4 codes by frame number and takes the
attended frames from its own sink_window_frames.  Per chunk the rebuilt window
must equal the oracle's byte for byte and the attention output must meet the
per-element bound of tests/test_gpu_attention.py."""
import numpy as np
import pytest

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import workloads as wl

from _util import bits

pytestmark = pytest.mark.gpu

HD = 128


def _assert_close(o_gpu, o_ref, E):
    o_gpu = o_gpu.astype(np.float64)
    tol = 2.0 ** -6 * E + 2.0 ** -8 * np.abs(o_ref)
    err = np.abs(o_gpu - o_ref)
    bad = ~(err <= tol)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{bad.sum()} of {bad.size} outside tolerance; first {i}: "
                             f"gpu {o_gpu[i]} ref {o_ref[i]} E {E[i]}")


@pytest.mark.parametrize("chunks,tpf,heads", [
    # 3-frame chunks with cuts after frames 12 and 27 (G = 3, H = 3, W = 9)
    ([(3, False)] * 4 + [(3, True)] + [(3, False)] * 4 + [(3, True)] + [(3, False)] * 2,
     16, 2),
    # mixed chunk lengths, a cut on the second chunk, back-to-back cuts
    ([(2, False), (3, True), (1, False), (3, False), (3, True), (2, True), (3, False),
      (3, False), (3, False)], 24, 3),
])
def test_multi_shot_sequence(orc, chunks, tpf, heads):
    G, H, W = 3, 3, 9
    n_slots = G + H + W
    plan = nv.SinkPlan(n_slots, G, H, W)
    cache = nv.KVCache(n_slots, tpf, heads, HD)
    ref_frames = orc.sink_window_frames(chunks, G, H, W)
    per = tpf * heads * HD
    # the oracle's frame store: NVFP4 codes, scales and s_t of every frame
    store = {p: ([], [], []) for p in ("k", "v")}
    f0 = 0
    for ci, ((n, cut), frames) in enumerate(zip(chunks, ref_frames)):
        dst, win = plan.next(n, cut)
        k = wl.kv_tensor(100 + 2 * ci, n * tpf, heads, HD)
        v = wl.kv_tensor(101 + 2 * ci, n * tpf, heads, HD)
        cache.quant_chunk(k.cuda(), v.cuda(), dst)
        for p, x in (("k", k), ("v", v)):
            c, s, t = orc.kv_quant_chunk(bits(x).reshape(-1), n, tpf, heads, HD)
            for f in range(n):
                store[p][0].append(c[f])
                store[p][1].append(s[f])
                store[p][2].append(t[f])
        f0 += n
        assert len(win) == len(frames)
        k_gpu, v_gpu = cache.dequant_window(win)
        ref = {}
        for p, got in (("k", k_gpu), ("v", v_gpu)):
            codes = np.stack(store[p][0]).reshape(f0, per // 2)
            sf = np.stack(store[p][1]).reshape(f0, per // 16)
            st = np.asarray(store[p][2], np.float32)
            ref[p] = orc.kv_dequant_window(codes, sf, st, frames, tpf, heads, HD)
            np.testing.assert_array_equal(bits(got), ref[p], err_msg=f"chunk {ci} {p} window")
        q = wl.randn((n * tpf, heads * HD), 6, 200 + ci)
        out = cache.window_attention(q.cuda(), win)
        o_ref, E = orc.window_attention(bits(q), ref["k"], ref["v"], HD ** -0.5)
        _assert_close(out.float().cpu().numpy().reshape(n * tpf, heads, HD), o_ref, E)
    assert nv.device_status() == 0
    plan.close()
