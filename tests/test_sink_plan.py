"""The library's multi-shot slot planner (nvfp4_sink_plan, host only, no GPU)
against the oracle's frame sets.

For random chunk / cut sequences the test keeps its own slot -> frame map from
the dst_slots the planner hands out (as nvfp4_kv_quant_chunk would fill the
slots), and checks for every chunk that the planner's window slot list names,
in order, exactly the frames the oracle says the chunk attends to, that each of
those frames is still in the slot it was written to (no slot still needed was
reused), and that the pool never holds more than G + H + W frames."""
import numpy as np
import pytest

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import _native as N


def _run(orc, chunks, n_slots, G, H, W):
    plan = nv.SinkPlan(n_slots, G, H, W)
    held = {}  # slot -> frame, as written through dst_slots
    f0 = 0
    ref = orc.sink_window_frames(chunks, G, H, W)
    for (n, cut), frames in zip(chunks, ref):
        dst, win = plan.next(n, cut)
        assert len(set(dst)) == n and all(0 <= s < n_slots for s in dst)
        # the chunk's slots did not hold a frame this chunk still attends
        assert not any(held.get(s) in frames for s in dst)
        for k, s in enumerate(dst):
            held[s] = f0 + k
        assert [held[s] for s in win] == frames
        assert len(win) <= G + H + W
        for s in range(n_slots):
            f = plan.frame_of_slot(s)
            assert f == -1 or f == held[s]
        f0 += n
    plan.close()


def test_bench_window(orc):
    """3-frame chunks, 3 global sinks, no shot sinks, 9-frame window in a
    15-slot pool: after the warm-up every chunk lists 3 sinks + 9 frames."""
    _run(orc, [(3, False)] * 20, 15, 3, 0, 9)
    plan = nv.SinkPlan(15, 3, 0, 9)
    for _ in range(10):
        dst, win = plan.next(3)
    assert len(win) == 12 and dst == win[-3:]


@pytest.mark.parametrize("seed", range(12))
def test_random_multi_shot_sequences(orc, seed):
    rng = np.random.default_rng(seed)
    G, H = int(rng.integers(0, 5)), int(rng.integers(0, 5))
    W = int(rng.integers(8, 16))
    n_slots = G + H + W + int(rng.integers(0, 4))
    chunks = [(int(rng.integers(1, 9)), bool(rng.random() < 0.2)) for _ in range(60)]
    _run(orc, chunks, n_slots, G, H, W)


def test_rejects():
    with pytest.raises(N.NVFP4Error):
        nv.SinkPlan(14, 3, 3, 9)  # fewer slots than G + H + W
    with pytest.raises(N.NVFP4Error):
        nv.SinkPlan(300, 3, 3, 9)  # more than the window list can hold
    plan = nv.SinkPlan(15, 3, 3, 9)
    for bad in (0, 9):
        with pytest.raises(N.NVFP4Error):
            plan.next(bad)
    small = nv.SinkPlan(8, 1, 1, 4)
    with pytest.raises(N.NVFP4Error):
        small.next(5)  # a chunk longer than the window
    dst, win = small.next(4)  # the plan is unchanged by the rejected calls
    assert dst == [0, 1, 2, 3] and win == [0, 1, 2, 3]
    assert small.frame_of_slot(-1) == -1 and small.frame_of_slot(8) == -1
