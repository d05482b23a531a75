"""Pins of the oracle's multi-shot sink window (no GPU).

Per chunk, the frames attended: the first G frames of the video (global sink,
kept for good), the first H frames of the current shot (shot sink, re-bound at
each cut: neurohive.io LongLive-2.0 article, inference section;
tailorednewshub.com article, "Sumidero de Atención Multi-Toma"), and the last W
frames up to the chunk's own (171host.com teardown, section 2.2: 3 global sink
frames, a 9-frame local window).  The worked examples below are written out by
hand from those sentences (3-frame chunks, G = 3, W = 9, H = 3 where shots are
used), not computed from the oracle's formula.
"""
import numpy as np


def test_single_shot_three_sinks_nine_window(orc):
    w = orc.sink_window_frames([(3, False)] * 11, 3, 0, 9)
    assert w[0] == [0, 1, 2]
    assert w[1] == [0, 1, 2, 3, 4, 5]
    assert w[2] == list(range(9))
    assert w[3] == list(range(12))                  # frames 0..2 are sinks and in the window
    assert w[4] == [0, 1, 2] + list(range(6, 15))   # 3 sinks + 9 window = 12 frames
    assert w[10] == [0, 1, 2] + list(range(24, 33))


def test_shot_sinks_rebound_at_a_cut(orc):
    chunks = [(3, False)] * 10 + [(3, True), (3, False), (3, False), (3, False)]
    w = orc.sink_window_frames(chunks, 3, 3, 9)
    # before the cut the shot sinks are the video's first frames (first shot)
    assert w[9] == [0, 1, 2] + list(range(21, 30))
    # the cut chunk (frames 30..32) starts the second shot
    assert w[10] == [0, 1, 2] + list(range(24, 33))
    assert w[11] == [0, 1, 2] + list(range(27, 36))
    assert w[12] == [0, 1, 2, 30, 31, 32] + list(range(33, 39))
    assert w[13] == [0, 1, 2, 30, 31, 32] + list(range(33, 42))  # 3 + 3 + 9 frames
    # a later cut (2-frame chunks from frame 42) replaces the shot sinks, the global ones stay
    w2 = orc.sink_window_frames(chunks + [(2, True)] + [(2, False)] * 5, 3, 3, 9)
    assert w2[-1] == [0, 1, 2, 42, 43, 44] + list(range(45, 54))
    # every chunk a cut: the shot sinks are the chunk's own frames
    w3 = orc.sink_window_frames(chunks + [(2, True)] * 6, 3, 3, 9)
    assert w3[-1] == [0, 1, 2] + list(range(45, 54))


def test_invariants_on_random_sequences(orc):
    rng = np.random.default_rng(0)
    for trial in range(40):
        G, H, W = int(rng.integers(0, 5)), int(rng.integers(0, 5)), int(rng.integers(8, 14))
        chunks = [(int(rng.integers(1, 9)), bool(rng.random() < 0.15)) for _ in range(30)]
        wins = orc.sink_window_frames(chunks, G, H, W)
        f0 = 0
        dropped = set()
        for (n, _), frames in zip(chunks, wins):
            f1 = f0 + n
            assert frames == sorted(set(frames))
            assert set(range(f0, f1)) <= set(frames)        # the chunk sees itself
            assert set(range(min(G, f1))) <= set(frames)    # global sinks stay
            assert len(frames) <= G + H + W
            assert not (set(frames) & dropped)              # a dropped frame never returns
            dropped |= set(range(f0)) - set(frames)
            f0 = f1
