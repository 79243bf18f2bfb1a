"""GPU: audio-in streaming (sf_stream_step_audio) against the oracle's
audio-in stream (oracle/streaming.py: window mel from the continuous signal,
normalised over the window, steps only on complete windows).  fp32 engine,
tiny model with xavier-scaled weights, free-running; the oracle's decision
margins are asserted to exceed the fp32 discrepancy; probabilities within
1e-4."""
import numpy as np
import pytest

import oracle as O
from oracle.streaming import stream_run_audio
from synth import synth_clip
from _helpers import make_engine, tiny_weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


@pytest.fixture(scope="module")
def w():
    return tiny_weights(xavier=True)


@pytest.fixture(scope="module")
def eng(w):
    e = make_engine(w, 0, 2, 2, max_batch=8)
    yield e
    b.sf_destroy(e)


def _schedule(n, first, step, ticks):
    """Samples received before each tick: nothing until `first`, then `step`
    more per tick, capped at n."""
    return [min(n, max(0, first + step * k)) for k in range(ticks)]


def _oracle(audio, n, w, pre, sched):
    taps = []
    probs, per_step = stream_run_audio(audio, n, w, pre, sched, taps=taps)
    margin = min([t["margin"] for t in taps] + [np.inf])
    return probs, per_step, margin


@pytest.mark.parametrize("preset", ["low", "ultra_low"])
def test_audio_in_streams_match_oracle(eng, w, preset):
    """Three streams in one batch with different lengths and arrival
    schedules (fine pieces, late start with coarse pieces, everything at
    once); one sf_stream_step_audio call per tick."""
    pre = O.PRESETS[preset]
    clips = [synth_clip([60, i], d, 4)[0] for i, d in enumerate([12.0, 9.3, 6.1])]
    ns = [len(c) for c in clips]
    n_buf = max(ns)
    audio = np.zeros((3, n_buf), np.float32)
    for i, c in enumerate(clips):
        audio[i, :len(c)] = c
    ticks = 400
    scheds = [_schedule(ns[0], 2000, 4000, ticks), _schedule(ns[1], 30000, 16000, ticks), [ns[2]] * ticks]
    d_audio = torch.from_numpy(audio).cuda()
    st = b.sf_stream_create(eng, (pre.chunk_len, pre.right_context, pre.fifo_len, pre.update_period,
                                  pre.spkcache_len), 3)
    cp = torch.zeros((3, pre.chunk_len, 4), device="cuda")
    outs = [[] for _ in range(3)]
    steps = [[] for _ in range(3)]
    T_enc = [1 + (n // 160 - 1) // 8 for n in ns]
    try:
        for k in range(ticks):
            if all(sum(len(o) for o in outs[i]) >= T_enc[i] for i in range(3)):
                break
            end = np.array([s[k] for s in scheds], np.int64)
            final = np.array([int(end[i] >= ns[i]) for i in range(3)], np.int32)
            n_out = b.sf_stream_step_audio(eng, st, d_audio, np.zeros(3, np.int64), end, final, cp)
            c = cp.cpu().numpy()
            for i in range(3):
                if sum(len(o) for o in outs[i]) < T_enc[i]:
                    steps[i].append(int(n_out[i]))
                outs[i].append(c[i, :n_out[i]])
        b.sf_check(eng)
    finally:
        b.sf_stream_destroy(st)
    for i in range(3):
        ref, per_step, margin = _oracle(clips[i], ns[i], w, pre, scheds[i])
        assert margin > 2e-6, margin
        got = np.concatenate(outs[i])
        assert got.shape == ref.shape == (T_enc[i], 4), i
        assert np.max(np.abs(got - ref)) <= 1e-4, i
        assert steps[i][:len(per_step)] == per_step, i      # same ticks emit the same frame counts


def test_audio_in_sliding_buffer(eng, w):
    """The caller keeps only recent audio: each tick's buffer row starts at
    the latest sample the next window may need (160 m0 - 257, rounded down to
    a multiple of 1000) and is refilled from there."""
    pre = O.PRESETS["low"]
    clip = synth_clip([61, 0], 8.0, 3)[0]
    n = len(clip)
    n_buf = 160 * 8 * (pre.chunk_len + pre.right_context + 1) + 12000   # window + slack for arrivals ahead
    sched = _schedule(n, 1600, 3200, 400)
    st = b.sf_stream_create(eng, (pre.chunk_len, pre.right_context, pre.fifo_len, pre.update_period,
                                  pre.spkcache_len), 1)
    cp = torch.zeros((1, pre.chunk_len, 4), device="cuda")
    T_enc = 1 + (n // 160 - 1) // 8
    outs, c0 = [], 0
    try:
        for k in range(400):
            if c0 >= T_enc:
                break
            m0 = 8 * (c0 - 1) if c0 > 0 else 0
            a0 = max(0, 160 * m0 - 257) // 1000 * 1000
            end = sched[k]
            assert end - a0 <= n_buf                   # the row holds everything received since a0
            row = np.zeros((1, n_buf), np.float32)
            seg = clip[a0:end]
            row[0, :len(seg)] = seg
            n_out = b.sf_stream_step_audio(eng, st, torch.from_numpy(row).cuda(), np.array([a0]), np.array([end]),
                                           np.array([int(end >= n)]), cp)
            outs.append(cp.cpu().numpy()[0, :n_out[0]])
            c0 += int(n_out[0])
        b.sf_check(eng)
    finally:
        b.sf_stream_destroy(st)
    ref, _, margin = _oracle(clip, n, w, pre, sched)
    assert margin > 2e-6
    got = np.concatenate(outs)
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) <= 1e-4


def test_audio_in_rejects_a_buffer_that_starts_too_late(eng):
    pre = O.PRESETS["low"]
    st = b.sf_stream_create(eng, (pre.chunk_len, pre.right_context, pre.fifo_len, pre.update_period,
                                  pre.spkcache_len), 1)
    try:
        row = torch.zeros((1, 40000), device="cuda")
        cp = torch.zeros((1, pre.chunk_len, 4), device="cuda")
        with pytest.raises(b.SFError):   # the first window needs samples from 0 on
            b.sf_stream_step_audio(eng, st, row, np.array([100]), np.array([40100]), np.array([0]), cp)
    finally:
        b.sf_stream_destroy(st)
