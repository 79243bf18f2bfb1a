"""Pins of the audio-in streaming oracle (window mel from raw audio with
per-window normalisation): the window front-end equals the pinned clip
front-end on the same frames; a stream whose whole clip fits one window
reduces to the feature-path stream; the result does not depend on how the
audio arrives; a step waits exactly until its last frame's samples are in."""
import numpy as np
import pytest

import oracle as O
from oracle.streaming import stream_run_audio, stream_step_audio, window_log_mel
from synth import TINY, make_weights, synth_clip


@pytest.fixture(scope="module")
def w():
    return make_weights(TINY, seed=0, xavier=True)


@pytest.mark.parametrize("n,m0,m1", [(40000, 0, 40), (40000, 120, 200), (40000, 200, 250), (4321, 0, 27)])
def test_window_mel_equals_clip_front_end(n, m0, m1):
    x = np.random.default_rng(n).standard_normal(n + 777)
    full = O.log_mel(O.stft_power(O.preemphasis(x[:n], n)))
    assert np.max(np.abs(window_log_mel(x, n, m0, m1) - full[:, m0:m1])) < 1e-12


def test_single_window_stream_equals_feature_stream(w):
    """Very high preset (340 + 40 frames of chunk + look-ahead) on a 9 s clip:
    one window covers the whole clip, so per-window normalisation is the clip
    normalisation and the audio-in step equals the feature-path step."""
    audio, _ = synth_clip([5, 0], 9.0, 3)
    n = len(audio)
    pre = O.PRESETS["very_high"]
    got, steps = stream_run_audio(audio, n, w, pre, [n])
    f, L = O.mel_features(audio[None], np.array([n]))
    ref, _ = O.stream_run(f[0], int(L[0]), w, pre)
    assert steps == [len(ref)]
    assert np.max(np.abs(got - ref)) < 1e-12


def test_output_independent_of_arrival_pattern(w):
    """Low preset, 7 s: audio arriving 0.1 s at a time or 0.9 s at a time
    (windows are computed only once all their samples are in) gives the
    same probabilities."""
    audio, _ = synth_clip([5, 1], 7.0, 2)
    n = len(audio)
    pre = O.Preset(6, 7, 16, 12, 24)
    fine = list(range(1600, n, 1600)) + [n] * 40
    coarse = list(range(14400, n, 14400)) + [n] * 40
    a, steps_a = stream_run_audio(audio, n, w, pre, fine)
    b, steps_b = stream_run_audio(audio, n, w, pre, coarse)
    assert a.shape == b.shape == (1 + (n // 160 - 1) // 8, 4)
    assert np.max(np.abs(a - b)) < 1e-12
    assert sum(steps_a) == sum(steps_b) == len(a)


def test_step_waits_for_its_last_frame(w):
    """The first Low-preset window (frames 0 .. 103) is complete once sample
    160 * 103 + 255 has arrived: one sample less and the step does nothing."""
    audio, _ = synth_clip([5, 2], 5.0, 2)
    pre = O.PRESETS["low"]
    need = 8 * (pre.chunk_len + pre.right_context)
    last = 160 * (need - 1) + 256            # samples [0, last) cover the last frame's support
    st = O.StreamState()
    assert stream_step_audio(st, audio, last - 1, False, w, pre) is None
    assert st.c0 == 0
    out = stream_step_audio(st, audio, last, False, w, pre)
    assert out is not None and out.shape == (pre.chunk_len, 4) and st.c0 == pre.chunk_len
