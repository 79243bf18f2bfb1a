"""GPU parity of the alternative front-end implementation (SF_OPT_MEL_PATH
= 0: radix-2 FFT through shared memory, one normalisation CTA per (clip,
bin)) against the oracle, on the cases the default path (1: FFT in
registers with warp shuffles, separate statistics and normalisation passes
over all SMs) is tested on elsewhere: clip, ragged batch, minimum length,
silence and a pure tone, the offline forward, the audio-in streaming step
(window mode) and one hour in one call.  Log-mel features within 1e-3,
probabilities within 1e-4 (fp32 engine)."""
import numpy as np
import pytest

import oracle as O
from oracle.streaming import stream_run_audio
from synth import clip_for_config, synth_batch, synth_clip
from _helpers import make_engine, tiny_weights, to_dev

pytestmark = pytest.mark.gpu
ALT_PATH = 0
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


def _engine(w, **kw):
    e = make_engine(w, 0, 2, 2, **kw)
    b.sf_set_option(e, b.SF_OPT_MEL_PATH, ALT_PATH)
    return e


@pytest.fixture(scope="module")
def eng():
    e = _engine(tiny_weights(xavier=True), max_batch=8)
    yield e
    b.sf_destroy(e)


def gpu_mel(e, audio, lens):
    T = 1 + audio.shape[1] // 160
    mel = torch.full((audio.shape[0], 128, T), float("nan"), device="cuda")
    ml = b.sf_mel(e, to_dev(audio), lens, mel)
    b.sf_check(e)
    return mel.cpu().numpy(), ml


@pytest.mark.parametrize("case", ["cfg0", "ragged", "short", "silence_tone"])
def test_mel_alt_path_parity(eng, case):
    if case == "cfg0":
        audio, lens, _ = clip_for_config(0)
    elif case == "ragged":
        audio, lens, _ = synth_batch(77, [3.3, 1.01, 7.777, 0.1])
    elif case == "short":
        a, _ = synth_clip(78, 0.1, 2)
        audio, lens = a[None], np.array([1600])
    else:
        n = 16000
        audio = np.zeros((2, n), np.float32)
        audio[1] = np.sin(2 * np.pi * 64 * 16000 / 512 * np.arange(n) / 16000).astype(np.float32)
        lens = np.array([n, n])
    got, ml = gpu_mel(eng, audio, lens)
    ref, L = O.mel_features(audio, lens)
    assert np.array_equal(ml, L)
    assert not np.isnan(got).any()
    assert np.max(np.abs(got - ref)) <= 1e-3
    for i, l in enumerate(L):
        assert np.all(got[i, :, l:] == 0)


def test_offline_forward_alt_path(eng):
    w = tiny_weights(xavier=True)
    audio, lens, _ = synth_batch(83, [6.0, 2.2])
    Tp = int(O.encoder_frames(audio.shape[1] // 160))
    probs = torch.zeros((2, Tp, 4), device="cuda")
    b.sf_forward_offline(eng, to_dev(audio), lens, probs)
    b.sf_check(eng)
    ref, _ = O.forward_offline(audio, lens, w)
    assert np.max(np.abs(probs.cpu().numpy() - ref)) <= 1e-4


def test_audio_in_stream_alt_path(eng):
    w = tiny_weights(xavier=True)
    pre = O.PRESETS["low"]
    clip = synth_clip([60, 0], 9.0, 3)[0]
    n = len(clip)
    sched = [min(n, 3000 + 4000 * k) for k in range(300)]
    st = b.sf_stream_create(eng, (pre.chunk_len, pre.right_context, pre.fifo_len, pre.update_period,
                                  pre.spkcache_len), 1)
    cp = torch.zeros((1, pre.chunk_len, 4), device="cuda")
    d_audio = to_dev(clip[None])
    T_enc = 1 + (n // 160 - 1) // 8
    outs = []
    try:
        for k in range(300):
            if sum(len(o) for o in outs) >= T_enc:
                break
            n_out = b.sf_stream_step_audio(eng, st, d_audio, np.zeros(1, np.int64), np.array([sched[k]]),
                                           np.array([int(sched[k] >= n)]), cp)
            outs.append(cp.cpu().numpy()[0, :n_out[0]])
        b.sf_check(eng)
    finally:
        b.sf_stream_destroy(st)
    taps = []
    ref, _ = stream_run_audio(clip, n, w, pre, sched, taps=taps)
    assert min(t["margin"] for t in taps) > 2e-6
    got = np.concatenate(outs)
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) <= 1e-4


def test_mel_alt_path_one_hour():
    from synth.audio import hour_of_audio
    x = hour_of_audio()
    n = len(x)
    e = make_engine(tiny_weights(), 1, 2, 2, max_batch=1, max_samples=n)
    b.sf_set_option(e, b.SF_OPT_MEL_PATH, ALT_PATH)
    try:
        got, ml = gpu_mel(e, x[None], np.array([n]))
    finally:
        b.sf_destroy(e)
    ref, L = O.mel_features(x[None], np.array([n]))
    assert int(ml[0]) == int(L[0]) == 360_000
    assert np.max(np.abs(got - ref)) <= 1e-3
