"""GPU parity for every streaming preset of the "Streaming Configurations"
table, for streams at different fill states in one batch, and for the tail
cases: all 16 mel-frame remainders x the 4 presets.

Tiny model (2 + 2 layers), fp32 mode, xavier-scaled weights (probabilities
spread over [0, 1]); each stream is compared with the oracle run on that
stream alone, with the oracle's decision margins asserted to exceed the
fp32 discrepancy (~1e-7).  Tolerance 1e-4 on probabilities."""
import numpy as np
import pytest

import oracle as O
from synth import synth_batch
from _helpers import make_engine, tiny_weights, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

PRESETS = {k: (p.chunk_len, p.right_context, p.fifo_len, p.update_period, p.spkcache_len)
           for k, p in O.PRESETS.items()}


@pytest.fixture(scope="module")
def w():
    return tiny_weights(xavier=True)


@pytest.fixture(scope="module")
def eng(w):
    e = make_engine(w, 0, 2, 2, max_batch=16)
    yield e
    b.sf_destroy(e)


def _oracle(feats, L, w, preset):
    taps = []
    ref, st = O.stream_run(feats, int(L), w, O.PRESETS[preset] if isinstance(preset, str) else preset, taps=taps)
    margin = min([t["margin"] for t in taps] + [np.inf])
    return ref, st, margin


def _step_all(eng, st, fd, L, cp, outs, n_steps=None):
    n = len(L)
    left = np.array([1 + (int(l) - 1) // 8 for l in L]) - np.array([sum(len(o) for o in outs[i]) for i in range(n)])
    k = 0
    while (left > 0).any() and (n_steps is None or k < n_steps):
        n_out = b.sf_stream_step(eng, st, fd, np.zeros(n, np.int64), L, cp)
        c = cp.cpu().numpy()
        for i in range(n):
            outs[i].append(c[i, :n_out[i]])
        left -= n_out
        k += 1


@pytest.mark.parametrize("preset,dur", [("high", 32.0), ("ultra_low", 40.0)])
def test_preset_free_running(eng, w, preset, dur):
    """High (124/1/124/124) and Ultra low (3/1/188/144): long enough for pops
    and several cache compressions."""
    audio, lens, _ = synth_batch(400 + len(preset), [dur, dur - 3.3], n_spk_choices=(4,))
    feats, L = O.mel_features(audio, lens)
    st = b.sf_stream_create(eng, PRESETS[preset], 2)
    cp = torch.zeros((2, PRESETS[preset][0], 4), device="cuda")
    outs = [[], []]
    try:
        _step_all(eng, st, to_dev(feats), L, cp, outs)
    finally:
        b.sf_stream_destroy(st)
    for i in range(2):
        ref, ost, margin = _oracle(feats[i], L[i], w, preset)
        assert margin > 2e-6, margin
        got = np.concatenate(outs[i])
        assert got.shape == ref.shape
        assert np.max(np.abs(got - ref)) <= 1e-4
        assert len(ost.cache_emb) == 188          # the run reached a compressed cache


def test_streams_at_different_fill_states(eng, w):
    """Three streams in one batch (custom preset 6/3/16/12/24); stream 1 is reset after 9 steps and starts
    over while the others keep their cache/FIFO, so every later step mixes
    streams at different fill states."""
    pre = O.Preset(6, 3, 16, 12, 24)
    audio, lens, _ = synth_batch(410, [9.0, 7.0, 8.0], n_spk_choices=(4,))
    feats, L = O.mel_features(audio, lens)
    fd = to_dev(feats)
    st = b.sf_stream_create(eng, (6, 3, 16, 12, 24), 3)
    cp = torch.zeros((3, 6, 4), device="cuda")
    outs = [[], [], []]
    try:
        _step_all(eng, st, fd, L, cp, outs, n_steps=9)
        b.sf_stream_reset(st, [1])
        outs[1] = []
        _step_all(eng, st, fd, L, cp, outs)
    finally:
        b.sf_stream_destroy(st)
    for i in range(3):
        ref, _, margin = _oracle(feats[i], L[i], w, pre)
        assert margin > 2e-6, margin
        got = np.concatenate(outs[i])
        assert got.shape == ref.shape, i
        assert np.max(np.abs(got - ref)) <= 1e-4, i


@pytest.mark.parametrize("preset", ["very_high", "high", "low", "ultra_low"])
def test_tail_cases_all_16_remainders(eng, w, preset):
    """16 streams whose mel lengths cover every remainder mod 16; each emits
    exactly 1 + (L-1)//8 frames in chunk_len pieces (last one short) and
    matches the oracle."""
    # two steps for the long-chunk presets (the second one short), a few for the others
    base = {"very_high": 345 * 8, "high": 130 * 8}.get(preset, 6 * 8)
    L = np.array([base + r for r in range(16)], np.int64)
    audio, lens, _ = synth_batch(420, [(l * 160 + 80) / 16000 for l in L])
    feats, L2 = O.mel_features(audio, lens)
    assert np.array_equal(L2, L)
    st = b.sf_stream_create(eng, PRESETS[preset], 16)
    cp = torch.zeros((16, PRESETS[preset][0], 4), device="cuda")
    outs = [[] for _ in range(16)]
    try:
        _step_all(eng, st, to_dev(feats), L, cp, outs)
    finally:
        b.sf_stream_destroy(st)
    cl = PRESETS[preset][0]
    for i in range(16):
        got = np.concatenate(outs[i])
        T = 1 + (int(L[i]) - 1) // 8
        assert len(got) == T
        sizes = [len(o) for o in outs[i] if len(o)]
        assert all(s == cl for s in sizes[:-1]) and 0 < sizes[-1] <= cl
        ref, _, margin = _oracle(feats[i], L[i], w, preset)
        assert margin > 2e-6, margin
        assert np.max(np.abs(got - ref)) <= 1e-4
