"""Pins for the oracle's front-end against facts the pages or mathematics fix."""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
from oracle import frontend as F

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_frame_counts_match_pages():
    g = json.load(open(os.path.join(GOLD, "frames.json")))
    for n, L in g["samples_to_mel"]:
        assert O.n_valid_frames(n) == L
    for L, T in g["mel_to_enc"]:
        assert int(O.encoder_frames(L)) == T
    # 10 ms stride x 8 = 80 ms per output frame
    assert 1000 * 160 // 16000 * 8 == g["ms_per_output_frame"]


def test_encoder_frames_is_three_stride2_stages():
    for L in range(1, 5000):
        l1 = 1 + (L - 1) // 2
        l2 = 1 + (l1 - 1) // 2
        l3 = 1 + (l2 - 1) // 2
        assert l3 == int(O.encoder_frames(L))


def test_preemphasis_impulse_and_length():
    x = np.zeros(32)
    x[5] = 1.0
    y = O.preemphasis(x, 20)
    ref = np.zeros(32)
    ref[5], ref[6] = 1.0, -0.97
    assert np.array_equal(y, ref)
    x = np.ones(10)
    y = O.preemphasis(x, 4)
    assert np.allclose(y, [1.0, 0.03, 0.03, 0.03, 0, 0, 0, 0, 0, 0])


def test_hann_symmetric_closed_forms():
    w = O.hann_window_512()
    assert np.all(w[:56] == 0) and np.all(w[456:] == 0)
    assert w[56] == 0.0 and abs(w[455]) < 1e-15
    assert np.allclose(w[56:456], w[56:456][::-1], atol=1e-15)
    # sum_{n=0}^{399} 0.5 - 0.5 cos(2 pi n / 399) = 200 - 0.5 * 1 = 199.5
    assert abs(w.sum() - 199.5) < 1e-10


@pytest.mark.parametrize("k", [3, 20, 64, 200, 250])
def test_pure_tone_peaks_in_its_bin(k):
    f = k * 16000 / 512
    n = np.arange(16000)
    y = np.sin(2 * np.pi * f * n / 16000)
    P = O.stft_power(y)
    interior = P[3:-3]
    assert np.all(np.argmax(interior, axis=1) == k)


def test_parseval_per_frame():
    rng = np.random.default_rng(5)
    y = rng.standard_normal(4000)
    P = O.stft_power(y)
    pad = np.concatenate([np.zeros(256), y, np.zeros(256)])
    w = O.hann_window_512()
    for t in (0, 3, 11, len(P) - 1):
        fr = pad[160 * t:160 * t + 512] * w
        # rfft power: bins 1..255 stand for two conjugate bins each
        tot = P[t, 0] + P[t, 256] + 2 * P[t, 1:256].sum()
        assert abs(tot - 512 * np.sum(fr ** 2)) <= 1e-9 * max(1.0, tot)


def test_direct_dft_agrees_with_fft():
    rng = np.random.default_rng(6)
    y = rng.standard_normal(3000)
    P = O.stft_power(y)
    pad = np.concatenate([np.zeros(256), y, np.zeros(256)])
    w = O.hann_window_512()
    fr = np.stack([pad[160 * t:160 * t + 512] * w for t in range(len(P))])
    ref = np.abs(np.fft.rfft(fr, axis=1)) ** 2
    assert np.max(np.abs(P - ref)) <= 1e-9 * np.max(ref)


def test_slaney_scale_closed_forms():
    assert abs(F._hz_to_mel_slaney(1000.0) - 15.0) < 1e-12
    assert abs(F._hz_to_mel_slaney(6400.0) - 42.0) < 1e-12       # 15 + 27 * ln(6.4)/ln(6.4)
    assert abs(F._hz_to_mel_slaney(300.0) - 4.5) < 1e-12         # linear part: f / (200/3)
    for m in (0.0, 3.0, 15.0, 30.0, 45.0):
        assert abs(F._hz_to_mel_slaney(F._mel_to_hz_slaney(m)) - m) < 1e-9


def test_mel_filterbank_partition_of_unity_and_sparsity():
    Fu, pts = O.slaney_mel_filterbank(normalize=False)
    fk = np.arange(257) * 16000 / 512
    inside = (fk >= pts[1]) & (fk <= pts[128])
    s = Fu.sum(axis=0)
    assert np.allclose(s[inside], 1.0, atol=1e-12)
    assert np.all(np.count_nonzero(Fu, axis=0) <= 2)
    Fn, _ = O.slaney_mel_filterbank(normalize=True)
    assert np.all(np.count_nonzero(Fn, axis=0) <= 2)
    # area normalisation: each triangle integrates to 1 over Hz (exact on a fine grid)
    for m in (10, 60, 100, 127):
        f = np.linspace(pts[m], pts[m + 2], 200001)
        tri = np.maximum(0, np.minimum((f - pts[m]) / (pts[m + 1] - pts[m]), (pts[m + 2] - f) / (pts[m + 2] - pts[m + 1])))
        area = np.trapezoid(tri * 2.0 / (pts[m + 2] - pts[m]), f)
        assert abs(area - 1.0) < 1e-6
        # the bin-sampled version approximates the same integral for wide filters
        if m >= 60:
            assert abs(Fn[m].sum() * 16000 / 512 - 1.0) < 0.05


def test_silence_gives_log_guard_and_zero_features():
    lm = O.log_mel(np.zeros((7, 257)))
    assert np.all(lm == math.log(2.0 ** -24))
    assert abs(lm[0, 0] - (-16.635532333438686)) < 1e-12
    feats, L = O.mel_features(np.zeros((1, 3200)), np.array([3200]))
    # (x - mean) is 0 up to the rounding of the mean of 20 equal values
    assert L[0] == 20 and np.max(np.abs(feats)) < 1e-8


def test_normalisation_moments_and_mask():
    rng = np.random.default_rng(7)
    lm = rng.standard_normal((128, 50)) * 3 + 2
    L = 41
    out = O.normalize_per_bin(lm, L)
    assert np.all(out[:, L:] == 0)
    v = out[:, :L]
    assert np.allclose(v.mean(axis=1), 0, atol=1e-12)
    sraw = lm[:, :L].std(axis=1, ddof=1)
    assert np.allclose(v.var(axis=1, ddof=1), (sraw / (sraw + 1e-5)) ** 2, rtol=1e-12)


def test_batch_padding_does_not_change_valid_frames():
    from synth import synth_clip
    a, _ = synth_clip(11, 1.3, 2)
    b, _ = synth_clip(12, 0.9, 3)
    n = max(len(a), len(b))
    x = np.zeros((2, n + 500))
    x[0, :len(a)] = a
    x[1, :len(b)] = b
    f2, L2 = O.mel_features(x, np.array([len(a), len(b)]))
    f1, L1 = O.mel_features(b[None], np.array([len(b)]))
    assert L2[1] == L1[0]
    assert np.allclose(f2[1, :, :L1[0]], f1[0, :, :L1[0]], atol=1e-12)
    assert np.all(f2[1, :, L1[0]:] == 0)


def test_fp32_oracle_close_to_fp64():
    from synth import clip_for_config
    a, ln, _ = clip_for_config(0)
    f64, _ = O.mel_features(a, ln)
    f32, _ = O.mel_features(a, ln, dt=np.float32)
    assert np.max(np.abs(f64 - f32)) < 1e-3
