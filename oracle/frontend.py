"""Oracle: log-mel front-end (plain definitions, direct DFT).

Source: "Streaming Sortformer Diarizer", Pipeline and Model Parameters
(16 kHz audio -> 128 mel bins, 25 ms window, 10 ms stride) and Exported
Methods / preprocessor (audio (N,) + length -> mel (1, 128, T) + mel_len).
The DSP constants the page leaves open are fixed by this engine's front-end
recipe: preemphasis 0.97, n_fft 512, 400-sample Hann window, hop 160, power
spectrum, 128 Slaney mel bins over 0-8 kHz, log(x + 2^-24), per-bin
mean/variance normalisation over the valid frames.

Readings where the pages are silent (each pinned by a test where a fact
allows):
  * preemphasis runs over the valid samples only; samples >= length are 0;
  * centred framing pads 256 zeros on each side (constant, not reflect);
  * the Hann window is the symmetric one, w[n] = 0.5 - 0.5 cos(2 pi n / 399),
    centred in the 512-sample frame (56 zeros each side);
  * valid frames L = floor(N / 160); the extra centred column is computed
    and masked to zero;
  * normalisation uses the unbiased variance over the L valid frames and
    adds 1e-5 to the standard deviation (not inside the square root).
"""
from __future__ import annotations

import numpy as np

SR = 16000
N_FFT = 512
WIN = 400
HOP = 160
N_MELS = 128
PREEMPH = 0.97
LOG_GUARD = 2.0 ** -24
NORM_EPS = 1e-5


def n_frames(n_samples_buffer: int) -> int:
    """Columns of the centred STFT of a buffer of N samples: 1 + N // hop."""
    return 1 + n_samples_buffer // HOP


def n_valid_frames(length: int) -> int:
    """Valid mel frames of a clip of ``length`` samples: floor(length / hop)."""
    return length // HOP


def preemphasis(x, length, dt=np.float64):
    """y[0] = x[0]; y[n] = x[n] - 0.97 x[n-1] for 0 < n < length; 0 beyond."""
    x = np.asarray(x, dt)
    y = np.zeros_like(x)
    if length > 0:
        y[0] = x[0]
        y[1:length] = x[1:length] - dt(PREEMPH) * x[0:length - 1]
    return y


def hann_window_512(dt=np.float64):
    """Symmetric 400-point Hann window zero-padded to 512 (56 each side)."""
    n = np.arange(WIN, dtype=np.float64)
    w = 0.5 - 0.5 * np.cos(2.0 * np.pi * n / (WIN - 1))
    out = np.zeros(N_FFT, np.float64)
    off = (N_FFT - WIN) // 2
    out[off:off + WIN] = w
    return out.astype(dt)


def stft_power(y, dt=np.float64):
    """|X[t, k]|^2 for k = 0..256 of the centred STFT of ``y`` (1-D buffer).

    Frame t covers zero-padded samples [hop*t, hop*t + 512) of ``y`` padded
    with 256 zeros on both sides, multiplied by the window; X is the direct
    DFT  X[k] = sum_m f[m] exp(-2 pi i k m / 512)."""
    y = np.asarray(y, dt)
    T = n_frames(len(y))
    pad = np.concatenate([np.zeros(N_FFT // 2, dt), y, np.zeros(N_FFT // 2, dt)])
    idx = HOP * np.arange(T)[:, None] + np.arange(N_FFT)[None, :]
    frames = pad[idx] * hann_window_512(dt)[None, :]
    m = np.arange(N_FFT)
    k = np.arange(N_FFT // 2 + 1)
    ang = -2.0 * np.pi * np.outer(m, k) / N_FFT
    cdt = np.complex128 if dt == np.float64 else np.complex64
    D = (np.cos(ang) + 1j * np.sin(ang)).astype(cdt)
    X = frames.astype(cdt) @ D
    return (X.real ** 2 + X.imag ** 2).astype(dt)


def _hz_to_mel_slaney(f):
    f = np.asarray(f, np.float64)
    f_sp = 200.0 / 3.0
    min_log_hz = 1000.0
    min_log_mel = min_log_hz / f_sp
    logstep = np.log(6.4) / 27.0
    return np.where(f >= min_log_hz, min_log_mel + np.log(np.maximum(f, 1e-300) / min_log_hz) / logstep, f / f_sp)


def _mel_to_hz_slaney(m):
    m = np.asarray(m, np.float64)
    f_sp = 200.0 / 3.0
    min_log_hz = 1000.0
    min_log_mel = min_log_hz / f_sp
    logstep = np.log(6.4) / 27.0
    return np.where(m >= min_log_mel, min_log_hz * np.exp(logstep * (m - min_log_mel)), f_sp * m)


def slaney_mel_filterbank(normalize=True):
    """(128, 257) Slaney filterbank over 0-8 kHz at the FFT bin frequencies
    k * 16000 / 512: triangles between consecutive points of 130 equally
    spaced Slaney-mel points, area-normalised by 2 / (f[m+2] - f[m])."""
    pts = _mel_to_hz_slaney(np.linspace(_hz_to_mel_slaney(0.0), _hz_to_mel_slaney(SR / 2), N_MELS + 2))
    fk = np.arange(N_FFT // 2 + 1) * SR / N_FFT
    F = np.zeros((N_MELS, N_FFT // 2 + 1))
    for m in range(N_MELS):
        lo = (fk - pts[m]) / (pts[m + 1] - pts[m])
        hi = (pts[m + 2] - fk) / (pts[m + 2] - pts[m + 1])
        F[m] = np.maximum(0.0, np.minimum(lo, hi))
        if normalize:
            F[m] *= 2.0 / (pts[m + 2] - pts[m])
    return F, pts


def log_mel(power, dt=np.float64):
    """log(F @ P + 2^-24): (T, 257) -> (128, T)."""
    F, _ = slaney_mel_filterbank()
    M = F.astype(dt) @ np.asarray(power, dt).T
    return np.log(M + dt(LOG_GUARD))


def normalize_per_bin(lm, L, dt=np.float64):
    """Per-bin normalisation over the first L frames; frames >= L become 0."""
    lm = np.asarray(lm, dt)
    out = np.zeros_like(lm)
    v = lm[:, :L]
    mu = v.mean(axis=1, keepdims=True)
    sd = np.sqrt(((v - mu) ** 2).sum(axis=1, keepdims=True) / (L - 1)) + dt(NORM_EPS)
    out[:, :L] = (v - mu) / sd
    return out


def mel_features(audio, lengths, dt=np.float64):
    """Batch front-end: audio (B, N_max) + lengths (B,) -> (features (B, 128,
    1 + N_max // 160), valid frame counts (B,) = lengths // 160)."""
    audio = np.atleast_2d(np.asarray(audio))
    B, N = audio.shape
    T = n_frames(N)
    out = np.zeros((B, N_MELS, T), dt)
    L = np.zeros(B, np.int64)
    for b in range(B):
        n = int(lengths[b])
        y = preemphasis(audio[b], n, dt)
        lm = log_mel(stft_power(y, dt), dt)
        L[b] = n_valid_frames(n)
        out[b] = normalize_per_bin(lm, int(L[b]), dt)
    return out, L
