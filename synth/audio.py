"""Seeded synthetic meeting audio (16 kHz mono float32).

Stand-in for the recordings the pages evaluate on (AMI meetings, the HF
example clip), which are not available here.  Structure follows the pages'
workloads: 2-4 speakers, overlapped speech, speakers arriving at different
times, silence between turns.

Recipe per clip:
  * each speaker: a harmonic tone (f0 ~ U(100, 250) Hz, 10 harmonics with
    amplitude 1/h, rendered from a wavetable) with 4 Hz amplitude modulation
    (1 + 0.5 sin(2 pi 4 t)), gated by a two-state on/off Markov chain whose
    state durations are exponential (means ``on_mean`` / ``off_mean``);
  * optional overlap target: ``off_mean`` is bisected (the underlying unit
    exponential draws stay fixed) until the overlapped share of speech frames
    (10 ms frames with >= 2 active speakers among those with >= 1) is within
    +-1 % of the target;
  * optional arrivals: each speaker is off until a first-on time ~ U(0, A);
  * mix = sum of speakers + white noise 30 dB below the mix RMS, then the
    clip is peak-normalised to 0.9.
"""
from __future__ import annotations

import numpy as np

SR = 16000
_TABLE_N = 8192
_TABLE = None


def _wavetable():
    global _TABLE
    if _TABLE is None:
        ph = np.arange(_TABLE_N) / _TABLE_N
        _TABLE = sum(np.sin(2 * np.pi * h * ph) / h for h in range(1, 11)).astype(np.float32)
    return _TABLE


def _intervals(e_on, e_off, start_on, on_mean, off_mean, dur, first_on):
    """On-intervals (seconds) of one speaker's Markov gate."""
    out = []
    t = first_on
    on = start_on if first_on == 0.0 else True
    i = j = 0
    while t < dur and i < len(e_on) and j < len(e_off):
        if on:
            d = on_mean * e_on[i]
            i += 1
            out.append((t, min(dur, t + d)))
        else:
            d = off_mean * e_off[j]
            j += 1
        t += d
        on = not on
    return out


def _frame_mask(iv, n_frames, hop_s=0.01):
    m = np.zeros(n_frames + 1, np.int32)
    for a, b in iv:
        ia = int(np.ceil(a / hop_s - 0.5))
        ib = int(np.ceil(b / hop_s - 0.5))
        ia, ib = max(ia, 0), min(ib, n_frames)
        if ib > ia:
            m[ia] += 1
            m[ib] -= 1
    return np.cumsum(m[:-1]) > 0


def _overlap_share(masks):
    act = np.sum(masks, axis=0)
    speech = np.count_nonzero(act >= 1)
    return 0.0 if speech == 0 else np.count_nonzero(act >= 2) / speech


def synth_clip(seed, dur_s, n_spk, overlap=None, arrival_max_s=0.0, on_mean=1.5, off_mean=1.5):
    """Return (audio float32 (N,), info dict).  ``seed`` may be an int or a
    sequence accepted by ``numpy.random.default_rng``."""
    rng = np.random.default_rng(seed)
    n = int(round(dur_s * SR))
    n_frames = n // 160
    k = int(2 * dur_s / 0.05) + 64
    spk = []
    for _ in range(n_spk):
        f0 = rng.uniform(100.0, 250.0)
        start_on = bool(rng.random() < 0.5)
        e_on = rng.exponential(1.0, k)
        e_off = rng.exponential(1.0, k)
        first_on = rng.uniform(0.0, arrival_max_s) if arrival_max_s > 0 else 0.0
        spk.append((f0, start_on, e_on, e_off, first_on))

    def schedule(off_m):
        return [_intervals(e_on, e_off, st, on_mean, off_m, dur_s, fo) for (_, st, e_on, e_off, fo) in spk]

    off_used = off_mean
    if overlap is not None and n_spk >= 2:
        lo, hi = np.log(0.05), np.log(500.0)
        for _ in range(60):
            mid = 0.5 * (lo + hi)
            ov = _overlap_share([_frame_mask(iv, n_frames) for iv in schedule(np.exp(mid))])
            off_used = float(np.exp(mid))
            if abs(ov - overlap) <= 0.01:
                break
            if ov > overlap:
                lo = mid
            else:
                hi = mid
    ivs = schedule(off_used)
    masks = [_frame_mask(iv, n_frames) for iv in ivs]
    achieved = _overlap_share(masks)

    t = np.arange(n, dtype=np.float64) / SR
    am = (1.0 + 0.5 * np.sin(2 * np.pi * 4.0 * t)).astype(np.float32)
    tab = _wavetable()
    mix = np.zeros(n, np.float32)
    for (f0, _, _, _, _), iv in zip(spk, ivs):
        gate = np.zeros(n + 1, np.int32)
        for a, b in iv:
            ia, ib = int(round(a * SR)), min(n, int(round(b * SR)))
            if ib > ia:
                gate[ia] += 1
                gate[ib] -= 1
        g = np.cumsum(gate[:-1]) > 0
        idx = (np.mod(f0 * t, 1.0) * _TABLE_N).astype(np.int64) % _TABLE_N
        mix += np.where(g, tab[idx], 0.0).astype(np.float32)
    mix *= am
    rms = float(np.sqrt(np.mean(mix.astype(np.float64) ** 2))) if n else 0.0
    noise = rng.standard_normal(n).astype(np.float32) * np.float32(rms * 10 ** (-30 / 20))
    x = mix + noise
    peak = float(np.max(np.abs(x))) if n else 0.0
    if peak > 0:
        x = x * np.float32(0.9 / peak)
    info = dict(n_spk=n_spk, overlap=achieved, off_mean=off_used,
                activity=np.stack(masks, 1) if masks else np.zeros((n_frames, 0), bool))
    return x.astype(np.float32), info


def synth_batch(seed, durs, n_spk_choices=(2, 3, 4), overlap=None, arrival_max_s=0.0):
    """Independent clips; clip i uses the seed sequence [seed, i].  Returns
    (padded audio (B, N_max) float32, lengths (B,) int64, infos)."""
    clips, infos = [], []
    rng = np.random.default_rng(seed)
    spk = rng.choice(n_spk_choices, size=len(durs)) if n_spk_choices is not None else None
    for i, d in enumerate(durs):
        ns = int(spk[i])
        a, info = synth_clip([seed, i], d, ns, overlap=overlap, arrival_max_s=arrival_max_s)
        clips.append(a)
        infos.append(info)
    nmax = max(len(c) for c in clips)
    out = np.zeros((len(clips), nmax), np.float32)
    for i, c in enumerate(clips):
        out[i, :len(c)] = c
    return out, np.array([len(c) for c in clips], np.int64), infos


def clip_for_config(idx, n_clips=None, dur_s=None):
    """Audio for the named workloads (audio seed = 1000 + workload index):

    0: 1 clip, 2 speakers, 2.0 s
    1: 1 clip, 4 speakers, 90 s, 15 % overlap
    2: 64 streams x 60 s, 2-4 speakers each
    3: 16 streams x 600 s, 4 speakers, 20 % overlap, arrivals U(0, 300 s)
    4: 32 clips, lengths U(5, 120) s, 2-4 speakers each

    ``n_clips``/``dur_s`` take a bounded subset (the first clips/streams,
    optionally shortened) of the same recipe.  Returns (audio (B, N_max),
    lengths (B,), infos)."""
    seed = 1000 + idx
    if idx == 0:
        a, info = synth_clip(seed, dur_s or 2.0, 2)
        return a[None], np.array([len(a)], np.int64), [info]
    if idx == 1:
        a, info = synth_clip(seed, dur_s or 90.0, 4, overlap=0.15)
        return a[None], np.array([len(a)], np.int64), [info]
    if idx == 2:
        n = n_clips or 64
        return synth_batch(seed, [dur_s or 60.0] * n)
    if idx == 3:
        n = n_clips or 16
        return synth_batch(seed, [dur_s or 600.0] * n, n_spk_choices=(4,), overlap=0.20, arrival_max_s=300.0)
    if idx == 4:
        rng = np.random.default_rng(seed)
        durs = rng.uniform(5.0, 120.0, size=32)
        durs = np.round(durs * SR) / SR
        n = n_clips or 32
        d = list(durs[:n]) if dur_s is None else [min(dur_s, x) for x in durs[:n]]
        return synth_batch([seed, 99], d)
    raise ValueError(idx)


def hour_of_audio(seed=1004, minutes=60):
    """Concatenated synthetic audio for the front-end throughput run: 60 s
    clips (2-4 speakers) joined end to end."""
    a, ln, _ = synth_batch([seed, 7], [60.0] * minutes)
    return np.concatenate([a[i, :ln[i]] for i in range(len(ln))])
