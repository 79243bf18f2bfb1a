"""Post-processing of frame probabilities into speaker segments (oracle).

Test infrastructure only (see oracle/__init__.py).

Source: the "Streaming Sortformer Diarizer" model card, section "Output":
the raw output is (B, T/8, 4) sigmoid probabilities, which diarize() turns
into [start_seconds, end_seconds, speaker_index] segments by VAD-style
thresholding and smoothing; NeMo API page, SortformerEncLabelModel.diarize
(postprocessing parameters come from an optional yaml, not given).

Reading (the pages name the steps but give no parameters or order): the
usual VAD post-processing parameters, applied per speaker in this order
  1. hysteresis binarisation: a frame run starts at the first frame with
     p > onset and ends before the first later frame with p <= offset
     (onset = offset = 0.5 by default: active <=> p > 0.5, the same
     activity test as the cache-compression reading);
  2. a run of frames a..b covers [a * 0.08, (b + 1) * 0.08) seconds (one
     encoder frame = 8 x 10 ms);
  3. padding: start - pad_onset (clamped at 0), end + pad_offset (clamped at
     the clip's end, n_frames * 0.08);
  4. merging: a segment whose start lies at or before the previous one's end,
     or whose gap to it is shorter than min_duration_off, joins it;
  5. filtering: merged segments shorter than min_duration_on are dropped.
Times are float64; the activity test compares float32 probabilities with
float32 thresholds (both sides take that decision in the same precision).
"""
from __future__ import annotations

import dataclasses

import numpy as np

FRAME_S = 0.08   # encoder frame period: 8 mel frames of 10 ms


@dataclasses.dataclass(frozen=True)
class SegParams:
    onset: float = 0.5
    offset: float = 0.5
    pad_onset: float = 0.0
    pad_offset: float = 0.0
    min_duration_on: float = 0.0
    min_duration_off: float = 0.0


def binarize(p, onset, offset):
    """Step 1: frame runs (a, b), inclusive, of one speaker's probabilities."""
    p = np.asarray(p, np.float32)
    on, off = np.float32(onset), np.float32(offset)
    runs, active, start = [], False, 0
    for t in range(len(p)):
        if not active and p[t] > on:
            active, start = True, t
        elif active and p[t] <= off:
            runs.append((start, t - 1))
            active = False
    if active:
        runs.append((start, len(p) - 1))
    return runs


def to_seconds(runs):
    """Step 2: frame runs to [start, end) seconds."""
    return [(a * FRAME_S, (b + 1) * FRAME_S) for a, b in runs]


def pad(segs, pad_onset, pad_offset, duration):
    """Step 3: widen every segment, clamped to [0, duration]."""
    return [(max(s - pad_onset, 0.0), min(e + pad_offset, duration)) for s, e in segs]


def merge(segs, min_duration_off):
    """Step 4: join a segment to the previous one when it starts at or before
    the previous end or the gap between them is shorter than
    min_duration_off.  Input in increasing start order."""
    out = []
    for s, e in segs:
        if out and (s <= out[-1][1] or s - out[-1][1] < min_duration_off):
            out[-1] = (out[-1][0], max(out[-1][1], e))
        else:
            out.append((s, e))
    return out


def drop_short(segs, min_duration_on):
    """Step 5: remove segments shorter than min_duration_on."""
    return [(s, e) for s, e in segs if e - s >= min_duration_on]


def speaker_segments(p, n_frames, params=SegParams()):
    """Segments of one speaker from its first n_frames probabilities."""
    runs = binarize(np.asarray(p)[:n_frames], params.onset, params.offset)
    segs = pad(to_seconds(runs), params.pad_onset, params.pad_offset, n_frames * FRAME_S)
    return drop_short(merge(segs, params.min_duration_off), params.min_duration_on)


def segments(probs, n_frames, params=SegParams()):
    """All speakers of one clip: probs (T', S) -> list of [start, end, speaker]
    sorted by start, then speaker (the diarize() output format)."""
    out = []
    for spk in range(probs.shape[1]):
        out.extend([s, e, spk] for s, e in speaker_segments(probs[:, spk], n_frames, params))
    out.sort(key=lambda x: (x[0], x[2]))
    return out
