"""Pins of the post-processing oracle (frame probabilities -> speaker
segments), independent of its own code: hand-worked cases
(tests/golden/segments.json), a closed form of the plain threshold computed
with array operations, and invariants of the smoothing that any correct
implementation satisfies."""
import json
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "segments.json")


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"][:40])
def test_golden_cases(case):
    probs = np.asarray(case["probs"], np.float32)
    got = O.segments(probs, len(probs), O.SegParams(**case["params"]))
    assert len(got) == len(case["expected"])
    for g, e in zip(got, case["expected"]):
        assert g[2] == e[2]
        assert abs(g[0] - e[0]) < 1e-9 and abs(g[1] - e[1]) < 1e-9


def _runs_closed_form(active):
    """Maximal runs of True via the sign changes of the padded indicator."""
    d = np.diff(np.concatenate([[0], active.astype(np.int8), [0]]))
    starts, ends = np.flatnonzero(d == 1), np.flatnonzero(d == -1) - 1
    return list(zip(starts.tolist(), ends.tolist()))


@pytest.mark.parametrize("seed", range(5))
def test_plain_threshold_is_the_runs_of_p_above_theta(seed):
    rng = np.random.default_rng(seed)
    p = rng.random(500).astype(np.float32)
    for theta in (0.5, 0.3, 0.9):
        assert O.binarize(p, theta, theta) == _runs_closed_form(p > np.float32(theta))


@pytest.mark.parametrize("seed", range(5))
def test_hysteresis_runs_contain_the_onset_runs_and_lie_inside_the_offset_runs(seed):
    rng = np.random.default_rng(100 + seed)
    # smooth-ish random curve so that hysteresis matters
    p = np.clip(np.convolve(rng.random(600), np.ones(7) / 7, mode="same") * 1.6 - 0.3, 0, 1).astype(np.float32)
    on, off = 0.6, 0.4
    runs = O.binarize(p, on, off)
    covered = np.zeros(len(p), bool)
    for a, b in runs:
        covered[a:b + 1] = True
        assert p[a] > on                       # a run starts above the onset
        assert np.all(p[a:b + 1] > off)       # and stays above the offset
        assert b == len(p) - 1 or p[b + 1] <= off
    assert np.all(covered[p > on])            # every frame above the onset is inside a run
    assert not np.any(covered[p <= off])


@pytest.mark.parametrize("seed", range(5))
def test_smoothing_invariants(seed):
    rng = np.random.default_rng(200 + seed)
    T = 400
    probs = np.clip(np.convolve(rng.random(T), np.ones(5) / 5, mode="same")[:, None] * 1.5
                    - rng.random((1, 4)) * 0.5, 0, 1).astype(np.float32)
    prm = O.SegParams(onset=0.55, offset=0.45, pad_onset=0.05, pad_offset=0.1,
                      min_duration_on=0.25, min_duration_off=0.2)
    segs = O.segments(probs, T, prm)
    assert segs == sorted(segs, key=lambda x: (x[0], x[2]))
    for spk in range(4):
        own = [(s, e) for s, e, k in segs if k == spk]
        for s, e in own:
            assert 0.0 <= s < e <= T * 0.08 + 1e-12
            assert e - s >= prm.min_duration_on
        for (s0, e0), (s1, e1) in zip(own, own[1:]):
            assert s1 - e0 >= prm.min_duration_off   # short gaps were closed
        # every onset frame lies in a segment unless its merged segment was
        # shorter than min_duration_on; with no duration filter all of them do
        loose = O.speaker_segments(probs[:, spk], T, O.SegParams(onset=0.55, offset=0.45, pad_onset=0.05,
                                                                  pad_offset=0.1, min_duration_off=0.2))
        for t in np.flatnonzero(probs[:, spk] > np.float32(0.55)):
            assert any(s <= t * 0.08 and (t + 1) * 0.08 <= e + 1e-12 for s, e in loose)


def test_no_padding_no_filter_gives_exact_frame_boundaries():
    probs = np.zeros((50, 1), np.float32)
    probs[10:20, 0] = 0.9
    probs[30:31, 0] = 0.9
    segs = O.segments(probs, 50)
    assert [(round(s / 0.08), round(e / 0.08)) for s, e, _ in segs] == [(10, 20), (30, 31)]


def test_length_limits_the_frames_read():
    probs = np.full((20, 1), 0.9, np.float32)
    assert O.segments(probs, 5) == [[0.0, 5 * 0.08, 0]]
    assert O.segments(probs, 0) == []
