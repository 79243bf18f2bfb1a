"""GPU: post-processing of frame probabilities into speaker segments
(sf_segments) against the oracle (oracle/postprocess.py).  Times are float64
evaluated with the same separately rounded operations on both sides and the
activity test compares float32 values, so segments and counts must agree
exactly."""
import json
import os

import numpy as np
import pytest

import oracle as O
from _helpers import make_engine, tiny_weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "segments.json")


@pytest.fixture(scope="module")
def eng():
    e = make_engine(tiny_weights(), 1, 2, 2, max_batch=64)
    yield e
    b.sf_destroy(e)


def _params(**kw):
    return O.SegParams(**kw), b.seg_params(**kw)


def _check(eng, probs, n_frames, kw, max_seg=256):
    op, gp = _params(**kw)
    segs, counts = b.sf_segments(eng, torch.from_numpy(probs).cuda(), n_frames, gp, max_seg=max_seg)
    b.sf_check(eng)
    segs, counts = segs.cpu().numpy(), counts.cpu().numpy()
    for i in range(probs.shape[0]):
        for s in range(4):
            ref = O.speaker_segments(probs[i, :, s], int(n_frames[i]), op)
            assert counts[i, s] == len(ref), (i, s)
            k = min(len(ref), max_seg)
            got = [tuple(x) for x in segs[i, s, :k]]
            assert got == ref[:k], (i, s)


def test_golden_cases_on_gpu(eng):
    for case in json.load(open(GOLDEN))["cases"]:
        p = np.asarray(case["probs"], np.float32)
        probs = np.zeros((1, len(p), 4), np.float32)
        probs[0, :, :p.shape[1]] = p
        _check(eng, probs, [len(p)], case["params"])


PARAM_SETS = [{}, {"onset": 0.6, "offset": 0.4},
              {"onset": 0.55, "offset": 0.45, "pad_onset": 0.05, "pad_offset": 0.1, "min_duration_on": 0.25,
               "min_duration_off": 0.2},
              {"pad_onset": 0.3, "pad_offset": 0.3, "min_duration_off": 1.0}]


@pytest.mark.parametrize("kw", PARAM_SETS, ids=lambda k: ",".join(f"{a}={v}" for a, v in k.items()) or "defaults")
def test_random_clips_match_oracle(eng, kw):
    """32 clips, ragged lengths (0, 1, multiples of 32 and not, up to 1500
    frames = 120 s), smooth random activity with plateaus at exactly the
    thresholds."""
    rng = np.random.default_rng(7)
    n, T = 32, 1500
    lens = np.array([0, 1, 31, 32, 33, 64, 96, 1500] + list(rng.integers(2, T, n - 8)), np.int32)
    x = rng.random((n, T + 8, 4))
    k = np.ones(9) / 9
    probs = np.stack([np.stack([np.convolve(x[i, :, s], k, mode="valid") for s in range(4)], -1)
                      for i in range(n)]).astype(np.float32)[:, :T]
    probs = np.clip((probs - 0.5) * 4 + 0.5, 0, 1).astype(np.float32)
    probs[:, ::17, :] = np.float32(0.5)    # exact-threshold frames
    probs[:, 5::23, :] = np.float32(0.6)
    _check(eng, probs, lens, kw)


def test_more_segments_than_storage(eng):
    probs = np.zeros((2, 400, 4), np.float32)
    probs[:, ::2, :] = 0.9                  # 200 one-frame runs per speaker
    _check(eng, probs, [400, 399], {}, max_seg=50)


def test_model_probabilities_to_segments(eng):
    """Probabilities of the model itself (the oracle's forward of the tiny
    model with xavier weights: values spread over [0, 1]) post-processed on
    the GPU and by the oracle."""
    from synth import synth_batch
    w = tiny_weights(xavier=True)
    audio, lens, _ = synth_batch(31, [12.0, 7.3], n_spk_choices=(4,))
    probs, tp = O.forward_offline(audio, lens, w)
    _check(eng, np.ascontiguousarray(probs, np.float32), tp.astype(np.int32),
           {"pad_onset": 0.08, "min_duration_on": 0.16, "min_duration_off": 0.24})


def test_rejects_bad_parameters(eng):
    probs = torch.zeros((1, 10, 4), device="cuda")
    with pytest.raises(b.SFError):
        b.sf_segments(eng, probs, [10], b.seg_params(onset=0.3, offset=0.6))     # onset < offset
    with pytest.raises(b.SFError):
        b.sf_segments(eng, probs, [11])                                          # longer than the buffer
    with pytest.raises(b.SFError):
        b.sf_segments(eng, probs, [10], b.seg_params(pad_onset=-1.0))
