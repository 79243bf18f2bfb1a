"""GPU parity of the Nemotron-3 variant's offline forward (sf_nem_*) against
the oracle (oracle/nemotron.py) on the same seeded inputs.

bf16 engine: speaker probabilities within 2e-2 (the tolerance of the bf16
mode), with xavier-scaled weights so the oracle's probabilities spread by
more than 4x the bound (a constant output fails); frames past each clip's
last 10 ms frame are exactly 0."""
import numpy as np
import pytest

from oracle import nemotron as N
from synth import NEM_FULL, NEM_TINY, make_nem_weights, synth_batch, weights_blob

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

TOL = 2e-2


def _engine(dims, max_batch, max_samples=1_920_000):
    w = make_nem_weights(dims, seed=0, xavier=True)
    cfg = b.nem_default_config(n_layers=dims.n_layers, max_batch=max_batch, max_samples=max_samples)
    return w, b.sf_nem_create(weights_blob(w), cfg)


def _run(eng, audio, lens):
    B, n = audio.shape
    probs = torch.full((B, n // 160, 8), float("nan"), device="cuda")
    out_len = b.sf_nem_forward_offline(eng, torch.from_numpy(audio).cuda(), lens, probs)
    return probs.cpu().numpy(), out_len


def _check(got, audio, lens, w, clips):
    L = np.asarray(lens) // 160
    for i in range(len(lens)):
        assert np.all(got[i, L[i]:] == 0), i
    for i in clips:
        ref, Lr = N.nem_forward_offline(audio[i:i + 1, :lens[i]], lens[i:i + 1], w)
        assert Lr[0] == L[i]
        assert float(ref.max() - ref.min()) > 4 * TOL
        err = float(np.max(np.abs(got[i, :L[i]] - ref[0, :L[i]])))
        assert err <= TOL, (i, err)


def test_nemotron_tiny_ragged_batch():
    w, eng = _engine(NEM_TINY, 4)
    try:
        audio, lens, _ = synth_batch(201, [9.0, 4.1, 0.3])
        got, out_len = _run(eng, audio, lens)
        got2, _ = _run(eng, audio, lens)
    finally:
        b.sf_nem_destroy(eng)
    assert list(out_len) == list(np.asarray(lens) // 160)
    assert np.array_equal(got, got2)                     # repeatable to the bit
    _check(got, audio, lens, w, range(3))


def test_nemotron_full_31_layers():
    w, eng = _engine(NEM_FULL, 2)
    try:
        audio, lens, _ = synth_batch(202, [20.0, 3.3])
        got, _ = _run(eng, audio, lens)
    finally:
        b.sf_nem_destroy(eng)
    _check(got, audio, lens, w, range(2))


def test_nemotron_beyond_one_wave():
    """8 clips of 100-120 s: 11,800 rows, beyond one wave of clusters, so the
    residual LayerNorms run as separate kernels; sampled clips vs the oracle."""
    w, eng = _engine(NEM_TINY, 8)
    try:
        audio, lens, _ = synth_batch(203, [120.0, 100.0, 110.0, 117.3, 101.0, 119.9, 105.5, 112.0])
        got, _ = _run(eng, audio, lens)
    finally:
        b.sf_nem_destroy(eng)
    _check(got, audio, lens, w, (1, 7))


def test_nemotron_argument_errors():
    w, eng = _engine(NEM_TINY, 2, max_samples=160_000)
    try:
        audio = torch.zeros((3, 32_000), device="cuda")
        probs = torch.zeros((3, 200, 8), device="cuda")
        with pytest.raises(b.SFError, match="SF_ESHAPE"):
            b.sf_nem_forward_offline(eng, audio, np.full(3, 32_000), probs)     # batch over max_batch
        with pytest.raises(b.SFError, match="SF_EINVAL"):
            b.sf_nem_forward_offline(eng, audio[:2], np.array([32_000, 1_000]), probs)   # clip under 1600
        with pytest.raises(b.SFError, match="SF_ESHAPE"):
            big = torch.zeros((1, 200_000), device="cuda")
            b.sf_nem_forward_offline(eng, big, np.array([200_000]), torch.zeros((1, 1250, 8), device="cuda"))
    finally:
        b.sf_nem_destroy(eng)
    with pytest.raises(b.SFError, match="SF_EINVAL"):
        b.sf_nem_create(weights_blob(w), b.nem_default_config(d_model=256))
    bad = dict(w)
    del bad["nem.head.bias"]
    with pytest.raises(b.SFError, match="SF_EFORMAT"):
        b.sf_nem_create(weights_blob(bad), b.nem_default_config(n_layers=2))
