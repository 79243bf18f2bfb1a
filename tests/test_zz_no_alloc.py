"""The allocation-free front-end, sf_mel_noalloc, against sf_mel and the oracle.

This entry point is for callers that cannot allocate device memory while
they compute features (a memory pool budgeted by someone else, a plugin in a
foreign CUDA context, a real-time thread that must not block in cudaMalloc).
It keeps its scratch in a static device array, so two calls in a row must
both give sf_mel's result: the second call reuses scratch the first one
left behind.  Both entry points run the same kernels on the same inputs, so
their features must be equal to the bit.  This file is collected last on
purpose."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import oracle as O  # noqa: E402
from synth import synth_batch  # noqa: E402
from _helpers import make_engine, tiny_weights, to_dev  # noqa: E402
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_mel_noalloc_matches_sf_mel_on_two_calls_in_a_row():
    eng = make_engine(tiny_weights(), 0, 2, 2, max_batch=8)
    try:
        cases = [synth_batch(301, [3.3, 1.01, 7.777]), synth_batch(302, [0.5, 12.0])]
        for n, (audio, lens, _) in enumerate(cases):
            a = to_dev(audio)
            T = 1 + audio.shape[1] // 160
            ref = torch.full((audio.shape[0], 128, T), float("nan"), device="cuda")
            got = torch.full_like(ref, float("nan"))
            ml_ref = b.sf_mel(eng, a, lens, ref)
            ml = b.sf_mel_noalloc(a, lens, got)
            torch.cuda.synchronize()
            assert np.array_equal(ml, ml_ref)
            g, r = got.cpu().numpy(), ref.cpu().numpy()
            assert not np.isnan(g).any()
            assert np.array_equal(g, r)                 # same kernels, same inputs
            if n == 0:
                feats, L = O.mel_features(audio, lens)
                assert np.array_equal(L, ml)
                assert np.max(np.abs(g - feats)) <= 1e-3   # the mel tolerance of the parity tests
    finally:
        b.sf_destroy(eng)


def test_mel_noalloc_first_call_in_a_fresh_process_before_any_engine():
    """The one-time set-up (scratch address, tables, the shared-memory
    attribute of the frame kernels) must not depend on an engine having been
    created on the device first."""
    code = (
        "import sys, numpy as np, torch; sys.path.insert(0, 'tests');"
        "import oracle as O; from synth import synth_batch;"
        "from streaming_speaker_diarization_b200 import binding as b;"
        "audio, lens, _ = synth_batch(303, [4.2, 2.5]);"
        "mel = torch.full((2, 128, 1 + audio.shape[1] // 160), float('nan'), device='cuda');"
        "ml = b.sf_mel_noalloc(torch.from_numpy(audio).cuda(), lens, mel); torch.cuda.synchronize();"
        "f, L = O.mel_features(audio, lens); assert np.array_equal(L, ml);"
        "err = float(np.max(np.abs(mel.cpu().numpy() - f))); assert err <= 1e-3, err; print('ok', err)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok")


def test_mel_noalloc_rejects_sizes_beyond_its_scratch():
    audio = to_dev(np.zeros((11, 1_920_000), np.float32))
    mel = torch.zeros((11, 128, 1 + 1_920_000 // 160), device="cuda")
    with pytest.raises(b.SFError, match="SF_ESHAPE"):
        b.sf_mel_noalloc(audio, np.full(11, 1_920_000), mel)   # 11 x 376 tiles > 4096
    small = to_dev(np.zeros((65, 1600), np.float32))
    with pytest.raises(b.SFError, match="SF_ESHAPE"):
        b.sf_mel_noalloc(small, np.full(65, 1600), torch.zeros((65, 128, 11), device="cuda"))   # > 64 clips
