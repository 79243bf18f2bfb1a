"""The allocation-free front-end, sf_mel_noalloc, against sf_mel.

This entry point is for callers that cannot allocate device memory while
they compute features (a memory pool budgeted by someone else, a plugin in a
foreign CUDA context, a real-time thread that must not block in cudaMalloc).
It keeps its scratch in a static device array, so two calls in a row must
both give sf_mel's result: the second call reuses scratch the first one
left behind.  This file is collected last on purpose."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from synth import synth_batch  # noqa: E402
from _helpers import make_engine, tiny_weights, to_dev  # noqa: E402
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


def test_mel_noalloc_matches_sf_mel_on_two_calls_in_a_row():
    eng = make_engine(tiny_weights(), 0, 2, 2, max_batch=8)
    try:
        cases = [synth_batch(301, [3.3, 1.01, 7.777]), synth_batch(302, [0.5, 12.0])]
        for audio, lens, _ in cases:
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
            assert np.max(np.abs(g - r)) <= 1e-3      # the mel tolerance of the parity tests
    finally:
        b.sf_destroy(eng)


def test_mel_noalloc_rejects_sizes_beyond_its_scratch():
    audio = to_dev(np.zeros((11, 1_920_000), np.float32))
    mel = torch.zeros((11, 128, 1 + 1_920_000 // 160), device="cuda")
    with pytest.raises(b.SFError, match="SF_ESHAPE"):
        b.sf_mel_noalloc(audio, np.full(11, 1_920_000), mel)   # 11 x 376 tiles > 4096
