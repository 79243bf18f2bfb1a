"""GPU failure detection without a fault: the bounded device wait that every
tcgen05 kernel uses, run on a barrier nothing completes, gives up after its
clock budget; the host reads SF_ETIMEOUT from sf_check, the error word is
cleared, and the same engine then runs a forward that matches the oracle.
Collected after the parity files: it makes a device wait run out, so it
runs once they have finished."""
import time

import numpy as np
import pytest

import oracle as O
from synth import clip_for_config
from _helpers import make_engine, tiny_weights, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


def test_bounded_wait_times_out_and_the_engine_stays_usable():
    w = tiny_weights()
    eng = make_engine(w, 1, 2, 2, max_batch=1)
    try:
        t0 = time.perf_counter()
        b.sf_selftest_wait(eng)
        with pytest.raises(b.SFError, match="SF_ETIMEOUT"):
            b.sf_check(eng)
        dt = time.perf_counter() - t0
        assert 0.3 < dt < 60, dt            # the wait ran for its budget, then returned
        b.sf_check(eng)                     # the word was cleared
        audio, lens, _ = clip_for_config(0)
        probs = torch.zeros((1, 25, 4), device="cuda")
        b.sf_forward_offline(eng, to_dev(audio), lens, probs)
        b.sf_check(eng)
        ref, _ = O.forward_offline(audio, lens, w)
        assert np.max(np.abs(probs.cpu().numpy() - ref)) <= 2e-2
    finally:
        b.sf_destroy(eng)
