"""GPU parity at full size, in the launch configurations bench.py times.

Full model (17 FastConformer + 18 Transformer layers), bf16, seeded N(0, 0.02)
weights.  Streaming workloads run with all their streams batched exactly as
in the benchmark; sampled streams are compared with the oracle run on that
stream alone (probabilities within 2e-2).  Only steps before the first FIFO
pop / cache compression are compared free-running: until then no step takes
a threshold decision, so the two runs see identical state structure."""
import numpy as np
import pytest

import oracle as O
from synth import clip_for_config
from _helpers import full_weights, make_engine, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


@pytest.fixture(scope="module")
def weights():
    return full_weights()


def _run_steps(eng, preset, audio, lens, n_steps):
    n = audio.shape[0]
    T = 1 + audio.shape[1] // 160
    mel = torch.empty((n, 128, T), device="cuda")
    ml = b.sf_mel(eng, to_dev(audio), lens, mel)
    st = b.sf_stream_create(eng, preset, n)
    cp = torch.zeros((n, preset[0], 4), device="cuda")
    outs = [[] for _ in range(n)]
    try:
        for _ in range(n_steps):
            n_out = b.sf_stream_step(eng, st, mel, np.zeros(n, np.int64), ml, cp)
            c = cp.cpu().numpy()
            for i in range(n):
                outs[i].append(c[i, :n_out[i]])
        b.sf_check(eng)
        sizes = []
        for i in (0, n - 1):
            v = b.sf_state_view()
            b.sf_stream_get_state(eng, st, i, v)
            sizes.append((v.n_cache, v.n_fifo, v.next_frame))
    finally:
        b.sf_stream_destroy(st)
    return [np.concatenate(o) for o in outs], ml, sizes


def test_low_preset_64_streams_first_12_steps(weights):
    """Low preset, 64 streams x 60 s (the benchmark's streaming workload)."""
    pre = O.PRESETS["low"]
    audio, lens, _ = clip_for_config(2)
    eng = make_engine(weights, 1, 17, 18, max_batch=64)
    try:
        got, ml, sizes = _run_steps(eng, (6, 7, 188, 144, 188), audio, lens, 12)
    finally:
        b.sf_destroy(eng)
    assert sizes[0] == (0, 72, 72) and sizes[1] == (0, 72, 72)
    for i in (0, 17, 63):
        f, L = O.mel_features(audio[i:i + 1, :lens[i]], lens[i:i + 1])
        st = O.StreamState()
        ref = np.concatenate([O.stream_step(st, f[0], int(L[0]), weights, pre) for _ in range(12)])
        assert got[i].shape == ref.shape == (72, 4)
        err = np.max(np.abs(got[i] - ref))
        assert err <= 2e-2, (i, err)


def test_very_high_preset_16_streams_first_step(weights):
    """Very high preset, 16 streams x 600 s: the first step (S = 380 frames,
    chunk 340 emitted) of sampled streams, then the state sizes after a
    second step (pop of 300 frames into a compressed 188-frame cache)."""
    pre = O.PRESETS["very_high"]
    audio, lens, _ = clip_for_config(3)
    eng = make_engine(weights, 1, 17, 18, max_batch=16, max_samples=int(audio.shape[1]))
    try:
        got, ml, sizes = _run_steps(eng, (340, 40, 40, 300, 188), audio, lens, 2)
    finally:
        b.sf_destroy(eng)
    assert sizes[0] == sizes[1] == (188, 40, 680)   # step 2 popped 340 of 380 FIFO frames; cache compressed to 188
    for i in (0, 15):
        f, L = O.mel_features(audio[i:i + 1, :lens[i]], lens[i:i + 1])
        st = O.StreamState()
        ref = O.stream_step(st, f[0], int(L[0]), weights, pre)
        assert ref.shape == (340, 4)
        err = np.max(np.abs(got[i][:340] - ref))
        assert err <= 2e-2, (i, err)


def test_offline_batch_32_clips(weights):
    """The variable-length batch: 32 clips of 5-120 s (seeded), padded to the
    longest, in one offline call of the full model (bf16).  Output lengths
    are 1 + (L - 1) // 8, padded rows are zero, and the shortest, a middle
    and the longest clip match the oracle run on that clip alone (2e-2)."""
    audio, lens, _ = clip_for_config(4)
    B, n_max = audio.shape
    eng = make_engine(weights, 1, 17, 18, max_batch=32, max_samples=int(n_max))
    try:
        Tp = int(O.encoder_frames(n_max // 160))
        probs = torch.full((B, Tp, 4), float("nan"), device="cuda")
        out_len = b.sf_forward_offline(eng, to_dev(audio), lens, probs)
        b.sf_check(eng)
    finally:
        b.sf_destroy(eng)
    got = probs.cpu().numpy()
    T = np.array([int(O.encoder_frames(int(n) // 160)) for n in lens])
    assert np.array_equal(np.asarray(out_len), T)
    for i in range(B):
        assert np.all(got[i, T[i]:] == 0), i
        assert np.all(np.isfinite(got[i])) and got[i].min() >= 0 and got[i].max() <= 1, i
    order = np.argsort(lens)
    for i in (int(order[0]), int(order[B // 2]), int(order[-1])):
        ref, tp = O.forward_offline(audio[i:i + 1, :lens[i]], lens[i:i + 1], weights)
        assert tp[0] == T[i]
        err = np.max(np.abs(got[i, :T[i]] - ref[0]))
        assert err <= 2e-2, (i, err)
