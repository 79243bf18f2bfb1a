"""GPU checks of the fused subsampling front (SF_OPT_SUB_PATH = 1: the 3x3
s2 conv's outputs computed on chip and fed straight into the first
depthwise conv).  It sums every output's taps in the order of the two-kernel
path and rounds the stage-1 values the same way, so pre_encode embeddings,
offline probabilities and streaming steps must equal path 0 to the bit;
the embeddings are also checked against the oracle.  Path 1 is the default;
path 0 stays selectable and is the bitwise reference here."""
import numpy as np
import pytest

import oracle as O
from synth import clip_for_config, synth_batch
from _helpers import act_dtype, make_engine, tiny_weights, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


def _pre_encode(eng, feats, starts, frames, precision):
    n = len(frames)
    T3 = int(max(O.encoder_frames(f) for f in frames))
    embs = torch.zeros((n, T3, 512), device="cuda", dtype=act_dtype(precision))
    b.sf_pre_encode(eng, to_dev(feats), np.arange(n) % feats.shape[0], starts, frames, embs, T3)
    b.sf_check(eng)
    return embs.float().cpu().numpy()


@pytest.mark.parametrize("precision", [0, 1])
def test_pre_encode_path1_equals_path0(precision):
    w = tiny_weights(xavier=True)
    eng = make_engine(w, precision, 2, 2)
    try:
        audio, lens, _ = synth_batch(80, [4.0, 2.5, 3.1])
        feats, L = O.mel_features(audio, lens)
        feats = feats.astype(np.float32)
        starts = np.array([0, 16, 7])
        frames = np.array([L[0], 101, 57])
        for_path = {}
        for path in (0, 1):
            b.sf_set_option(eng, b.SF_OPT_SUB_PATH, path)
            for_path[path] = _pre_encode(eng, feats, starts, frames, precision)
        assert np.array_equal(for_path[0], for_path[1])
        for i in range(3):
            ref = O.subsample(feats[i, :, starts[i]:starts[i] + frames[i]].T.astype(np.float64), w)
            g = for_path[1][i, :len(ref)]
            rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
            assert rel < (1e-5 if precision == 0 else 3e-2), (i, rel)
    finally:
        b.sf_destroy(eng)


def test_offline_and_stream_path1_equal_path0():
    """bf16 tiny model: a ragged offline batch and four Low-preset steps of
    two streams give the same bits on both paths."""
    w = tiny_weights(xavier=True)
    eng = make_engine(w, 1, 2, 2)
    try:
        audio, lens, _ = synth_batch(84, [7.5, 3.3])
        Tp = int(O.encoder_frames(audio.shape[1] // 160))
        out = {}
        for path in (0, 1):
            b.sf_set_option(eng, b.SF_OPT_SUB_PATH, path)
            probs = torch.zeros((2, Tp, 4), device="cuda")
            b.sf_forward_offline(eng, to_dev(audio), lens, probs)
            mel = torch.empty((2, 128, 1 + audio.shape[1] // 160), device="cuda")
            ml = b.sf_mel(eng, to_dev(audio), lens, mel)
            st = b.sf_stream_create(eng, (6, 7, 188, 144, 188), 2)
            cp = torch.zeros((2, 6, 4), device="cuda")
            steps = []
            try:
                for _ in range(4):
                    b.sf_stream_step(eng, st, mel, np.zeros(2, np.int64), ml, cp)
                    steps.append(cp.cpu().numpy().copy())
            finally:
                b.sf_stream_destroy(st)
            b.sf_check(eng)
            out[path] = (probs.cpu().numpy(), np.stack(steps))
        assert np.array_equal(out[0][0], out[1][0])
        assert np.array_equal(out[0][1], out[1][1])
    finally:
        b.sf_destroy(eng)


def test_full_batch_path1_equals_path0():
    """The 32-clip variable-length batch through the first two subsampling
    stages of the full-size front (bf16): same bits on both paths."""
    audio, lens, _ = clip_for_config(4, n_clips=8)
    w = tiny_weights()
    eng = make_engine(w, 1, 2, 2, max_batch=8, max_samples=int(audio.shape[1]))
    try:
        feats = torch.empty((8, 128, 1 + audio.shape[1] // 160), device="cuda")
        ml = b.sf_mel(eng, to_dev(audio), lens, feats)
        T3 = int(O.encoder_frames(int(ml.max())))
        res = {}
        for path in (0, 1):
            b.sf_set_option(eng, b.SF_OPT_SUB_PATH, path)
            embs = torch.zeros((8, T3, 512), device="cuda", dtype=torch.bfloat16)
            b.sf_pre_encode(eng, feats, np.arange(8), np.zeros(8, np.int64), ml, embs, T3)
            b.sf_check(eng)
            res[path] = embs.float().cpu().numpy()
        assert np.array_equal(res[0], res[1])
    finally:
        b.sf_destroy(eng)
