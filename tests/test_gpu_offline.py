"""GPU parity: front-end, pre_encode, encode and the offline forward through
the C ABI, element by element against the oracle on the same seeded inputs.

Tolerances: log-mel features 1e-3 abs; speaker probabilities 1e-4 abs in the
fp32 mode and 2e-2 abs in the bf16 mode.  Intermediate embeddings, which have
no stated tolerance, are compared by relative L2 error: fp32 1e-5 (fp32
accumulation over K <= 4096 terms), bf16 3e-2 (bf16 operands carry a relative
rounding of 2^-9 per element; errors compound over the stacked layers)."""
import numpy as np
import pytest

import oracle as O
from synth import clip_for_config, synth_batch, synth_clip
from _helpers import act_dtype, bf16_round, full_weights, make_engine, tiny_weights, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


def rel_l2(a, ref):
    return float(np.linalg.norm(np.asarray(a, np.float64) - ref) / max(np.linalg.norm(ref), 1e-30))


@pytest.fixture(scope="module")
def eng_fp32():
    e = make_engine(tiny_weights(), 0, 2, 2)
    yield e
    b.sf_destroy(e)


@pytest.fixture(scope="module")
def eng_fp32_x():
    e = make_engine(tiny_weights(xavier=True), 0, 2, 2)
    yield e
    b.sf_destroy(e)


@pytest.fixture(scope="module")
def eng_bf16_x():
    e = make_engine(tiny_weights(xavier=True), 1, 2, 2)
    yield e
    b.sf_destroy(e)


def gpu_mel(eng, audio, lens):
    a = to_dev(audio)
    T = 1 + audio.shape[1] // 160
    mel = torch.full((audio.shape[0], 128, T), float("nan"), device="cuda")
    ml = b.sf_mel(eng, a, lens, mel)
    torch.cuda.synchronize()
    return mel.cpu().numpy(), ml


@pytest.mark.parametrize("case", ["cfg0", "ragged", "short"])
def test_mel_parity(eng_fp32, case):
    if case == "cfg0":
        audio, lens, _ = clip_for_config(0)
    elif case == "ragged":      # several clips, lengths not multiples of the hop, > several 32-frame tiles
        audio, lens, _ = synth_batch(77, [3.3, 1.01, 7.777, 0.1])
    else:                       # minimum length (1600 samples = 10 frames)
        a, _ = synth_clip(78, 0.1, 2)
        audio, lens = a[None], np.array([1600])
    got, ml = gpu_mel(eng_fp32, audio, lens)
    ref, L = O.mel_features(audio, lens)
    assert np.array_equal(ml, L)
    assert not np.isnan(got).any()
    err = np.max(np.abs(got - ref))
    assert err <= 1e-3, err
    for i, l in enumerate(L):
        assert np.all(got[i, :, l:] == 0)


def test_mel_silence_and_pure_tone(eng_fp32):
    n = 16000
    x = np.zeros((2, n), np.float32)
    x[1] = np.sin(2 * np.pi * 64 * 16000 / 512 * np.arange(n) / 16000).astype(np.float32)
    got, _ = gpu_mel(eng_fp32, x, np.array([n, n]))
    assert np.max(np.abs(got[0])) < 1e-3          # silence -> normalised features 0
    ref, _ = O.mel_features(x, np.array([n, n]))
    assert np.max(np.abs(got[1] - ref[1])) <= 1e-3


def _pre_encode(eng, feats, starts, frames, precision):
    n = len(frames)
    T3 = int(max(O.encoder_frames(f) for f in frames))
    embs = torch.zeros((n, T3, 512), device="cuda", dtype=act_dtype(precision))
    b.sf_pre_encode(eng, to_dev(feats), np.arange(n) % feats.shape[0], starts, frames, embs, T3)
    torch.cuda.synchronize()
    return embs.float().cpu().numpy()


@pytest.mark.parametrize("precision", [0, 1])
def test_pre_encode_parity(precision, eng_fp32_x, eng_bf16_x):
    eng = eng_fp32_x if precision == 0 else eng_bf16_x
    w = tiny_weights(xavier=True)
    audio, lens, _ = synth_batch(80, [4.0, 2.5, 3.1])
    feats, L = O.mel_features(audio, lens)
    starts = np.array([0, 16, 7])
    frames = np.array([L[0], 101, 57])           # ragged: odd lengths, offsets, several tiles
    got = _pre_encode(eng, feats.astype(np.float32), starts, frames, precision)
    for i in range(3):
        ref = O.subsample(feats[i, :, starts[i]:starts[i] + frames[i]].T, w)
        g = got[i, :len(ref)]
        tol = 1e-5 if precision == 0 else 3e-2
        assert rel_l2(g, ref) < tol, (i, rel_l2(g, ref))


@pytest.mark.parametrize("precision", [0, 1])
def test_encode_parity_xavier(precision, eng_fp32_x, eng_bf16_x):
    """encode() on given embeddings, three packed sequences of ragged
    lengths (1, 70, 130 rows: one-row sequence, tile tails)."""
    eng = eng_fp32_x if precision == 0 else eng_bf16_x
    w = tiny_weights(xavier=True)
    rng = np.random.default_rng(5)
    lens = [1, 70, 130]
    X = rng.standard_normal((sum(lens), 512)).astype(np.float32)
    if precision == 1:
        X = bf16_round(X)
    preds = torch.zeros((sum(lens), 4), device="cuda")
    b.sf_encode(eng, to_dev(X, act_dtype(precision)), lens, preds)
    torch.cuda.synchronize()
    got = preds.cpu().numpy()
    off = 0
    for n in lens:
        ref = O.encode(X[off:off + n].astype(np.float64), w)
        err = np.max(np.abs(got[off:off + n] - ref))
        assert err <= (1e-4 if precision == 0 else 2e-2), (n, err)
        off += n


def test_offline_fp32_tiny_cfg0(eng_fp32):
    """Tiny offline workload (2 s, 2 + 2 layers, fp32): probabilities 1e-4."""
    w = tiny_weights()
    audio, lens, _ = clip_for_config(0)
    probs = torch.full((1, 25, 4), float("nan"), device="cuda")
    ol = b.sf_forward_offline(eng_fp32, to_dev(audio), lens, probs)
    torch.cuda.synchronize()
    ref, tp = O.forward_offline(audio, lens, w)
    assert ol[0] == tp[0] == 25
    err = np.max(np.abs(probs.cpu().numpy() - ref))
    assert err <= 1e-4, err


def test_offline_fp32_ragged_batch(eng_fp32_x):
    """Variable-length batch: padded rows are zero, valid rows match."""
    w = tiny_weights(xavier=True)
    audio, lens, _ = synth_batch(81, [1.7, 5.3, 0.45])
    Tp = int(O.encoder_frames(audio.shape[1] // 160))
    probs = torch.full((3, Tp, 4), float("nan"), device="cuda")
    ol = b.sf_forward_offline(eng_fp32_x, to_dev(audio), lens, probs)
    torch.cuda.synchronize()
    ref, tp = O.forward_offline(audio, lens, w)
    got = probs.cpu().numpy()
    assert list(ol) == list(tp)
    for i in range(3):
        assert np.max(np.abs(got[i, :tp[i]] - ref[i, :tp[i]])) <= 1e-4
        assert np.all(got[i, tp[i]:] == 0)


def test_offline_host_entry_matches_device_entry(eng_fp32_x):
    audio, lens, _ = synth_batch(82, [2.2, 3.0])
    Tp = int(O.encoder_frames(audio.shape[1] // 160))
    probs = torch.zeros((2, Tp, 4), device="cuda")
    b.sf_forward_offline(eng_fp32_x, to_dev(audio), lens, probs)
    torch.cuda.synchronize()
    host = np.zeros((2, Tp, 4), np.float32)
    b.sf_forward_offline_host(eng_fp32_x, np.ascontiguousarray(audio), lens, host)
    assert np.array_equal(host, probs.cpu().numpy())


def test_offline_bf16_full_cfg1():
    """Full model (17 + 18 layers) bf16 on the 90 s workload clip, in the
    benchmark's launch shape: with xavier-scaled weights (probabilities
    spread over ~[0.2, 0.8], so a constant output fails) all 1125 frames
    within 2e-2 of the fp64 oracle; with the benchmark's N(0, 0.02) weights
    (probabilities at 0.5 +- 0.015) a shape and range check only."""
    audio, lens, _ = clip_for_config(1)
    for xavier in (True, False):
        w = full_weights(xavier=xavier)
        eng = make_engine(w, 1, 17, 18, max_batch=1)
        try:
            probs = torch.full((1, 1125, 4), float("nan"), device="cuda")
            b.sf_forward_offline(eng, to_dev(audio), lens, probs)
            b.sf_check(eng)
            got = probs.cpu().numpy()
        finally:
            b.sf_destroy(eng)
        assert np.all(np.isfinite(got)) and got.min() >= 0 and got.max() <= 1
        if xavier:
            ref, tp = O.forward_offline(audio, lens, w)
            assert tp[0] == 1125
            assert float(ref.max() - ref.min()) > 0.08     # 4 x the bound
            err = np.max(np.abs(got - ref))
            assert err <= 2e-2, err


def test_offline_bf16_full_xavier_sampled_frames():
    """Full model with O(1) activations (xavier weights): a ragged batch in
    the launch shape of the benchmark; every output row of the shortest clip
    and sampled rows of the others against the oracle."""
    w = full_weights(xavier=True)
    eng = make_engine(w, 1, 17, 18, max_batch=4)
    try:
        audio, lens, _ = synth_batch(83, [12.0, 3.3])
        Tp = int(O.encoder_frames(audio.shape[1] // 160))
        probs = torch.zeros((2, Tp, 4), device="cuda")
        b.sf_forward_offline(eng, to_dev(audio), lens, probs)
        torch.cuda.synchronize()
        ref, tp = O.forward_offline(audio, lens, w)
        got = probs.cpu().numpy()
        for i in range(2):
            err = np.max(np.abs(got[i, :tp[i]] - ref[i, :tp[i]]))
            assert err <= 2e-2, (i, err)
    finally:
        b.sf_destroy(eng)


def test_mel_one_hour():
    """Front-end on 1 h of audio in one call (57.6M samples, 360,001 STFT
    columns, 360,000 valid frames; the front-end throughput workload): every
    feature against the oracle's front-end on the same hour (1e-3)."""
    from synth.audio import hour_of_audio
    x = hour_of_audio()
    n = len(x)
    eng = make_engine(tiny_weights(), 1, 2, 2, max_batch=1, max_samples=n)
    try:
        got, ml = gpu_mel(eng, x[None], np.array([n]))
        b.sf_check(eng)
    finally:
        b.sf_destroy(eng)
    ref, L = O.mel_features(x[None], np.array([n]))
    assert int(ml[0]) == int(L[0]) == 360_000 and got.shape == ref.shape == (1, 128, 360_001)
    assert np.all(got[0, :, 360_000] == 0)
    err = np.max(np.abs(got - ref))
    assert err <= 1e-3, err


def test_fp32_engines_of_different_lengths_coexist():
    """Two fp32 engines in one process: one for clips up to 120 s, then one
    for clips up to 10 s.  The first still runs a 75 s clip (938 encoder
    frames: longer attention rows than any sequence of the second engine)
    after the second was made; probabilities within 1e-4."""
    w = tiny_weights(xavier=True)
    e1 = make_engine(w, 0, 2, 2, max_batch=1)
    e2 = make_engine(w, 0, 2, 2, max_batch=1, max_samples=160_000)
    try:
        audio, lens, _ = synth_batch(91, [75.0])
        T = int(O.encoder_frames(audio.shape[1] // 160))
        probs = torch.zeros((1, T, 4), device="cuda")
        b.sf_forward_offline(e1, to_dev(audio), lens, probs)
        b.sf_check(e1)
        ref, tp = O.forward_offline(audio, lens, w)
        assert tp[0] == T == 938
        assert np.max(np.abs(probs.cpu().numpy()[0] - ref[0])) <= 1e-4
    finally:
        b.sf_destroy(e2)
        b.sf_destroy(e1)


def test_fp32_engine_length_bound():
    """fp32 attention keeps a score row per warp in shared memory: 14,000
    encoder frames at most (max_samples 17,920,159); one sample more is
    rejected at creation."""
    w = tiny_weights()
    with pytest.raises(b.SFError, match="SF_ESHAPE"):
        make_engine(w, 0, 2, 2, max_batch=1, max_samples=17_920_160)
    b.sf_destroy(make_engine(w, 0, 2, 2, max_batch=1, max_samples=17_920_159))


def test_bad_arguments_rejected(eng_fp32):
    audio = to_dev(np.zeros((1, 1000), np.float32))
    probs = torch.zeros((1, 10, 4), device="cuda")
    with pytest.raises(b.SFError, match="SF_ESHAPE|SF_EINVAL"):
        b.sf_forward_offline(eng_fp32, audio, np.array([1000]), probs)       # below 1600 samples
    audio = to_dev(np.zeros((1, 4000), np.float32))
    with pytest.raises(b.SFError, match="SF_EINVAL"):
        b.sf_forward_offline(eng_fp32, audio, np.array([4001]), probs)       # length > buffer


def test_offline_forward_programmatic_launch_is_bitwise_equal():
    """With programmatic dependent launch (SF_OPT_PDL = 1) each GEMM loads
    its first weight tiles before waiting for the previous kernel, and the
    single-wave GEMMs run with half the operand ring so that two CTAs fit on
    an SM; the arithmetic is unchanged, so the bf16 forward is bitwise equal
    to the one with plain stream ordering (full model, 90 s clip)."""
    w = full_weights(xavier=True)
    eng = make_engine(w, 1, 17, 18, max_batch=1)
    try:
        audio, lens, _ = clip_for_config(1)
        outs = []
        for pdl in (0, 1, 0, 1):
            b.sf_set_option(eng, b.SF_OPT_PDL, pdl)
            probs = torch.full((1, 1125, 4), float("nan"), device="cuda")
            b.sf_forward_offline(eng, to_dev(audio), lens, probs)
            b.sf_check(eng)
            outs.append(probs.cpu().numpy())
    finally:
        b.sf_destroy(eng)
    assert np.all(np.isfinite(outs[1]))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


@pytest.mark.parametrize("lens_s,force", [([9.0, 4.1, 0.3], 1), ([60.0] * 6 + [41.3, 7.7], 2)])
def test_fused_transformer_layer_vs_unfused_and_oracle(lens_s, force):
    """The Transformer layers with everything after the attention in one
    kernel (cluster of four CTAs per 128-row block) against the separate
    projections and LayerNorms (same bf16 operands: within 1e-2) and against
    the oracle (2e-2), on a ragged batch whose 128-row blocks straddle
    sequences; the second case has 5,112 rows (more clusters than one wave,
    SF_OPT_TF_FUSE = 2)."""
    w = tiny_weights(xavier=True)
    audio, lens, _ = synth_batch(87, lens_s)
    B = len(lens_s)
    eng = make_engine(w, 1, 2, 2, max_batch=B)
    try:
        Tp = int(O.encoder_frames(audio.shape[1] // 160))
        outs = []
        for fuse in (force, 0):
            b.sf_set_option(eng, b.SF_OPT_TF_FUSE, fuse)
            p = torch.full((B, Tp, 4), float("nan"), device="cuda")
            b.sf_forward_offline(eng, to_dev(audio), lens, p)
            b.sf_check(eng)
            outs.append(p.cpu().numpy())
    finally:
        b.sf_destroy(eng)
    T = np.array([int(O.encoder_frames(int(n) // 160)) for n in lens])
    for i in range(B):
        assert np.all(outs[0][i, T[i]:] == 0)
    assert np.max(np.abs(outs[0] - outs[1])) <= 1e-2
    for i in (0, B - 1):
        ref, tp = O.forward_offline(audio[i:i + 1, :lens[i]], lens[i:i + 1], w)
        assert np.max(np.abs(outs[0][i, :T[i]] - ref[0])) <= 2e-2, i
