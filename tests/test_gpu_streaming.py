"""GPU parity of the streaming path through the C ABI.

Selection and FIFO/cache bookkeeping are compared bit-exactly given the same
scores; chunk probabilities within 1e-4 (fp32 mode) / 2e-2 (bf16 mode).
Where a free-running stream is compared with the oracle, the oracle's
decision margins (|p - 0.5|, argmax gaps, top-k score gaps) are asserted to
exceed the fp32 discrepancy, so the two runs take the same decisions."""
import numpy as np
import pytest

import oracle as O
from oracle import streaming as OS
from synth import synth_batch, synth_clip
from _helpers import (act_dtype, bf16_round, get_state, make_engine, oracle_states as _oracle_states, set_state,
                      tiny_weights, to_dev)

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402


@pytest.fixture(scope="module")
def eng32():
    e = make_engine(tiny_weights(), 0, 2, 2, max_batch=8)
    yield e
    b.sf_destroy(e)


@pytest.fixture(scope="module")
def eng32x():
    e = make_engine(tiny_weights(xavier=True), 0, 2, 2, max_batch=8)
    yield e
    b.sf_destroy(e)


@pytest.fixture(scope="module")
def eng16():
    e = make_engine(tiny_weights(), 1, 2, 2, max_batch=8)
    yield e
    b.sf_destroy(e)


@pytest.mark.parametrize("seed", range(6))
def test_select_topk_bit_exact(eng32, seed):
    rng = np.random.default_rng(seed)
    n_sets, stride, k = 5, 400, int(rng.integers(1, 60))
    n = rng.integers(0, stride + 1, size=n_sets)
    n[0] = stride
    sc = rng.standard_normal((n_sets, stride, 4)).astype(np.float32)
    sc[rng.random(sc.shape) < 0.6] = -np.inf
    sc[:, ::7] = np.round(sc[:, ::7])                      # exact ties
    sc[1, :50] = 0.25                                       # long tie run
    src = torch.zeros((n_sets, 4 * k), dtype=torch.int32, device="cuda")
    b.sf_select_topk(eng32, to_dev(sc), n, k, src)
    torch.cuda.synchronize()
    got = src.cpu().numpy()
    for i in range(n_sets):
        sel = O.select_topk(sc[i, :n[i]].astype(np.float64), k)
        ref = list(np.sort(np.concatenate(sel)).astype(int))   # a frame kept by two speakers appears twice
        for s in range(4):
            ref += [-1 - s] * (k - len(sel[s]))
        assert list(got[i]) == ref


@pytest.mark.parametrize("precision", [0, 1])
def test_bookkeeping_bit_exact_given_scores(precision, eng32, eng16):
    """Teacher-forced state update: oracle state before each step, oracle
    window predictions and new embeddings in; the GPU's scores are handed to
    the oracle's update so both select from identical scores.  Sizes, slot
    sources, cache/FIFO contents and predictions must then match exactly."""
    eng = eng32 if precision == 0 else eng16
    w = tiny_weights()
    pre = OS.Preset(6, 3, 16, 12, 24)
    a, _ = synth_clip(90, 9.0, 4)
    f, L = O.mel_features(a[None], np.array([len(a)]))
    states, taps = _oracle_states(w, f[0], int(L[0]), pre, 40)
    st = b.sf_stream_create(eng, (pre.chunk_len, pre.right_context, pre.fifo_len, pre.update_period,
                                  pre.spkcache_len), 1)
    rnd = (lambda x: x) if precision == 0 else bf16_round
    n_comp = 0
    try:
        for k, (s0, tp) in enumerate(zip(states, taps)):
            s0 = s0.copy()
            for key in ("cache_emb", "fifo_emb"):
                setattr(s0, key, rnd(getattr(s0, key).astype(np.float32)).astype(np.float64))
            for key in ("cache_preds", "fifo_preds"):
                setattr(s0, key, getattr(s0, key).astype(np.float32).astype(np.float64))
            s0.sil_mean = s0.sil_mean.astype(np.float32).astype(np.float64)
            set_state(eng, st, 0, s0, precision)
            P = tp["P"].astype(np.float32)
            new = rnd(tp["new"].astype(np.float32))
            stride = pre.spkcache_len + pre.fifo_len + pre.chunk_len
            scores = torch.full((1, stride, 4), float("nan"), device="cuda")
            src = torch.full((1, pre.spkcache_len), -99, dtype=torch.int32, device="cuda")
            b.sf_stream_update(eng, st, to_dev(P), to_dev(new[None], act_dtype(precision)), len(new), [len(new)],
                               scores, src)
            torch.cuda.synchronize()
            g = get_state(eng, st, 0, precision, pre.spkcache_len, pre.fifo_len + pre.chunk_len)
            ref = s0.copy()
            gsc = scores[0].cpu().numpy().astype(np.float64)
            nC = len(s0.cache_emb) + tp["popped"]
            info = OS.state_update(ref, P.astype(np.float64), new.astype(np.float64), tp["n_chunk"], pre,
                                   scores=gsc[:nC] if tp["compressed"] else None)
            assert (g["n_c"], g["n_f"]) == (len(ref.cache_emb), len(ref.fifo_emb)), k
            assert np.array_equal(g["cache_emb"], ref.cache_emb.astype(np.float32)), k
            assert np.array_equal(g["fifo_emb"], ref.fifo_emb.astype(np.float32)), k
            assert np.array_equal(g["cache_preds"], ref.cache_preds.astype(np.float32)), k
            assert np.array_equal(g["fifo_preds"], ref.fifo_preds.astype(np.float32)), k
            assert g["sil_count"] == ref.sil_count
            assert np.max(np.abs(g["sil_mean"] - ref.sil_mean)) <= 1e-5
            if tp["compressed"]:
                n_comp += 1
                assert list(src[0].cpu().numpy()) == list(info["src"]), k
                osc = OS.compress_scores(P.astype(np.float64)[len(s0.cache_emb):][:0])  # noqa: F841
                ref_sc = OS.compress_scores(np.concatenate([s0.cache_preds, P[len(s0.cache_emb):][:tp["popped"]]]))
                fin = np.isfinite(ref_sc)
                assert np.array_equal(fin, np.isfinite(gsc[:nC]))
                assert np.max(np.abs(gsc[:nC][fin] - ref_sc[fin])) <= 1e-5
        assert n_comp >= 3
    finally:
        b.sf_stream_destroy(st)


def _run_gpu_stream(eng, preset, feats, L, n_steps=None):
    n = feats.shape[0]
    st = b.sf_stream_create(eng, preset, n)
    out = [[] for _ in range(n)]
    cp = torch.zeros((n, preset[0], 4), device="cuda")
    fd = to_dev(feats)
    steps = 0
    try:
        while True:
            active = [i for i in range(n) if sum(len(o) for o in out[i]) < 1 + (L[i] - 1) // 8]
            if not active or (n_steps is not None and steps >= n_steps):
                break
            n_out = b.sf_stream_step(eng, st, fd, np.zeros(n, np.int64), L, cp)
            torch.cuda.synchronize()
            c = cp.cpu().numpy()
            for i in range(n):
                out[i].append(c[i, :n_out[i]])
                assert np.all(c[i, n_out[i]:] == 0)
            steps += 1
        return [np.concatenate(o) for o in out], st
    except Exception:
        b.sf_stream_destroy(st)
        raise


def test_stream_fp32_free_running_matches_oracle(eng32x):
    """Two streams of different lengths, small preset with several cache
    compressions; every emitted frame within 1e-4, final states equal.
    Xavier-scaled weights spread the probabilities over [0, 1], so every
    threshold/argmax/top-k decision sits well clear of fp32 rounding (the
    margin is asserted: the GPU's fp32 error is ~1e-7)."""
    eng32 = eng32x
    w = tiny_weights(xavier=True)
    pre = OS.Preset(6, 3, 16, 12, 24)
    audio, lens, _ = synth_batch(91, [11.0, 7.3], n_spk_choices=(4,))
    feats, L = O.mel_features(audio, lens)
    got, st = _run_gpu_stream(eng32, (6, 3, 16, 12, 24), feats.astype(np.float32), L)
    try:
        for i in range(2):
            taps = []
            ref, ost = O.stream_run(feats[i], int(L[i]), w, pre, taps=taps)
            margin = min(t["margin"] for t in taps)
            assert margin > 2e-6, margin            # decisions are far from fp32 noise
            assert got[i].shape == ref.shape
            assert np.max(np.abs(got[i] - ref)) <= 1e-4
            g = get_state(eng32, st, i, 0, 24, 22)
            assert (g["n_c"], g["n_f"], g["c0"]) == (len(ost.cache_emb), len(ost.fifo_emb), ost.c0)
            assert g["finished"] == 1
            assert np.max(np.abs(g["cache_preds"] - ost.cache_preds)) <= 1e-4
            assert np.max(np.abs(g["cache_emb"] - ost.cache_emb)) <= 1e-4
    finally:
        b.sf_stream_destroy(st)


def test_single_chunk_stream_equals_offline(eng32):
    """A clip shorter than one chunk (Very high preset): the step's output
    is the offline forward's, bit for bit."""
    audio, lens, _ = synth_batch(92, [2.0])
    feats, L = O.mel_features(audio, lens)
    got, st = _run_gpu_stream(eng32, (340, 40, 40, 300, 188), feats.astype(np.float32), L)
    b.sf_stream_destroy(st)
    probs = torch.zeros((1, 25, 4), device="cuda")
    # the offline path through the engine's own front-end
    b.sf_forward_offline(eng32, to_dev(audio), lens, probs)
    torch.cuda.synchronize()
    ref_off = probs.cpu().numpy()[0]
    # compare through the oracle (features differ only by fp32 rounding) and exactly against sf_encode
    assert np.max(np.abs(got[0] - ref_off)) <= 1e-4
    emb = torch.zeros((1, 25, 512), device="cuda")
    b.sf_pre_encode(eng32, to_dev(feats), [0], [0], [int(L[0])], emb, 25)
    pr = torch.zeros((25, 4), device="cuda")
    b.sf_encode(eng32, emb[0].contiguous(), [25], pr)
    torch.cuda.synchronize()
    assert np.array_equal(got[0], pr.cpu().numpy())


def test_reset_replays_bit_identically(eng32):
    audio, lens, _ = synth_batch(93, [6.0])
    feats, L = O.mel_features(audio, lens)
    pre = (4, 2, 10, 6, 12)
    n = feats.shape[0]
    st = b.sf_stream_create(eng32, pre, n)
    fd = to_dev(feats)
    cp = torch.zeros((n, 4, 4), device="cuda")
    try:
        runs = []
        for _ in range(2):
            outs = []
            for _ in range(18):               # 6 s -> 75 frames -> 19 chunks of 4
                b.sf_stream_step(eng32, st, fd, [0], L, cp)
                outs.append(cp.cpu().numpy().copy())
            runs.append(np.stack(outs))
            b.sf_stream_reset(st)
        assert np.array_equal(runs[0], runs[1])
    finally:
        b.sf_stream_destroy(st)


def test_stream_bf16_teacher_forced_low_preset(eng16):
    """Low preset (6/7/188/144/188) at full state sizes, bf16: each step
    starts from the oracle's state; chunk probabilities within 2e-2."""
    w = tiny_weights()
    pre = O.PRESETS["low"]
    a, _ = synth_clip(94, 40.0, 3)
    f, L = O.mel_features(a[None], np.array([len(a)]))
    L = int(L[0])
    states, taps = _oracle_states(w, f[0], L, pre, 60)
    st = b.sf_stream_create(eng16, (6, 7, 188, 144, 188), 1)
    fd = to_dev(f.astype(np.float32))
    cp = torch.zeros((1, 6, 4), device="cuda")
    try:
        for k in list(range(0, 60, 7)) + [31, 55, 56]:
            if k >= len(states):
                continue
            set_state(eng16, st, 0, states[k], 1)
            n_out = b.sf_stream_step(eng16, st, fd, [0], [L], cp)
            torch.cuda.synchronize()
            ref = taps[k]["P"][taps[k]["n_c"] + taps[k]["n_f"]:][:taps[k]["n_chunk"]]
            assert n_out[0] == len(ref)
            assert np.max(np.abs(cp.cpu().numpy()[0, :n_out[0]] - ref)) <= 2e-2, k
            g = get_state(eng16, st, 0, 1, 188, 194)
            assert (g["n_c"], g["n_f"]) == (len(states[k + 1].cache_emb), len(states[k + 1].fifo_emb))
    finally:
        b.sf_stream_destroy(st)


def test_stream_errors(eng32):
    st = b.sf_stream_create(eng32, (6, 7, 188, 144, 188), 1)
    try:
        f = to_dev(np.zeros((1, 128, 20), np.float32))
        cp = torch.zeros((1, 6, 4), device="cuda")
        with pytest.raises(b.SFError, match="SF_ESHAPE"):
            b.sf_stream_step(eng32, st, f, [0], [200], cp)   # window beyond the buffer
        with pytest.raises(b.SFError):
            b.sf_stream_create(eng32, (6, 7, 188, 144, 190), 1)   # cache length not a multiple of 4
    finally:
        b.sf_stream_destroy(st)
