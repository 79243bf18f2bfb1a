"""GPU: the Transformer self-attention with four key groups per CTA
(sf_attention_mha path 2; SF_OPT_ATTN_PATH 2 in the engine) against a
float64 evaluation of the same bf16 operands, and the engine's offline
forward on that path against the oracle.  Tolerances as for the two-group
kernel: 1.5e-2 on outputs of magnitude <= ~1, 2e-2 on probabilities.

These run only with SF_TEST_NEW_PATHS=1 in the environment: the default
engine keeps two key groups until this kernel has been measured."""
import os

import numpy as np
import pytest

import oracle as O
from synth import synth_batch
from _helpers import bf16_round, make_engine, tiny_weights, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(os.environ.get("SF_TEST_NEW_PATHS") != "1",
                                 reason="kernel paths not yet default run with SF_TEST_NEW_PATHS=1")]
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

E, H, HD = 192, 8, 24
RAGGED = [1, 2, 63, 64, 65, 127, 128, 129, 191, 255, 256, 257, 322, 1125]


def _reference(qkv, lens):
    offs = np.concatenate([[0], np.cumsum(lens)])
    out = []
    for s in range(len(lens)):
        X = qkv[offs[s]:offs[s + 1]].astype(np.float64)
        res = np.zeros((len(X), E))
        for h in range(H):
            q, k = X[:, h * HD:(h + 1) * HD], X[:, E + h * HD:E + (h + 1) * HD]
            v = X[:, 2 * E + h * HD:2 * E + (h + 1) * HD]
            sc = q @ k.T / np.sqrt(HD)
            p = np.exp(sc - sc.max(axis=1, keepdims=True))
            res[:, h * HD:(h + 1) * HD] = (p / p.sum(axis=1, keepdims=True)) @ v
        out.append(res)
    return np.concatenate(out)


def test_mha_four_groups_ragged():
    eng = make_engine(tiny_weights(), 1, 2, 2, max_batch=16)
    try:
        qkv = bf16_round(np.random.default_rng(7).standard_normal((sum(RAGGED), 3 * E)).astype(np.float32))
        ctx = torch.full((sum(RAGGED), E), float("nan"), device="cuda", dtype=torch.bfloat16)
        b.sf_attention_mha(eng, torch.from_numpy(qkv).cuda().to(torch.bfloat16), np.asarray(RAGGED, np.int32), ctx,
                           path=2)
        b.sf_check(eng)
        got = ctx.float().cpu().numpy()
    finally:
        b.sf_destroy(eng)
    assert np.isfinite(got).all()
    assert np.max(np.abs(got - _reference(qkv, RAGGED))) <= 1.5e-2


def test_offline_forward_attention_path2():
    w = tiny_weights(xavier=True)
    eng = make_engine(w, 1, 2, 2)
    try:
        b.sf_set_option(eng, b.SF_OPT_ATTN_PATH, 2)
        audio, lens, _ = synth_batch(86, [14.0, 4.1])
        Tp = int(O.encoder_frames(audio.shape[1] // 160))
        probs = torch.zeros((2, Tp, 4), device="cuda")
        b.sf_forward_offline(eng, to_dev(audio), lens, probs)
        b.sf_check(eng)
        ref, tp = O.forward_offline(audio, lens, w)
        got = probs.cpu().numpy()
        for i in range(2):
            assert np.max(np.abs(got[i, :tp[i]] - ref[i, :tp[i]])) <= 2e-2, i
    finally:
        b.sf_destroy(eng)
