"""GPU: the Transformer encoder's self-attention alone (sf_attention_mha),
tcgen05 kernel and mma.sync kernel, against a float64 evaluation of the same
bf16 operands ("Streaming Sortformer Diarizer" model card: 18-layer
Transformer, d_model 192, 8 heads of 24):

    out_i = sum_j softmax_j(q_i . k_j / sqrt(24)) v_j

Both kernels round the softmax weights to bf16 for P.V and the output to
bf16; 1.5e-2 absolute on outputs of magnitude <= ~1."""
import numpy as np
import pytest

from _helpers import bf16_round, make_engine, tiny_weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

E, H, HD = 192, 8, 24


@pytest.fixture(scope="module")
def eng():
    e = make_engine(tiny_weights(), 1, 2, 2, max_batch=64)
    yield e
    b.sf_destroy(e)


def _inputs(seed, lens):
    rng = np.random.default_rng(seed)
    return bf16_round(rng.standard_normal((int(sum(lens)), 3 * E)).astype(np.float32))


def _reference(qkv, lens, seqs):
    offs = np.concatenate([[0], np.cumsum(lens)])
    out = {}
    for s in seqs:
        X = qkv[offs[s]:offs[s + 1]].astype(np.float64)
        res = np.zeros((len(X), E))
        for h in range(H):
            q = X[:, h * HD:(h + 1) * HD]
            k = X[:, E + h * HD:E + (h + 1) * HD]
            v = X[:, 2 * E + h * HD:2 * E + (h + 1) * HD]
            sc = q @ k.T / np.sqrt(HD)
            sc -= sc.max(axis=1, keepdims=True)
            p = np.exp(sc)
            p /= p.sum(axis=1, keepdims=True)
            res[:, h * HD:(h + 1) * HD] = p @ v
        out[s] = res
    return out


def _run(eng, qkv, lens, path):
    ctx = torch.full((int(sum(lens)), E), float("nan"), device="cuda", dtype=torch.bfloat16)
    b.sf_attention_mha(eng, torch.from_numpy(qkv).cuda().to(torch.bfloat16), np.asarray(lens, np.int32), ctx, path=path)
    b.sf_check(eng)
    return ctx.float().cpu().numpy()


RAGGED = [1, 2, 63, 64, 65, 127, 128, 129, 191, 322, 1125]


@pytest.mark.parametrize("path", [1, 0])
def test_mha_ragged(eng, path):
    qkv = _inputs(3, RAGGED)
    got = _run(eng, qkv, RAGGED, path)
    assert np.isfinite(got).all()
    ref = _reference(qkv, RAGGED, range(len(RAGGED)))
    offs = np.concatenate([[0], np.cumsum(RAGGED)])
    for s in range(len(RAGGED)):
        err = np.max(np.abs(got[offs[s]:offs[s + 1]] - ref[s]))
        assert err <= 1.5e-2, (RAGGED[s], err)


def test_mha_streaming_batch(eng):
    """64 windows of 322 frames (the Low-preset streaming step): sampled
    windows against float64, all windows tcgen05 vs mma.sync."""
    lens = [322] * 64
    qkv = _inputs(4, lens)
    got = _run(eng, qkv, lens, 1)
    ref = _reference(qkv, lens, [0, 40, 63])
    for s in (0, 40, 63):
        assert np.max(np.abs(got[322 * s:322 * (s + 1)] - ref[s])) <= 1.5e-2, s
    assert np.max(np.abs(got - _run(eng, qkv, lens, 0))) <= 2e-2


@pytest.mark.parametrize("lens", [[1125], [1, 65, 700, 3], [129, 1500]])
def test_mha_key_split(eng, lens):
    """Few (query tile, head) units: the tcgen05 kernel splits each unit's
    keys over a cluster of CTAs (4 for one 1125-frame clip) and merges them;
    sequences shorter than the split leave some CTAs without key tiles.
    Against float64, bitwise repeatable, and close to the mma.sync kernel."""
    qkv = _inputs(5, lens)
    got = _run(eng, qkv, lens, 1)
    assert np.isfinite(got).all()
    ref = _reference(qkv, lens, range(len(lens)))
    offs = np.concatenate([[0], np.cumsum(lens)])
    for s in range(len(lens)):
        err = np.max(np.abs(got[offs[s]:offs[s + 1]] - ref[s]))
        assert err <= 1.5e-2, (lens[s], err)
    assert np.array_equal(got, _run(eng, qkv, lens, 1))
    assert np.max(np.abs(got - _run(eng, qkv, lens, 0))) <= 2e-2
