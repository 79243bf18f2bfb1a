"""GPU: the relative-position self-attention alone (sf_attention_relpos), the
tcgen05 kernel and the mma.sync kernel, against a float64 evaluation of the
same bf16 operands ("Streaming Sortformer Diarizer" model card: FastConformer
relative-position MHSA, d_model 512, 8 heads of 64):

    out_i = sum_j softmax_j(((q_i + u) . k_j + (q_i + v) . p_(i-j)) / 8) v_j

q + u and q + v are rounded to bf16 as the kernels feed them to the tensor
cores.  Both kernels also round the softmax weights to bf16 for P.V and the
output to bf16: |error| <= ~2^-8 relative to max |v| bounds both; the test
uses 1.5e-2 absolute on outputs of magnitude <= ~1."""
import numpy as np
import pytest

from _helpers import bf16_round, make_engine, tiny_weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

D, H, HD = 512, 8, 64


@pytest.fixture(scope="module")
def eng():
    e = make_engine(tiny_weights(), 1, 2, 2, max_batch=64)
    yield e
    b.sf_destroy(e)


def _inputs(seed, lens, R):
    rng = np.random.default_rng(seed)
    M = int(sum(lens))
    qkv = bf16_round(rng.standard_normal((M, 3 * D)).astype(np.float32))
    ptab = bf16_round(rng.standard_normal((2 * R - 1, D)).astype(np.float32))
    u = (0.5 * rng.standard_normal(D)).astype(np.float32)
    v = (0.5 * rng.standard_normal(D)).astype(np.float32)
    return qkv, ptab, u, v


def _reference(qkv, ptab, R, u, v, lens, seqs):
    """Rows of the sequences in `seqs` (float64, brute force per head)."""
    offs = np.concatenate([[0], np.cumsum(lens)])
    out = {}
    for s in seqs:
        L, o0 = int(lens[s]), int(offs[s])
        X = qkv[o0:o0 + L].astype(np.float64)
        res = np.zeros((L, D))
        idx = np.arange(L)[:, None] - np.arange(L)[None, :] + R - 1
        for h in range(H):
            c = slice(h * HD, (h + 1) * HD)
            q = X[:, c]
            k = X[:, D + h * HD:D + (h + 1) * HD]
            vv = X[:, 2 * D + h * HD:2 * D + (h + 1) * HD]
            qu = bf16_round((q + u[c]).astype(np.float32)).astype(np.float64)
            qv = bf16_round((q + v[c]).astype(np.float32)).astype(np.float64)
            bd_all = qv @ ptab[:, c].astype(np.float64).T          # (L, 2R - 1)
            bd = np.take_along_axis(bd_all, idx, axis=1)
            sc = (qu @ k.T + bd) / 8.0
            sc -= sc.max(axis=1, keepdims=True)
            p = np.exp(sc)
            p /= p.sum(axis=1, keepdims=True)
            res[:, c] = p @ vv
        out[s] = res
    return out


def _run(eng, qkv, ptab, R, u, v, lens, path):
    M = int(sum(lens))
    ctx = torch.full((M, D), float("nan"), device="cuda", dtype=torch.bfloat16)
    b.sf_attention_relpos(eng, torch.from_numpy(qkv).cuda().to(torch.bfloat16),
                          torch.from_numpy(ptab).cuda().to(torch.bfloat16), R, torch.from_numpy(u).cuda(),
                          torch.from_numpy(v).cuda(), np.asarray(lens, np.int32), ctx, path=path)
    b.sf_check(eng)
    return ctx.float().cpu().numpy()


# ragged lengths around the 64-key and 128-query tile sizes, a one-key
# sequence, a streaming window (322) and a long offline sequence (1125)
RAGGED = [1, 2, 63, 64, 65, 127, 128, 129, 191, 322, 1125]


@pytest.mark.parametrize("path", [1, 0])
def test_relpos_attention_ragged(eng, path):
    R = 1200
    qkv, ptab, u, v = _inputs(5, RAGGED, R)
    got = _run(eng, qkv, ptab, R, u, v, RAGGED, path)
    assert np.isfinite(got).all()
    ref = _reference(qkv, ptab, R, u, v, RAGGED, range(len(RAGGED)))
    offs = np.concatenate([[0], np.cumsum(RAGGED)])
    for s in range(len(RAGGED)):
        err = np.max(np.abs(got[offs[s]:offs[s + 1]] - ref[s]))
        assert err <= 1.5e-2, (RAGGED[s], err)


def test_relpos_attention_streaming_batch(eng):
    """64 windows of 322 frames (the Low-preset streaming step, M = 20608):
    sampled windows against float64, all windows tcgen05 vs mma.sync."""
    lens = [322] * 64
    R = 756
    qkv, ptab, u, v = _inputs(6, lens, R)
    got = _run(eng, qkv, ptab, R, u, v, lens, 1)
    ref = _reference(qkv, ptab, R, u, v, lens, [0, 31, 63])
    for s in (0, 31, 63):
        assert np.max(np.abs(got[322 * s:322 * (s + 1)] - ref[s])) <= 1.5e-2, s
    other = _run(eng, qkv, ptab, R, u, v, lens, 0)
    assert np.max(np.abs(got - other)) <= 2e-2


def test_relpos_attention_rejects_bad_input(eng):
    qkv, ptab, u, v = _inputs(7, [10], 16)
    with pytest.raises(b.SFError):
        _run(eng, qkv, ptab, 16, u, v, [17], 1)      # longer than R
    with pytest.raises(b.SFError):
        _run(eng, qkv, ptab, 16, u, v, [10], 2)      # unknown path


@pytest.mark.parametrize("L", [1125, 300, 100, 65])
def test_relpos_attention_key_split(eng, L):
    """One sequence: fewer (query tile, head) units than SMs, so each unit's
    keys are split over up to 4 CTAs (1125: 2 splits of 9 key tiles; 300: 4
    splits over 5 tiles; 100 and 65: 2 splits of one tile) and the partial
    softmax states are merged by the last CTA."""
    R = 1200
    qkv, ptab, u, v = _inputs(11 + L, [L], R)
    got = _run(eng, qkv, ptab, R, u, v, [L], 1)
    ref = _reference(qkv, ptab, R, u, v, [L], [0])[0]
    assert np.max(np.abs(got - ref)) <= 1.5e-2
    again = _run(eng, qkv, ptab, R, u, v, [L], 1)
    assert np.array_equal(got, again)            # merge order fixed: bitwise repeatable
