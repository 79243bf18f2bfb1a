"""Pins for the Nemotron-3 variant's oracle: closed forms, brute force and
invariants of each step (stacking, rotary embedding, attention, layers,
the transposed-conv head), with non-zero weights where the step has any."""
import math

import numpy as np
import pytest

from oracle import nemotron as N
from synth import NEM_FULL, NEM_TINY, make_nem_weights, nem_manifest


def test_stacking_order_and_count():
    L = 21
    x = np.arange(L * 3, dtype=np.float64).reshape(L, 3)       # 3 "mel bins" to read the order by eye
    s = N.stack_frames(x, stack=8)
    assert s.shape == (3, 24)                                    # ceil(21 / 8) encoder frames
    assert list(s[0, :6]) == [0, 1, 2, 3, 4, 5]                  # frame 0 then frame 1 (frame-major)
    assert list(s[1, :3]) == list(x[8])
    assert np.all(s[2, 5 * 3:] == 0) and list(s[2, :3]) == list(x[16])   # frames 21-23 past the clip
    for L in (1, 7, 8, 9, 3600):
        assert N.stack_frames(np.zeros((L, 128))).shape[0] == math.ceil(L / 8)


def test_rope_closed_forms_and_relative_position():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((6, 2, 8))
    k = rng.standard_normal((6, 2, 8))
    assert np.allclose(N.rope(q, np.zeros(6)), q)                        # position 0: identity
    # one pair (i, i + 4) at angle p * base^(-2i/8) is a plane rotation
    p, i = 5.0, 1
    th = p * 10000.0 ** (-2.0 * i / 8)
    r = N.rope(q[:1], [p])
    a, b = q[0, 0, i], q[0, 0, i + 4]
    assert np.isclose(r[0, 0, i], a * math.cos(th) - b * math.sin(th))
    assert np.isclose(r[0, 0, i + 4], b * math.cos(th) + a * math.sin(th))
    assert np.allclose(np.linalg.norm(N.rope(q, np.arange(6) * 7.0), axis=-1), np.linalg.norm(q, axis=-1))
    # scores depend only on the relative position: shifting both by c changes nothing
    pos = np.array([0, 3, 4, 9, 11, 20], np.float64)
    s0 = np.einsum("ihd,jhd->hij", N.rope(q, pos), N.rope(k, pos))
    s1 = np.einsum("ihd,jhd->hij", N.rope(q, pos + 37.0), N.rope(k, pos + 37.0))
    assert np.allclose(s0, s1, atol=1e-10)


def _small_weights(d=16, H=2, ff=24, seed=4):
    rng = np.random.default_rng(seed)
    p = "nem.layers.0."
    w = {}
    for q in ("q", "k", "v", "o"):
        w[p + f"att.{q}.weight"] = rng.standard_normal((d, d)) * 0.4
        w[p + f"att.{q}.bias"] = rng.standard_normal(d) * 0.3
    w[p + "ln1.weight"], w[p + "ln1.bias"] = 1 + 0.2 * rng.standard_normal(d), 0.1 * rng.standard_normal(d)
    w[p + "ln2.weight"], w[p + "ln2.bias"] = 1 + 0.2 * rng.standard_normal(d), 0.1 * rng.standard_normal(d)
    w[p + "ff.linear1.weight"], w[p + "ff.linear1.bias"] = rng.standard_normal((ff, d)) / 4, rng.standard_normal(ff) * 0.1
    w[p + "ff.linear2.weight"], w[p + "ff.linear2.bias"] = rng.standard_normal((d, ff)) / 5, rng.standard_normal(d) * 0.1
    return w, p


def _brute_rope_mha(x, w, p, H):
    S, d = len(x), len(x[0])
    dk = d // H
    lin = lambda n: [[sum(x[i][c] * w[p + f"att.{n}.weight"][o][c] for c in range(d)) + w[p + f"att.{n}.bias"][o]  # noqa: E731
                      for o in range(d)] for i in range(S)]
    q, k, v = lin("q"), lin("k"), lin("v")

    def rot(vec, h, pos):
        out = list(vec)
        for i in range(dk // 2):
            th = pos * 10000.0 ** (-2.0 * i / dk)
            a, b = vec[h * dk + i], vec[h * dk + i + dk // 2]
            out[h * dk + i] = a * math.cos(th) - b * math.sin(th)
            out[h * dk + i + dk // 2] = b * math.cos(th) + a * math.sin(th)
        return out
    ctx = [[0.0] * d for _ in range(S)]
    for h in range(H):
        qr = [rot(q[i], h, i) for i in range(S)]
        kr = [rot(k[j], h, j) for j in range(S)]
        for i in range(S):
            s = [sum(qr[i][h * dk + c] * kr[j][h * dk + c] for c in range(dk)) / math.sqrt(dk) for j in range(S)]
            mx = max(s)
            e = [math.exp(t - mx) for t in s]
            z = sum(e)
            for j in range(S):
                for c in range(dk):
                    ctx[i][h * dk + c] += e[j] / z * v[j][h * dk + c]
    return np.array([[sum(ctx[i][c] * w[p + "att.o.weight"][o][c] for c in range(d)) + w[p + "att.o.bias"][o]
                      for o in range(d)] for i in range(S)])


@pytest.mark.parametrize("S", [1, 2, 7])
def test_rope_attention_vs_brute_force(S, monkeypatch):
    w, p = _small_weights()
    x = np.random.default_rng(S).standard_normal((S, 16))
    out = N.rope_mha(x, w, p, H=2)
    assert np.max(np.abs(out - _brute_rope_mha(x.tolist(), w, p, 2))) < 1e-11
    if S > 1:   # a planted mistake (no rotation) must change the result: the positions matter
        monkeypatch.setattr(N, "rope", lambda t, pos, base=N.ROPE_BASE: t)
        assert np.max(np.abs(out - N.rope_mha(x, w, p, H=2))) > 1e-3


def test_pre_ln_layer_vs_loop_and_zero_weights():
    w, p = _small_weights()
    x = np.random.default_rng(11).standard_normal((5, 16)) * 2
    out = N.nem_layer(x, w, 0, H=2)
    ln = lambda t, g, b: (t - t.mean(-1, keepdims=True)) / np.sqrt(t.var(-1, keepdims=True) + 1e-5) * g + b  # noqa: E731
    a = x + _brute_rope_mha(ln(x, w[p + "ln1.weight"], w[p + "ln1.bias"]).tolist(), w, p, 2)
    hid = ln(a, w[p + "ln2.weight"], w[p + "ln2.bias"]) @ w[p + "ff.linear1.weight"].T + w[p + "ff.linear1.bias"]
    hid = hid / (1 + np.exp(-hid))
    ref = a + hid @ w[p + "ff.linear2.weight"].T + w[p + "ff.linear2.bias"]
    assert np.max(np.abs(out - ref)) < 1e-10
    z = {k: (np.zeros_like(v) if not k.endswith(("ln1.weight", "ln2.weight")) else v) for k, v in w.items()}
    assert np.max(np.abs(N.nem_layer(x, z, 0, H=2) - x)) < 1e-14     # pre-LN with zero weights: identity


def test_head_is_a_non_overlapping_transposed_conv():
    rng = np.random.default_rng(3)
    d, S, K = 6, 8, 8
    w = {"nem.head.weight": rng.standard_normal((d, S, K)), "nem.head.bias": rng.standard_normal(S)}
    x = rng.standard_normal((4, d))
    z = N.nem_head(x, w, logits=True)
    assert z.shape == (32, 8)
    for t in range(4):
        for k in range(K):
            for s in range(S):
                ref = sum(x[t, c] * w["nem.head.weight"][c, s, k] for c in range(d)) + w["nem.head.bias"][s]
                assert abs(z[8 * t + k, s] - ref) < 1e-12


def test_forward_shapes_and_parameter_count():
    assert 97e6 < sum(int(np.prod(s)) for _, s, _ in nem_manifest(NEM_FULL)) < 100e6   # "~100M parameters"
    w = make_nem_weights(NEM_TINY, xavier=True)
    from synth import synth_batch
    audio, lens, _ = synth_batch(5, [2.0, 0.73])
    p, L = N.nem_forward_offline(audio, lens, w)
    assert list(L) == [200, 73] and p.shape == (2, 200, 8)
    assert np.all(p[1, 73:] == 0) and np.all((p[:, :73] > 0) & (p[:, :73] < 1))
    assert float(p[0].max() - p[0].min()) > 0.1            # xavier weights: probabilities spread
