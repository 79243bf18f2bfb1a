"""Pins for the oracle's encoder layers: closed forms, brute force, and an
independent re-derivation of the relative-position shift."""
import math

import numpy as np
import pytest
import scipy.signal
import scipy.special

import oracle as O
from oracle import model as M
from synth import TINY, make_weights


def _zero_like(w):
    z = {}
    for k, v in w.items():
        if k.endswith(("ln.weight", "ln1.weight", "ln2.weight", "out_ln.weight", "bn.running_var", "bn.weight")):
            z[k] = np.ones_like(v)
        else:
            z[k] = np.zeros_like(v)
    return z


def _brute_rel_attention(x, w, p, H):
    """Pure-loop rel-pos attention with the sinusoid recomputed per (i, j)."""
    S, d = x.shape
    dk = d // H
    Wq, bq = w[p + "att.linear_q.weight"], w[p + "att.linear_q.bias"]
    Wk, bk = w[p + "att.linear_k.weight"], w[p + "att.linear_k.bias"]
    Wv, bv = w[p + "att.linear_v.weight"], w[p + "att.linear_v.bias"]
    Wp = w[p + "att.linear_pos.weight"]
    u, vb = w[p + "att.pos_bias_u"], w[p + "att.pos_bias_v"]
    q = [[sum(x[i][c] * Wq[o][c] for c in range(d)) + bq[o] for o in range(d)] for i in range(S)]
    k = [[sum(x[i][c] * Wk[o][c] for c in range(d)) + bk[o] for o in range(d)] for i in range(S)]
    v = [[sum(x[i][c] * Wv[o][c] for c in range(d)) + bv[o] for o in range(d)] for i in range(S)]

    def pos(r):
        pe = [0.0] * d
        for m in range(d // 2):
            a = r * 10000.0 ** (-2.0 * m / d)
            pe[2 * m], pe[2 * m + 1] = np.sin(a), np.cos(a)
        return [sum(pe[c] * Wp[o][c] for c in range(d)) for o in range(d)]

    ctx = [[0.0] * d for _ in range(S)]
    for h in range(H):
        for i in range(S):
            s = []
            for j in range(S):
                pr = pos(i - j)
                ac = sum((q[i][h * dk + c] + u[h][c]) * k[j][h * dk + c] for c in range(dk))
                bd = sum((q[i][h * dk + c] + vb[h][c]) * pr[h * dk + c] for c in range(dk))
                s.append((ac + bd) / np.sqrt(dk))
            mx = max(s)
            e = [np.exp(t - mx) for t in s]
            z = sum(e)
            for j in range(S):
                for c in range(dk):
                    ctx[i][h * dk + c] += e[j] / z * v[j][h * dk + c]
    Wo, bo = w[p + "att.linear_out.weight"], w[p + "att.linear_out.bias"]
    return np.array([[sum(ctx[i][c] * Wo[o][c] for c in range(d)) + bo[o] for o in range(d)] for i in range(S)])


def _small_att_weights(d=16, H=2, seed=3):
    rng = np.random.default_rng(seed)
    p = "enc.layers.0."
    w = {}
    for q in ("q", "k", "v", "out"):
        w[p + f"att.linear_{q}.weight"] = rng.standard_normal((d, d)) * 0.3
        w[p + f"att.linear_{q}.bias"] = rng.standard_normal(d) * 0.3
    w[p + "att.linear_pos.weight"] = rng.standard_normal((d, d)) * 0.3
    w[p + "att.pos_bias_u"] = rng.standard_normal((H, d // H)) * 0.3
    w[p + "att.pos_bias_v"] = rng.standard_normal((H, d // H)) * 0.3
    return w, p


@pytest.mark.parametrize("S", [1, 2, 5, 8])
def test_rel_pos_attention_vs_brute_force(S):
    w, p = _small_att_weights()
    x = np.random.default_rng(S).standard_normal((S, 16))
    out = M.rel_pos_mhsa(x, w, p, H=2)
    ref = _brute_rel_attention(x, w, p, H=2)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_rel_shift_by_pad_and_view_equals_i_minus_j():
    """The page's rel_shift (pad one zero column, view as (2S, S) over the
    pe rows ordered r = S-1 .. -(S-1), drop a row, view back, keep S
    columns) selects relative distance r = i - j for score (i, j)."""
    S = 7
    rng = np.random.default_rng(1)
    # bd_desc[i, c] is the score of query i against relative position r = S-1-c
    bd_desc = rng.standard_normal((S, 2 * S - 1))
    padded = np.concatenate([np.zeros((S, 1)), bd_desc], axis=1)       # (S, 2S)
    shifted = padded.reshape(2 * S, S)[1:].reshape(S, 2 * S - 1)[:, :S]
    for i in range(S):
        for j in range(S):
            c = S - 1 - (i - j)
            assert shifted[i, j] == bd_desc[i, c]


def test_rel_pos_table_rows():
    pe = M.rel_pos_table(5, 8)
    assert pe.shape == (9, 8)
    assert np.allclose(pe[4], [0, 1, 0, 1, 0, 1, 0, 1])              # r = 0
    assert np.allclose(pe[:, 0::2] ** 2 + pe[:, 1::2] ** 2, 1.0)
    assert np.allclose(pe[4 + 3, 0], np.sin(3.0))                    # r = 3, m = 0
    assert np.allclose(pe[4 - 2, 2], np.sin(-2.0 * 10000 ** (-2 / 8)))


def test_single_frame_attention_is_value_path():
    w, p = _small_att_weights()
    x = np.random.default_rng(9).standard_normal((1, 16))
    out = M.rel_pos_mhsa(x, w, p, H=2)
    v = x @ w[p + "att.linear_v.weight"].T + w[p + "att.linear_v.bias"]
    ref = v @ w[p + "att.linear_out.weight"].T + w[p + "att.linear_out.bias"]
    assert np.max(np.abs(out - ref)) < 1e-13


def test_softmax_rows_sum_to_one_and_zero_pos_reduces_to_sdpa():
    w, p = _small_att_weights()
    x = np.random.default_rng(4).standard_normal((6, 16))
    _, probs = M.rel_pos_mhsa(x, w, p, H=2, return_probs=True)
    for a in probs:
        assert np.allclose(a.sum(axis=1), 1.0, atol=1e-14)
    w0 = dict(w)
    w0[p + "att.linear_pos.weight"] = np.zeros((16, 16))
    w0[p + "att.pos_bias_u"] = np.zeros((2, 8))
    w0[p + "att.pos_bias_v"] = np.zeros((2, 8))
    out = M.rel_pos_mhsa(x, w0, p, H=2)
    q = (x @ w[p + "att.linear_q.weight"].T + w[p + "att.linear_q.bias"]).reshape(6, 2, 8)
    k = (x @ w[p + "att.linear_k.weight"].T + w[p + "att.linear_k.bias"]).reshape(6, 2, 8)
    v = (x @ w[p + "att.linear_v.weight"].T + w[p + "att.linear_v.bias"]).reshape(6, 2, 8)
    ctx = np.concatenate([scipy.special.softmax(q[:, h] @ k[:, h].T / np.sqrt(8), axis=1) @ v[:, h] for h in range(2)], 1)
    ref = ctx @ w[p + "att.linear_out.weight"].T + w[p + "att.linear_out.bias"]
    assert np.max(np.abs(out - ref)) < 1e-13


def test_zero_weight_layers_closed_forms(tiny_weights):
    z = _zero_like(tiny_weights)
    x = np.random.default_rng(2).standard_normal((9, 512)) * 2 + 0.5
    ln = lambda t: (t - t.mean(-1, keepdims=True)) / np.sqrt(t.var(-1, keepdims=True) + 1e-5)  # noqa: E731
    assert np.max(np.abs(M.conformer_layer(x, z, 0) - ln(x))) < 1e-12
    y = np.random.default_rng(3).standard_normal((9, 192))
    assert np.max(np.abs(M.transformer_layer(y, z, 0) - ln(ln(y)))) < 1e-12
    zh = dict(z)
    zh["head.fc2.bias"] = np.array([0.3, -1.0, 0.0, 2.0])
    assert np.allclose(M.head(y, zh), 1 / (1 + np.exp(-zh["head.fc2.bias"]))[None, :], atol=1e-15)


def test_subsampling_vs_scipy_correlate(tiny_weights):
    """Independent restatement: scipy 2-D cross-correlation per channel,
    stride 2 by slicing, masking by running on the valid rows only."""
    w = tiny_weights
    rng = np.random.default_rng(8)
    L = 37
    x = rng.standard_normal((L, 128))
    p = "enc.pre_encode."

    def conv(inp, k):
        full = scipy.signal.correlate2d(np.pad(inp, 1), k, mode="valid")
        return full[::2, ::2]

    c1 = np.stack([conv(x, w[p + "conv1.weight"][c, 0]) + w[p + "conv1.bias"][c] for c in range(256)], -1)
    h = np.maximum(c1, 0)
    for s in (1, 2):
        d = np.stack([conv(h[:, :, c], w[p + f"dw{s}.weight"][c, 0]) + w[p + f"dw{s}.bias"][c] for c in range(256)], -1)
        h = np.maximum(np.einsum("tfc,oc->tfo", d, w[p + f"pw{s}.weight"]) + w[p + f"pw{s}.bias"], 0)
    T3 = h.shape[0]
    assert T3 == int(O.encoder_frames(L)) and h.shape[1] == 16
    flat = np.stack([h[t].T.reshape(-1) for t in range(T3)])          # torch order: c * 16 + f
    ref = flat @ w[p + "out.weight"].T + w[p + "out.bias"]
    out = M.subsample(x, w)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_conv_module_depthwise_vs_numpy_convolve(tiny_weights_xavier):
    """Depthwise conv (k=9, zero pad 4) against numpy.convolve per channel."""
    w = tiny_weights_xavier
    p = "enc.layers.1.conv."
    rng = np.random.default_rng(12)
    x = rng.standard_normal((13, 512))
    out = M._conv_module(x, w, p, np.float64)
    h = x @ w[p + "pointwise1.weight"].T + w[p + "pointwise1.bias"]
    g = h[:, :512] / (1 + np.exp(-h[:, 512:]))
    c = np.stack([np.convolve(g[:, ch], w[p + "depthwise.weight"][ch][::-1], mode="same") for ch in range(512)], 1)
    c = (c + w[p + "depthwise.bias"]) / np.sqrt(1 + 1e-5)
    c = c / (1 + np.exp(-c))
    ref = c @ w[p + "pointwise2.weight"].T + w[p + "pointwise2.bias"]
    assert np.max(np.abs(out - ref)) < 1e-12


def test_fp32_oracle_close_to_fp64(tiny_weights):
    from synth import clip_for_config
    a, ln, _ = clip_for_config(0)
    p64, _ = O.forward_offline(a, ln, tiny_weights)
    p32, _ = O.forward_offline(a, ln, tiny_weights, dt=np.float32)
    assert np.max(np.abs(p64 - p32)) < 1e-5


def test_parameter_count_matches_117m():
    w = make_weights(TINY)
    per_conf = sum(v.size for k, v in w.items() if k.startswith("enc.layers.0."))
    per_tf = sum(v.size for k, v in w.items() if k.startswith("tf.layers.0."))
    rest = sum(v.size for k, v in w.items() if not k.startswith(("enc.layers.", "tf.layers.")))
    total = 17 * per_conf + 18 * per_tf + rest
    # "Speaker diarization model (117M params)"; ~470 MB fp32 export
    assert 116.5e6 < total < 118.5e6
    assert abs(total * 4 / 1e6 - 470) < 5


# --------------------------------------------------------------------------
# Transformer layer and macaron FFN with non-zero weights.  The model is the
# "Streaming Sortformer Diarizer" page's Pipeline: an 18-layer Transformer of
# width 192 with 8 heads (head size 24) after Linear 512->192; post-LN with a
# ReLU FFN 192->768->192 (the workload's "post-LN Transformer layers").

def _tf_weights(seed=21, e=192, ff=768, scale=0.15):
    """Non-zero weights for one Transformer layer, strong enough that every
    softmax row is far from uniform (score spread of several units)."""
    rng = np.random.default_rng(seed)
    p = "tf.layers.0."
    w = {}
    for q in ("q", "k", "v", "o"):
        w[p + f"att.{q}.weight"] = rng.standard_normal((e, e)) * scale
        w[p + f"att.{q}.bias"] = rng.standard_normal(e) * scale
    w[p + "ff.linear1.weight"] = rng.standard_normal((ff, e)) * (1 / np.sqrt(e))
    w[p + "ff.linear1.bias"] = rng.standard_normal(ff) * 0.1
    w[p + "ff.linear2.weight"] = rng.standard_normal((e, ff)) * (1 / np.sqrt(ff))
    w[p + "ff.linear2.bias"] = rng.standard_normal(e) * 0.1
    for ln in ("ln1", "ln2"):
        w[p + f"{ln}.weight"] = 1 + 0.2 * rng.standard_normal(e)
        w[p + f"{ln}.bias"] = 0.2 * rng.standard_normal(e)
    return w, p


def _loop_linear(x, Wm, b):
    return [[sum(row[c] * Wm[o][c] for c in range(len(row))) + b[o] for o in range(len(b))] for row in x]


def _brute_mha(x, w, p, H, scale_dim=None, head_cols=None):
    """Pure-loop multi-head attention: head h uses feature columns
    head_cols(h, c) (default h * dk + c), scores divided by sqrt(scale_dim)
    (default the head size).  The two options only exist so the pins below
    can show that a wrong scale or head split would be caught."""
    S, e = len(x), len(x[0])
    dk = e // H
    scale_dim = dk if scale_dim is None else scale_dim
    col = head_cols or (lambda h, c: h * dk + c)
    q = _loop_linear(x, w[p + "q.weight"], w[p + "q.bias"])
    k = _loop_linear(x, w[p + "k.weight"], w[p + "k.bias"])
    v = _loop_linear(x, w[p + "v.weight"], w[p + "v.bias"])
    ctx = [[0.0] * e for _ in range(S)]
    for h in range(H):
        for i in range(S):
            s = [sum(q[i][col(h, c)] * k[j][col(h, c)] for c in range(dk)) / math.sqrt(scale_dim) for j in range(S)]
            mx = max(s)
            ex = [math.exp(t - mx) for t in s]
            z = sum(ex)
            for j in range(S):
                for c in range(dk):
                    ctx[i][col(h, c)] += ex[j] / z * v[j][col(h, c)]
    return np.array(_loop_linear(ctx, w[p + "o.weight"], w[p + "o.bias"]))


def _loop_layer_norm(row, g, b, eps=1e-5):
    n = len(row)
    mu = sum(row) / n
    var = sum((t - mu) ** 2 for t in row) / n
    return [(row[c] - mu) / math.sqrt(var + eps) * g[c] + b[c] for c in range(n)]


@pytest.mark.parametrize("S", [1, 3, 8])
def test_transformer_mha_vs_brute_force(S):
    w, p = _tf_weights()
    x = np.random.default_rng(30 + S).standard_normal((S, 192))
    out = M._mha(x, w, p + "att.", 8, np.float64)
    ref = _brute_mha(x.tolist(), w, p + "att.", 8)
    assert np.max(np.abs(out - ref)) < 1e-10
    if S > 1:
        # planted mistakes the comparison must see: scale 1/sqrt(192) instead
        # of 1/sqrt(24), and heads taken as interleaved columns c * H + h
        wrong_scale = _brute_mha(x.tolist(), w, p + "att.", 8, scale_dim=192)
        wrong_split = _brute_mha(x.tolist(), w, p + "att.", 8, head_cols=lambda h, c: c * 8 + h)
        assert np.max(np.abs(out - wrong_scale)) > 1e-2
        assert np.max(np.abs(out - wrong_split)) > 1e-2


def test_transformer_mha_is_rel_pos_mhsa_without_positions():
    """With linear_pos, pos_bias_u and pos_bias_v zero, the conformer's
    relative-position attention (pinned against brute force above) is plain
    scaled dot-product attention: the Transformer's MHA must equal it."""
    w, p = _tf_weights(seed=5)
    q = "enc.layers.0."
    wr = {}
    for a, b in (("q", "q"), ("k", "k"), ("v", "v"), ("out", "o")):
        wr[q + f"att.linear_{a}.weight"] = w[p + f"att.{b}.weight"]
        wr[q + f"att.linear_{a}.bias"] = w[p + f"att.{b}.bias"]
    wr[q + "att.linear_pos.weight"] = np.zeros((192, 192))
    wr[q + "att.pos_bias_u"] = np.zeros((8, 24))
    wr[q + "att.pos_bias_v"] = np.zeros((8, 24))
    x = np.random.default_rng(6).standard_normal((11, 192))
    out = M._mha(x, w, p + "att.", 8, np.float64)
    ref = M.rel_pos_mhsa(x, wr, q, 8)
    assert np.max(np.abs(out - ref)) < 1e-12
    _, probs = M.rel_pos_mhsa(x, wr, q, 8, return_probs=True)
    assert min(float(a.max()) for a in probs) > 0.3     # attention far from uniform (1/11)


@pytest.mark.parametrize("S", [1, 4])
def test_transformer_layer_vs_loop_post_ln(S):
    """Post-LN order written out with loops: y = LN1(x + MHA(x)),
    out = LN2(y + W2 relu(W1 y + b1) + b2)."""
    w, p = _tf_weights(seed=9)
    x = np.random.default_rng(40 + S).standard_normal((S, 192))
    out = M.transformer_layer(x, w, 0)
    a = _brute_mha(x.tolist(), w, p + "att.", 8)
    y = [_loop_layer_norm([x[i][c] + a[i][c] for c in range(192)], w[p + "ln1.weight"], w[p + "ln1.bias"])
         for i in range(S)]
    h = [[max(t, 0.0) for t in row] for row in _loop_linear(y, w[p + "ff.linear1.weight"], w[p + "ff.linear1.bias"])]
    f = _loop_linear(h, w[p + "ff.linear2.weight"], w[p + "ff.linear2.bias"])
    ref = np.array([_loop_layer_norm([y[i][c] + f[i][c] for c in range(192)], w[p + "ln2.weight"], w[p + "ln2.bias"])
                    for i in range(S)])
    assert np.max(np.abs(out - ref)) < 1e-10
    # pre-LN (LN before each sublayer) is a different layer: must not match
    pre = x + M._mha(M.layer_norm(x, w[p + "ln1.weight"], w[p + "ln1.bias"]), w, p + "att.", 8, np.float64)
    assert np.max(np.abs(out - pre)) > 1e-2


def test_macaron_ffn_half_step_and_swish(tiny_weights_xavier):
    """A conformer layer whose attention and conv module have zero weights
    (their residual branches add their output biases, zero here) and whose
    second FFN is zero reduces to LN(x + FFN1(LN(x)) / 2) with
    FFN(h) = W2 swish(W1 h + b1) + b2; the FFN is written out with loops."""
    w = dict(tiny_weights_xavier)
    p = "enc.layers.0."
    for k in list(w):
        if k.startswith(p) and (".att." in k or ".conv." in k or ".ff2." in k) and not k.endswith(
                ("ln.weight", "ln.bias", "bn.running_var", "bn.weight")):
            w[k] = np.zeros_like(w[k])
    rng = np.random.default_rng(13)
    x = rng.standard_normal((3, 512))
    out = M.conformer_layer(x, w, 0)
    g1 = np.ones(512)
    z1 = np.zeros(512)
    ln_x = [_loop_layer_norm(list(r), g1, z1) for r in x]
    h = _loop_linear(ln_x, w[p + "ff1.linear1.weight"], w[p + "ff1.linear1.bias"])
    h = [[t / (1 + math.exp(-t)) for t in row] for row in h]
    f = _loop_linear(h, w[p + "ff1.linear2.weight"], w[p + "ff1.linear2.bias"])
    ref = np.array([_loop_layer_norm([x[i][c] + 0.5 * f[i][c] for c in range(512)], g1, z1) for i in range(3)])
    assert np.max(np.abs(out - ref)) < 1e-10
    full_step = np.array([_loop_layer_norm([x[i][c] + f[i][c] for c in range(512)], g1, z1) for i in range(3)])
    assert np.max(np.abs(out - full_step)) > 1e-2
