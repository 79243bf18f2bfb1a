"""Oracle: ConvSubsampling, FastConformer, encoder_proj, Transformer, head.

Sources: "Streaming Sortformer Diarizer" (Pipeline; torch.export Fixes 3, 4,
5 and 6 for MaskedConvSequential, the (c, f) flattening order, the
1 + (L-1)//8 frame count and the rel_shift gather) and the NeMo Speaker
Diarization API (``forward``, ``forward_infer``, ``frontend_encoder``).

Each function is the plain definition of its layer for ONE sequence of
valid frames (no padding); batching with masks is the engine's business and
must reproduce these values on the valid rows.  Readings where the pages
are silent:
  * subsampling: conv3x3 s2 1->256 + ReLU, then twice [depthwise 3x3 s2 +
    pointwise 256->256 + ReLU]; padding 1; time rows beyond each stage's
    length are zero (that is what running on exactly the valid rows gives);
    no input scaling;
  * conformer layer is the macaron block: x += FFN1/2, x += MHSA, x += Conv,
    x += FFN2/2, x = LN(x); LN eps 1e-5; FFN = W2 swish(W1 h + b1) + b2;
  * rel-pos MHSA: s[i, j] = ((q_i + u) . k_j + (q_i + v) . p_(i-j)) / sqrt(dk)
    with the sinusoidal table pe[r, 2m] = sin(r w_m), pe[r, 2m+1] = cos(r w_m),
    w_m = 10000^(-2m/d), projected by linear_pos (no bias);
  * conv module: pw 512->1024 + GLU (first half * sigmoid(second half)),
    depthwise k=9 (zero padding 4), BatchNorm with running statistics,
    swish, pw 512->512;
  * transformer layer is post-LN with no positional encoding;
  * head: sigmoid(W2 relu(W1 x + b1) + b2).
Real-checkpoint outputs: parity unpinned (no values printed on the pages).
"""
from __future__ import annotations

import numpy as np

from .frontend import mel_features

LN_EPS = 1e-5
BN_EPS = 1e-5


def W(w, name, dt):
    return np.asarray(w[name], dt)


def encoder_frames(L):
    """Encoder frames after 8x subsampling of L mel frames: 1 + (L-1)//8."""
    return 1 + (np.asarray(L) - 1) // 8


def layer_norm(x, g, b, eps=LN_EPS):
    mu = x.mean(-1, keepdims=True)
    var = ((x - mu) ** 2).mean(-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + b


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _swish(z):
    return z * _sigmoid(z)


def _conv3x3_s2(x, w, b, depthwise):
    """x (T, F, Cin) -> (1+(T-1)//2, 1+(F-1)//2, Cout); zero padding 1.
    w: (Cout, 1, 3, 3).  Full conv only for Cin == 1 (first stage)."""
    T, F, _ = x.shape
    To, Fo = 1 + (T - 1) // 2, 1 + (F - 1) // 2
    xp = np.zeros((T + 2, F + 2, x.shape[2]), x.dtype)
    xp[1:T + 1, 1:F + 1] = x
    out = np.zeros((To, Fo, w.shape[0]), x.dtype)
    for dt_ in range(3):
        for df in range(3):
            patch = xp[dt_:dt_ + 2 * To:2, df:df + 2 * Fo:2, :]   # (To, Fo, Cin)
            if depthwise:
                out += patch * w[:, 0, dt_, df][None, None, :]
            else:
                out += patch[:, :, 0:1] * w[:, 0, dt_, df][None, None, :]
    return out + b[None, None, :]


def subsample(feats_tf, w, dt=np.float64):
    """ConvSubsampling 8x of one clip's valid features (L, 128) -> (T', 512)."""
    p = "enc.pre_encode."
    x = np.asarray(feats_tf, dt)[:, :, None]
    x = np.maximum(_conv3x3_s2(x, W(w, p + "conv1.weight", dt), W(w, p + "conv1.bias", dt), False), 0)
    for s in (1, 2):
        x = _conv3x3_s2(x, W(w, p + f"dw{s}.weight", dt), W(w, p + f"dw{s}.bias", dt), True)
        x = np.maximum(x @ W(w, p + f"pw{s}.weight", dt).T + W(w, p + f"pw{s}.bias", dt), 0)
    T3, F3, C = x.shape
    feat = x.transpose(0, 2, 1).reshape(T3, C * F3)       # feature index c*F + f
    return feat @ W(w, p + "out.weight", dt).T + W(w, p + "out.bias", dt)


def rel_pos_table(S, d, dt=np.float64):
    """pe rows for relative distances r = -(S-1) .. S-1 (row r + S - 1)."""
    r = np.arange(-(S - 1), S, dtype=np.float64)[:, None]
    m = np.arange(d // 2, dtype=np.float64)[None, :]
    ang = r * np.power(10000.0, -2.0 * m / d)
    pe = np.zeros((2 * S - 1, d))
    pe[:, 0::2] = np.sin(ang)
    pe[:, 1::2] = np.cos(ang)
    return pe.astype(dt)


def rel_pos_mhsa(x, w, p, H, dt=np.float64, return_probs=False):
    """Relative-position MHSA over one sequence x (S, d)."""
    S, d = x.shape
    dk = d // H
    q = (x @ W(w, p + "att.linear_q.weight", dt).T + W(w, p + "att.linear_q.bias", dt)).reshape(S, H, dk)
    k = (x @ W(w, p + "att.linear_k.weight", dt).T + W(w, p + "att.linear_k.bias", dt)).reshape(S, H, dk)
    v = (x @ W(w, p + "att.linear_v.weight", dt).T + W(w, p + "att.linear_v.bias", dt)).reshape(S, H, dk)
    P = (rel_pos_table(S, d, dt) @ W(w, p + "att.linear_pos.weight", dt).T).reshape(2 * S - 1, H, dk)
    u = W(w, p + "att.pos_bias_u", dt)
    vb = W(w, p + "att.pos_bias_v", dt)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    ridx = (i - j) + (S - 1)                       # row of p_(i-j)
    ctx = np.zeros((S, H, dk), dt)
    probs = []
    for h in range(H):
        ac = (q[:, h] + u[h]) @ k[:, h].T
        bd_full = (q[:, h] + vb[h]) @ P[:, h].T    # (S, 2S-1): every relative distance
        bd = np.take_along_axis(bd_full, ridx, axis=1)
        s = (ac + bd) / np.sqrt(dt(dk))
        s = s - s.max(axis=1, keepdims=True)
        a = np.exp(s)
        a /= a.sum(axis=1, keepdims=True)
        probs.append(a)
        ctx[:, h] = a @ v[:, h]
    out = ctx.reshape(S, d) @ W(w, p + "att.linear_out.weight", dt).T + W(w, p + "att.linear_out.bias", dt)
    return (out, probs) if return_probs else out


def _ffn(x, w, p, dt):
    h = _swish(x @ W(w, p + "linear1.weight", dt).T + W(w, p + "linear1.bias", dt))
    return h @ W(w, p + "linear2.weight", dt).T + W(w, p + "linear2.bias", dt)


def _conv_module(x, w, p, dt):
    D = x.shape[1]
    h = x @ W(w, p + "pointwise1.weight", dt).T + W(w, p + "pointwise1.bias", dt)
    g = h[:, :D] * _sigmoid(h[:, D:])
    kw = W(w, p + "depthwise.weight", dt)             # (D, K)
    K = kw.shape[1]
    pad = (K - 1) // 2
    S = g.shape[0]
    gp = np.zeros((S + 2 * pad, D), dt)
    gp[pad:pad + S] = g
    c = np.zeros((S, D), dt)
    for t in range(K):
        c += gp[t:t + S] * kw[:, t][None, :]
    c += W(w, p + "depthwise.bias", dt)
    c = (c - W(w, p + "bn.running_mean", dt)) / np.sqrt(W(w, p + "bn.running_var", dt) + BN_EPS) \
        * W(w, p + "bn.weight", dt) + W(w, p + "bn.bias", dt)
    c = _swish(c)
    return c @ W(w, p + "pointwise2.weight", dt).T + W(w, p + "pointwise2.bias", dt)


def conformer_layer(x, w, l, H=8, dt=np.float64):
    p = f"enc.layers.{l}."
    ln = lambda t, z: layer_norm(z, W(w, p + t + ".weight", dt), W(w, p + t + ".bias", dt))  # noqa: E731
    x = x + 0.5 * _ffn(ln("ff1.ln", x), w, p + "ff1.", dt)
    x = x + rel_pos_mhsa(ln("att.ln", x), w, p, H, dt)
    x = x + _conv_module(ln("conv.ln", x), w, p + "conv.", dt)
    x = x + 0.5 * _ffn(ln("ff2.ln", x), w, p + "ff2.", dt)
    return ln("out_ln", x)


def _mha(x, w, p, H, dt):
    S, e = x.shape
    dk = e // H
    q = (x @ W(w, p + "q.weight", dt).T + W(w, p + "q.bias", dt)).reshape(S, H, dk)
    k = (x @ W(w, p + "k.weight", dt).T + W(w, p + "k.bias", dt)).reshape(S, H, dk)
    v = (x @ W(w, p + "v.weight", dt).T + W(w, p + "v.bias", dt)).reshape(S, H, dk)
    ctx = np.zeros((S, H, dk), dt)
    for h in range(H):
        s = (q[:, h] @ k[:, h].T) / np.sqrt(dt(dk))
        s = s - s.max(axis=1, keepdims=True)
        a = np.exp(s)
        a /= a.sum(axis=1, keepdims=True)
        ctx[:, h] = a @ v[:, h]
    return ctx.reshape(S, e) @ W(w, p + "o.weight", dt).T + W(w, p + "o.bias", dt)


def transformer_layer(x, w, l, H=8, dt=np.float64):
    p = f"tf.layers.{l}."
    x = layer_norm(x + _mha(x, w, p + "att.", H, dt), W(w, p + "ln1.weight", dt), W(w, p + "ln1.bias", dt))
    f = np.maximum(x @ W(w, p + "ff.linear1.weight", dt).T + W(w, p + "ff.linear1.bias", dt), 0)
    f = f @ W(w, p + "ff.linear2.weight", dt).T + W(w, p + "ff.linear2.bias", dt)
    return layer_norm(x + f, W(w, p + "ln2.weight", dt), W(w, p + "ln2.bias", dt))


def head(x, w, dt=np.float64, logits=False):
    h = np.maximum(x @ W(w, "head.fc1.weight", dt).T + W(w, "head.fc1.bias", dt), 0)
    z = h @ W(w, "head.fc2.weight", dt).T + W(w, "head.fc2.bias", dt)
    return z if logits else _sigmoid(z)


def _count(w, prefix):
    return len({k.split(".")[2] for k in w if k.startswith(prefix)})


def encode(X, w, dt=np.float64, H=8, taps=None):
    """Pre-encode embeddings (S, 512) -> speaker probabilities (S, 4):
    conformer layers, encoder_proj, transformer layers, head.  ``taps``
    (a dict) receives the intermediate tensors for layer-wise comparisons."""
    x = np.asarray(X, dt)
    for l in range(_count(w, "enc.layers.")):
        x = conformer_layer(x, w, l, H, dt)
        if taps is not None:
            taps[f"conformer{l}"] = x
    x = x @ W(w, "proj.weight", dt).T + W(w, "proj.bias", dt)
    if taps is not None:
        taps["proj"] = x
    for l in range(_count(w, "tf.layers.")):
        x = transformer_layer(x, w, l, H, dt)
        if taps is not None:
            taps[f"transformer{l}"] = x
    if taps is not None:
        taps["logits"] = head(x, w, dt, logits=True)
    return head(x, w, dt)


def forward_offline(audio, lengths, w, dt=np.float64, taps=None):
    """forward(audio, lengths) -> (probs (B, T'_max, 4), T' (B,)); frames
    beyond each clip's T' are 0.  ``taps`` (list of dicts, one per clip)
    receives intermediates."""
    feats, L = mel_features(audio, lengths, dt)
    Tp = encoder_frames(L)
    out = np.zeros((len(L), int(Tp.max()), 4), dt)
    for b in range(len(L)):
        emb = subsample(feats[b, :, :L[b]].T, w, dt)
        t = None
        if taps is not None:
            t = {"mel": feats[b], "pre_encode": emb}
            taps.append(t)
        out[b, :Tp[b]] = encode(emb, w, dt, taps=t)
    return out, Tp
