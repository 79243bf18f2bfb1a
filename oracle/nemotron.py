"""Oracle for the Nemotron-3 diarization variant (offline forward).

Test infrastructure only: the GPU engine never imports or calls this.

Sources: "Enable Nemotron-3-Diarization on MLX, CUDA, XNNPACK, and Vulkan"
(model description: 16 kHz mono audio, 128-bin mel features stacked to an
80 ms encoder frame rate, a 31-layer Transformer with RoPE, a Conv1D
upsampling head giving per-speaker activity at 10 ms, up to 8 speakers);
Transformers "Nemotron 3 Diarization" (logits of shape (1, frames, 8), one
frame every 10 ms; positions restart at 0 for each window the encoder sees).
Readings where the pages are silent (each written out below):
  * features: the Sortformer front-end of ``oracle.frontend`` (the same
    128-bin log-mel with per-bin normalisation);
  * stacking: encoder frame t is the concatenation of mel frames 8t .. 8t+7
    (frame-major: feature index k * 128 + f), frames past the clip zero,
    T' = ceil(L / 8); then a Linear 1024 -> 512 with bias;
  * Transformer: d 512, 8 heads of 64, pre-LN layers
    x += MHA(LN1(x)); x += FFN(LN2(x)), FFN = W2 swish(W1 h + b1) + b2, a
    final LayerNorm; projections with biases; LayerNorm eps 1e-5;
  * RoPE on queries and keys, "rotate half" pairing (dimension i with
    i + 32 in each head), angle p * 10000^(-2i/64) for position p counted
    from the sequence start;
  * head: a transposed 1-D convolution 512 -> 8 speakers with kernel =
    stride = 8 (no overlap), i.e. output frame 8t + k of speaker s is
    sum_c x[t, c] W[c, s, k] + b[s]; then a sigmoid; outputs past the clip's
    L mel frames are dropped.
Parity against a released checkpoint is unpinned (no weights or outputs on
the pages)."""
from __future__ import annotations

import numpy as np

from .frontend import mel_features
from .model import layer_norm

ROPE_BASE = 10000.0


def _w(w, name, dt):
    return np.asarray(w[name], dt)


def stack_frames(feats_tf, stack=8, dt=np.float64):
    """(L, n_mels) valid frames -> (ceil(L / stack), stack * n_mels)."""
    x = np.asarray(feats_tf, dt)
    L, F = x.shape
    T = (L + stack - 1) // stack
    pad = np.zeros((T * stack, F), dt)
    pad[:L] = x
    return pad.reshape(T, stack * F)          # row t = frames 8t .. 8t+7, frame-major


def rope(x, pos, base=ROPE_BASE):
    """Rotary embedding of x (S, H, dk) at positions pos (S,): rotate-half
    pairs (i, i + dk/2) by the angle pos * base^(-2i/dk)."""
    S, H, dk = x.shape
    half = dk // 2
    inv = np.power(base, -2.0 * np.arange(half) / dk)
    ang = np.asarray(pos, np.float64)[:, None] * inv[None, :]          # (S, half)
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1).astype(x.dtype)


def rope_mha(x, w, p, H, dt=np.float64, return_probs=False):
    """Multi-head self-attention with RoPE over one sequence x (S, d)."""
    S, d = x.shape
    dk = d // H
    proj = lambda n: (x @ _w(w, p + f"att.{n}.weight", dt).T + _w(w, p + f"att.{n}.bias", dt)).reshape(S, H, dk)  # noqa: E731
    pos = np.arange(S)
    q, k, v = rope(proj("q"), pos), rope(proj("k"), pos), proj("v")
    ctx = np.zeros((S, H, dk), dt)
    probs = []
    for h in range(H):
        s = (q[:, h] @ k[:, h].T) / np.sqrt(dt(dk))
        s = s - s.max(axis=1, keepdims=True)
        a = np.exp(s)
        a /= a.sum(axis=1, keepdims=True)
        probs.append(a)
        ctx[:, h] = a @ v[:, h]
    out = ctx.reshape(S, d) @ _w(w, p + "att.o.weight", dt).T + _w(w, p + "att.o.bias", dt)
    return (out, probs) if return_probs else out


def _swish(z):
    return z / (1.0 + np.exp(-z))


def nem_layer(x, w, l, H=8, dt=np.float64):
    p = f"nem.layers.{l}."
    ln = lambda t, z: layer_norm(z, _w(w, p + t + ".weight", dt), _w(w, p + t + ".bias", dt))  # noqa: E731
    x = x + rope_mha(ln("ln1", x), w, p, H, dt)
    h = _swish(ln("ln2", x) @ _w(w, p + "ff.linear1.weight", dt).T + _w(w, p + "ff.linear1.bias", dt))
    return x + h @ _w(w, p + "ff.linear2.weight", dt).T + _w(w, p + "ff.linear2.bias", dt)


def nem_head(x, w, dt=np.float64, logits=False):
    """(T', d) -> (8 T', n_spk): transposed conv, kernel = stride = 8."""
    W = _w(w, "nem.head.weight", dt)                    # (d, n_spk, k)
    b = _w(w, "nem.head.bias", dt)
    d, n_spk, K = W.shape
    z = np.einsum("tc,csk->tks", np.asarray(x, dt), W) + b[None, None, :]
    z = z.reshape(-1, n_spk)                            # frame 8t + k
    return z if logits else 1.0 / (1.0 + np.exp(-z))


def nem_encode(feats_tf, w, n_layers, H=8, dt=np.float64, taps=None):
    """Valid mel frames (L, 128) of one clip -> probabilities (L, n_spk)."""
    L = feats_tf.shape[0]
    x = stack_frames(feats_tf, dt=dt) @ _w(w, "nem.stack.weight", dt).T + _w(w, "nem.stack.bias", dt)
    if taps is not None:
        taps["stack"] = x
    for l in range(n_layers):
        x = nem_layer(x, w, l, H, dt)
        if taps is not None:
            taps[f"layer{l}"] = x
    x = layer_norm(x, _w(w, "nem.final_ln.weight", dt), _w(w, "nem.final_ln.bias", dt))
    return nem_head(x, w, dt)[:L]


def nem_forward_offline(audio, lengths, w, dt=np.float64):
    """Probabilities (B, L_max, n_spk) at 10 ms and L (B,): frames at and
    beyond a clip's L are 0."""
    n_layers = len({k.split(".")[2] for k in w if k.startswith("nem.layers.")})
    feats, L = mel_features(audio, lengths, dt)
    n_spk = w["nem.head.bias"].shape[0]
    out = np.zeros((len(L), int(L.max()), n_spk), dt)
    for b in range(len(L)):
        out[b, :L[b]] = nem_encode(feats[b, :, :L[b]].T, w, n_layers, dt=dt)
    return out, L
