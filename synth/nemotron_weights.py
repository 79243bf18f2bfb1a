"""Seeded random weights for the Nemotron-3 diarization variant.

The model card ("Enable Nemotron-3-Diarization on MLX, CUDA, XNNPACK, and
Vulkan", model description) gives: about 100M parameters, up to 8 speakers,
128-bin mel features stacked to an 80 ms encoder frame rate, a 31-layer
Transformer with rotary position embedding (RoPE), and a Conv1D upsampling
head producing per-speaker activity at 10 ms.  Widths are not printed; the
readings here are d_model 512, 8 heads of 64, FFN 2048 (31 x 12 x 512^2 ~
97.5M, ~98.3M with the stacking projection and head), pre-LN layers with a
final LayerNorm, and a transposed 1-D convolution with kernel = stride = 8
as the head (one 512 -> 8 x 8 map per encoder frame).

Drawn like ``synth.weights``: every matrix and bias N(0, std) (or each
matrix / sqrt(fan_in) with ``xavier``) from ``default_rng(seed)`` in
manifest order; LayerNorm gamma 1, beta 0.  The blob format is the same
SFW1 container (``synth.weights.weights_blob``)."""
from __future__ import annotations

import dataclasses
from collections import OrderedDict

import numpy as np


@dataclasses.dataclass(frozen=True)
class NemDims:
    n_layers: int = 31
    d_model: int = 512
    n_heads: int = 8
    ff: int = 2048
    n_mels: int = 128
    stack: int = 8          # mel frames per encoder frame (10 ms -> 80 ms)
    n_spk: int = 8
    upsample: int = 8       # output frames per encoder frame (80 ms -> 10 ms)


NEM_FULL = NemDims()
NEM_TINY = NemDims(n_layers=2)


def nem_manifest(d: NemDims):
    m = []
    D, F = d.d_model, d.ff
    m += [("nem.stack.weight", (D, d.stack * d.n_mels), "n"), ("nem.stack.bias", (D,), "n")]
    for l in range(d.n_layers):
        p = f"nem.layers.{l}."
        m += [(p + "ln1.weight", (D,), "one"), (p + "ln1.bias", (D,), "zero")]
        for q in ("q", "k", "v", "o"):
            m += [(p + f"att.{q}.weight", (D, D), "n"), (p + f"att.{q}.bias", (D,), "n")]
        m += [(p + "ln2.weight", (D,), "one"), (p + "ln2.bias", (D,), "zero"),
              (p + "ff.linear1.weight", (F, D), "n"), (p + "ff.linear1.bias", (F,), "n"),
              (p + "ff.linear2.weight", (D, F), "n"), (p + "ff.linear2.bias", (D,), "n")]
    m += [("nem.final_ln.weight", (D,), "one"), ("nem.final_ln.bias", (D,), "zero")]
    # ConvTranspose1d(D -> n_spk, kernel = stride = upsample): weight [D][n_spk][upsample]
    m += [("nem.head.weight", (D, d.n_spk, d.upsample), "n"), ("nem.head.bias", (d.n_spk,), "n")]
    return m


def make_nem_weights(d: NemDims = NEM_FULL, seed: int = 0, std: float = 0.02, xavier: bool = False):
    rng = np.random.default_rng(seed)
    w = OrderedDict()
    for name, shape, kind in nem_manifest(d):
        if kind == "n":
            a = rng.standard_normal(size=shape, dtype=np.float32)
            if xavier and len(shape) >= 2:
                fan_in = shape[0] if name.endswith("head.weight") else int(np.prod(shape[1:]))
                a *= np.float32(1.0 / np.sqrt(fan_in))
            else:
                a *= np.float32(std)
        elif kind == "one":
            a = np.ones(shape, np.float32)
        else:
            a = np.zeros(shape, np.float32)
        w[name] = a
    return w
