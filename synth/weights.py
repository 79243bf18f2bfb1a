"""Seeded random weights for the Streaming Sortformer diarizer.

Shapes follow the model description on the "Streaming Sortformer Diarizer"
page (Pipeline and Model Parameters tables): ConvSubsampling 8x with 256
channels, FastConformer d=512 with 8 heads, Linear 512->192, Transformer
d=192 with 8 heads and FFN 768, and a Linear-ReLU-Linear head to 4 speakers.

Every matrix, bias and positional bias is drawn N(0, std) from
``numpy.random.default_rng(seed)`` in manifest order; LayerNorm gamma=1,
beta=0; BatchNorm running_mean=0, running_var=1, weight=1, bias=0 (these are
not drawn).  Tensors are float32.

The on-disk/in-memory blob (``weights_blob``) is a container format of this
project ("SFW1"): little-endian, 64-byte aligned payloads:

    char[4]  magic "SFW1"
    u32      n_tensors
    u64      data_offset        (from the start of the blob)
    n_tensors x {
        u16  name_len; char name[name_len];
        u8   ndim;     u32 dims[ndim];
        u64  offset              (from data_offset, bytes, 64-aligned)
    }
    payload: float32 tensors at their offsets
"""
from __future__ import annotations

import dataclasses
import struct
from collections import OrderedDict

import numpy as np


@dataclasses.dataclass(frozen=True)
class ModelDims:
    n_conformer: int = 17
    n_transformer: int = 18
    d_model: int = 512
    tf_d_model: int = 192
    n_heads: int = 8
    ff_mult: int = 4
    tf_ff: int = 768
    conv_kernel: int = 9
    sub_channels: int = 256
    n_mels: int = 128
    n_spk: int = 4


FULL = ModelDims()
TINY = ModelDims(n_conformer=2, n_transformer=2)

# init kinds: "n" = normal(0, std) draw, "one" = ones, "zero" = zeros
def manifest(d: ModelDims):
    """Ordered (name, shape, kind) list; the draw order defines the weights."""
    m = []
    C, D, E = d.sub_channels, d.d_model, d.tf_d_model
    F = d.n_mels // 8  # frequency rows after three stride-2 stages
    pre = "enc.pre_encode."
    m += [(pre + "conv1.weight", (C, 1, 3, 3), "n"), (pre + "conv1.bias", (C,), "n")]
    for s in (1, 2):
        m += [(pre + f"dw{s}.weight", (C, 1, 3, 3), "n"), (pre + f"dw{s}.bias", (C,), "n"),
              (pre + f"pw{s}.weight", (C, C), "n"), (pre + f"pw{s}.bias", (C,), "n")]
    m += [(pre + "out.weight", (D, C * F), "n"), (pre + "out.bias", (D,), "n")]
    dff = D * d.ff_mult
    dk = D // d.n_heads
    for l in range(d.n_conformer):
        p = f"enc.layers.{l}."

        def ffn(tag):
            return [(p + f"{tag}.ln.weight", (D,), "one"), (p + f"{tag}.ln.bias", (D,), "zero"),
                    (p + f"{tag}.linear1.weight", (dff, D), "n"), (p + f"{tag}.linear1.bias", (dff,), "n"),
                    (p + f"{tag}.linear2.weight", (D, dff), "n"), (p + f"{tag}.linear2.bias", (D,), "n")]
        m += ffn("ff1")
        m += [(p + "att.ln.weight", (D,), "one"), (p + "att.ln.bias", (D,), "zero")]
        for q in ("q", "k", "v", "out"):
            m += [(p + f"att.linear_{q}.weight", (D, D), "n"), (p + f"att.linear_{q}.bias", (D,), "n")]
        m += [(p + "att.linear_pos.weight", (D, D), "n"),
              (p + "att.pos_bias_u", (d.n_heads, dk), "n"), (p + "att.pos_bias_v", (d.n_heads, dk), "n")]
        m += [(p + "conv.ln.weight", (D,), "one"), (p + "conv.ln.bias", (D,), "zero"),
              (p + "conv.pointwise1.weight", (2 * D, D), "n"), (p + "conv.pointwise1.bias", (2 * D,), "n"),
              (p + "conv.depthwise.weight", (D, d.conv_kernel), "n"), (p + "conv.depthwise.bias", (D,), "n"),
              (p + "conv.bn.running_mean", (D,), "zero"), (p + "conv.bn.running_var", (D,), "one"),
              (p + "conv.bn.weight", (D,), "one"), (p + "conv.bn.bias", (D,), "zero"),
              (p + "conv.pointwise2.weight", (D, D), "n"), (p + "conv.pointwise2.bias", (D,), "n")]
        m += ffn("ff2")
        m += [(p + "out_ln.weight", (D,), "one"), (p + "out_ln.bias", (D,), "zero")]
    m += [("proj.weight", (E, D), "n"), ("proj.bias", (E,), "n")]
    for l in range(d.n_transformer):
        p = f"tf.layers.{l}."
        for q in ("q", "k", "v", "o"):
            m += [(p + f"att.{q}.weight", (E, E), "n"), (p + f"att.{q}.bias", (E,), "n")]
        m += [(p + "ln1.weight", (E,), "one"), (p + "ln1.bias", (E,), "zero"),
              (p + "ff.linear1.weight", (d.tf_ff, E), "n"), (p + "ff.linear1.bias", (d.tf_ff,), "n"),
              (p + "ff.linear2.weight", (E, d.tf_ff), "n"), (p + "ff.linear2.bias", (E,), "n"),
              (p + "ln2.weight", (E,), "one"), (p + "ln2.bias", (E,), "zero")]
    m += [("head.fc1.weight", (E, E), "n"), ("head.fc1.bias", (E,), "n"),
          ("head.fc2.weight", (d.n_spk, E), "n"), ("head.fc2.bias", (d.n_spk,), "n")]
    return m


def make_weights(d: ModelDims = FULL, seed: int = 0, std: float = 0.02, xavier: bool = False):
    """Draw the weights.  ``xavier=True`` scales each drawn matrix by
    1/sqrt(fan_in) instead of ``std`` (biases keep ``std``): a second parity
    input whose activations stay O(1) through every layer."""
    rng = np.random.default_rng(seed)
    w = OrderedDict()
    for name, shape, kind in manifest(d):
        if kind == "n":
            a = rng.standard_normal(size=shape, dtype=np.float32)
            if xavier and len(shape) >= 2 and not name.endswith(("pos_bias_u", "pos_bias_v")):
                fan_in = int(np.prod(shape[1:]))
                a *= np.float32(1.0 / np.sqrt(fan_in))
            else:
                a *= np.float32(std)
        elif kind == "one":
            a = np.ones(shape, np.float32)
        else:
            a = np.zeros(shape, np.float32)
        w[name] = a
    return w


def weights_blob(w) -> bytes:
    """Serialise a weight dict into the SFW1 container (see module docstring)."""
    entries = []
    off = 0
    for name, a in w.items():
        a = np.ascontiguousarray(a, dtype=np.float32)
        entries.append((name, a, off))
        off += (a.nbytes + 63) // 64 * 64
    hdr = bytearray()
    for name, a, o in entries:
        nb = name.encode()
        hdr += struct.pack("<H", len(nb)) + nb
        hdr += struct.pack("<B", a.ndim) + struct.pack(f"<{a.ndim}I", *a.shape)
        hdr += struct.pack("<Q", o)
    head_len = 4 + 4 + 8 + len(hdr)
    data_off = (head_len + 63) // 64 * 64
    out = bytearray(data_off + off)
    out[0:4] = b"SFW1"
    out[4:8] = struct.pack("<I", len(entries))
    out[8:16] = struct.pack("<Q", data_off)
    out[16:16 + len(hdr)] = hdr
    mv = memoryview(out)
    for name, a, o in entries:
        mv[data_off + o: data_off + o + a.nbytes] = a.tobytes()
    return bytes(out)
