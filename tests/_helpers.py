"""Shared helpers for the GPU parity tests (engine creation, dtype moves)."""
import numpy as np

from synth import TINY, FULL, make_weights, weights_blob


def bf16_round(a):
    """Round float array to bfloat16 (nearest even), returned as float32."""
    a = np.ascontiguousarray(a, np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def make_engine(weights, precision, n_conf, n_tf, max_batch=8, max_samples=1_920_000):
    from streaming_speaker_diarization_b200 import binding as b
    cfg = b.default_config(n_conformer=n_conf, n_transformer=n_tf, precision=precision, max_batch=max_batch,
                           max_samples=max_samples)
    return b.sf_create(weights_blob(weights), cfg)


def act_dtype(precision):
    import torch
    return torch.bfloat16 if precision == 1 else torch.float32


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    return t.to(dtype) if dtype is not None else t


def tiny_weights(xavier=False):
    return make_weights(TINY, seed=0, xavier=xavier)


def full_weights(xavier=False):
    return make_weights(FULL, seed=0, xavier=xavier)
