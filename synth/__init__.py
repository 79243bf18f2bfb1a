"""Seeded synthetic inputs shared by the CUDA engine's tests/bench and the CPU oracle.

This package only *draws* inputs: random weights in a fixed manifest order and
synthetic multi-speaker audio.  It holds none of the diarization arithmetic
(no filterbanks, convolutions, attention or cache logic); both the oracle and
the CUDA path consume what it produces, each with its own implementation.
"""
from .weights import ModelDims, TINY, FULL, manifest, make_weights, weights_blob  # noqa: F401
from .audio import synth_clip, synth_batch, clip_for_config  # noqa: F401
from .nemotron_weights import NemDims, NEM_FULL, NEM_TINY, nem_manifest, make_nem_weights  # noqa: F401
