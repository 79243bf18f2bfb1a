"""CPU oracle for the Streaming Sortformer forward pass.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the engine computes, written from the pages (the
"Streaming Sortformer Diarizer" model description, the NeMo Speaker
Diarization API and the Transformers "Nemotron 3 Diarization" streaming
notes), and of the Nemotron-3 variant's offline forward (``nemotron``).  Only the tests, the smoke check and the benchmark's CPU-baseline leg
may import it; the engine never does, and this package imports nothing from
the engine.  It shares no code with the CUDA path: only the seeded input
generators in ``synth`` feed both.

Precision: float64 by default (``dt=np.float32`` gives the fp32 variant).

Pinning (tests/test_oracle_*.py): every function here is checked against
facts fixed by the pages or by mathematics (frame-count formulas, the preset
latency table, pure-tone STFT peaks, Parseval, mel partition of unity,
closed forms of zero-weight layers, brute-force attention and subset
enumeration on tiny inputs).  What no such fact pins is marked
"parity unpinned" in the function's docstring: the real checkpoint's
outputs (the pages print none) and the exact cache-compression scoring of
the released v2.1 model (the pages name it but give no formula).
"""
from .frontend import (preemphasis, hann_window_512, stft_power, slaney_mel_filterbank,  # noqa: F401
                       log_mel, normalize_per_bin, mel_features, n_frames, n_valid_frames)
from .model import (encoder_frames, subsample, rel_pos_table, rel_pos_mhsa, conformer_layer,  # noqa: F401
                    transformer_layer, head, encode, forward_offline, layer_norm, W)
from .streaming import (Preset, PRESETS, StreamState, compress_scores, select_topk,  # noqa: F401
                        compress_cache, stream_step, stream_run, state_update)
from .postprocess import SegParams, binarize, speaker_segments, segments  # noqa: F401
from .nemotron import (stack_frames, rope, rope_mha, nem_layer, nem_head, nem_encode,  # noqa: F401
                       nem_forward_offline)
