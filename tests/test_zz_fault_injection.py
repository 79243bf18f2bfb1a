"""Host-side fault injection through the C ABI: null and misaligned
pointers, sizes beyond the configured maxima, audio under the 1600-sample
minimum, bad presets, unknown options and a step after every stream has
finished.  Each call must return its documented status and enqueue nothing,
and the engine must keep working afterwards (a final forward matches the
oracle).  Collected after the parity files."""
import ctypes

import numpy as np
import pytest

import oracle as O
from synth import clip_for_config
from _helpers import make_engine, tiny_weights, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

SF_EINVAL, SF_ESHAPE, SF_ESTATE = 1, 2, 5


@pytest.fixture(scope="module")
def setup():
    w = tiny_weights()
    eng = make_engine(w, 1, 2, 2, max_batch=2, max_samples=64000)
    yield w, eng
    b.sf_destroy(eng)


def _st():
    return b._stream(None)


def test_null_pointers(setup):
    _, eng = setup
    audio = torch.zeros((1, 32000), device="cuda")
    probs = torch.zeros((1, 25, 4), device="cuda")
    mel = torch.zeros((1, 128, 201), device="cuda")
    lens = np.array([32000], np.int64)
    lp = lens.ctypes.data
    assert b.lib.sf_forward_offline(eng, None, lp, 1, 32000, probs.data_ptr(), None, _st()) == SF_EINVAL
    assert b.lib.sf_forward_offline(eng, audio.data_ptr(), None, 1, 32000, probs.data_ptr(), None, _st()) == SF_EINVAL
    assert b.lib.sf_forward_offline(eng, audio.data_ptr(), lp, 1, 32000, None, None, _st()) == SF_EINVAL
    assert b.lib.sf_mel(eng, audio.data_ptr(), lp, 1, 32000, None, None, _st()) == SF_EINVAL
    assert b.lib.sf_forward_offline(None, audio.data_ptr(), lp, 1, 32000, probs.data_ptr(), None, _st()) == SF_EINVAL
    assert b.lib.sf_mel(eng, audio.data_ptr(), lp, 1, 32000, mel.data_ptr(), None, _st()) == 0


def test_sizes_beyond_the_configuration(setup):
    _, eng = setup
    audio = torch.zeros((3, 70000), device="cuda")
    probs = torch.zeros((3, 100, 4), device="cuda")
    lens3 = np.full(3, 32000, np.int64)
    # three clips on an engine made for two; a buffer longer than max_samples; no clip at all
    assert b.lib.sf_forward_offline(eng, audio.data_ptr(), lens3.ctypes.data, 3, 32000, probs.data_ptr(), None,
                                    _st()) == SF_ESHAPE
    lens1 = np.array([32000], np.int64)
    assert b.lib.sf_forward_offline(eng, audio.data_ptr(), lens1.ctypes.data, 1, 70000, probs.data_ptr(), None,
                                    _st()) == SF_ESHAPE
    assert b.lib.sf_forward_offline(eng, audio.data_ptr(), lens1.ctypes.data, 0, 32000, probs.data_ptr(), None,
                                    _st()) == SF_ESHAPE
    # a clip under the 1600-sample minimum, and one longer than its buffer
    short = np.array([1599], np.int64)
    assert b.lib.sf_forward_offline(eng, audio.data_ptr(), short.ctypes.data, 1, 32000, probs.data_ptr(), None,
                                    _st()) == SF_EINVAL
    over = np.array([32001], np.int64)
    assert b.lib.sf_forward_offline(eng, audio.data_ptr(), over.ctypes.data, 1, 32000, probs.data_ptr(), None,
                                    _st()) == SF_EINVAL


@pytest.mark.parametrize("preset,n,code", [
    ((0, 7, 188, 144, 188), 1, SF_EINVAL),      # empty chunk
    ((6, -1, 188, 144, 188), 1, SF_EINVAL),     # negative look-ahead
    ((6, 7, -4, 144, 188), 1, SF_EINVAL),       # negative FIFO
    ((6, 7, 188, 0, 188), 1, SF_EINVAL),        # no update period
    ((6, 7, 188, 144, 192), 1, SF_EINVAL),      # cache longer than the model's 188
    ((6, 7, 188, 144, 186), 1, SF_EINVAL),      # cache not a multiple of the 4 speakers
    ((6, 7, 188, 144, 188), 0, SF_ESHAPE),      # no streams
    ((6, 7, 188, 144, 188), 3, SF_ESHAPE),      # more streams than max_batch
])
def test_bad_presets(setup, preset, n, code):
    _, eng = setup
    p = b.sf_preset(*preset)
    h = ctypes.c_void_p()
    assert b.lib.sf_stream_create(eng, ctypes.byref(p), n, ctypes.byref(h)) == code
    assert not h.value


def test_unknown_options_and_values(setup):
    _, eng = setup
    assert b.lib.sf_set_option(eng, 99, 1) == SF_EINVAL
    for opt, bad in ((b.SF_OPT_GEMM_PATH, 4), (b.SF_OPT_ATTN_PATH, 3), (b.SF_OPT_GEMM_PAIR_BN, 64),
                     (b.SF_OPT_MEL_PATH, 2), (b.SF_OPT_SUB_PATH, -1)):
        assert b.lib.sf_set_option(eng, opt, bad) == SF_EINVAL


def test_misaligned_attention_operands(setup):
    _, eng = setup
    qkv = torch.zeros((64 * 576 + 8,), device="cuda", dtype=torch.bfloat16)
    ctx = torch.zeros((64 * 192 + 8,), device="cuda", dtype=torch.bfloat16)
    lens = np.array([64], np.int32)
    assert b.lib.sf_attention_mha(eng, qkv.data_ptr() + 2, lens.ctypes.data, 1, ctx.data_ptr(), 1, _st()) == SF_EINVAL
    assert b.lib.sf_attention_mha(eng, qkv.data_ptr(), lens.ctypes.data, 1, ctx.data_ptr() + 2, 1, _st()) == SF_EINVAL


def test_step_after_the_last_chunk(setup):
    """A 2 s clip with the Very high preset finishes in one step; the next
    step has no stream left and returns SF_ESTATE without touching state."""
    w, eng = setup
    audio, lens, _ = clip_for_config(0)
    mel = torch.empty((1, 128, 1 + audio.shape[1] // 160), device="cuda")
    ml = b.sf_mel(eng, to_dev(audio), lens, mel)
    st = b.sf_stream_create(eng, (340, 40, 40, 300, 188), 1)
    cp = torch.zeros((1, 340, 4), device="cuda")
    try:
        n_out = b.sf_stream_step(eng, st, mel, np.zeros(1, np.int64), ml, cp)
        assert int(n_out[0]) == 25
        with pytest.raises(b.SFError, match="SF_ESTATE"):
            b.sf_stream_step(eng, st, mel, np.zeros(1, np.int64), ml, cp)
        v = b.sf_state_view()
        b.sf_stream_get_state(eng, st, 0, v)
        assert (v.n_cache, v.n_fifo, v.next_frame, v.finished) == (0, 25, 25, 1)
    finally:
        b.sf_stream_destroy(st)


def test_engine_still_works_after_the_rejections(setup):
    w, eng = setup
    audio, lens, _ = clip_for_config(0)
    probs = torch.zeros((1, 25, 4), device="cuda")
    b.sf_forward_offline(eng, to_dev(audio), lens, probs)
    b.sf_check(eng)
    ref, _ = O.forward_offline(audio, lens, w)
    assert np.max(np.abs(probs.cpu().numpy() - ref)) <= 2e-2


def test_stream_outliving_its_engine():
    """The engine destroyed first: its stream is detached; stepping it or
    reading its state returns SF_EINVAL, resetting and destroying it work."""
    eng = make_engine(tiny_weights(), 1, 2, 2, max_batch=1)
    p = b.sf_preset(6, 7, 188, 144, 188)
    h = ctypes.c_void_p()
    assert b.lib.sf_stream_create(eng, ctypes.byref(p), 1, ctypes.byref(h)) == 0
    st = h.value
    b.sf_destroy(eng)
    mel = torch.zeros((1, 128, 201), device="cuda")
    cp = torch.zeros((1, 6, 4), device="cuda")
    start, end = np.zeros(1, np.int64), np.array([200], np.int64)
    n_out = np.zeros(1, np.int32)
    assert b.lib.sf_stream_step(st, mel.data_ptr(), 201, start.ctypes.data, end.ctypes.data, cp.data_ptr(),
                                n_out.ctypes.data, _st()) == SF_EINVAL
    v = b.sf_state_view()
    assert b.lib.sf_stream_get_state(st, 0, ctypes.byref(v), _st()) == SF_EINVAL
    assert b.lib.sf_stream_reset(st, None, 0) == 0
    assert b.lib.sf_stream_destroy(st) == 0
