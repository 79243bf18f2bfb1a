"""Checkpoint / resume of streaming state: two streams run k steps, their
state (cache and FIFO embeddings and predictions, silence mean and count,
next frame) is exported with sf_stream_get_state, the stream object is
destroyed, a new one is filled with sf_stream_set_state, and the remaining
steps must give the same bits as an uninterrupted run.  The new stream
object may reuse the destroyed one's host address: its steps must not
replay graphs that were captured with the destroyed stream's buffers.  A small preset
(chunk 6, look-ahead 3, FIFO 16, update 12, cache 24) makes the run cross
FIFO pops and cache compressions on both sides of the checkpoint.
Collected after the parity files."""
import numpy as np
import pytest

from synth import synth_batch
from _helpers import make_engine, tiny_weights, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402

PRESET = (6, 3, 16, 12, 24)


def _export(eng, st, sid):
    cap_c, cap_f = PRESET[4], PRESET[2] + PRESET[0]
    bufs = dict(ce=torch.zeros((cap_c, 512), device="cuda"), cp=torch.zeros((cap_c, 4), device="cuda"),
                fe=torch.zeros((cap_f, 512), device="cuda"), fp=torch.zeros((cap_f, 4), device="cuda"),
                sm=torch.zeros(512, device="cuda"))
    v = b.sf_state_view()
    v.d_cache_emb, v.d_cache_preds = bufs["ce"].data_ptr(), bufs["cp"].data_ptr()
    v.d_fifo_emb, v.d_fifo_preds, v.d_sil_mean = bufs["fe"].data_ptr(), bufs["fp"].data_ptr(), bufs["sm"].data_ptr()
    b.sf_stream_get_state(eng, st, sid, v)
    return v, bufs


def test_resume_from_exported_state_is_bit_identical():
    eng = make_engine(tiny_weights(xavier=True), 0, 2, 2, max_batch=2)
    try:
        audio, lens, _ = synth_batch(95, [9.0, 6.5])
        mel = torch.empty((2, 128, 1 + audio.shape[1] // 160), device="cuda")
        ml = b.sf_mel(eng, to_dev(audio), lens, mel)
        zero = np.zeros(2, np.int64)
        cp = torch.zeros((2, PRESET[0], 4), device="cuda")

        def run(st, n_steps):
            outs = []
            for _ in range(n_steps):
                n_out = b.sf_stream_step(eng, st, mel, zero, ml, cp)
                outs.append((n_out.copy(), cp.cpu().numpy().copy()))
            return outs

        T_enc = 1 + (ml - 1) // 8
        n_steps = int(np.max((T_enc + PRESET[0] - 1) // PRESET[0]))
        k = n_steps // 2
        st = b.sf_stream_create(eng, PRESET, 2)
        try:
            full = run(st, n_steps - 1)          # all but the last step, in both runs
        finally:
            b.sf_stream_destroy(st)

        st = b.sf_stream_create(eng, PRESET, 2)
        try:
            first = run(st, k)
            saved = [_export(eng, st, i) for i in range(2)]
            assert saved[0][0].n_cache > 0 and saved[0][0].n_fifo > 0   # the checkpoint holds a cache and a FIFO
        finally:
            b.sf_stream_destroy(st)
        st = b.sf_stream_create(eng, PRESET, 2)
        try:
            for i, (v, _) in enumerate(saved):
                b.sf_stream_set_state(eng, st, i, v)
            rest = run(st, n_steps - 1 - k)
        finally:
            b.sf_stream_destroy(st)
        b.sf_check(eng)
        resumed = first + rest
        assert len(resumed) == len(full)
        for (na, pa), (nb, pb) in zip(full, resumed):
            assert np.array_equal(na, nb)
            for i in range(2):
                assert np.array_equal(pa[i, :na[i]], pb[i, :nb[i]])
    finally:
        b.sf_destroy(eng)
