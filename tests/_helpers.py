"""Shared helpers for the GPU parity tests (engine creation, dtype moves,
streaming state injection and read-back)."""
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


def oracle_states(w, feats, L, preset, upto):
    """The oracle's stream over at most `upto` steps: states[k] is the state
    before step k (one more state than steps: the last is the state after
    the final step), taps[k] step k's window probabilities and embeddings."""
    import oracle as O
    st = O.StreamState()
    states, taps = [], []
    while st.c0 < 1 + (L - 1) // 8 and len(taps) < upto:
        states.append(st.copy())
        O.stream_step(st, feats, L, w, preset, taps=taps)
    states.append(st.copy())
    return states, taps


def set_state(eng, st, sid, ost, precision):
    import torch
    from streaming_speaker_diarization_b200 import binding as b
    dt = act_dtype(precision)
    keep = []

    def dev(a, d=None):
        t = to_dev(a if len(a) else np.zeros((1,) + a.shape[1:]), d)
        keep.append(t)
        return t.data_ptr()
    v = b.sf_state_view()
    v.n_cache, v.n_fifo, v.next_frame = len(ost.cache_emb), len(ost.fifo_emb), ost.c0
    v.finished, v.sil_count = 0, ost.sil_count
    v.d_cache_emb, v.d_cache_preds = dev(ost.cache_emb, dt), dev(ost.cache_preds)
    v.d_fifo_emb, v.d_fifo_preds = dev(ost.fifo_emb, dt), dev(ost.fifo_preds)
    v.d_sil_mean = dev(ost.sil_mean)
    b.sf_stream_set_state(eng, st, sid, v)
    torch.cuda.synchronize()


def get_state(eng, st, sid, precision, cap_c, cap_f):
    import torch
    from streaming_speaker_diarization_b200 import binding as b
    dt = act_dtype(precision)
    t = dict(ce=torch.zeros((cap_c, 512), device="cuda", dtype=dt), cp=torch.zeros((cap_c, 4), device="cuda"),
             fe=torch.zeros((cap_f, 512), device="cuda", dtype=dt), fp=torch.zeros((cap_f, 4), device="cuda"),
             sm=torch.zeros(512, device="cuda"))
    v = b.sf_state_view()
    v.d_cache_emb, v.d_cache_preds = t["ce"].data_ptr(), t["cp"].data_ptr()
    v.d_fifo_emb, v.d_fifo_preds, v.d_sil_mean = t["fe"].data_ptr(), t["fp"].data_ptr(), t["sm"].data_ptr()
    b.sf_stream_get_state(eng, st, sid, v)
    nc, nf = v.n_cache, v.n_fifo
    return dict(n_c=nc, n_f=nf, c0=v.next_frame, finished=v.finished, sil_count=v.sil_count,
                cache_emb=t["ce"][:nc].float().cpu().numpy(), cache_preds=t["cp"][:nc].cpu().numpy(),
                fifo_emb=t["fe"][:nf].float().cpu().numpy(), fifo_preds=t["fp"][:nf].cpu().numpy(),
                sil_mean=t["sm"].cpu().numpy())
