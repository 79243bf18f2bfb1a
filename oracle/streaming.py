"""Oracle: streaming step over [speaker cache | FIFO | chunk] and cache
compression.

Sources: "Streaming Sortformer Diarizer" (Streaming Architecture: the
concatenation, the 188-frame speaker cache of single-speaker-dominant frames
picked by log-odds importance scoring, per-speaker top frames plus silence
placeholders on overflow, FIFO frames popping into the cache, pre_encode on
the new chunk only; Streaming Configurations table) and the NeMo Speaker
Diarization API (``forward_streaming_step``: streaming-state fields
spkcache / spkcache_lengths / spkcache_preds / fifo / fifo_lengths /
fifo_preds; ``forward_for_export``).  The Transformers "Nemotron 3
Diarization" streaming notes fix that look-ahead frames are attended to but
not emitted.

Readings (the pages give the structure, not these details):
  * chunk window: encoder frames [c0, c0 + chunk_len + right_context),
    clipped at the clip end, with one encoder frame (8 mel frames) of left
    context when c0 > 0 whose output is dropped; chunk outputs
    cl' = min(chunk_len, n) and look-ahead rc' = n - cl' of the n new frames;
  * after the encoder, FIFO predictions are refreshed with the current
    window's values; cache predictions stay as they were when the frames
    entered the cache;
  * the chunk's cl' embeddings and predictions are appended to the FIFO; when
    the FIFO holds more than fifo_len frames, the oldest
    n = min(max(update_period, |FIFO| - fifo_len), |FIFO|) frames pop;
  * popped frames whose four probabilities are all < 0.5 update a running
    mean silence embedding;
  * candidates C = cache ++ popped (in that order); if |C| <= spkcache_len
    the cache becomes C, else it is compressed;
  * compression score of frame t for speaker s (p clamped to [1e-6, 1-1e-6]):
        log(p_ts / (1 - p_ts)) + sum_{s' != s} log(1 - p_ts'),
    defined only for s = argmax_s p_ts (lowest s on ties) with p_ts > 0.5
    (else -inf); each speaker keeps its top k = spkcache_len // 4 frames by
    (score descending, candidate index ascending); empty slots become
    placeholders (silence mean embedding, zero predictions); the new cache is
    the kept frames in candidate order followed by the placeholders in
    speaker order.
The scoring formula is this engine's definition: parity unpinned against
the released v2.1 model (its scoring parameters are named, not given).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .model import encode, subsample

P_CLAMP = 1e-6


@dataclasses.dataclass(frozen=True)
class Preset:
    chunk_len: int
    right_context: int
    fifo_len: int
    update_period: int
    spkcache_len: int = 188

    @property
    def latency_s(self):
        """Input-buffer latency: (chunk_len + right_context) x 80 ms."""
        return (self.chunk_len + self.right_context) * 0.08


PRESETS = {
    "very_high": Preset(340, 40, 40, 300, 188),
    "high": Preset(124, 1, 124, 124, 188),
    "low": Preset(6, 7, 188, 144, 188),
    "ultra_low": Preset(3, 1, 188, 144, 188),
}


@dataclasses.dataclass
class StreamState:
    d: int = 512
    n_spk: int = 4
    dt: type = np.float64

    def __post_init__(self):
        self.cache_emb = np.zeros((0, self.d), self.dt)
        self.cache_preds = np.zeros((0, self.n_spk), self.dt)
        self.fifo_emb = np.zeros((0, self.d), self.dt)
        self.fifo_preds = np.zeros((0, self.n_spk), self.dt)
        self.sil_mean = np.zeros(self.d, self.dt)
        self.sil_count = 0
        self.c0 = 0

    def copy(self):
        s = StreamState(self.d, self.n_spk, self.dt)
        for k in ("cache_emb", "cache_preds", "fifo_emb", "fifo_preds", "sil_mean"):
            setattr(s, k, getattr(self, k).copy())
        s.sil_count, s.c0 = self.sil_count, self.c0
        return s


def compress_scores(preds):
    """Masked log-odds importance scores (n, 4); -inf where frame t is not a
    candidate for speaker s."""
    p = np.asarray(preds, np.float64)
    pc = np.clip(p, P_CLAMP, 1.0 - P_CLAMP)
    l1m = np.log(1.0 - pc)
    sc = np.log(pc / (1.0 - pc)) + (l1m.sum(axis=1, keepdims=True) - l1m)
    top = np.argmax(p, axis=1)                  # first maximum
    ok = p[np.arange(len(p)), top] > 0.5
    out = np.full_like(sc, -np.inf)
    rows = np.nonzero(ok)[0]
    out[rows, top[rows]] = sc[rows, top[rows]]
    return out


def select_topk(scores, k):
    """Per speaker: candidate indices of the top k by (score desc, index asc)
    among finite scores; returns a list (one array per speaker, ascending
    index order)."""
    sel = []
    n = scores.shape[0]
    for s in range(scores.shape[1]):
        cand = np.nonzero(np.isfinite(scores[:, s]))[0]
        order = np.lexsort((cand, -scores[cand, s]))   # primary: -score, secondary: index
        sel.append(np.sort(cand[order[:k]]))
        assert len(sel[-1]) <= min(k, n)
    return sel


def compress_cache(C_emb, C_preds, sil_mean, cache_len, scores=None):
    """Compress candidates to exactly cache_len frames.  Returns (emb, preds,
    slot source list) where a slot source is a candidate index, or -1 - s
    for a placeholder of speaker s."""
    n_spk = C_preds.shape[1]
    k = cache_len // n_spk
    sc = compress_scores(C_preds) if scores is None else scores
    sel = select_topk(sc, k)
    keep = np.sort(np.concatenate(sel)) if sel else np.zeros(0, np.int64)
    src = list(int(i) for i in keep)
    for s in range(n_spk):
        src += [-1 - s] * (k - len(sel[s]))
    emb = np.stack([C_emb[i] if i >= 0 else sil_mean for i in src]).astype(C_emb.dtype)
    pr = np.stack([C_preds[i] if i >= 0 else np.zeros(n_spk) for i in src]).astype(C_preds.dtype)
    return emb, pr, np.array(src, np.int64)


def chunk_window(c0, L, preset):
    """Mel-frame window [m0, m1) of the step starting at encoder frame c0 and
    its left-context frame count lc."""
    lc = 1 if c0 > 0 else 0
    m0 = 8 * (c0 - lc)
    m1 = min(8 * (c0 + preset.chunk_len + preset.right_context), L)
    return lc, m0, m1


def state_update(st, P, chunk_embs, n_chunk, preset, scores=None):
    """State update after the encoder ran on [cache | FIFO | chunk]:
    P (S, 4) are the window's probabilities, chunk_embs the new frames'
    pre-encode embeddings, n_chunk = cl'.  ``scores`` overrides the
    compression scores (used to compare bookkeeping given identical
    scores).  Mutates ``st``; returns an info dict."""
    n_c, n_f = len(st.cache_emb), len(st.fifo_emb)
    chunk_probs = P[n_c + n_f: n_c + n_f + n_chunk]
    st.fifo_preds = P[n_c: n_c + n_f].astype(st.dt).copy()
    st.fifo_emb = np.concatenate([st.fifo_emb, chunk_embs[:n_chunk]])
    st.fifo_preds = np.concatenate([st.fifo_preds, chunk_probs.astype(st.dt)])
    info = {"popped": 0, "compressed": False, "src": None, "scores": None, "margin": np.inf}
    if len(st.fifo_emb) > preset.fifo_len:
        npop = min(max(preset.update_period, len(st.fifo_emb) - preset.fifo_len), len(st.fifo_emb))
        pe, pp = st.fifo_emb[:npop], st.fifo_preds[:npop]
        st.fifo_emb, st.fifo_preds = st.fifo_emb[npop:], st.fifo_preds[npop:]
        info["margin"] = float(np.min(np.abs(pp - 0.5)))
        sil = np.all(pp < 0.5, axis=1)
        m = int(sil.sum())
        if m:
            st.sil_mean = (st.sil_mean * st.sil_count + pe[sil].sum(axis=0)) / (st.sil_count + m)
            st.sil_count += m
        C_emb = np.concatenate([st.cache_emb, pe])
        C_preds = np.concatenate([st.cache_preds, pp])
        info["popped"] = npop
        if len(C_emb) <= preset.spkcache_len:
            st.cache_emb, st.cache_preds = C_emb, C_preds
        else:
            sc = compress_scores(C_preds) if scores is None else scores
            st.cache_emb, st.cache_preds, src = compress_cache(C_emb, C_preds, st.sil_mean,
                                                               preset.spkcache_len, sc)
            info.update(compressed=True, src=src, scores=sc, cand_preds=C_preds,
                        margin=min(info["margin"], _decision_margin(C_preds, sc, preset.spkcache_len // 4)))
    return info


def _decision_margin(P, sc, k):
    """Smallest distance of any float decision to its threshold: |p - 0.5|
    over the frames, the gap between the two largest probabilities of a
    frame whose largest probability exceeds 0.5 (the argmax decides its
    speaker), and the score gap at each speaker's top-k boundary."""
    m = float(np.min(np.abs(P - 0.5))) if P.size else np.inf
    if P.shape[1] > 1 and P.size:
        s = np.sort(P, axis=1)
        live = s[:, -1] > 0.5
        if live.any():
            m = min(m, float(np.min(s[live, -1] - s[live, -2])))
    if sc is not None:
        for s_ in range(sc.shape[1]):
            f = np.sort(sc[np.isfinite(sc[:, s_]), s_])[::-1]
            if len(f) > k:
                m = min(m, float(f[k - 1] - f[k]))
    return m


def stream_step(st, feats, L, w, preset, dt=np.float64, taps=None):
    """One streaming step for one stream on its normalised features
    (128, >= L).  Returns the chunk probabilities (cl', 4); updates ``st``."""
    T_enc = 1 + (L - 1) // 8
    if st.c0 >= T_enc:
        raise ValueError("stream finished")
    lc, m0, m1 = chunk_window(st.c0, L, preset)
    embs = subsample(np.asarray(feats[:, m0:m1], dt).T, w, dt)
    new = embs[lc:]
    n = len(new)
    cl = min(preset.chunk_len, n)
    X = np.concatenate([st.cache_emb, st.fifo_emb, new])
    n_c, n_f = len(st.cache_emb), len(st.fifo_emb)
    P = encode(X, w, dt)
    out = P[n_c + n_f: n_c + n_f + cl].copy()
    info = state_update(st, P, new, cl, preset)
    st.c0 += cl
    if taps is not None:
        taps.append(dict(X=X, P=P, n_c=n_c, n_f=n_f, lc=lc, m0=m0, m1=m1, new=new, n_chunk=cl, **info))
    return out


def stream_run(feats, L, w, preset, dt=np.float64, taps=None, max_steps=None):
    """All steps of one stream; returns (probs (T', 4), final state)."""
    st = StreamState(dt=dt)
    T_enc = 1 + (L - 1) // 8
    outs = []
    steps = 0
    while st.c0 < T_enc and (max_steps is None or steps < max_steps):
        outs.append(stream_step(st, feats, L, w, preset, dt, taps))
        steps += 1
    return np.concatenate(outs), st


# ---------------------------------------------------------------- audio in
# Source: the Transformers "Nemotron 3 Diarization" streaming notes (the
# processor is called on successive audio slices, the last one flagged as the
# end of the session) and the NeMo API (streaming over features).  Reading:
# a step's mel window is computed from the stream's continuous signal as the
# offline front-end computes it (preemphasis from the stream start, centred
# frames, zeros past the samples received so far) and normalised per bin over
# the window's own frames (the clip normalisation applied to the window).

def window_log_mel(audio, n_avail, m0, m1, dt=np.float64):
    """Log-mel (128, m1 - m0) of frames m0 .. m1-1 of the first n_avail
    samples of a stream: frame t is the 400-point Hann-windowed, 512-point
    zero-padded segment centred on sample 160 t of the preemphasised signal
    (zeros outside [0, n_avail)), power spectrum by direct DFT, Slaney mel,
    log(x + 2^-24)."""
    from .frontend import hann_window_512, log_mel, preemphasis
    y = preemphasis(np.asarray(audio[:n_avail], dt), n_avail, dt)
    need = 160 * (m1 - 1) + 512                       # last padded sample used
    ypad = np.zeros(max(need, n_avail + 512), dt)
    ypad[256:256 + n_avail] = y
    win = hann_window_512(dt)
    frames = np.stack([ypad[160 * t: 160 * t + 512] for t in range(m0, m1)]) * win
    k = np.arange(257)[:, None] * np.arange(512)[None, :]
    X = frames @ np.exp(-2j * np.pi * k / 512).T
    return log_mel(np.abs(X) ** 2, dt)


def stream_step_audio(st, audio, n_avail, final, w, preset, dt=np.float64, taps=None):
    """One audio-in step of one stream with n_avail samples received (final:
    no more will come).  Returns the chunk probabilities, or None when the
    window is not complete yet (its last frame's samples have not all
    arrived) and the stream is not final."""
    from .frontend import normalize_per_bin
    L = n_avail // 160
    c0 = st.c0
    need = 8 * (c0 + preset.chunk_len + preset.right_context)
    lc, m0, m1 = chunk_window(c0, L, preset)
    if not final and n_avail < 160 * need + 96:
        return None
    if m1 <= 8 * c0:
        return None
    feats = np.zeros((128, m1), dt)
    feats[:, m0:m1] = normalize_per_bin(window_log_mel(audio, n_avail, m0, m1, dt), m1 - m0, dt)
    return stream_step(st, feats, m1, w, preset, dt, taps)


def stream_run_audio(audio, n_total, w, preset, arrivals, dt=np.float64, taps=None):
    """A stream fed by audio arriving in pieces: arrivals = increasing sample
    counts received before each step (the last equal to n_total, marked
    final).  Steps every arrival until the stream finishes; returns (probs
    (T', 4), emitted frames per step)."""
    st = StreamState(dt=dt)
    T_enc = 1 + (n_total // 160 - 1) // 8
    outs, per_step = [], []
    k = 0
    while st.c0 < T_enc:
        n_avail = int(arrivals[min(k, len(arrivals) - 1)])
        final = n_avail >= n_total
        out = stream_step_audio(st, audio, n_avail, final, w, preset, dt, taps)
        per_step.append(0 if out is None else len(out))
        if out is not None:
            outs.append(out)
        if out is None and final:
            break
        k += 1
    return (np.concatenate(outs) if outs else np.zeros((0, 4), dt)), per_step
