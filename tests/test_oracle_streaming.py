"""Pins for the oracle's streaming state machine and cache compression."""
import itertools
import json
import os

import numpy as np
import pytest

import oracle as O
from oracle import streaming as S
from synth import synth_clip

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_preset_latencies_match_table():
    g = json.load(open(os.path.join(GOLD, "presets.json")))["presets"]
    for name, row in g.items():
        p = O.PRESETS[name]
        assert (p.chunk_len, p.right_context, p.fifo_len, p.update_period, p.spkcache_len) == \
            (row["chunk_len"], row["right_context"], row["fifo_len"], row["update_period"], row["spkcache_len"])
        assert abs(p.latency_s - row["latency_s"]) < 1e-9


def test_score_closed_form_and_golden_selection():
    g = json.load(open(os.path.join(GOLD, "compress_small.json")))
    preds = np.array(g["preds"])
    sc = O.compress_scores(preds)
    assert abs(sc[0, 0] - g["expected_score_t0_s0"]) < 1e-12
    assert np.isneginf(sc[4]).all()                      # no probability above 0.5
    assert np.isneginf(sc[0, 1:]).all()                  # only the argmax speaker scores
    emb = np.arange(len(preds))[:, None] * np.ones((1, 3))
    sil = np.full(3, -7.0)
    e, p, src = O.compress_cache(emb, preds, sil, g["cache_len"])
    assert list(src) == g["expected_src"]
    assert np.array_equal(e[:3, 0], [0, 3, 5]) and np.all(e[3] == -7.0)
    assert np.all(p[3] == 0)


def _brute_select(scores, k):
    sel = []
    for s in range(scores.shape[1]):
        cand = [t for t in range(len(scores)) if np.isfinite(scores[t, s])]
        m = min(k, len(cand))
        best = None
        for sub in itertools.combinations(cand, m):
            key = sorted(((-scores[t, s], t) for t in sub))
            if best is None or key < best[0]:
                best = (key, sub)
        sel.append(sorted(best[1]) if best else [])
    return sel


@pytest.mark.parametrize("seed", range(12))
def test_topk_vs_brute_force_enumeration(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 21))
    preds = rng.uniform(0, 1, (n, 4))
    if seed % 3 == 0:                                   # exact ties in score
        preds[n // 2] = preds[0]
    sc = O.compress_scores(preds)
    for k in (1, 2, 3):
        got = [list(a) for a in O.select_topk(sc, k)]
        assert got == _brute_select(sc, k)


def test_selection_monotone_in_own_probability():
    rng = np.random.default_rng(21)
    for _ in range(30):
        preds = rng.uniform(0, 1, (15, 4))
        sc = O.compress_scores(preds)
        sel = O.select_topk(sc, 2)
        for s in range(4):
            for t in sel[s]:
                p2 = preds.copy()
                p2[t, s] = min(1.0, p2[t, s] + 0.05)
                assert t in O.select_topk(O.compress_scores(p2), 2)[s]


def _feats(seed, dur, nspk=3):
    a, _ = synth_clip(seed, dur, nspk)
    f, L = O.mel_features(a[None], np.array([len(a)]))
    return f[0], int(L[0])


def test_single_step_equals_offline(tiny_weights):
    f, L = _feats(31, 2.0)
    ref = O.encode(O.subsample(f[:, :L].T, tiny_weights), tiny_weights)
    probs, st = O.stream_run(f, L, tiny_weights, O.PRESETS["very_high"])
    assert probs.shape == ref.shape == (25, 4)
    assert np.array_equal(probs, ref)


def test_chunk_embeddings_equal_offline_embeddings(tiny_weights):
    """The left-context frame makes each chunk's pre-encode embeddings equal
    to the offline ones (receptive field of the three stride-2 convs)."""
    f, L = _feats(32, 3.05)
    full = O.subsample(f[:, :L].T, tiny_weights)
    pre = S.Preset(5, 3, 8, 4, 12)
    st = O.StreamState()
    taps = []
    while st.c0 < len(full):
        c0 = st.c0
        O.stream_step(st, f, L, tiny_weights, pre, taps=taps)
        new = taps[-1]["new"]
        assert np.max(np.abs(new - full[c0:c0 + len(new)])) < 1e-12


@pytest.mark.parametrize("name", ["very_high", "high", "low", "ultra_low"])
def test_output_counts_per_preset(name):
    pre = O.PRESETS[name]
    for Tp in (1, 2, 7, 100, 341, 999):
        c0, outs = 0, []
        while c0 < Tp:
            n = min(pre.chunk_len + pre.right_context, Tp - c0)
            cl = min(pre.chunk_len, n)
            outs.append(cl)
            c0 += cl
        assert sum(outs) == Tp
        assert all(o == pre.chunk_len for o in outs[:-1])


def test_all_sixteen_remainders_output_lengths(tiny_weights):
    """Frame-count remainders mod 16 of the mel length: total streamed
    outputs = 1 + (L-1)//8 for each."""
    pre = S.Preset(3, 1, 6, 4, 8)
    a, _ = synth_clip(40, 0.8, 2)
    full, L0 = O.mel_features(a[None], np.array([len(a)]))
    for r in range(16):
        L = 48 + r
        probs, _ = O.stream_run(full[0], L, tiny_weights, pre)
        assert len(probs) == 1 + (L - 1) // 8


def test_cache_and_fifo_bounds_and_rollover(tiny_weights):
    pre = S.Preset(chunk_len=6, right_context=2, fifo_len=16, update_period=12, spkcache_len=24)
    f, L = _feats(33, 12.0, 4)
    st = O.StreamState()
    taps = []
    T = 1 + (L - 1) // 8
    n_comp = 0
    out = []
    while st.c0 < T:
        out.append(O.stream_step(st, f, L, tiny_weights, pre, taps=taps))
        assert len(st.cache_emb) <= pre.spkcache_len
        assert len(st.fifo_emb) <= pre.fifo_len
        assert len(st.cache_emb) == len(st.cache_preds) and len(st.fifo_emb) == len(st.fifo_preds)
        n_comp += taps[-1]["compressed"]
        if taps[-1]["compressed"]:
            assert len(st.cache_emb) == pre.spkcache_len
            src = taps[-1]["src"]
            real = src[src >= 0]
            assert np.all(np.diff(real) > 0)            # kept frames stay in candidate order
            ph = src[src < 0]
            assert np.all(np.diff(-1 - ph) >= 0)        # placeholders in speaker order
    assert n_comp >= 3
    assert sum(len(o) for o in out) == T


def test_state_sizes_do_not_depend_on_data(tiny_weights, tiny_weights_xavier):
    pre = S.Preset(4, 2, 10, 6, 12)
    f, L = _feats(34, 5.0)
    sizes = []
    for w in (tiny_weights, tiny_weights_xavier):
        st = O.StreamState()
        seq = []
        while st.c0 < 1 + (L - 1) // 8:
            O.stream_step(st, f, L, w, pre)
            seq.append((len(st.cache_emb), len(st.fifo_emb), st.c0))
        sizes.append(seq)
    assert sizes[0] == sizes[1]


def test_low_preset_first_compression_at_full_sizes(tiny_weights):
    """Low preset at its real sizes: the FIFO first overflows after 32
    chunks, pops 144 frames into the cache, and the cache first compresses
    when a second pop would take it past 188."""
    pre = O.PRESETS["low"]
    f, L = _feats(35, 60.0, 3)
    st = O.StreamState()
    taps = []
    steps = 0
    while steps < 57:
        O.stream_step(st, f, L, tiny_weights, pre, taps=taps)
        steps += 1
    pops = [i for i, t in enumerate(taps) if t["popped"]]
    assert pops[0] == 31 and taps[31]["popped"] == 144
    assert pops[1] == 55
    assert taps[55]["compressed"] and len(st.cache_emb) == 188
    assert not any(t["compressed"] for t in taps[:55])
