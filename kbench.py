"""Kernel micro-benchmarks through the C ABI's single-op entry points.

    python kbench.py gemm M N K [--epi E] [--path P] [--reps R]
    python kbench.py attn N_SEQ LEN [--path P] [--reps R]
    python kbench.py mha N_SEQ LEN [--path P] [--reps R]
    python kbench.py mel SECONDS [--clips B] [--path P] [--reps R]
    python kbench.py ln M N K [--xnorm X] [--double] [--reps R]
    python kbench.py stream N_STREAMS STEPS [--preset C R F U S]
    python kbench.py nem SECONDS [--clips B] [--layers L] [--reps R]

`gemm` runs sf_gemm_bf16 (E: 1 f32 out, 2 bf16 out, 3 residual update, 4
swish, 5 gated linear unit; P: SF_OPT_GEMM_PATH, 1 = tcgen05 with CTA pairs
where faster, 2 = CTA pairs always, 3 = single CTAs, 0 = mma.sync); `attn`
runs sf_attention_relpos and `mha` sf_attention_mha on N_SEQ packed
sequences of LEN rows (P: 1 tcgen05, 0 mma.sync); `mel` runs sf_mel on B
clips of SECONDS of audio each (P: SF_OPT_MEL_PATH); `ln` runs
sf_gemm_bf16_ln, the residual projection with the LayerNorm after it fused
into the epilogue (X: 1 = the residual stream receives the normalised row;
--double: a second LayerNorm into the bf16 output); `stream` runs STEPS
streaming steps of N_STREAMS streams (a 2 + 2-layer bf16 engine, random
normalised features, default the Low preset 6/7/188/144/188): the state
update and cache compression kernels at full state sizes; `nem` runs
sf_nem_forward_offline, the Nemotron-3 variant's offline forward (L layers,
default all 31; weights N(0, 0.02)) on B clips of SECONDS each.  Operands are seeded random values on the device; three warm-up
launches, then REPS launches queued behind a GPU sleep (so host launch
overhead is hidden) and timed with CUDA events on the current stream.  Also
the driver for single-kernel ncu captures (small REPS)."""
from __future__ import annotations

import argparse

import numpy as np


def _engine(b, max_batch):
    from synth import TINY, make_weights, weights_blob
    cfg = b.default_config(n_conformer=TINY.n_conformer, n_transformer=TINY.n_transformer, precision=1,
                           max_batch=max_batch)
    return b.sf_create(weights_blob(make_weights(TINY, seed=0)), cfg)


def _time(torch, fn, reps):
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(2_000_000)
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / reps


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    sub = ap.add_subparsers(dest="op", required=True)
    g = sub.add_parser("gemm")
    g.add_argument("M", type=int)
    g.add_argument("N", type=int)
    g.add_argument("K", type=int)
    g.add_argument("--epi", type=int, default=2)
    g.add_argument("--path", type=int, default=1)
    g.add_argument("--reps", type=int, default=20)
    a = sub.add_parser("attn")
    a.add_argument("n_seq", type=int)
    a.add_argument("length", type=int)
    a.add_argument("--path", type=int, default=1)
    a.add_argument("--reps", type=int, default=20)
    m = sub.add_parser("mha")
    m.add_argument("n_seq", type=int)
    m.add_argument("length", type=int)
    m.add_argument("--path", type=int, default=1)
    m.add_argument("--reps", type=int, default=20)
    f = sub.add_parser("mel")
    f.add_argument("seconds", type=float)
    f.add_argument("--clips", type=int, default=1)
    f.add_argument("--path", type=int, default=1)
    f.add_argument("--reps", type=int, default=10)
    n = sub.add_parser("ln")
    n.add_argument("M", type=int)
    n.add_argument("N", type=int)
    n.add_argument("K", type=int)
    n.add_argument("--xnorm", type=int, default=0)
    n.add_argument("--double", action="store_true")
    n.add_argument("--reps", type=int, default=20)
    t = sub.add_parser("stream")
    t.add_argument("n_streams", type=int)
    t.add_argument("steps", type=int)
    t.add_argument("--preset", type=int, nargs=5, default=[6, 7, 188, 144, 188])
    v = sub.add_parser("nem")
    v.add_argument("seconds", type=float)
    v.add_argument("--clips", type=int, default=1)
    v.add_argument("--layers", type=int, default=31)
    v.add_argument("--reps", type=int, default=10)
    args = ap.parse_args(argv)

    import torch
    from streaming_speaker_diarization_b200 import binding as b
    gen = torch.Generator(device="cuda").manual_seed(0)
    if args.op == "gemm":
        eng = _engine(b, 8)
        M, N, K = args.M, args.N, args.K
        if args.path == 0:
            args.epi = 1   # the mma.sync kernel writes f32 only
        b.sf_set_option(eng, b.SF_OPT_GEMM_PATH, args.path)
        A = torch.randn(M, K, device="cuda", generator=gen).to(torch.bfloat16)
        W = torch.randn(N, K, device="cuda", generator=gen).to(torch.bfloat16)
        cols = N // 2 if args.epi == 5 else N
        C = torch.zeros(M, cols, device="cuda", dtype=torch.float32 if args.epi in (1, 3) else torch.bfloat16)
        path = args.epi if args.path else 0   # sf_gemm_bf16 path: the epilogue, or 0 = mma.sync
        ms = _time(torch, lambda: b.sf_gemm_bf16(eng, A, W, C, path=path), args.reps)
        print(f"gemm M={M} N={N} K={K} epi={args.epi} path={args.path}: {ms * 1e3:.1f} us/launch, "
              f"{2 * M * N * K / ms / 1e9:.1f} TFLOP/s")
    elif args.op == "ln":
        eng = _engine(b, 8)
        M, N, K = args.M, args.N, args.K
        A = (torch.randn(M, K, device="cuda", generator=gen) / K ** 0.5).to(torch.bfloat16)
        W = torch.randn(N, K, device="cuda", generator=gen).to(torch.bfloat16)
        x = torch.randn(M, N, device="cuda", generator=gen)
        h = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
        g, bb = torch.ones(N, device="cuda"), torch.zeros(N, device="cuda")
        two = args.double
        ms = _time(torch, lambda: b.sf_gemm_bf16_ln(eng, A, W, x, g, bb, h, alpha=0.5, xnorm=1 if two else args.xnorm,
                                                     g2=g if two else None, b2=bb if two else None), args.reps)
        print(f"gemm+ln M={M} N={N} K={K} xnorm={args.xnorm} double={two}: {ms * 1e3:.1f} us/launch, "
              f"{2 * M * N * K / ms / 1e9:.1f} TFLOP/s")
    elif args.op == "stream":
        n, pre = args.n_streams, tuple(args.preset)
        eng = _engine(b, n)
        T = 8 * (pre[0] * args.steps + pre[1]) + 8
        feats = torch.randn(n, 128, T, device="cuda", generator=gen)
        st = b.sf_stream_create(eng, pre, n)
        cp = torch.zeros(n, pre[0], 4, device="cuda")
        zero, end = np.zeros(n, np.int64), np.full(n, T, np.int64)
        for _ in range(3):   # capture the step graphs
            b.sf_stream_step(eng, st, feats, zero, end, cp)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b.sf_stream_reset(st)
        e0.record()
        for _ in range(args.steps):
            b.sf_stream_step(eng, st, feats, zero, end, cp)
        e1.record()
        torch.cuda.synchronize()
        b.sf_stream_destroy(st)
        print(f"stream n={n} preset={pre}: {args.steps} steps, {e0.elapsed_time(e1) / args.steps * 1e3:.1f} us/step")
    elif args.op == "nem":
        from synth import NemDims, make_nem_weights, weights_blob
        B, n = args.clips, int(args.seconds * 16000)
        eng = b.sf_nem_create(weights_blob(make_nem_weights(NemDims(n_layers=args.layers), seed=0)),
                              b.nem_default_config(n_layers=args.layers, max_batch=B, max_samples=n))
        audio = 0.1 * torch.randn(B, n, device="cuda", generator=gen)
        lens = np.full(B, n, np.int64)
        probs = torch.zeros(B, n // 160, 8, device="cuda")
        ms = _time(torch, lambda: b.sf_nem_forward_offline(eng, audio, lens, probs), args.reps)
        b.sf_nem_destroy(eng)
        print(f"nem {B} x {args.seconds} s, {args.layers} layers: {ms * 1e3:.1f} us/forward, "
              f"{B * args.seconds / ms * 1e3:.0f} audio-s/s")
        return   # a Nemotron engine: not an sf_engine handle for the checks below
    elif args.op == "mel":
        n = int(args.seconds * 16000)
        B = args.clips
        from synth import TINY, make_weights, weights_blob
        cfg = b.default_config(n_conformer=TINY.n_conformer, n_transformer=TINY.n_transformer, precision=1,
                               max_batch=B, max_samples=n)
        eng = b.sf_create(weights_blob(make_weights(TINY, seed=0)), cfg)
        b.sf_set_option(eng, b.SF_OPT_MEL_PATH, args.path)
        audio = 0.1 * torch.randn(B, n, device="cuda", generator=gen)
        T = 1 + n // 160
        mel = torch.empty(B, 128, T, device="cuda")
        lens = np.full(B, n, np.int64)
        ms = _time(torch, lambda: b.sf_mel(eng, audio, lens, mel), args.reps)
        alg = B * (4.0 * n + 4.0 * 128 * T)
        print(f"mel B={B} x {args.seconds:g} s path={args.path}: {ms * 1e3:.1f} us/call, "
              f"{B * args.seconds / (ms / 1e3):.0f} audio-s/s, {alg / (ms / 1e3) / 1e9:.1f} GB/s algorithmic")
    elif args.op == "mha":
        n, L = args.n_seq, args.length
        eng = _engine(b, max(n, 8))
        qkv = torch.randn(n * L, 576, device="cuda", generator=gen).to(torch.bfloat16)
        ctx = torch.empty(n * L, 192, device="cuda", dtype=torch.bfloat16)
        lens = np.full(n, L, np.int32)
        ms = _time(torch, lambda: b.sf_attention_mha(eng, qkv, lens, ctx, path=args.path), args.reps)
        flops = 2 * 2 * n * L * L * 192
        print(f"mha n={n} L={L} path={args.path}: {ms * 1e3:.1f} us/launch, {flops / ms / 1e9:.1f} TFLOP/s "
              f"(2 x 2 x L^2 x 192 per sequence)")
    else:
        n, L = args.n_seq, args.length
        eng = _engine(b, max(n, 8))
        R = max(L, 756)
        qkv = torch.randn(n * L, 1536, device="cuda", generator=gen).to(torch.bfloat16)
        ptab = torch.randn(2 * R - 1, 512, device="cuda", generator=gen).to(torch.bfloat16)
        u = 0.5 * torch.randn(512, device="cuda", generator=gen)
        v = 0.5 * torch.randn(512, device="cuda", generator=gen)
        ctx = torch.empty(n * L, 512, device="cuda", dtype=torch.bfloat16)
        lens = np.full(n, L, np.int32)
        ms = _time(torch, lambda: b.sf_attention_relpos(eng, qkv, ptab, R, u, v, lens, ctx, path=args.path), args.reps)
        flops = 3 * 2 * n * L * L * 512
        print(f"attn n={n} L={L} path={args.path}: {ms * 1e3:.1f} us/launch, {flops / ms / 1e9:.1f} TFLOP/s "
              f"(3 x 2 x L^2 x 512 per sequence)")
    b.sf_check(eng)
    b.sf_destroy(eng)


if __name__ == "__main__":
    main()
