"""Benchmark of the Sortformer engine: audio-seconds per second (RTFx).

Workload (one step): the offline forward of one 90 s, 16 kHz synthetic
meeting clip (4 speakers, 15 % overlap; audio seed 1001) through the full
model (ConvSubsampling, 17 FastConformer layers, 18 Transformer layers,
head), bf16 weights/activations with fp32 accumulation, random weights
N(0, 0.02) from seed 0: front-end -> probabilities, all in the engine's
kernels.  Inputs are resident in HBM when the timed region starts; L2 is
flushed (256 MiB write) between timed steps.

Also in the line: the two streaming workloads (`streaming`: Low preset 64 x
60 s, Very high preset 16 x 600 s), the variable-length batch of 32 clips
(`batch`), the Nemotron-3 variant on the same 90 s clip (`nemotron`) and the
front-end alone on 1 h of audio (`frontend_1h`, HBM roofline).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): the path has no exchange step, so
every rank runs its own replica of the workload ("replicas only"); value =
audio processed by all ranks / max-over-ranks device time.

--impl reference times the CPU oracle (test infrastructure, fp64 numpy) on
this machine's host cores, each step a bounded sample of the same workload
(the first 10 s of the clip).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "audio-sec/sec (RTFx) offline & streaming at 1 B200; % of bf16 tensor/HBM roofline"
UNIT = "audio-s/s"
CONFIG = {"workload": "offline forward, 1 clip x 90 s (16 kHz, 4 speakers, 15% overlap), full Sortformer "
                      "(17 FastConformer + 18 Transformer layers), bf16, fp32 accumulation",
          "audio_s": 90.0, "batch": 1, "mel_frames": 9000, "encoder_frames": 1125,
          "l2": "flushed between timed steps (256 MiB write)"}


# DRAM bytes (read + write) per projection launch of the offline forward,
# from an ncu launch list of this workload (710.4 MB over the 142 GEMM
# launches of one forward, the residual + LayerNorm epilogues included);
# valid only for the GEMM sources it was taken with, null once they change.
GEMM_TRAFFIC = {"bytes_per_launch": 710.39e6 / 142,
                "sources_sha256": "6adad731e4c712ce20106c3898e98d3fea44b47bdebe8191fbb7a019e63bdabe"}


# Warp instructions one sf_mel call on the 1 h workload issues (front-end
# path 1: frame, statistics and normalisation kernels; ncu
# smsp__inst_executed.sum, 438.2M + 4.1M + 25.0M), valid only for the
# front-end source it was taken with.  The call is bound by instruction
# issue (the FFT), not by HBM: its issue roofline is 148 SMs x 4 schedulers
# x one warp instruction per clock x 1965 MHz.
FRONTEND_INST = {"warp_inst_per_call": 467.33e6,
                 "sources_sha256": "edb41f3764b09c48b0e44751b1cddb013dde6b4fa3aba91f82a005ee84a5d525"}
ISSUE_PEAK = 148 * 4 * 1.965e9   # warp instructions per second


def frontend_inst_per_call():
    import hashlib
    try:
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "streaming_speaker_diarization_b200", "csrc",
                               "frontend.cu"), "rb") as fh:
            h = hashlib.sha256(fh.read()).hexdigest()
    except OSError:
        return None
    return FRONTEND_INST["warp_inst_per_call"] if h == FRONTEND_INST["sources_sha256"] else None


def gemm_traffic_per_launch():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "streaming_speaker_diarization_b200", "csrc")
    try:
        for f in ("gemm_tc.cu", "tcgen05.cuh", "epilogue.cuh", "epilogue_tma.cuh"):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return GEMM_TRAFFIC["bytes_per_launch"] if h.hexdigest() == GEMM_TRAFFIC["sources_sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# NVML clock-event reason bits (nvmlClocksEventReason*) reported in the line
_REASON_BITS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
                0x80: "hw_power_brake_slowdown"}


def summarize_samples(samples):
    """Summary of in-process clock samples [(sm_mhz, max_sm_mhz, reason_bits)]:
    median SM clock, max clock, and every throttle reason seen active."""
    sm = [float(a) for a, _, _ in samples]
    reasons = set()
    for _, _, bits in samples:
        for bit, name in _REASON_BITS.items():
            if bits & bit:
                reasons.add(name)
    return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": float(samples[-1][1]) if samples else None,
            "reasons": sorted(reasons), "samples": len(sm)}


class Clocks:
    """Clocks and throttle reasons sampled DURING a timed region.  A thread
    polls NVML every millisecond (reading only), so regions of tens of
    milliseconds still get samples; without NVML, nvidia-smi is sampled
    every 200 ms (raw samples under `out_dir`, default the temporary
    directory)."""

    def __init__(self, idx, out_dir=None):
        import threading
        self.samples, self.p = [], None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.stop_ev = threading.Event()

            def poll():
                while not self.stop_ev.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx,
                                             int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        pass
                    time.sleep(0.001)
            self.t = threading.Thread(target=poll, daemon=True)
            self.t.start()
            self.mode = "nvml"
            return
        except Exception:
            self.mode = "nvidia-smi"
        import tempfile
        self.path = os.path.join(out_dir or tempfile.gettempdir(), f"sf_bench_clocks_rank{idx}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(idx), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.mode == "nvml":
            self.stop_ev.set()
            self.t.join(timeout=5)
            return dict(summarize_samples(self.samples), source="nvml, 1 ms polling during the timed region")
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.close()
        with open(self.path) as f:
            return dict(parse_clocks(f), source="nvidia-smi, 200 ms polling during the timed region")


def parse_clocks(lines):
    """Summary of nvidia-smi samples (index, clocks.sm, clocks.max.sm, power,
    active reasons, then hw_slowdown, hw_thermal_slowdown,
    sw_thermal_slowdown, sw_power_cap as Active / Not Active): median SM
    clock, max clock, and every throttle reason seen active."""
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            mx = float(f[2])
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


def cpu_baseline(audio, seconds=30.0):
    import oracle as O
    from synth import FULL, make_weights
    w = make_weights(FULL, seed=0)
    n = int(seconds * 16000)
    t0 = time.perf_counter()
    O.forward_offline(audio[:, :n], np.array([n]), w)
    dt = time.perf_counter() - t0
    return {"value": seconds / dt, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"first {seconds:.0f} s of the 90 s workload clip, full model, fp64 numpy, one pass "
                      f"({dt:.1f} s)"}


# Algorithmic work of the model per encoder frame of a sequence of S frames
# (2 flops per multiply-add): conformer layer 12.06 MF of projections (FFN
# 2 x 2 x 512 x 2048 x 2, Q/K/V/out 4 x 512^2 x 2, conv pointwise 512 x 1024
# x 2 + 512^2 x 2) + 3 x 2 x 512 x S of attention (AC, BD, P.V);
# Transformer layer 0.885 MF (Q/K/V/out 4 x 192^2 x 2, FFN 2 x 192 x 768 x 2)
# + 2 x 2 x 192 x S; encoder_proj 2 x 512 x 192; head 2 x 192 x (192 + 4);
# subsampling 16.23 MF per encoder frame it produces.  The relative-position
# projections are weights-only (computed once when the engine is created)
# and are not counted.
CONF_MF, TF_MF, PROJ_HEAD_MF, SUB_MF = 12.059136e6, 0.884736e6, 0.196608e6 + 0.075264e6, 16.23e6


def model_flops(S, new_frames, n_conf=17, n_tf=18):
    """Flops of one encoder pass over a sequence of S frames of which
    new_frames came out of the subsampling in this pass."""
    per = n_conf * (CONF_MF + 3072.0 * S) + n_tf * (TF_MF + 768.0 * S) + PROJ_HEAD_MF
    return S * per + new_frames * SUB_MF


def stream_plan(preset, total_frames):
    """Per step of one stream: (S, window embeddings) for a clip of
    total_frames encoder frames under preset (chunk, right context, FIFO,
    update period, cache).  The sizes do not depend on the data: the window
    holds cl' = min(chunk, left) chunk frames and rc' = min(right, left - cl')
    look-ahead frames after [cache | FIFO]; the chunk joins the FIFO, which
    pops max(update period, overflow) frames into the cache once it is over
    its length; the cache is compressed back to its length when it overflows."""
    cl, rc, fl, up, cap = preset
    n_c = n_f = c0 = 0
    out = []
    while c0 < total_frames:
        c = min(cl, total_frames - c0)
        r = min(rc, total_frames - c0 - c)
        out.append((n_c + n_f + c + r, c + r))
        n_f += c
        c0 += c
        if n_f > fl:
            n = min(max(up, n_f - fl), n_f)
            n_f -= n
            n_c = min(n_c + n, cap)
    return out


STREAM_WORKLOADS = [
    # (name, preset chunk/right/fifo/update/cache, workload index, streams, seconds)
    ("Low preset (6/7/188/144/188, 1.04 s latency), 64 streams x 60 s, 2-4 speakers", (6, 7, 188, 144, 188), 2, 64, 60.0),
    ("Very high preset (340/40/40/300/188, 30.4 s latency), 16 streams x 600 s, 4 speakers, 20% overlap, arrivals",
     (340, 40, 40, 300, 188), 3, 16, 600.0),
]


def set_options(b, eng, args):
    """The kernel-selection options of the command line on one engine."""
    b.sf_set_option(eng, b.SF_OPT_PDL, args.pdl)
    b.sf_set_option(eng, b.SF_OPT_MEL_PATH, args.mel_path)
    b.sf_set_option(eng, b.SF_OPT_SUB_PATH, args.sub_path)
    b.sf_set_option(eng, b.SF_OPT_ATTN_PATH, args.attn_path)
    b.sf_set_option(eng, b.SF_OPT_TF_FUSE, args.tf_fuse)
    b.sf_set_option(eng, b.SF_OPT_LN_FUSE, args.ln_fuse)


def streaming_bench(b, torch, eng_blob, rank, world, local, args, clocks_dir=None):
    """Streaming throughput: front-end over each stream's clip, then every
    step of every stream (pre_encode on the new window, encoder on
    [cache | FIFO | chunk], state update) until all streams finish.  A first
    pass captures each step shape's CUDA graph; the streams are reset and the
    second pass is timed with CUDA events (clocks sampled meanwhile).  A
    third pass brackets only the state-update and selection launches with
    events: the cache compression's microseconds per step; a fourth brackets
    the projection GEMMs: their class throughput in the step.  The roofline is
    the model's algorithmic flops (model_flops over every stream's steps)
    over the timed pass."""
    from streaming_speaker_diarization_b200 import dist as sd
    from synth import clip_for_config
    out = []
    for name, preset, idx, n_total, dur in STREAM_WORKLOADS:
        lo, hi = sd.shard(n_total, rank, world)
        n = hi - lo
        audio_np, lens, _ = clip_for_config(idx)
        audio_np, lens = np.ascontiguousarray(audio_np[lo:hi]), lens[lo:hi]
        eng = b.sf_create(eng_blob, b.default_config(max_batch=max(n, 1), max_samples=int(audio_np.shape[1])))
        set_options(b, eng, args)
        audio = torch.from_numpy(audio_np).cuda()
        T = 1 + audio_np.shape[1] // 160
        mel = torch.empty((n, 128, T), device="cuda")
        cp = torch.zeros((n, preset[0], 4), device="cuda")
        st = b.sf_stream_create(eng, preset, n)
        zero = np.zeros(n, np.int64)

        def one_pass(times=None):
            ml = b.sf_mel(eng, audio, lens, mel)
            left = 1 + (ml - 1) // 8          # encoder frames each stream still has to emit
            while (left > 0).any():
                if times is not None:
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                n_out = b.sf_stream_step(eng, st, mel, zero, ml, cp)
                if times is not None:
                    e1.record()
                    times.append((e0, e1))
                left -= n_out
            return ml

        one_pass()
        b.sf_stream_reset(st)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps = []
        clk = Clocks(local, clocks_dir)
        t0.record()
        one_pass(steps)
        t1.record()
        torch.cuda.synchronize()
        clocks = clk.stop()
        ms = t0.elapsed_time(t1)
        step_ms = [a.elapsed_time(c) for a, c in steps]
        # compression: events around the state-update and selection launches only
        b.sf_stream_reset(st)
        b.sf_profile_read(eng, reset=True)
        b.sf_profile_enable(eng, 2 * ((1 << 11) | (1 << 13)))
        one_pass()
        torch.cuda.synchronize()
        upd = b.sf_profile_read(eng, reset=True)
        # the projection GEMMs: events around the GEMM launches only (class 3)
        b.sf_stream_reset(st)
        b.sf_profile_enable(eng, 2 * (1 << 3))
        one_pass()
        torch.cuda.synchronize()
        gm = b.sf_profile_read(eng, reset=True).get("gemm", (0, 0.0, 0.0, 0.0))
        b.sf_profile_enable(eng, 0)
        upd_ms = sum(v[1] for k, v in upd.items() if k in ("state_update", "select_topk"))
        audio_s = float(lens.sum()) / 16000.0
        value = sd.throughput(audio_s, ms)
        frames = [int(1 + (int(l) // 160 - 1) // 8) for l in lens]
        flops = sum(model_flops(S, new) for f in frames for S, new in stream_plan(preset, f))
        max_ms = sd.max_over_ranks(ms)
        pk, kind = peaks()
        tf = sd.sum_over_ranks(flops) / (max_ms / 1000.0) / 1e12
        peak_tf = pk["bf16_tflops_sustained"] if max_ms > 1000.0 else pk["bf16_tflops"]
        out.append({"workload": name, "value": value, "unit": UNIT, "streams": n_total, "steps": len(step_ms),
                    "ms_total": max_ms, "step_ms_p50": float(np.median(step_ms)),
                    "step_ms_p95": float(np.percentile(step_ms, 95)),
                    "encoder_frames_per_s": sd.sum_over_ranks(sum(frames)) / (max_ms / 1000.0),
                    "roofline": {"bound": "tensor", "kernel": "whole step (model flops)", "achieved": tf,
                                 "peak": peak_tf, "unit": "TFLOP/s", "frac": tf / peak_tf,
                                 "flops_total": flops,
                                 "peak_kind": f"{kind} bf16 {'sustained' if max_ms > 1000.0 else 'burst'}"},
                    "compression_us_per_step": 1000.0 * upd_ms / max(len(step_ms), 1),
                    "gemm": {"launches": int(gm[0]), "ms": gm[1], "share_of_pass": gm[1] / max_ms if max_ms else None,
                             "tflops": gm[2] / (gm[1] / 1000.0) / 1e12 if gm[1] else None,
                             "frac": (gm[2] / (gm[1] / 1000.0) / 1e12) / pk["bf16_tflops"] if gm[1] else None,
                             "peak_kind": f"{kind} bf16 burst",
                             "note": "events around the GEMM launches of a separate pass (they add a few us each)"},
                    "clocks": clocks})
        b.sf_stream_destroy(st)
        b.sf_destroy(eng)
        del audio, mel
        torch.cuda.empty_cache()
    return out


def frontend_bench(b, torch, blob, steps, warmup, mel_path=1):
    """Front-end alone (preemphasis, centred STFT, power, Slaney mel, log,
    per-bin normalisation) on 1 h of audio in one sf_mel call: 57.6M samples
    -> 128 x 360,001 features.  Audio resident on the device, CUDA events per
    call on the launching stream; the 230 MB input and 184 MB output exceed
    L2, which is also flushed between calls.  Roofline: HBM, algorithmic
    bytes = 4 B per sample in + 128 x 4 B per feature column out."""
    from synth.audio import hour_of_audio
    x = hour_of_audio()
    n = len(x)
    T = 1 + n // 160
    eng = b.sf_create(blob, b.default_config(max_batch=1, max_samples=n))
    b.sf_set_option(eng, b.SF_OPT_MEL_PATH, mel_path)
    try:
        audio = torch.from_numpy(x[None]).cuda()
        mel = torch.empty((1, 128, T), device="cuda")
        lens = np.array([n], np.int64)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        st = torch.cuda.current_stream()
        for _ in range(warmup):
            b.sf_mel(eng, audio, lens, mel)
        b.sf_check(eng)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(st)
            b.sf_mel(eng, audio, lens, mel)
            ev[i][1].record(st)
        torch.cuda.synchronize()
        b.sf_check(eng)
    finally:
        b.sf_destroy(eng)
    ms = [a.elapsed_time(c) for a, c in ev]
    med = float(np.median(ms))
    alg = 4.0 * n + 4.0 * 128 * T
    pk, kind = peaks()
    gbs = alg / (med / 1000.0) / 1e9
    inst = frontend_inst_per_call()
    issue = None if inst is None else {
        "bound": "alu", "kernel": "front-end call (warp instructions issued, FFT-dominated)",
        "achieved": inst / (med / 1000.0), "peak": ISSUE_PEAK, "unit": "warp instructions/s",
        "frac": inst / (med / 1000.0) / ISSUE_PEAK, "inst_per_call": inst,
        "peak_kind": "148 SMs x 4 schedulers x 1 issue per clock x 1965 MHz"}
    return {"workload": "front-end only, 1 h of audio (60 x 60 s clips joined), 57.6M samples -> 128 x 360,001",
            "value": 3600.0 / (med / 1000.0), "unit": UNIT, "ms_p50": med, "ms_p95": float(np.percentile(ms, 95)),
            "calls": steps, "mel_path": mel_path,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "bytes_per_call": alg, "peak_kind": f"{kind} copy"},
            "roofline_issue": issue}


def batch_bench(b, torch, blob, steps, warmup, local, args, clocks_dir=None):
    """The variable-length offline batch: 32 clips of 5-120 s (seeded),
    padded to the longest, one sf_forward_offline call per step (front-end
    to probabilities).  Audio resident on the device, L2 flushed between
    steps, CUDA events per step on the launching stream."""
    from synth import clip_for_config
    audio_np, lens, _ = clip_for_config(4)
    B, n_max = audio_np.shape
    eng = b.sf_create(blob, b.default_config(max_batch=B, max_samples=int(n_max)))
    set_options(b, eng, args)
    try:
        audio = torch.from_numpy(audio_np).cuda()
        Tp = 1 + (n_max // 160 - 1) // 8
        probs = torch.zeros((B, Tp, 4), device="cuda")
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        st = torch.cuda.current_stream()
        for _ in range(warmup):
            b.sf_forward_offline(eng, audio, lens, probs)
        b.sf_check(eng)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        clk = Clocks(local, clocks_dir)
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(st)
            b.sf_forward_offline(eng, audio, lens, probs)
            ev[i][1].record(st)
        torch.cuda.synchronize()
        clocks = clk.stop()
        b.sf_check(eng)
    finally:
        b.sf_destroy(eng)
    ms = [a.elapsed_time(c) for a, c in ev]
    med = float(np.median(ms))
    audio_s = float(lens.sum()) / 16000.0
    frames = [int(1 + (int(l) // 160 - 1) // 8) for l in lens]
    flops = sum(model_flops(f, f) for f in frames)
    pk, kind = peaks()
    tf = flops / (med / 1000.0) / 1e12
    return {"workload": "offline variable-length batch, 32 clips of 5-120 s (seeded), padded to the longest, "
                        "full model, bf16", "value": audio_s / (med / 1000.0), "unit": UNIT,
            "audio_s": audio_s, "clips": B, "ms_p50": med, "ms_p95": float(np.percentile(ms, 95)), "calls": steps,
            "encoder_frames_per_s": sum(frames) / (med / 1000.0),
            "roofline": {"bound": "tensor", "kernel": "whole forward (model flops)", "achieved": tf,
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"],
                         "flops_per_call": flops, "peak_kind": f"{kind} bf16 burst"},
            "clocks": clocks}


def nem_model_flops(T, n_layers=31):
    """Flops of the Nemotron-3 variant's offline forward over one clip of T
    encoder frames (80 ms): stacking projection 2 x 1024 x 512, per layer
    Q|K|V + output 4 x 2 x 512^2 and FFN 2 x 2 x 512 x 2048 per frame plus
    2 x 2 x 512 x T of attention, head 2 x 512 x 64."""
    per = 2.0 * 1024 * 512 + n_layers * (8.0 * 512 ** 2 + 4.0 * 512 * 2048 + 2048.0 * T) + 2.0 * 512 * 64
    return T * per


def nemotron_bench(b, torch, steps, warmup, local, clocks_dir=None):
    """The Nemotron-3 variant (31 RoPE Transformer layers, 8 speakers at
    10 ms) on the same 90 s clip: offline forward per step, audio resident on
    the device, L2 flushed between steps, CUDA events; weights N(0, 0.02)."""
    from synth import NEM_FULL, clip_for_config, make_nem_weights, weights_blob
    audio_np, lens, _ = clip_for_config(1)
    eng = b.sf_nem_create(weights_blob(make_nem_weights(NEM_FULL, seed=0)), b.nem_default_config(max_batch=1))
    try:
        audio = torch.from_numpy(audio_np).cuda()
        probs = torch.zeros((1, audio_np.shape[1] // 160, 8), device="cuda")
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        st = torch.cuda.current_stream()
        for _ in range(warmup):
            b.sf_nem_forward_offline(eng, audio, lens, probs)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        clk = Clocks(local, clocks_dir)
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(st)
            b.sf_nem_forward_offline(eng, audio, lens, probs)
            ev[i][1].record(st)
        torch.cuda.synchronize()
        clocks = clk.stop()
    finally:
        b.sf_nem_destroy(eng)
    ms = [a.elapsed_time(c) for a, c in ev]
    med = float(np.median(ms))
    T = (int(lens[0]) // 160 + 7) // 8
    flops = nem_model_flops(T)
    pk, kind = peaks()
    tf = flops / (med / 1000.0) / 1e12
    return {"workload": "Nemotron-3 variant offline, 1 clip x 90 s (the headline clip), 31 RoPE Transformer layers "
                        "d 512, 8 speakers every 10 ms, bf16", "value": 90.0 / (med / 1000.0), "unit": UNIT,
            "ms_p50": med, "ms_p95": float(np.percentile(ms, 95)), "calls": steps,
            "output_frames_per_s": (int(lens[0]) // 160) / (med / 1000.0),
            "roofline": {"bound": "tensor", "kernel": "whole forward (model flops)", "achieved": tf,
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"],
                         "flops_per_call": flops, "peak_kind": f"{kind} bf16 burst"},
            "clocks": clocks}


def oracle_subsets(w):
    """The oracle (numpy, fp64 unless stated) on declared subsets of every
    workload, each timed once on this machine's host cores: the 90 s clip
    complete (fp64, then fp32), the front-end on 1 h complete, 2 Low-preset
    streams x their first 20 steps, 1 Very-high-preset stream x 3 steps, and
    the first 4 clips of the variable-length batch."""
    import oracle as O
    from synth import clip_for_config
    from synth.audio import hour_of_audio
    out = []

    def rec(name, sample, audio_s, dt, **kw):
        out.append(dict({"workload": name, "sample": sample, "value": audio_s / dt, "unit": UNIT, "seconds": dt},
                        **kw))

    a, ln, _ = clip_for_config(1)
    t0 = time.perf_counter()
    O.forward_offline(a, ln, w)
    rec("offline 90 s clip", "complete", 90.0, time.perf_counter() - t0)
    t0 = time.perf_counter()
    O.forward_offline(a, ln, w, dt=np.float32)
    rec("offline 90 s clip, oracle in fp32", "complete", 90.0, time.perf_counter() - t0)

    x = hour_of_audio()
    t0 = time.perf_counter()
    O.mel_features(x[None], np.array([len(x)]))
    rec("front-end only, 1 h of audio", "complete", len(x) / 16000.0, time.perf_counter() - t0)
    del x

    for idx, name, preset, n_streams, n_steps in ((2, "Low preset, 64 x 60 s", "low", 2, 20),
                                                   (3, "Very high preset, 16 x 600 s", "very_high", 1, 3)):
        a, ln, _ = clip_for_config(idx, n_clips=n_streams)
        pre = O.PRESETS[preset]
        feats, L = O.mel_features(a, ln)
        t0 = time.perf_counter()
        frames = 0
        for i in range(n_streams):
            st = O.StreamState()
            for _ in range(n_steps):
                frames += len(O.stream_step(st, feats[i], int(L[i]), w, pre))
        dt = time.perf_counter() - t0
        rec(name, f"{n_streams} stream(s) x first {n_steps} steps (front-end untimed)", frames * 0.08, dt,
            stream_steps_per_s=n_streams * n_steps / dt)

    a, ln, _ = clip_for_config(4, n_clips=4)
    t0 = time.perf_counter()
    O.forward_offline(a, ln, w)
    rec("variable-length batch, 32 clips of 5-120 s", "first 4 clips", float(ln.sum()) / 16000.0,
        time.perf_counter() - t0)
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle as O
    from synth import FULL, clip_for_config, make_weights
    w = make_weights(FULL, seed=0)
    audio, _, _ = clip_for_config(1)
    n = 10 * 16000
    x = audio[:, :n]
    for _ in range(args.warmup):
        O.forward_offline(x, np.array([n]), w)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.forward_offline(x, np.array([n]), w)
        times.append(time.perf_counter() - t0)
    ms = 1000 * float(np.mean(times))
    v = 10.0 / (ms / 1000)
    cores = len(os.sched_getaffinity(0))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": CONFIG,
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "each step: first 10 s of the 90 s workload clip, full model, fp64 numpy"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if getattr(args, "oracle_subsets", False):
        line["subsets"] = oracle_subsets(w)
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pdl", type=int, default=1, help="programmatic dependent launch between kernels (0/1)")
    ap.add_argument("--no-streaming", action="store_true", help="skip the streaming workloads")
    ap.add_argument("--no-frontend", action="store_true", help="skip the 1 h front-end-only run")
    ap.add_argument("--no-batch", action="store_true", help="skip the 32-clip variable-length batch")
    ap.add_argument("--no-nemotron", action="store_true", help="skip the Nemotron-3 variant's offline forward")
    ap.add_argument("--mel-path", type=int, default=1, choices=[0, 1], help="front-end implementation (SF_OPT_MEL_PATH)")
    ap.add_argument("--attn-path", type=int, default=1, choices=[0, 1], help="attention kernels (SF_OPT_ATTN_PATH)")
    ap.add_argument("--sub-path", type=int, default=1, choices=[0, 1],
                    help="subsampling conv1 + first depthwise implementation (SF_OPT_SUB_PATH)")
    ap.add_argument("--tf-fuse", type=int, default=1, choices=[0, 1, 2],
                    help="fused Transformer layers (SF_OPT_TF_FUSE: 1 where one wave covers the rows, 2 always)")
    ap.add_argument("--ln-fuse", type=int, default=1, choices=[0, 1], help="LayerNorm in the residual epilogue")
    ap.add_argument("--clocks-dir", default=None, help="where to keep the raw nvidia-smi clock samples")
    ap.add_argument("--oracle-subsets", action="store_true",
                    help="with --impl reference: also time the oracle on declared subsets of every workload")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    from streaming_speaker_diarization_b200 import binding as b
    from synth import FULL, clip_for_config, make_weights, weights_blob

    audio_np, lens, _ = clip_for_config(1)
    w = make_weights(FULL, seed=0)
    eng = b.sf_create(weights_blob(w), b.default_config(max_batch=1))
    set_options(b, eng, args)
    st = torch.cuda.current_stream()
    audio = torch.from_numpy(audio_np).cuda()
    probs = torch.zeros((1, 1125, 4), device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        b.sf_forward_offline(eng, audio, lens, probs)
    torch.cuda.synchronize()
    b.sf_profile_read(eng, reset=True)

    # timed region: per-step CUDA events on the launching stream, L2 flushed between steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    clk = Clocks(local, args.clocks_dir)
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(st)
        b.sf_forward_offline(eng, audio, lens, probs)
        ev[i][1].record(st)
    barrier()
    clocks = clk.stop()
    step_ms = [a.elapsed_time(c) for a, c in ev]
    stats = b.sf_profile_read(eng, reset=True)
    launches = int(sum(v[0] for v in stats.values()))
    from streaming_speaker_diarization_b200 import dist as sd
    total_ms = float(sum(step_ms))
    max_ms = sd.max_over_ranks(total_ms, "cuda")
    audio_s = 90.0 * args.steps * world
    value = sd.throughput(90.0 * args.steps, total_ms, "cuda")

    # per-kernel attribution: the same K steps again with CUDA events around
    # every launch (shares), then with events around the GEMM launches only
    # (the roofline's kernel time, without event nodes between the others)
    b.sf_profile_enable(eng, 1)
    for i in range(args.steps):
        flush.zero_()
        b.sf_forward_offline(eng, audio, lens, probs)
    torch.cuda.synchronize()
    prof = b.sf_profile_read(eng, reset=True)
    b.sf_profile_enable(eng, 2 * (1 << 3))      # class 3 = gemm
    for i in range(args.steps):
        flush.zero_()
        b.sf_forward_offline(eng, audio, lens, probs)
    torch.cuda.synchronize()
    prof_gemm = b.sf_profile_read(eng, reset=True)
    b.sf_profile_enable(eng, 0)

    # end to end through the host-memory entry point (H2D + compute + D2H every step)
    h_audio = torch.from_numpy(audio_np).pin_memory()
    h_probs = torch.zeros((1, 1125, 4)).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    b.sf_forward_offline_host(eng, h_audio.numpy(), lens, h_probs.numpy())
    barrier()
    for i in range(args.steps):
        flush.zero_()
        e2e_ev[i][0].record(st)
        b.sf_forward_offline_host(eng, h_audio.numpy(), lens, h_probs.numpy())
        e2e_ev[i][1].record(st)
    barrier()
    e2e_ms = float(sum(a.elapsed_time(c) for a, c in e2e_ev))
    e2e_value = sd.throughput(90.0 * args.steps, e2e_ms, "cuda")

    pk, pk_kind = peaks()
    g = prof_gemm.get("gemm", (0, 0.0, 0.0, 0.0))
    traffic = gemm_traffic_per_launch()
    timed_s = max_ms / 1000.0
    peak_tf = pk["bf16_tflops_sustained"] if timed_s > 1.0 else pk["bf16_tflops"]
    achieved = (g[2] / (g[1] / 1000.0)) / 1e12 if g[1] > 0 else None
    roof = {"bound": "tensor", "kernel": "gemm (all projection launches)", "achieved": achieved, "peak": peak_tf,
            "unit": "TFLOP/s", "frac": (achieved / peak_tf) if achieved else None, "traffic": traffic,
            "traffic_unit": "bytes per launch (DRAM read + write, mean over the forward's projections)",
            "peak_kind": f"{pk_kind} bf16 {'sustained' if timed_s > 1.0 else 'burst'}",
            "launches_per_step": g[0] / args.steps if args.steps else None,
            "ms_per_step": g[1] / args.steps if args.steps else None}
    kernels = {k: {"launches": int(v[0]), "ms": round(v[1], 4),
                   "tflops": round(v[2] / (v[1] / 1000) / 1e12, 2) if v[1] > 0 and v[2] > 0 else None,
                   "gbs": round(v[3] / (v[1] / 1000) / 1e9, 1) if v[1] > 0 and v[3] > 0 else None}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(CONFIG, parallelism=f"replicas x{world}", mel_path=args.mel_path, sub_path=args.sub_path,
                           attn_path=args.attn_path, tf_fuse=args.tf_fuse, ln_fuse=args.ln_fuse, pdl=args.pdl),
            "roofline": roof, "clocks": clocks, "gpu_launches": launches,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(audio_np.nbytes),
                    "d2h_bytes_per_step": int(h_probs.numel() * 4)},
            "step_ms_p50": float(np.median(step_ms)), "step_ms_p95": float(np.percentile(step_ms, 95)),
            "kernels": kernels}
    b.sf_destroy(eng)
    if not args.no_streaming:
        line["streaming"] = streaming_bench(b, torch, weights_blob(w), rank, world, local, args, args.clocks_dir)
    if not args.no_nemotron and world == 1:
        line["nemotron"] = nemotron_bench(b, torch, args.steps, max(args.warmup, 3), local, args.clocks_dir)
    if not args.no_batch and world == 1:
        line["batch"] = batch_bench(b, torch, weights_blob(w), args.steps, max(args.warmup, 3), local, args,
                                    args.clocks_dir)
    if not args.no_frontend:
        line["frontend_1h"] = frontend_bench(b, torch, weights_blob(w), max(args.steps, 5), max(args.warmup, 3),
                                             args.mel_path)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(audio_np)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
