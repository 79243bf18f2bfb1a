"""ctypes binding of libsf.so (include/sf.h), argument marshalling only.

Every call below forwards to the C function of the same name.  Device
buffers are torch CUDA tensors (their data pointers are passed), host arrays
are numpy arrays, and `stream` defaults to torch's current CUDA stream.
The library must have been built (``build.py``); importing this module on a
machine without it raises immediately -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsf.so")

SF_FP32, SF_BF16 = 0, 1
SF_OPT_GRAPHS, SF_OPT_PDL, SF_OPT_GEMM_PATH, SF_OPT_GEMM_PAIR_BN, SF_OPT_ATTN_PATH, SF_OPT_MEL_PATH = 1, 2, 3, 4, 5, 6
SF_OPT_SUB_PATH = 7
SF_OPT_LN_FUSE = 8
SF_OPT_TF_FUSE = 9
STATUS = {0: "SF_OK", 1: "SF_EINVAL", 2: "SF_ESHAPE", 3: "SF_ENOMEM", 4: "SF_ECUDA", 5: "SF_ESTATE",
          6: "SF_ETIMEOUT", 7: "SF_EDEVICE", 8: "SF_EFORMAT"}

_CFG_INT_FIELDS = ["sample_rate", "n_mels", "n_fft", "win_length", "hop_length", "subsampling", "d_model",
                   "tf_d_model", "n_conformer", "n_transformer", "n_heads", "ff_mult", "tf_ff", "conv_kernel",
                   "n_spk", "spkcache_len", "precision", "max_batch"]


class sf_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in _CFG_INT_FIELDS] + [("max_samples", ctypes.c_int64)]


class sf_preset(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("chunk_len", "right_context", "fifo_len", "update_period", "spkcache_len")]


class sf_state_view(ctypes.Structure):
    _fields_ = [("n_cache", ctypes.c_int), ("n_fifo", ctypes.c_int), ("next_frame", ctypes.c_int64),
                ("finished", ctypes.c_int), ("sil_count", ctypes.c_int),
                ("d_cache_emb", ctypes.c_void_p), ("d_cache_preds", ctypes.c_void_p),
                ("d_fifo_emb", ctypes.c_void_p), ("d_fifo_preds", ctypes.c_void_p), ("d_sil_mean", ctypes.c_void_p)]


class sf_seg_params(ctypes.Structure):
    _fields_ = [("onset", ctypes.c_float), ("offset", ctypes.c_float), ("pad_onset", ctypes.c_double),
                ("pad_offset", ctypes.c_double), ("min_duration_on", ctypes.c_double),
                ("min_duration_off", ctypes.c_double)]


class sf_nem_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("ff", ctypes.c_int), ("n_spk", ctypes.c_int),
                ("max_batch", ctypes.c_int), ("max_samples", ctypes.c_int64)]


class sf_kernel_stat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


EXPORTED = ["sf_default_config", "sf_create", "sf_create_from_file", "sf_destroy", "sf_get_metadata",
            "sf_last_error", "sf_status_str", "sf_mel", "sf_pre_encode", "sf_encode", "sf_forward_offline",
            "sf_forward_offline_host", "sf_stream_create", "sf_stream_destroy", "sf_stream_reset",
            "sf_stream_window", "sf_stream_step", "sf_stream_get_state", "sf_stream_set_state",
            "sf_stream_update", "sf_select_topk", "sf_profile_enable", "sf_profile_read", "sf_mel_noalloc",
            "sf_check", "sf_gemm_bf16", "sf_set_option", "sf_attention_relpos", "sf_default_seg_params",
            "sf_segments", "sf_stream_step_audio", "sf_attention_mha", "sf_selftest_wait", "sf_gemm_bf16_ln", "sf_nem_default_config", "sf_nem_create",
            "sf_nem_destroy", "sf_nem_forward_offline", "sf_nem_last_error"]


class SFError(RuntimeError):
    pass


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsf.so not built ({LIB_PATH}); run streaming_speaker_diarization_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, VP = ctypes.POINTER, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
    sig = {
        "sf_default_config": ([P(sf_config)], I),
        "sf_create": ([VP, ctypes.c_uint64, P(sf_config), P(VP)], I),
        "sf_create_from_file": ([ctypes.c_char_p, P(sf_config), P(VP)], I),
        "sf_destroy": ([VP], I),
        "sf_get_metadata": ([VP, P(sf_config)], I),
        "sf_last_error": ([VP], ctypes.c_char_p),
        "sf_status_str": ([I], ctypes.c_char_p),
        "sf_mel": ([VP, VP, VP, I, I64, VP, VP, VP], I),
        "sf_pre_encode": ([VP, VP, I, I64, VP, VP, VP, I, VP, I64, VP], I),
        "sf_encode": ([VP, VP, VP, I, VP, VP], I),
        "sf_forward_offline": ([VP, VP, VP, I, I64, VP, VP, VP], I),
        "sf_forward_offline_host": ([VP, VP, VP, I, I64, VP, VP, VP], I),
        "sf_stream_create": ([VP, P(sf_preset), I, P(VP)], I),
        "sf_stream_destroy": ([VP], I),
        "sf_stream_reset": ([VP, VP, I], I),
        "sf_stream_window": ([VP, I, I64, P(I64), P(I64)], I),
        "sf_stream_step": ([VP, VP, I64, VP, VP, VP, VP, VP], I),
        "sf_stream_get_state": ([VP, I, P(sf_state_view), VP], I),
        "sf_stream_set_state": ([VP, I, P(sf_state_view), VP], I),
        "sf_stream_update": ([VP, VP, VP, I64, VP, VP, VP, VP, VP], I),
        "sf_select_topk": ([VP, VP, VP, I, I, I, VP, VP], I),
        "sf_profile_enable": ([VP, I], I),
        "sf_profile_read": ([VP, P(sf_kernel_stat), I, P(I), I], I),
        "sf_mel_noalloc": ([VP, VP, I, I64, VP, VP, VP], I),
        "sf_check": ([VP, VP], I),
        "sf_selftest_wait": ([VP, VP], I),
        "sf_set_option": ([VP, I, I], I),
        "sf_gemm_bf16": ([VP, VP, I, VP, I, I, I, VP, VP, I, VP], I),
        "sf_gemm_bf16_ln": ([VP, VP, I, VP, I, I, I, VP, ctypes.c_float, VP, VP, VP, VP, VP, I, VP, VP], I),
        "sf_attention_relpos": ([VP, VP, VP, I, VP, VP, VP, I, VP, I, VP], I),
        "sf_default_seg_params": ([P(sf_seg_params)], I),
        "sf_segments": ([VP, VP, I, VP, I, P(sf_seg_params), I, VP, VP, VP], I),
        "sf_stream_step_audio": ([VP, VP, I64, VP, VP, VP, VP, VP, VP], I),
        "sf_attention_mha": ([VP, VP, VP, I, VP, I, VP], I),
        "sf_nem_default_config": ([P(sf_nem_config)], I),
        "sf_nem_create": ([VP, ctypes.c_uint64, P(sf_nem_config), P(VP)], I),
        "sf_nem_destroy": ([VP], I),
        "sf_nem_forward_offline": ([VP, VP, VP, I, I64, VP, VP, VP], I),
        "sf_nem_last_error": ([VP], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


lib = _load()


def _ptr(t):
    """Device pointer of a torch tensor, host pointer of a numpy array, or None."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        assert t.flags["C_CONTIGUOUS"]
        return t.ctypes.data
    if isinstance(t, int):
        return t
    assert t.is_contiguous()
    return t.data_ptr()


def _stream(s):
    if s is not None:
        return s
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(rc, eng=None):
    if rc != 0:
        msg = lib.sf_last_error(eng).decode() if eng else ""
        raise SFError(f"{STATUS.get(rc, rc)}: {msg}")


def default_config(**kw):
    c = sf_config()
    _check(lib.sf_default_config(ctypes.byref(c)))
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def sf_create(blob: bytes, cfg: sf_config):
    h = ctypes.c_void_p()
    buf = ctypes.create_string_buffer(blob, len(blob))
    rc = lib.sf_create(ctypes.cast(buf, ctypes.c_void_p), len(blob), ctypes.byref(cfg), ctypes.byref(h))
    if rc != 0:
        raise SFError(f"sf_create: {STATUS.get(rc, rc)}")
    return h.value


def sf_destroy(eng):
    _check(lib.sf_destroy(eng))


def sf_get_metadata(eng):
    c = sf_config()
    _check(lib.sf_get_metadata(eng, ctypes.byref(c)), eng)
    return c


def sf_mel(eng, audio, lengths, mel, stream=None):
    lengths = np.ascontiguousarray(lengths, np.int64)
    out_len = np.zeros_like(lengths)
    B, N = audio.shape
    _check(lib.sf_mel(eng, _ptr(audio), _ptr(lengths), B, N, _ptr(mel), _ptr(out_len), _stream(stream)), eng)
    return out_len


def sf_mel_noalloc(audio, lengths, mel, stream=None):
    """Allocation-free front-end (no engine); same result as sf_mel."""
    lengths = np.ascontiguousarray(lengths, np.int64)
    out_len = np.zeros_like(lengths)
    B, N = audio.shape
    _check(lib.sf_mel_noalloc(_ptr(audio), _ptr(lengths), B, N, _ptr(mel), _ptr(out_len), _stream(stream)))
    return out_len


def sf_pre_encode(eng, feats, buf_idx, start, frames, embs, emb_stride, stream=None):
    buf_idx = np.ascontiguousarray(buf_idx, np.int32)
    start = np.ascontiguousarray(start, np.int64)
    frames = np.ascontiguousarray(frames, np.int64)
    n_buf, _, t_buf = feats.shape
    _check(lib.sf_pre_encode(eng, _ptr(feats), n_buf, t_buf, _ptr(buf_idx), _ptr(start), _ptr(frames), len(frames),
                             _ptr(embs), emb_stride, _stream(stream)), eng)


def sf_encode(eng, embs, seq_len, preds, stream=None):
    seq_len = np.ascontiguousarray(seq_len, np.int32)
    _check(lib.sf_encode(eng, _ptr(embs), _ptr(seq_len), len(seq_len), _ptr(preds), _stream(stream)), eng)


def sf_forward_offline(eng, audio, lengths, probs, stream=None):
    lengths = np.ascontiguousarray(lengths, np.int64)
    out_len = np.zeros_like(lengths)
    B, N = audio.shape
    _check(lib.sf_forward_offline(eng, _ptr(audio), _ptr(lengths), B, N, _ptr(probs), _ptr(out_len),
                                  _stream(stream)), eng)
    return out_len


def sf_forward_offline_host(eng, audio, lengths, probs, stream=None):
    lengths = np.ascontiguousarray(lengths, np.int64)
    out_len = np.zeros_like(lengths)
    B, N = audio.shape
    _check(lib.sf_forward_offline_host(eng, _ptr(audio), _ptr(lengths), B, N, _ptr(probs), _ptr(out_len),
                                       _stream(stream)), eng)
    return out_len


def sf_stream_create(eng, preset, n_streams):
    p = sf_preset(*preset) if not isinstance(preset, sf_preset) else preset
    h = ctypes.c_void_p()
    _check(lib.sf_stream_create(eng, ctypes.byref(p), n_streams, ctypes.byref(h)), eng)
    return h.value


def sf_stream_destroy(st):
    _check(lib.sf_stream_destroy(st))


def sf_stream_reset(st, ids=None):
    if ids is None:
        _check(lib.sf_stream_reset(st, None, 0))
    else:
        ids = np.ascontiguousarray(ids, np.int32)
        _check(lib.sf_stream_reset(st, _ptr(ids), len(ids)))


def sf_stream_window(st, sid, total):
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(lib.sf_stream_window(st, sid, total, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def sf_stream_step(eng, st, feats, feat_start, feat_end, chunk_probs, stream=None):
    feat_start = np.ascontiguousarray(feat_start, np.int64)
    feat_end = np.ascontiguousarray(feat_end, np.int64)
    n_out = np.zeros(len(feat_start), np.int32)
    _check(lib.sf_stream_step(st, _ptr(feats), feats.shape[-1], _ptr(feat_start), _ptr(feat_end), _ptr(chunk_probs),
                              _ptr(n_out), _stream(stream)), eng)
    return n_out


def sf_stream_step_audio(eng, st, audio, audio_start, audio_end, final, chunk_probs, stream=None):
    """audio: device f32 [n_streams, n_buf]; returns frames emitted per stream."""
    audio_start = np.ascontiguousarray(audio_start, np.int64)
    audio_end = np.ascontiguousarray(audio_end, np.int64)
    final = np.ascontiguousarray(final, np.int32)
    n_out = np.zeros(len(audio_start), np.int32)
    _check(lib.sf_stream_step_audio(st, _ptr(audio), audio.shape[1], _ptr(audio_start), _ptr(audio_end), _ptr(final),
                                    _ptr(chunk_probs), _ptr(n_out), _stream(stream)), eng)
    return n_out


def sf_stream_get_state(eng, st, sid, view, stream=None):
    _check(lib.sf_stream_get_state(st, sid, ctypes.byref(view), _stream(stream)), eng)
    return view


def sf_stream_set_state(eng, st, sid, view, stream=None):
    _check(lib.sf_stream_set_state(st, sid, ctypes.byref(view), _stream(stream)), eng)


def sf_stream_update(eng, st, preds, new_embs, new_stride, n_new, scores=None, src=None, scores_in=None,
                     stream=None):
    n_new = np.ascontiguousarray(n_new, np.int32)
    _check(lib.sf_stream_update(st, _ptr(preds), _ptr(new_embs), new_stride, _ptr(n_new), _ptr(scores), _ptr(src),
                                _ptr(scores_in), _stream(stream)), eng)


def sf_select_topk(eng, scores, n, k, src, stream=None):
    n = np.ascontiguousarray(n, np.int32)
    n_sets, stride, _ = scores.shape
    _check(lib.sf_select_topk(eng, _ptr(scores), _ptr(n), n_sets, stride, k, _ptr(src), _stream(stream)), eng)


def sf_profile_enable(eng, enable=1):
    """0 = off, 1 = every kernel class, 2 * mask = the classes in mask."""
    _check(lib.sf_profile_enable(eng, int(enable)), eng)


def sf_profile_read(eng, reset=True):
    """Per kernel class: dict name -> (launches, ms, flops, bytes)."""
    arr = (sf_kernel_stat * 32)()
    n = ctypes.c_int()
    _check(lib.sf_profile_read(eng, arr, 32, ctypes.byref(n), int(bool(reset))), eng)
    return {arr[i].name.decode(): (arr[i].launches, arr[i].ms, arr[i].flops, arr[i].bytes) for i in range(n.value)}


def sf_check(eng, stream=None):
    _check(lib.sf_check(eng, _stream(stream)), eng)


def sf_selftest_wait(eng, stream=None):
    """Enqueue the failure-detection self-test (a bounded device wait that
    runs out after about 2 s); the next sf_check raises SF_ETIMEOUT."""
    _check(lib.sf_selftest_wait(eng, _stream(stream)), eng)


def sf_gemm_bf16(eng, A, W, C, bias=None, path=1, stream=None):
    M, K = A.shape
    N = W.shape[0]
    _check(lib.sf_gemm_bf16(eng, _ptr(A), A.stride(0), _ptr(W), M, N, K, _ptr(bias), _ptr(C), path,
                            _stream(stream)), eng)


def sf_gemm_bf16_ln(eng, A, W, x, g, b, h, bias=None, alpha=1.0, xnorm=0, g2=None, b2=None, stream=None):
    """Residual projection + LayerNorm in one launch: see sf.h."""
    M, K = A.shape
    N = W.shape[0]
    _check(lib.sf_gemm_bf16_ln(eng, _ptr(A), A.stride(0), _ptr(W), M, N, K, _ptr(bias), ctypes.c_float(alpha),
                               _ptr(x), _ptr(g), _ptr(b), _ptr(g2), _ptr(b2), int(xnorm), _ptr(h), _stream(stream)),
           eng)


def sf_attention_relpos(eng, qkv, ptab, R, u, v, seq_len, ctx, path=1, stream=None):
    seq_len = np.ascontiguousarray(seq_len, np.int32)
    _check(lib.sf_attention_relpos(eng, _ptr(qkv), _ptr(ptab), R, _ptr(u), _ptr(v), _ptr(seq_len), len(seq_len),
                                   _ptr(ctx), path, _stream(stream)), eng)


def sf_attention_mha(eng, qkv, seq_len, ctx, path=1, stream=None):
    seq_len = np.ascontiguousarray(seq_len, np.int32)
    _check(lib.sf_attention_mha(eng, _ptr(qkv), _ptr(seq_len), len(seq_len), _ptr(ctx), path, _stream(stream)), eng)


def seg_params(**kw):
    p = sf_seg_params()
    _check(lib.sf_default_seg_params(ctypes.byref(p)))
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def sf_segments(eng, probs, n_frames, params=None, max_seg=256, stream=None):
    """probs: device f32 [n, T, 4]; returns (segs f64 [n, 4, max_seg, 2], counts i32 [n, 4]) on the device."""
    import torch
    n, T = probs.shape[0], probs.shape[1]
    n_frames = np.ascontiguousarray(n_frames, np.int32)
    segs = torch.zeros((n, 4, max_seg, 2), dtype=torch.float64, device=probs.device)
    counts = torch.zeros((n, 4), dtype=torch.int32, device=probs.device)
    p = params if params is not None else seg_params()
    _check(lib.sf_segments(eng, _ptr(probs), T, _ptr(n_frames), n, ctypes.byref(p), max_seg, _ptr(segs),
                           _ptr(counts), _stream(stream)), eng)
    return segs, counts


def sf_set_option(eng, option, value):
    _check(lib.sf_set_option(eng, option, value), eng)


# ---------------------------------------------------------- Nemotron-3 variant

def nem_default_config(**kw):
    c = sf_nem_config()
    _check(lib.sf_nem_default_config(ctypes.byref(c)))
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def sf_nem_create(blob, cfg):
    out = ctypes.c_void_p()
    rc = lib.sf_nem_create(blob, len(blob), ctypes.byref(cfg), ctypes.byref(out))
    if rc != 0:
        raise SFError(f"{STATUS.get(rc, rc)}: sf_nem_create")
    return out


def sf_nem_destroy(eng):
    _check(lib.sf_nem_destroy(eng))


def sf_nem_forward_offline(eng, audio, lengths, probs, stream=None):
    """audio: device f32 [B, n_max]; probs: device f32 [B, n_max // 160, 8]."""
    lengths = np.ascontiguousarray(lengths, np.int64)
    out_len = np.zeros_like(lengths)
    B, N = audio.shape
    rc = lib.sf_nem_forward_offline(eng, _ptr(audio), _ptr(lengths), B, N, _ptr(probs), _ptr(out_len),
                                    _stream(stream))
    if rc != 0:
        raise SFError(f"{STATUS.get(rc, rc)}: {lib.sf_nem_last_error(eng).decode()}")
    return out_len
