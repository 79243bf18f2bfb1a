"""CPU checks of the C-ABI library: it loads, and exports every entry point
include/sf.h declares (no compute calls: there is no GPU here)."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    src = open(os.path.join(ROOT, "include", "sf.h")).read()
    return sorted(set(re.findall(r"^SF_API\s+[\w\s\*]+?\b(sf_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib_path():
    from streaming_speaker_diarization_b200 import build
    return build.build()


def test_header_declares_the_boundary():
    names = declared()
    for n in ("sf_create", "sf_mel", "sf_forward_offline", "sf_stream_step", "sf_stream_reset"):
        assert n in names
    assert len(names) >= 21


def test_library_exports_every_declared_symbol(lib_path):
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True, check=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if l.strip()}
    missing = [n for n in declared() if n not in syms]
    assert not missing, missing


def test_binding_loads_and_covers_the_header(lib_path):
    from streaming_speaker_diarization_b200 import binding as b
    assert sorted(b.EXPORTED) == declared()
    c = b.default_config()
    assert (c.n_conformer, c.n_transformer, c.d_model, c.tf_d_model, c.spkcache_len, c.max_samples) == \
        (17, 18, 512, 192, 188, 1920000)
    assert b.lib.sf_status_str(2) == b"size out of range"


def test_create_without_device_fails_cleanly(lib_path):
    """No GPU here: sf_create must return an error code, not crash."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from streaming_speaker_diarization_b200 import binding as b
    from synth import TINY, make_weights, weights_blob
    with pytest.raises(b.SFError):
        b.sf_create(weights_blob(make_weights(TINY)), b.default_config(n_conformer=2, n_transformer=2))


def test_header_is_plain_c(tmp_path):
    """include/sf.h compiles as strict C99 and as C++17 (no torch or CUDA
    types in the boundary)."""
    import shutil
    src = tmp_path / "use_sf.c"
    src.write_text('#include "sf.h"\nint main(void) { sf_config c; sf_seg_params p;\n'
                   '  return sf_default_config(&c) + sf_default_seg_params(&p); }\n')
    inc = os.path.join(ROOT, "include")
    for cc, std, lang in (("gcc", "-std=c99", "c"), ("g++", "-std=c++17", "c++")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not available")
        r = subprocess.run([cc, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-x", lang, "-I", inc, "-c", str(src),
                            "-o", str(tmp_path / f"o_{lang}.o")], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_host_only_entries_work_without_a_device(lib_path):
    """Defaults and status strings are host functions: usable on a machine
    without a GPU."""
    from streaming_speaker_diarization_b200 import binding as b
    p = b.seg_params()
    assert (p.onset, p.offset, p.pad_onset, p.pad_offset, p.min_duration_on, p.min_duration_off) == \
        (0.5, 0.5, 0.0, 0.0, 0.0, 0.0)
    q = b.seg_params(onset=0.7, min_duration_off=0.2)
    assert abs(q.onset - 0.7) < 1e-7 and q.min_duration_off == 0.2 and q.offset == 0.5
    c = b.default_config()
    assert c.sample_rate == 16000 and c.n_conformer == 17 and c.n_transformer == 18
    assert b.lib.sf_status_str(0)
