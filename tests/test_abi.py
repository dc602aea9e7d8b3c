"""The C-ABI library: it loads, exports every symbol the header declares, and rejects bad
arguments before touching a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kie():
    from bandwidth_bound_stream_b200 import build
    build.build_kie()
    from bandwidth_bound_stream_b200 import kie as k
    return k


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(kie_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(kie):
    declared = _declared()
    assert declared, "no declarations found"
    missing = [n for n in sorted(declared) if not hasattr(kie.lib, n)]
    assert not missing, missing
    assert declared == set(kie.EXPORTS)


def test_defaults_and_status_strings(kie):
    c = kie.KieConfig()
    kie.lib.kie_config_defaults(ctypes.byref(c))
    assert c.max_ctx == 4096 and c.modes == kie.KIE_MODE_BATCH1 and abs(c.rms_eps - 1e-5) < 1e-9
    assert kie.lib.kie_status_string(kie.KIE_ERR_CAPACITY) == b"capacity exceeded"


def test_create_rejects_bad_shapes_without_a_gpu(kie):
    from bandwidth_bound_stream_b200 import synth
    h = ctypes.c_void_p()
    w = kie.KieWeights()
    cfg = kie.config(synth.TINY)
    assert kie.lib.kie_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == kie.KIE_ERR_ARG  # null weights
    dummy = (ctypes.c_void_p * 18)(*([16] * 18))
    w = kie.KieWeights(16, ctypes.cast(dummy, ctypes.POINTER(ctypes.c_void_p)), 16, 16)
    for field, bad in [("d_model", 100), ("head_dim", 48), ("n_kv_heads", 3), ("max_ctx", 0), ("dtype", 7)]:
        c = kie.config(synth.TINY)
        setattr(c, field, bad)
        assert kie.lib.kie_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == kie.KIE_ERR_ARG, field
        assert not h.value


def test_flash_decode_argument_checks(kie):
    assert kie.flash_decode_scratch_bytes(16, 8, 128, 1280) > 0
    assert kie.flash_decode_scratch_bytes(16, 3, 128, 10) == -1
    assert kie.flash_decode(16, 16, 16, 16, 8, 100, 10, 10, 0, 16, 16, 1 << 20) == kie.KIE_ERR_ARG  # head_dim
    assert kie.flash_decode(16, 16, 16, 16, 8, 128, 10, 5, 0, 16, 16, 1 << 20) == kie.KIE_ERR_ARG  # stride < ctx
    assert kie.flash_decode(16, 16, 16, 16, 8, 128, 10, 10, 0, 16, 16, 8) == kie.KIE_ERR_ARG  # scratch too small
