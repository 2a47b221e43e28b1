"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point declared in include/*.h, lays out the weight blob exactly as
the input generator packs it, and rejects bad arguments before touching the
device."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

from oracle import w2v_oracle as O
from speech_encoder_b200 import w2v as B
from synth import inputs as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        for m in re.finditer(r"\b(w2v_[a-z0-9_]+)\s*\(", txt):
            names.add(m.group(1))
    return names


def test_library_builds_and_exports_every_declared_symbol():
    from speech_encoder_b200.build import build
    path = build()
    assert os.path.exists(path)
    L = B.lib()
    declared = _declared_symbols()
    assert {"w2v_create", "w2v_forward", "w2v_ctc_greedy", "w2v_destroy"} <= declared
    for name in declared:
        assert hasattr(L, name), name


def test_num_frames_matches_closed_form():
    for n in list(range(0, 2000, 7)) + [16000, 59200, 160000, 256000, 320000, 399, 400, 719, 720]:
        assert B.w2v_num_frames(n) == O.num_frames(n), n


@pytest.mark.parametrize("shape", [S.BASE, S.LARGE, S.small_shape(), S.small_shape(conv_norm="layer", stable=True,
                                                                                   conv_bias=True)])
def test_manifest_matches_input_generator(shape):
    cfg = B.make_config(shape, 256000, 1)
    lib_m = B.w2v_weight_manifest(cfg)
    gen_m = S.weight_manifest(shape)
    assert [(n, tuple(s)) for n, s, _ in lib_m] == [(n, tuple(s)) for n, s in gen_m]
    off = 0
    for (n, s, o) in lib_m:
        assert o == off, n
        off += int(np.prod(s))
    assert B.w2v_weight_count(cfg) == off


def test_invalid_configs_rejected_on_host():
    L = B.lib()
    good = B.make_config(S.BASE, 256000, 1)
    assert L.w2v_weight_count(ctypes.byref(good)) > 0
    for field, bad in [("d_model", 700), ("n_heads", 5), ("d_ffn", 100), ("vocab", 0), ("blank_id", 32),
                       ("conv_norm", 2), ("max_samples", 399), ("max_batch", 0), ("ln_eps", 0.0), ("n_layers", -1)]:
        cfg = B.make_config(S.BASE, 256000, 1)
        setattr(cfg, field, bad)
        assert L.w2v_weight_count(ctypes.byref(cfg)) == 0, field
        h = ctypes.c_void_p()
        blob = np.zeros(4, np.float32)
        assert L.w2v_create(ctypes.byref(cfg), blob.ctypes.data, blob.size, ctypes.byref(h)) == B.W2V_EINVAL, field
        assert not h.value


def test_blob_size_mismatch_and_null_args():
    L = B.lib()
    cfg = B.make_config(S.small_shape(), 16000, 1)
    h = ctypes.c_void_p()
    blob = np.zeros(10, np.float32)
    assert L.w2v_create(ctypes.byref(cfg), blob.ctypes.data, blob.size, ctypes.byref(h)) == B.W2V_ESHAPE
    assert L.w2v_create(ctypes.byref(cfg), None, 0, ctypes.byref(h)) == B.W2V_EINVAL
    assert L.w2v_create(ctypes.byref(cfg), blob.ctypes.data, blob.size, None) == B.W2V_EINVAL
    assert L.w2v_forward(None, None, 16000, 1, None, None) == B.W2V_EINVAL
    assert L.w2v_ctc_greedy(None, None, 1, 1, 1, None, None, None) == B.W2V_EINVAL
    assert L.w2v_sync(None, None) == B.W2V_EINVAL
    L.w2v_destroy(None)
    err = np.zeros(1, np.int32)
    assert L.w2v_op_gemm(None, None, 1, 1, 64, None, None, 0, None, 0, 0, 0, 1, None, None) == B.W2V_EINVAL
    assert L.w2v_op_wait_probe(None, 1000, None) == B.W2V_EINVAL
    assert L.w2v_op_layernorm(None, 0, None, 1, 512, None, None, 1e-5, 0, None) == B.W2V_EINVAL


def test_create_without_gpu_reports_device_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible")
    sh = S.small_shape()
    blob = S.pack_blob(sh, S.init_weights(sh, 0))
    cfg = B.make_config(sh, 16000, 1)
    L = B.lib()
    h = ctypes.c_void_p()
    assert L.w2v_create(ctypes.byref(cfg), blob.ctypes.data, blob.size, ctypes.byref(h)) == B.W2V_EDEVICE


def test_num_windows_host_arithmetic():
    assert B.w2v_num_windows(256000, 256000) == 1
    assert B.w2v_num_windows(256001, 256000) == 2
    assert B.w2v_num_windows(1, 160000) == 1
    assert B.w2v_num_windows(0, 160000) == 0
    assert B.w2v_num_windows(10, 0) == 0


def _prototypes():
    """name -> parameter count of every w2v_* function declared in include/*.h."""
    protos = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for m in re.finditer(r"\b(w2v_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", txt, flags=re.S):
            params = m.group(2).strip()
            protos[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_signatures_match_the_headers():
    # every entry point the binding types must take as many arguments as the
    # header declares (guards the ctypes table against drift)
    protos = _prototypes()
    L = B.lib()
    typed = [n for n in protos if getattr(getattr(L, n), "argtypes", None) is not None]
    assert len(typed) >= 20
    for n in typed:
        assert len(getattr(L, n).argtypes) == protos[n], (n, len(getattr(L, n).argtypes), protos[n])


def test_host_side_argument_checks_need_no_device():
    L = B.lib()
    assert L.w2v_window_pcm(None, 10, 4, None, None) == B.W2V_EINVAL
    buf = ctypes.create_string_buffer(64)
    cfg = B.make_config(S.small_shape(), 48000, 1)
    h = ctypes.c_void_p()
    assert L.w2v_create_from_safetensors(b"/nonexistent/model.safetensors", ctypes.byref(cfg), ctypes.byref(h),
                                         buf, 64) == B.W2V_EINVAL
    assert h.value is None and b"cannot open" in buf.value
    blob = np.zeros(B.w2v_weight_count(cfg), dtype=np.float32)
    assert L.w2v_pack_safetensors(b"x", ctypes.byref(cfg), blob.ctypes.data, blob.size - 1, buf, 64) == B.W2V_ESHAPE
