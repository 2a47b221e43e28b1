"""Thin ctypes binding of libw2v.so: the C entry points under the same names,
with argument marshalling only (torch tensors -> device pointers, the current
torch CUDA stream -> cudaStream_t).  Every step of the forward pass runs in the
library's CUDA kernels; if the library is missing this module raises instead
of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libw2v.so")

W2V_OK, W2V_EINVAL, W2V_ESHAPE, W2V_ENOMEM, W2V_ECUDA, W2V_EDEVICE, W2V_ETIMEOUT = range(7)
_NAMES = {0: "W2V_OK", 1: "W2V_EINVAL", 2: "W2V_ESHAPE", 3: "W2V_ENOMEM", 4: "W2V_ECUDA", 5: "W2V_EDEVICE",
          6: "W2V_ETIMEOUT"}


class W2VError(RuntimeError):
    def __init__(self, code: int, msg: str = ""):
        super().__init__(f"{_NAMES.get(code, code)}: {msg}")
        self.code = code


class w2v_config(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int), ("n_layers", ctypes.c_int), ("n_heads", ctypes.c_int), ("d_ffn", ctypes.c_int),
        ("vocab", ctypes.c_int), ("blank_id", ctypes.c_int), ("conv_norm", ctypes.c_int), ("conv_bias", ctypes.c_int),
        ("stable_layer_norm", ctypes.c_int), ("gelu_tanh", ctypes.c_int), ("max_samples", ctypes.c_int),
        ("max_batch", ctypes.c_int), ("ln_eps", ctypes.c_float), ("use_cuda_graph", ctypes.c_int),
    ]


class w2v_kernel_time(ctypes.Structure):
    _fields_ = [("klass", ctypes.c_int), ("ms", ctypes.c_float), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


_lib: Optional[ctypes.CDLL] = None
VP, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Loads libw2v.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m speech_encoder_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "w2v_num_frames": (I, [I]),
        "w2v_weight_count": (SZ, [ctypes.POINTER(w2v_config)]),
        "w2v_weight_num_entries": (I, [ctypes.POINTER(w2v_config)]),
        "w2v_weight_entry": (I, [ctypes.POINTER(w2v_config), I, ctypes.c_char_p, SZ, ctypes.POINTER(I),
                                 ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(SZ)]),
        "w2v_create": (I, [ctypes.POINTER(w2v_config), VP, SZ, ctypes.POINTER(VP)]),
        "w2v_num_windows": (I, [I, I]),
        "w2v_window_pcm": (I, [VP, I, I, VP, VP]),
        "w2v_pack_safetensors": (I, [ctypes.c_char_p, ctypes.POINTER(w2v_config), VP, SZ, ctypes.c_char_p, SZ]),
        "w2v_create_from_safetensors": (I, [ctypes.c_char_p, ctypes.POINTER(w2v_config), ctypes.POINTER(VP),
                                            ctypes.c_char_p, SZ]),
        "w2v_forward": (I, [VP, VP, I, I, VP, VP]),
        "w2v_ctc_greedy": (I, [VP, VP, I, I, I, VP, VP, VP]),
        "w2v_sync": (I, [VP, VP]),
        "w2v_forward_varlen": (I, [VP, VP, ctypes.POINTER(I), I, VP, VP]),
        "w2v_ctc_greedy_varlen": (I, [VP, VP, ctypes.POINTER(I), I, VP, VP, VP]),
        "w2v_debug_read": (I, [VP, I, VP, SZ, ctypes.POINTER(SZ), VP]),
        "w2v_last_error": (I, [VP, ctypes.c_char_p, SZ]),
        "w2v_destroy": (None, [VP]),
        "w2v_transcribe": (I, [VP, VP, I, I, I, VP, VP, VP]),
        "w2v_ctc_greedy_static": (I, [VP, I, I, I, I, I, VP, VP, VP]),
        "w2v_last_launch_count": (I, [VP]),
        "w2v_kernel_class_name": (ctypes.c_char_p, [I]),
        "w2v_profile_forward": (I, [VP, VP, I, I, VP, VP, ctypes.POINTER(w2v_kernel_time), I, ctypes.POINTER(I)]),
        "w2v_time_class": (I, [VP, VP, I, I, VP, I, I, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(I),
                               ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double), VP]),
        "w2v_op_gemm": (I, [VP, VP, I, I, I, VP, VP, I, VP, I, I, I, I, VP, VP]),
        "w2v_op_attention": (I, [VP, VP, VP, VP, I, I, I, I, VP, VP]),
        "w2v_op_layernorm": (I, [VP, I, VP, I, I, VP, VP, ctypes.c_float, I, VP]),
        "w2v_op_wait_probe": (I, [VP, ctypes.c_uint64, VP]),
        "w2v_op_pointwise": (I, [I, VP, I, ctypes.c_float, ctypes.c_float, VP, VP]),
        "w2v_fold_layernorm_linear": (I, [VP, I, I, VP, VP, VP, VP, VP, VP]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_config(shape, max_samples: int, max_batch: int = 1, use_cuda_graph: bool = True) -> w2v_config:
    """Builds the C config struct from a model shape (fields as in synth.inputs.ModelShape)."""
    return w2v_config(shape.d_model, shape.n_layers, shape.n_heads, shape.d_ffn, shape.vocab, shape.blank_id,
                      0 if shape.conv_norm == "group" else 1, int(shape.conv_bias), int(shape.stable_layer_norm),
                      int(shape.gelu_tanh), int(max_samples), int(max_batch), float(shape.ln_eps),
                      int(use_cuda_graph))


def w2v_num_frames(n_samples: int) -> int:
    return lib().w2v_num_frames(int(n_samples))


def w2v_weight_count(cfg: w2v_config) -> int:
    return lib().w2v_weight_count(ctypes.byref(cfg))


def w2v_weight_manifest(cfg: w2v_config):
    """[(name, shape, offset)] as the library lays out the weight blob."""
    L = lib()
    n = L.w2v_weight_num_entries(ctypes.byref(cfg))
    if n < 0:
        raise W2VError(W2V_EINVAL, "invalid config")
    out = []
    buf = ctypes.create_string_buffer(128)
    for i in range(n):
        nd = ctypes.c_int()
        shp = (ctypes.c_int64 * 3)()
        off = ctypes.c_size_t()
        rc = L.w2v_weight_entry(ctypes.byref(cfg), i, buf, 128, ctypes.byref(nd), shp, ctypes.byref(off))
        if rc:
            raise W2VError(rc, "w2v_weight_entry")
        out.append((buf.value.decode(), tuple(int(shp[j]) for j in range(nd.value)), int(off.value)))
    return out


def w2v_num_windows(n_samples: int, window: int) -> int:
    return lib().w2v_num_windows(int(n_samples), int(window))


def w2v_window_pcm(pcm, window: int, out=None, stream=None):
    """pcm: float32 CUDA tensor [n] of one raw clip.  Returns the normalised,
    zero-padded windows [num_windows, window] (see include/w2v.h)."""
    import torch
    n = pcm.numel()
    nw = w2v_num_windows(n, window)
    if out is None:
        out = torch.empty((nw, window), dtype=torch.float32, device=pcm.device)
    _check(lib().w2v_window_pcm(_ptr(pcm), int(n), int(window), _ptr(out), _stream(stream)), None, "w2v_window_pcm")
    return out


def w2v_pack_safetensors(path: str, cfg: w2v_config) -> np.ndarray:
    """The float32 weight blob of a single-file safetensors checkpoint (host only)."""
    blob = np.empty(w2v_weight_count(cfg), dtype=np.float32)
    err = ctypes.create_string_buffer(512)
    rc = lib().w2v_pack_safetensors(os.fsencode(path), ctypes.byref(cfg), blob.ctypes.data, blob.size, err, 512)
    if rc != W2V_OK:
        raise W2VError(rc, f"w2v_pack_safetensors: {err.value.decode(errors='replace')}")
    return blob


def w2v_create_from_safetensors(path: str, cfg: w2v_config) -> int:
    h = VP()
    err = ctypes.create_string_buffer(512)
    rc = lib().w2v_create_from_safetensors(os.fsencode(path), ctypes.byref(cfg), ctypes.byref(h), err, 512)
    if rc != W2V_OK:
        raise W2VError(rc, f"w2v_create_from_safetensors: {err.value.decode(errors='replace')}")
    return h.value


def _check(rc: int, handle=None, what: str = ""):
    if rc == W2V_OK:
        return
    msg = what
    if handle:
        buf = ctypes.create_string_buffer(512)
        lib().w2v_last_error(handle, buf, 512)
        msg = f"{what}: {buf.value.decode(errors='replace')}"
    raise W2VError(rc, msg)


def w2v_create(cfg: w2v_config, blob: np.ndarray) -> int:
    blob = np.ascontiguousarray(blob, dtype=np.float32)
    h = ctypes.c_void_p()
    rc = lib().w2v_create(ctypes.byref(cfg), blob.ctypes.data, blob.size, ctypes.byref(h))
    _check(rc, None, "w2v_create")
    return h.value


def w2v_forward(model: int, pcm, n_samples: int, batch: int, logits, stream=None) -> None:
    _check(lib().w2v_forward(model, _ptr(pcm), int(n_samples), int(batch), _ptr(logits), _stream(stream)), model,
           "w2v_forward")


def _int_array(values):
    vals = [int(v) for v in values]
    return (ctypes.c_int * len(vals))(*vals), len(vals)


def w2v_forward_varlen(model: int, pcm, n_samples, logits, stream=None) -> None:
    arr, n = _int_array(n_samples)
    _check(lib().w2v_forward_varlen(model, _ptr(pcm), arr, n, _ptr(logits), _stream(stream)), model,
           "w2v_forward_varlen")


def w2v_ctc_greedy_varlen(model: int, logits, frames, tokens, n_tokens, stream=None) -> None:
    arr, n = _int_array(frames)
    _check(lib().w2v_ctc_greedy_varlen(model, _ptr(logits), arr, n, _ptr(tokens), _ptr(n_tokens), _stream(stream)),
           model, "w2v_ctc_greedy_varlen")


def w2v_ctc_greedy(model: int, logits, batch: int, T: int, t_valid: int, tokens, n_tokens, stream=None) -> None:
    _check(lib().w2v_ctc_greedy(model, _ptr(logits), int(batch), int(T), int(t_valid), _ptr(tokens), _ptr(n_tokens),
                                _stream(stream)), model, "w2v_ctc_greedy")


def w2v_ctc_greedy_static(logits, batch: int, T: int, vocab: int, t_valid: int, blank_id: int, tokens, n_tokens,
                          stream=None) -> int:
    """Allocation-free greedy CTC decode (no model handle); returns the status code."""
    return lib().w2v_ctc_greedy_static(_ptr(logits), int(batch), int(T), int(vocab), int(t_valid), int(blank_id),
                                       _ptr(tokens), _ptr(n_tokens), _stream(stream))


def w2v_sync(model: int, stream=None) -> None:
    _check(lib().w2v_sync(model, _stream(stream)), model, "w2v_sync")


def w2v_debug_read(model: int, which: int, dst, stream=None) -> int:
    nbytes = ctypes.c_size_t()
    n = dst.numel() * dst.element_size()
    _check(lib().w2v_debug_read(model, int(which), _ptr(dst), n, ctypes.byref(nbytes), _stream(stream)), model,
           "w2v_debug_read")
    return int(nbytes.value)


def w2v_transcribe(model: int, pcm_host: np.ndarray, t_valid: int, tokens_host: np.ndarray,
                   n_tokens_host: np.ndarray, stream=None) -> None:
    """pcm_host: float32 [batch, n] (pinned for speed); tokens_host int32 [batch, t_valid]; n_tokens_host int32 [batch]."""
    batch, n = pcm_host.shape
    _check(lib().w2v_transcribe(model, pcm_host.ctypes.data, int(n), int(batch), int(t_valid), tokens_host.ctypes.data,
                                n_tokens_host.ctypes.data, _stream(stream)), model, "w2v_transcribe")


def w2v_last_launch_count(model: int) -> int:
    return lib().w2v_last_launch_count(model)


def w2v_kernel_class_name(klass: int) -> str:
    return lib().w2v_kernel_class_name(int(klass)).decode()


def w2v_profile_forward(model: int, pcm, n_samples: int, batch: int, logits, stream=None, max_out: int = 4096):
    """Returns [(class_name, ms, flops, bytes)] per kernel launch, in launch order."""
    buf = (w2v_kernel_time * max_out)()
    n = ctypes.c_int()
    _check(lib().w2v_profile_forward(model, _ptr(pcm), int(n_samples), int(batch), _ptr(logits), _stream(stream), buf,
                                     max_out, ctypes.byref(n)), model, "w2v_profile_forward")
    return [(w2v_kernel_class_name(buf[i].klass), float(buf[i].ms), float(buf[i].flops), float(buf[i].bytes))
            for i in range(n.value)]


KERNEL_CLASSES = ["gn_moments", "conv0_norm_gelu", "conv_gemm", "conv_layernorm", "fp_layernorm", "proj_gemm",
                  "posconv", "enc_layernorm", "qkv_gemm", "attention", "out_gemm", "ffn1_gemm", "ffn2_gemm",
                  "lm_head_gemm", "argmax", "ctc_collapse"]


def w2v_time_class(model: int, pcm, n_samples: int, batch: int, logits, klass, reps: int = 10, stream=None):
    """(us_per_launch, launches_per_forward, flops_per_launch, bytes_per_launch) of one kernel class."""
    k = KERNEL_CLASSES.index(klass) if isinstance(klass, str) else int(klass)
    us = ctypes.c_float()
    n = ctypes.c_int()
    fl = ctypes.c_double()
    by = ctypes.c_double()
    _check(lib().w2v_time_class(model, _ptr(pcm), int(n_samples), int(batch), _ptr(logits), k, int(reps),
                                ctypes.byref(us), ctypes.byref(n), ctypes.byref(fl), ctypes.byref(by),
                                _stream(stream)), model, "w2v_time_class")
    return float(us.value), int(n.value), float(fl.value), float(by.value)


def w2v_destroy(model: int) -> None:
    if model:
        lib().w2v_destroy(model)


def w2v_op_gemm(A, B, M, N, K, bias, residual, res_f32, out, out_f32, act, err, bn=0, splits=1, stream=None) -> int:
    return lib().w2v_op_gemm(_ptr(A), _ptr(B), M, N, K, _ptr(bias), _ptr(residual), res_f32, _ptr(out), out_f32,
                             act, bn, splits, _ptr(err), _stream(stream))


def w2v_op_attention(q, k, vt, out, batch, T, H, t_pad, err, stream=None) -> int:
    return lib().w2v_op_attention(_ptr(q), _ptr(k), _ptr(vt), _ptr(out), batch, T, H, t_pad, _ptr(err),
                                  _stream(stream))


def w2v_op_layernorm(x, in_f32, y, rows, cols, gamma, beta, eps, act, stream=None) -> int:
    return lib().w2v_op_layernorm(_ptr(x), in_f32, _ptr(y), rows, cols, _ptr(gamma), _ptr(beta), float(eps), act,
                                  _stream(stream))


def w2v_fold_layernorm_linear(W: np.ndarray, bias, gamma: np.ndarray, beta: np.ndarray):
    """Host-side LayerNorm -> Linear fold (see include/w2v_ops.h): returns
    (fp16 weight W diag(gamma), bias + W beta, column sums of the fp16 weight)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    bt = np.ascontiguousarray(beta, dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    wf = np.empty((N, K), dtype=np.float16)
    bo = np.empty(N, dtype=np.float32)
    cs = np.empty(N, dtype=np.float32)
    rc = lib().w2v_fold_layernorm_linear(W.ctypes.data, N, K, None if b is None else b.ctypes.data, g.ctypes.data,
                                         bt.ctypes.data, wf.ctypes.data, bo.ctypes.data, cs.ctypes.data)
    _check(rc, None, "w2v_fold_layernorm_linear")
    return wf, bo, cs


def w2v_op_pointwise(fn: int, x, y, c: float = 1.0, b: float = 0.0, stream=None) -> int:
    return lib().w2v_op_pointwise(int(fn), _ptr(x), int(x.numel()), float(c), float(b), _ptr(y), _stream(stream))


def w2v_op_wait_probe(err, limit_ns: int, stream=None) -> int:
    return lib().w2v_op_wait_probe(_ptr(err), int(limit_ns), _stream(stream))


class Model:
    """Owns one w2v_model handle.  Tensors are torch CUDA tensors."""

    def __init__(self, shape, blob: Optional[np.ndarray], max_samples: int, max_batch: int = 1,
                 use_cuda_graph: bool = True, safetensors: Optional[str] = None):
        """Weights from `blob` (float32, manifest order) or, with blob None,
        from the single-file safetensors checkpoint at `safetensors`."""
        self.shape = shape
        self.cfg = make_config(shape, max_samples, max_batch, use_cuda_graph)
        if blob is None:
            if safetensors is None:
                raise ValueError("give a weight blob or a safetensors path")
            self.handle = w2v_create_from_safetensors(safetensors, self.cfg)
        else:
            self.handle = w2v_create(self.cfg, blob)

    def forward(self, pcm, logits=None, stream=None):
        """pcm: float32 CUDA tensor [batch, n].  Returns logits [batch, T, vocab]."""
        import torch
        batch, n = pcm.shape
        T = w2v_num_frames(n)
        if logits is None:
            logits = torch.empty((batch, T, self.shape.vocab), dtype=torch.float32, device=pcm.device)
        w2v_forward(self.handle, pcm, n, batch, logits, stream)
        return logits

    def ctc_greedy(self, logits, t_valid: int, tokens=None, n_tokens=None, stream=None):
        import torch
        batch, T, _ = logits.shape
        if tokens is None:
            tokens = torch.empty((batch, max(t_valid, 1)), dtype=torch.int32, device=logits.device)
        if n_tokens is None:
            n_tokens = torch.empty((batch,), dtype=torch.int32, device=logits.device)
        w2v_ctc_greedy(self.handle, logits, batch, T, t_valid, tokens, n_tokens, stream)
        return tokens, n_tokens

    def forward_varlen(self, clips, logits=None, stream=None):
        """clips: list of 1-D float32 CUDA tensors (one per clip, any lengths).
        Returns (logits [sum T_c, vocab], frames [T_c])."""
        import torch
        lens = [int(c.numel()) for c in clips]
        frames = [w2v_num_frames(n) for n in lens]
        pcm = torch.cat([c.reshape(-1) for c in clips]).contiguous()
        if logits is None:
            logits = torch.empty((sum(frames), self.shape.vocab), dtype=torch.float32, device=pcm.device)
        w2v_forward_varlen(self.handle, pcm, lens, logits, stream)
        return logits, frames

    def ctc_greedy_varlen(self, logits, frames, stream=None):
        """Tokens of each clip of a packed forward_varlen output: a list of int32
        CUDA tensors (one per clip), after a stream sync."""
        import torch
        tokens = torch.empty((max(sum(frames), 1),), dtype=torch.int32, device=logits.device)
        n_tokens = torch.empty((len(frames),), dtype=torch.int32, device=logits.device)
        w2v_ctc_greedy_varlen(self.handle, logits, frames, tokens, n_tokens, stream)
        self.sync(stream)
        out, off = [], 0
        for c, T in enumerate(frames):
            out.append(tokens[off:off + int(n_tokens[c])])
            off += T
        return out

    def sync(self, stream=None):
        w2v_sync(self.handle, stream)

    def close(self):
        if self.handle:
            w2v_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
