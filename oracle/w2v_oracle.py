"""fp64 CPU oracle of the wav2vec2-style CTC forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline / reference arm may import this module.  It shares no code with
the CUDA library and imports nothing from it.

It is the plain definition of each step, written out in numpy float64, in the
order the model applies them, with no blocking, fusion or re-association beyond
what a library matmul does internally.  Sources for each step:

* Conv feature encoder, GroupNorm on layer 0 or per-frame LayerNorm on every
  layer, conv bias optional: TensorRT-Model-Connect wav2vec2 README, section
  "Wav2Vec2 CTC layouts" (group-normalised and per-frame layer-normalised
  feature encoders, with or without convolution bias); the LiteRT wav2vec2
  discussion, "Rewrites for the GPU" (feature-extractor GroupNorm).  Kernel
  sizes (10,3,3,3,3,2,2), strides (5,2,2,2,2,2,2), 512 channels: the workload
  description of the model.
* GroupNorm statistics are taken over every time step of the clip (README,
  section "FP8 quantization study", Kernel-time paragraph: "a group norm over
  every time step of the clip").
* GELU exact, or the tanh form: LiteRT discussion, "Rewrites for the GPU",
  first bullet.
* Positional conv with the weight-norm folded to a static weight: LiteRT
  discussion, third bullet.  Kernel 128, 16 groups.
* Blocks in post-norm or stable pre-norm order, encoder-level norm after the
  blocks for stable checkpoints: README, "Wav2Vec2 CTC layouts".
* Attention is plain SDPA with no mask: LiteRT discussion, fourth bullet.
* lm_head, per-frame argmax and CTC collapse: README, "Results" (CTC ids).

Readings taken where the pages are silent:
* eps 1e-5 with biased variance for every norm;
* for post-norm the encoder LN sits once after the positional-conv add and
  before block 1 (the pages state only that stable checkpoints apply it after
  the blocks);
* the positional conv pads 64 zeros on each side, drops the last output frame
  (even kernel), has a bias, and is followed by GELU and the residual add;
* the tanh-GELU variant replaces every GELU of the model (conv encoder,
  positional conv, FFN);
* attention scale 1/sqrt(64), biases on q/k/v/out, no mask, no dropout;
* GroupNorm statistics of a zero-padded fixed window are taken over all of its
  conv-0 frames, zeros included;
* argmax ties go to the lowest index; collapse merges repeats first and then
  drops blank (id 0, also for the 2341-token head).

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, brute-force loops on tiny shapes, torch fp64
library routines and (when ``transformers`` is importable) an independent
whole-model implementation loaded with the same tensors.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np
from numpy.lib.stride_tricks import sliding_window_view
from scipy.special import erf

CONV_KERNELS = (10, 3, 3, 3, 3, 2, 2)
CONV_STRIDES = (5, 2, 2, 2, 2, 2, 2)
POS_K = 128
POS_G = 16
HEAD_DIM = 64


def conv_out_len(n: int, k: int, s: int) -> int:
    """Output length of an unpadded strided conv: floor((n - k)/s) + 1, or 0."""
    return (n - k) // s + 1 if n >= k else 0


def num_frames(n_samples: int) -> int:
    """Frame count after the 7 conv layers, by applying each layer's rule in turn."""
    n = n_samples
    for k, s in zip(CONV_KERNELS, CONV_STRIDES):
        n = conv_out_len(n, k, s)
    return n


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2))."""
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def conv1d(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray], stride: int) -> np.ndarray:
    """Unpadded strided conv, time-major.

    x: [L, C_in], w: [C_out, C_in, k] -> y: [L_out, C_out] with
    y[t, c] = sum_{ci, j} w[c, ci, j] * x[stride*t + j, ci] (+ b[c]).
    """
    k = w.shape[2]
    L = x.shape[0]
    T = conv_out_len(L, k, stride)
    win = sliding_window_view(x, k, axis=0)[: (T - 1) * stride + 1: stride]  # [T, C_in, k]
    y = win.reshape(T, -1) @ w.reshape(w.shape[0], -1).T
    if b is not None:
        y = y + b
    return y


def group_norm_per_channel(y: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    """GroupNorm with one group per channel over [T, C]: each channel is
    normalised with its mean and (biased) variance over all T time steps."""
    mu = y.mean(axis=0)
    var = ((y - mu) ** 2).mean(axis=0)
    return (y - mu) / np.sqrt(var + eps) * g + b


def layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm over the last axis, biased variance."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + b


def _act(shape) :
    return gelu_tanh if shape.gelu_tanh else gelu


def feature_encoder(shape, W: Dict[str, np.ndarray], pcm: np.ndarray, taps: Optional[dict] = None) -> np.ndarray:
    """7 conv layers.  group layout: GN on layer 0 then GELU, GELU only on 1-6.
    layer layout: conv (+bias) -> per-frame LN over 512 channels -> GELU on every layer."""
    act = _act(shape)
    x = pcm.astype(np.float64)[:, None]
    for i, s in enumerate(CONV_STRIDES):
        y = conv1d(x, W[f"conv{i}.weight"], W.get(f"conv{i}.bias"), s)
        if shape.conv_norm == "group":
            if i == 0:
                y = group_norm_per_channel(y, W["conv0.norm.weight"], W["conv0.norm.bias"], shape.ln_eps)
        else:
            y = layer_norm(y, W[f"conv{i}.norm.weight"], W[f"conv{i}.norm.bias"], shape.ln_eps)
        x = act(y)
        if taps is not None:
            taps[f"conv{i}"] = x
    return x


def feature_projection(shape, W, x: np.ndarray) -> np.ndarray:
    """LN over the 512 conv channels, then Linear 512 -> d."""
    y = layer_norm(x, W["fp.norm.weight"], W["fp.norm.bias"], shape.ln_eps)
    return y @ W["fp.proj.weight"].T + W["fp.proj.bias"]


def positional_conv(shape, W, x: np.ndarray) -> np.ndarray:
    """Grouped conv, kernel 128, 16 groups, stride 1, 64 zeros padded on each
    side of time, last output frame dropped (even kernel), bias, then GELU.
    Returns the positional term p; the caller adds it to x."""
    T, d = x.shape
    m = d // POS_G
    w = W["pos_conv.weight"]                      # [d, m, 128]
    xp = np.zeros((T + 2 * (POS_K // 2), d))
    xp[POS_K // 2: POS_K // 2 + T] = x
    p = np.empty((T, d))
    for g in range(POS_G):
        xs = xp[:, g * m:(g + 1) * m]             # [T+128, m]
        y = conv1d(xs, w[g * m:(g + 1) * m], None, 1)   # [T+1, m]
        p[:, g * m:(g + 1) * m] = y[:T]
    p = p + W["pos_conv.bias"]
    return _act(shape)(p)


def softmax_rows(s: np.ndarray) -> np.ndarray:
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def self_attention(shape, W, p: str, h: np.ndarray) -> np.ndarray:
    """Multi-head SDPA with no mask over all T frames, head dim 64, scale 1/8,
    q/k/v/out projections with bias."""
    T, d = h.shape
    H = shape.n_heads
    q = h @ W[p + "attn.q.weight"].T + W[p + "attn.q.bias"]
    k = h @ W[p + "attn.k.weight"].T + W[p + "attn.k.bias"]
    v = h @ W[p + "attn.v.weight"].T + W[p + "attn.v.bias"]
    dh = d // H
    o = np.empty((T, d))
    for hh in range(H):
        sl = slice(hh * dh, (hh + 1) * dh)
        P = softmax_rows(q[:, sl] @ k[:, sl].T / np.sqrt(dh))
        o[:, sl] = P @ v[:, sl]
    return o @ W[p + "attn.out.weight"].T + W[p + "attn.out.bias"]


def feed_forward(shape, W, p: str, h: np.ndarray) -> np.ndarray:
    a = _act(shape)(h @ W[p + "ffn.in.weight"].T + W[p + "ffn.in.bias"])
    return a @ W[p + "ffn.out.weight"].T + W[p + "ffn.out.bias"]


def encoder(shape, W, x: np.ndarray, taps: Optional[dict] = None) -> np.ndarray:
    eps = shape.ln_eps
    h = x + positional_conv(shape, W, x)
    if taps is not None:
        taps["posconv"] = h
    if not shape.stable_layer_norm:
        h = layer_norm(h, W["enc.norm.weight"], W["enc.norm.bias"], eps)
        for l in range(shape.n_layers):
            p = f"layers.{l}."
            h = layer_norm(h + self_attention(shape, W, p, h), W[p + "attn_norm.weight"], W[p + "attn_norm.bias"], eps)
            h = layer_norm(h + feed_forward(shape, W, p, h), W[p + "ffn_norm.weight"], W[p + "ffn_norm.bias"], eps)
            if taps is not None:
                taps[f"block{l}"] = h
    else:
        for l in range(shape.n_layers):
            p = f"layers.{l}."
            h = h + self_attention(shape, W, p, layer_norm(h, W[p + "attn_norm.weight"], W[p + "attn_norm.bias"], eps))
            h = h + feed_forward(shape, W, p, layer_norm(h, W[p + "ffn_norm.weight"], W[p + "ffn_norm.bias"], eps))
            if taps is not None:
                taps[f"block{l}"] = h
        h = layer_norm(h, W["enc.norm.weight"], W["enc.norm.bias"], eps)
    return h


def to_f64(weights: Dict[str, np.ndarray], round_fp16: bool = False) -> Dict[str, np.ndarray]:
    """Promote the float32 weights to float64; optionally round matrix weights
    through fp16 first (a debug aid that separates weight rounding from
    kernel error)."""
    out = {}
    for k, v in weights.items():
        a = np.asarray(v, dtype=np.float32)
        if round_fp16 and a.ndim >= 2:
            a = a.astype(np.float16).astype(np.float32)
        out[k] = a.astype(np.float64)
    return out


def forward(shape, W64: Dict[str, np.ndarray], pcm: np.ndarray, taps: Optional[dict] = None) -> np.ndarray:
    """One clip: PCM [n] -> logits [T, V] (float64)."""
    if num_frames(pcm.shape[0]) < 1:
        raise ValueError("clip shorter than the 400-sample receptive field")
    x = feature_encoder(shape, W64, pcm, taps)
    x = feature_projection(shape, W64, x)
    if taps is not None:
        taps["proj"] = x
    h = encoder(shape, W64, x, taps)
    if taps is not None:
        taps["final"] = h
    return h @ W64["lm_head.weight"].T + W64["lm_head.bias"]


def argmax_lowest(logits: np.ndarray) -> np.ndarray:
    """Per-frame argmax; among equal maxima the lowest index wins."""
    return np.argmax(logits, axis=-1).astype(np.int32)  # numpy returns the first maximum


def ctc_collapse(ids, blank: int = 0) -> List[int]:
    """Greedy CTC: merge runs of equal ids, then drop the blank id."""
    out: List[int] = []
    prev = None
    for a in ids:
        a = int(a)
        if a != prev and a != blank:
            out.append(a)
        prev = a
    return out


def ctc_greedy(logits: np.ndarray, t_valid: int, blank: int = 0) -> List[int]:
    return ctc_collapse(argmax_lowest(logits[:t_valid]), blank)
