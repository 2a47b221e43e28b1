"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module holds no arithmetic of the model itself.  It only defines:

* the model shapes (wav2vec2-base and wav2vec2-large stable-layer-norm, as the
  TensorRT-Model-Connect wav2vec2 README, section "Wav2Vec2 CTC layouts",
  describes them: group- or layer-normalised conv encoders, with or without
  conv bias, post-norm or stable pre-norm blocks, 1024-wide 24-layer model with
  a 2341-token CTC head),
* the five workloads (clip lengths, seeds, GELU variant),
* the PCM recipe: summed sinusoids plus Gaussian noise, normalised to zero
  mean / unit variance (the input normalisation a runtime applies before the
  model; "Input normalized like the runtime", same README, section "Method"),
* the random-init weight draws, in a fixed manifest order.

The recipe constants (frequency band 100-4000 Hz, noise std 0.1, Kaiming-normal
conv init, N(0, 0.02) linear init, LN gamma 1 / beta 0) are the workload
description; the pages give no waveform, so these stand in for the pages'
LibriSpeech clips, which are not available here.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import numpy as np

SAMPLE_RATE = 16000
CONV_CHANNELS = 512
CONV_KERNELS = (10, 3, 3, 3, 3, 2, 2)
CONV_STRIDES = (5, 2, 2, 2, 2, 2, 2)
POS_CONV_KERNEL = 128
POS_CONV_GROUPS = 16


@dataclasses.dataclass(frozen=True)
class ModelShape:
    name: str
    d_model: int
    n_layers: int
    n_heads: int
    d_ffn: int
    vocab: int
    blank_id: int
    conv_norm: str          # "group": GroupNorm(512, 512) on conv layer 0; "layer": per-frame LN on every conv layer
    conv_bias: bool
    stable_layer_norm: bool  # False: post-norm blocks, encoder LN before blocks; True: pre-norm, encoder LN after
    gelu_tanh: bool = False
    ln_eps: float = 1e-5

    def with_(self, **kw) -> "ModelShape":
        return dataclasses.replace(self, **kw)


BASE = ModelShape("wav2vec2-base", 768, 12, 12, 3072, 32, 0, "group", False, False)
LARGE = ModelShape("wav2vec2-large-stable", 1024, 24, 16, 4096, 2341, 0, "layer", True, True)


def weight_manifest(shape: ModelShape) -> List[Tuple[str, Tuple[int, ...]]]:
    """Names and shapes of every weight tensor, in blob order.

    The order is the order of the forward pass.  PyTorch layouts: Conv1d weight
    [C_out, C_in/groups, k], Linear weight [out, in].  q/k/v are separate
    tensors as in the checkpoints; the positional conv weight is the already
    folded static weight g*v/||v||.
    """
    C, d, F, V = CONV_CHANNELS, shape.d_model, shape.d_ffn, shape.vocab
    m: List[Tuple[str, Tuple[int, ...]]] = []
    for i, k in enumerate(CONV_KERNELS):
        cin = 1 if i == 0 else C
        m.append((f"conv{i}.weight", (C, cin, k)))
        if shape.conv_bias:
            m.append((f"conv{i}.bias", (C,)))
        if shape.conv_norm == "layer" or i == 0:
            m.append((f"conv{i}.norm.weight", (C,)))
            m.append((f"conv{i}.norm.bias", (C,)))
    m += [("fp.norm.weight", (C,)), ("fp.norm.bias", (C,)),
          ("fp.proj.weight", (d, C)), ("fp.proj.bias", (d,)),
          ("pos_conv.weight", (d, d // POS_CONV_GROUPS, POS_CONV_KERNEL)), ("pos_conv.bias", (d,)),
          ("enc.norm.weight", (d,)), ("enc.norm.bias", (d,))]
    for l in range(shape.n_layers):
        p = f"layers.{l}."
        for nm in ("q", "k", "v", "out"):
            m.append((p + f"attn.{nm}.weight", (d, d)))
            m.append((p + f"attn.{nm}.bias", (d,)))
        m += [(p + "attn_norm.weight", (d,)), (p + "attn_norm.bias", (d,)),
              (p + "ffn.in.weight", (F, d)), (p + "ffn.in.bias", (F,)),
              (p + "ffn.out.weight", (d, F)), (p + "ffn.out.bias", (d,)),
              (p + "ffn_norm.weight", (d,)), (p + "ffn_norm.bias", (d,))]
    m += [("lm_head.weight", (V, d)), ("lm_head.bias", (V,))]
    return m


def init_weights(shape: ModelShape, seed: int = 0, affine_noise: bool = False) -> Dict[str, np.ndarray]:
    """Random-init weights, float32, drawn from one seeded stream in manifest order.

    Conv weights: Kaiming-normal, std sqrt(2 / fan_in), fan_in = (C_in/groups)*k
    (the positional conv included).  Linear weights and every bias: N(0, 0.02).
    Norm gamma = 1, beta = 0; with ``affine_noise`` gamma = 1 + N(0, 0.1),
    beta = N(0, 0.1) so that the affine terms are exercised.
    """
    rng = np.random.default_rng(seed)
    out: Dict[str, np.ndarray] = {}
    for name, shp in weight_manifest(shape):
        if name.endswith("norm.weight"):
            a = 1.0 + (rng.normal(0.0, 0.1, shp) if affine_noise else np.zeros(shp))
        elif name.endswith("norm.bias"):
            a = rng.normal(0.0, 0.1, shp) if affine_noise else np.zeros(shp)
        elif name.endswith(".bias"):
            a = rng.normal(0.0, 0.02, shp)
        elif name.startswith("conv") or name.startswith("pos_conv"):
            fan_in = shp[1] * shp[2]
            a = rng.standard_normal(shp, dtype=np.float32) * np.float32(np.sqrt(2.0 / fan_in))
        else:
            a = rng.standard_normal(shp, dtype=np.float32) * np.float32(0.02)
        out[name] = np.ascontiguousarray(a, dtype=np.float32)
    return out


def pack_blob(shape: ModelShape, weights: Dict[str, np.ndarray]) -> np.ndarray:
    """Concatenate the weights (float32) in manifest order into one flat blob."""
    parts = []
    for name, shp in weight_manifest(shape):
        a = np.asarray(weights[name], dtype=np.float32)
        if a.shape != tuple(shp):
            raise ValueError(f"{name}: shape {a.shape} != {shp}")
        parts.append(a.reshape(-1))
    return np.concatenate(parts)


def synth_pcm(n_samples: int, seed: int) -> np.ndarray:
    """One clip: 3 sinusoids (f ~ U(100, 4000) Hz, phase ~ U(0, 2pi), amplitude 1)
    plus N(0, 0.1^2) noise at 16 kHz, then normalised to zero mean and unit
    variance (eps 1e-7), stored as float32."""
    rng = np.random.default_rng(seed)
    f = rng.uniform(100.0, 4000.0, 3)
    ph = rng.uniform(0.0, 2.0 * np.pi, 3)
    t = np.arange(n_samples, dtype=np.float64) / SAMPLE_RATE
    x = np.zeros(n_samples)
    for i in range(3):
        x += np.sin(2.0 * np.pi * f[i] * t + ph[i])
    x += rng.normal(0.0, 0.1, n_samples)
    x = (x - x.mean()) / np.sqrt(x.var() + 1e-7)
    return x.astype(np.float32)


def pad_to_window(x: np.ndarray, window: int) -> np.ndarray:
    """Zero-pad a clip at the end to a fixed window length."""
    if x.shape[0] > window:
        raise ValueError("clip longer than window")
    out = np.zeros(window, dtype=np.float32)
    out[: x.shape[0]] = x
    return out


@dataclasses.dataclass
class Workload:
    """A list of forward calls.  Each call is (pcm[batch, n] float32, n_valid per clip)."""
    name: str
    model: ModelShape
    calls: List[Tuple[np.ndarray, List[int]]]
    weight_seed: int = 0

    @property
    def audio_seconds(self) -> float:
        return sum(int(p.shape[0]) * int(p.shape[1]) for p, _ in self.calls) / SAMPLE_RATE


def c4_lengths() -> List[int]:
    return [int(v) for v in np.random.default_rng(4).integers(32000, 320001, size=8)]


def workload(name: str) -> Workload:
    """The five workloads.

    c0  base, 1 s (16000 samples, seed 0), exact GELU
    c1  base, tanh-GELU, fixed 16 s window (256000 samples): a full 16 s clip
        (seed 10) and a 3.7 s clip (59200 samples, seed 1) zero-padded to the
        window and decoded over its valid frames
    c2  base, exact GELU, 16 clips of 10 s (seeds 200..215) in one batch
    c3  large stable-layer-norm, 16 s (seed 3)
    c4  large, 8 true-length clips, n_i ~ U[32000, 320000] (seed 4), clip seeds
        400+i, issued one after another
    """
    if name == "c0":
        return Workload(name, BASE, [(synth_pcm(16000, 0)[None], [16000])])
    if name == "c1":
        m = BASE.with_(gelu_tanh=True)
        full = synth_pcm(256000, 10)[None]
        short = pad_to_window(synth_pcm(59200, 1), 256000)[None]
        return Workload(name, m, [(full, [256000]), (short, [59200])])
    if name == "c2":
        pcm = np.stack([synth_pcm(160000, 200 + i) for i in range(16)])
        return Workload(name, BASE, [(pcm, [160000] * 16)])
    if name == "c3":
        return Workload(name, LARGE, [(synth_pcm(256000, 3)[None], [256000])])
    if name == "c4":
        calls = []
        for i, n in enumerate(c4_lengths()):
            calls.append((synth_pcm(n, 400 + i)[None], [n]))
        return Workload(name, LARGE, calls)
    raise KeyError(name)


def small_shape(conv_norm="group", stable=False, conv_bias=False, gelu_tanh=False,
                d_model=256, n_layers=2, n_heads=4, d_ffn=512, vocab=40) -> ModelShape:
    """A reduced model for fast tests: real conv frontend, narrow encoder
    (head dim stays 64, pos-conv groups stay 16)."""
    return ModelShape("small", d_model, n_layers, n_heads, d_ffn, vocab, 0, conv_norm,
                      conv_bias, stable, gelu_tanh)
