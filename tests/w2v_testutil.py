"""Shared helpers of the GPU parity tests: cached oracle results, the
tolerance checks, and model construction through the C ABI."""
from __future__ import annotations

import functools

import numpy as np

from oracle import w2v_oracle as O
from synth import inputs as S

# Tolerances of the fp16-compute path against the fp64 oracle (logits):
MAX_ABS = 3e-2
MEAN_ABS = 2e-3
ARGMAX_AGREE = 0.995
MARGIN = 0.1


@functools.lru_cache(maxsize=8)
def weights(shape: S.ModelShape, seed: int = 0, affine_noise: bool = False):
    return S.init_weights(shape, seed, affine_noise)


@functools.lru_cache(maxsize=4)
def weights64(shape: S.ModelShape, seed: int = 0, affine_noise: bool = False):
    return O.to_f64(weights(shape, seed, affine_noise))


def oracle_logits(shape, pcm_1d: np.ndarray, seed: int = 0, affine_noise: bool = False, taps=None) -> np.ndarray:
    return O.forward(shape, weights64(shape, seed, affine_noise), pcm_1d, taps)


@functools.lru_cache(maxsize=64)
def oracle_workload_clip(name: str, call: int, clip: int) -> np.ndarray:
    w = S.workload(name)
    pcm, _ = w.calls[call]
    return oracle_logits(w.model, pcm[clip])


def compare_logits(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Asserts the logits tolerances; returns a dict of the measured errors."""
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite logits"
    d = np.abs(got.astype(np.float64) - ref)
    top2 = np.sort(ref, axis=-1)[:, -2:] if ref.shape[-1] > 1 else np.concatenate([ref, ref - 1], -1)
    margin = top2[:, 1] - top2[:, 0]
    sel = margin > MARGIN
    agree = float(np.mean(np.argmax(got, -1)[sel] == np.argmax(ref, -1)[sel])) if sel.any() else 1.0
    stats = dict(max_abs=float(d.max()), mean_abs=float(d.mean()), agree=agree, n_margin=int(sel.sum()))
    assert stats["max_abs"] <= MAX_ABS, (what, stats)
    assert stats["mean_abs"] <= MEAN_ABS, (what, stats)
    assert agree >= ARGMAX_AGREE, (what, stats)
    return stats


def make_model(shape, max_samples, max_batch=1, seed=0, affine_noise=False, use_cuda_graph=True):
    from speech_encoder_b200 import w2v as B
    blob = S.pack_blob(shape, weights(shape, seed, affine_noise))
    return B.Model(shape, blob, max_samples=max_samples, max_batch=max_batch, use_cuda_graph=use_cuda_graph)
