"""The create-time LayerNorm fold of the post-norm blocks (host only): the
library's folded weight, bias and column sums match their definitions, and
with them the GEMM-side formula rstd * (x W''^T - mean * colsum) + bias'
reproduces LayerNorm(x) -> Linear up to the fp16 rounding of the weight."""
import numpy as np
import pytest

from oracle import w2v_oracle as O
from speech_encoder_b200 import w2v as B


@pytest.mark.parametrize("N,K", [(96, 256), (40, 768), (1, 1)])
def test_fold_outputs_match_their_definitions(N, K):
    rng = np.random.default_rng(N + K)
    W = rng.standard_normal((N, K)).astype(np.float32) * 0.05
    bias = rng.standard_normal(N).astype(np.float32) * 0.1
    gamma = (1 + 0.2 * rng.standard_normal(K)).astype(np.float32)
    beta = (0.2 * rng.standard_normal(K)).astype(np.float32)
    wf, bo, cs = B.w2v_fold_layernorm_linear(W, bias, gamma, beta)
    # fp16 of the float32 product, round to nearest even (numpy's cast rounds so)
    assert np.array_equal(wf, (W * gamma[None, :]).astype(np.float16))
    np.testing.assert_allclose(bo, bias.astype(np.float64) + W.astype(np.float64) @ beta.astype(np.float64),
                               rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(cs, wf.astype(np.float64).sum(axis=1), rtol=1e-6, atol=1e-7)
    _, bo0, _ = B.w2v_fold_layernorm_linear(W, None, gamma, beta)
    np.testing.assert_allclose(bo0, W.astype(np.float64) @ beta.astype(np.float64), rtol=1e-6, atol=1e-7)


def test_folded_gemm_formula_equals_layernorm_then_linear():
    rng = np.random.default_rng(5)
    N, K, rows, eps = 64, 256, 50, 1e-5
    W = rng.standard_normal((N, K)).astype(np.float32) * 0.05
    bias = rng.standard_normal(N).astype(np.float32) * 0.1
    gamma = (1 + 0.2 * rng.standard_normal(K)).astype(np.float32)
    beta = (0.2 * rng.standard_normal(K)).astype(np.float32)
    x = (rng.standard_normal((rows, K)) * 2 + 0.3).astype(np.float64)  # un-normalised rows, offset mean
    wf, bo, cs = B.w2v_fold_layernorm_linear(W, bias, gamma, beta)
    mean = x.mean(axis=1, keepdims=True)
    rstd = 1 / np.sqrt(x.var(axis=1, keepdims=True) + eps)
    got = rstd * (x @ wf.astype(np.float64).T - mean * cs.astype(np.float64)[None, :]) + bo.astype(np.float64)
    ref = O.layer_norm(x, gamma.astype(np.float64), beta.astype(np.float64), eps) @ W.astype(np.float64).T + bias
    # the only approximation is the fp16 rounding of W * gamma (relative 2^-11 per element)
    assert np.abs(got - ref).max() < 2e-3 * np.abs(ref).max()
    # a plausible slip (dropping the mean term, or the beta term) is far outside that bound
    bad = rstd * (x @ wf.astype(np.float64).T) + bo
    assert np.abs(bad - ref).max() > 10 * np.abs(got - ref).max()


def test_fold_rejects_bad_arguments():
    with pytest.raises(B.W2VError):
        B.w2v_fold_layernorm_linear(np.zeros((0, 4), np.float32), None, np.ones(4), np.zeros(4))
