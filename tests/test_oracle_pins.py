"""Pins of the fp64 oracle against things other than itself.

Each test ties one oracle function to a closed form, an invariant, a brute-force
loop on a tiny shape, a torch float64 library routine, or (for the whole model)
an independent implementation loaded with the same tensors.  A dropped term, a
wrong sign, an off-by-one tap or a transposed operand in the oracle fails at
least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import w2v_oracle as O
from synth import inputs as S

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        return [l.strip() for l in f if l.strip() and not l.startswith("#")]


# ---------------------------------------------------------------- frame count
def test_frame_count_golden():
    for row in _rows("frame_counts.txt"):
        n, t = map(int, row.split())
        assert O.num_frames(n) == t, (n, t)


def test_frame_count_closed_form_all_lengths():
    # The layer-by-layer recursion equals floor((n-400)/320)+1 (receptive field
    # 400 samples, hop 320) for every n below 400000, and 0 below 400.
    n = np.arange(0, 400000, dtype=np.int64)
    L = n.copy()
    for k, s in zip(O.CONV_KERNELS, O.CONV_STRIDES):
        L = np.where(L >= k, (L - k) // s + 1, 0)
    closed = np.where(n >= 400, (n - 400) // 320 + 1, 0)
    assert np.array_equal(L, closed)
    for v in (0, 399, 400, 16000, 12345, 399999):
        assert O.num_frames(int(v)) == closed[v]


# ----------------------------------------------------------------------- conv
def _conv_brute(x, w, b, s):
    L, Ci = x.shape
    Co, _, k = w.shape
    T = (L - k) // s + 1
    y = np.zeros((T, Co))
    for t in range(T):
        for c in range(Co):
            acc = 0.0
            for ci in range(Ci):
                for j in range(k):
                    acc += w[c, ci, j] * x[s * t + j, ci]
            y[t, c] = acc + (b[c] if b is not None else 0.0)
    return y


@pytest.mark.parametrize("k,s", [(10, 5), (3, 2), (2, 2), (4, 1)])
def test_conv_brute_force(k, s):
    rng = np.random.default_rng(1)
    x = rng.normal(size=(50, 3))
    w = rng.normal(size=(4, 3, k))
    b = rng.normal(size=4)
    assert np.allclose(O.conv1d(x, w, b, s), _conv_brute(x, w, b, s), atol=1e-12)
    assert np.allclose(O.conv1d(x, w, None, s), _conv_brute(x, w, None, s), atol=1e-12)


def test_conv_delta_input_returns_taps():
    # A unit impulse at sample 0 of channel ci gives y[0, c] = w[c, ci, 0];
    # an impulse at sample j (j < stride) gives y[0, c] = w[c, ci, j].
    rng = np.random.default_rng(2)
    w = rng.normal(size=(5, 2, 10))
    for j in range(10):
        x = np.zeros((40, 2))
        x[j, 1] = 1.0
        y = O.conv1d(x, w, None, 5)
        assert np.allclose(y[0], w[:, 1, j])


def test_conv_matches_torch():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(301, 7))
    w = rng.normal(size=(6, 7, 3))
    b = rng.normal(size=6)
    ref = F.conv1d(torch.tensor(x.T[None]), torch.tensor(w), torch.tensor(b), stride=2)[0].numpy().T
    assert np.allclose(O.conv1d(x, w, b, 2), ref, atol=1e-12)


# ---------------------------------------------------------------------- norms
def test_group_norm_invariants_and_torch():
    rng = np.random.default_rng(4)
    y = rng.normal(3.0, 2.0, size=(200, 16)) * rng.uniform(0.5, 4, 16)
    z = O.group_norm_per_channel(y, np.ones(16), np.zeros(16), 1e-5)
    assert np.allclose(z.mean(0), 0, atol=1e-12)
    assert np.allclose(z.var(0), 1, atol=1e-5)  # var/(var+eps)
    g, b = rng.normal(size=16), rng.normal(size=16)
    ref = F.group_norm(torch.tensor(y.T[None]), 16, torch.tensor(g), torch.tensor(b), eps=1e-5)[0].numpy().T
    assert np.allclose(O.group_norm_per_channel(y, g, b, 1e-5), ref, atol=1e-12)


def test_layer_norm_invariants_and_torch():
    rng = np.random.default_rng(5)
    x = rng.normal(2.0, 3.0, size=(33, 96))
    z = O.layer_norm(x, np.ones(96), np.zeros(96), 1e-5)
    assert np.allclose(z.mean(-1), 0, atol=1e-12)
    assert np.allclose(z.var(-1), 1, atol=1e-5)
    g, b = rng.normal(size=96), rng.normal(size=96)
    ref = F.layer_norm(torch.tensor(x), (96,), torch.tensor(g), torch.tensor(b), eps=1e-5).numpy()
    assert np.allclose(O.layer_norm(x, g, b, 1e-5), ref, atol=1e-12)


# ----------------------------------------------------------------------- GELU
def test_gelu_golden_values():
    for row in _rows("gelu_values.txt"):
        x, ge, gt = map(float, row.split())
        assert abs(float(O.gelu(np.float64(x))) - ge) < 1e-15
        assert abs(float(O.gelu_tanh(np.float64(x))) - gt) < 1e-15


def test_gelu_identities():
    x = np.linspace(-8, 8, 4001)
    # x*Phi(x) - (-x)*Phi(-x) = x (Phi(x) + Phi(-x)) = x
    assert np.allclose(O.gelu(x) - O.gelu(-x), x, atol=1e-14)
    assert np.allclose(O.gelu_tanh(x) - O.gelu_tanh(-x), x, atol=1e-14)
    d = np.abs(O.gelu(np.linspace(-6, 6, 1200001)) - O.gelu_tanh(np.linspace(-6, 6, 1200001)))
    assert 4.70e-4 < d.max() < 4.76e-4
    xt = torch.tensor(x)
    assert np.allclose(O.gelu(x), F.gelu(xt).numpy(), atol=1e-15)
    assert np.allclose(O.gelu_tanh(x), F.gelu(xt, approximate="tanh").numpy(), atol=1e-15)


# ------------------------------------------------------------- positional conv
def _pos_shape(d):
    return S.small_shape(d_model=d)


def test_posconv_delta_tap_shifts():
    # Weight = identity channel map at a single tap j, zero bias: before GELU
    # the output at t is x[t + j - 64] (zero outside [0, T)).
    d, T = 32, 150
    m = d // 16
    rng = np.random.default_rng(6)
    x = rng.normal(size=(T, d))
    for j in (0, 1, 63, 64, 65, 127):
        w = np.zeros((d, m, 128))
        for c in range(d):
            w[c, c % m, j] = 1.0
        W = {"pos_conv.weight": w, "pos_conv.bias": np.zeros(d)}
        shape = _pos_shape(d)
        p = O.positional_conv(shape, W, x)
        sh = np.zeros((T, d))
        for t in range(T):
            src = t + j - 64
            if 0 <= src < T:
                sh[t] = x[src]
        assert p.shape == (T, d)
        assert np.allclose(p, O.gelu(sh), atol=1e-14), j


def test_posconv_matches_torch():
    d, T = 64, 97
    rng = np.random.default_rng(7)
    x = rng.normal(size=(T, d))
    w = rng.normal(size=(d, d // 16, 128)) * 0.05
    b = rng.normal(size=d)
    W = {"pos_conv.weight": w, "pos_conv.bias": b}
    ref = F.conv1d(torch.tensor(x.T[None]), torch.tensor(w), torch.tensor(b), padding=64, groups=16)[0, :, :-1]
    ref = F.gelu(ref).numpy().T
    assert np.allclose(O.positional_conv(_pos_shape(d), W, x), ref, atol=1e-12)


# ------------------------------------------------------------------ attention
def _attn_weights(d, rng, zero_q=False):
    W = {}
    for nm in ("q", "k", "v", "out"):
        W[f"l.attn.{nm}.weight"] = rng.normal(size=(d, d)) * 0.3
        W[f"l.attn.{nm}.bias"] = rng.normal(size=d) * 0.1
    if zero_q:
        W["l.attn.q.weight"][:] = 0
        W["l.attn.q.bias"][:] = 0
    return W


def test_attention_brute_force_tiny():
    T, H, dh = 3, 2, 4
    d = H * dh
    rng = np.random.default_rng(8)
    h = rng.normal(size=(T, d))
    W = _attn_weights(d, rng)
    sh = S.small_shape(d_model=d, n_heads=H)
    got = O.self_attention(sh, W, "l.", h)
    q = h @ W["l.attn.q.weight"].T + W["l.attn.q.bias"]
    k = h @ W["l.attn.k.weight"].T + W["l.attn.k.bias"]
    v = h @ W["l.attn.v.weight"].T + W["l.attn.v.bias"]
    o = np.zeros((T, d))
    for hh in range(H):
        for i in range(T):
            sc = [sum(q[i, hh * dh + e] * k[j, hh * dh + e] for e in range(dh)) / math.sqrt(dh) for j in range(T)]
            mx = max(sc)
            ex = [math.exp(s - mx) for s in sc]
            z = sum(ex)
            for e in range(dh):
                o[i, hh * dh + e] = sum(ex[j] / z * v[j, hh * dh + e] for j in range(T))
    ref = o @ W["l.attn.out.weight"].T + W["l.attn.out.bias"]
    assert np.allclose(got, ref, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(9)
    H, dh = 2, 64
    d = H * dh
    sh = S.small_shape(d_model=d, n_heads=H)
    # q == 0: uniform weights, output is the mean of V rows (then out_proj).
    h = rng.normal(size=(7, d))
    W = _attn_weights(d, rng, zero_q=True)
    v = h @ W["l.attn.v.weight"].T + W["l.attn.v.bias"]
    ref = np.tile(v.mean(0), (7, 1)) @ W["l.attn.out.weight"].T + W["l.attn.out.bias"]
    assert np.allclose(O.self_attention(sh, W, "l.", h), ref, atol=1e-12)
    # T == 1: output is V itself.
    W = _attn_weights(d, rng)
    h1 = rng.normal(size=(1, d))
    v1 = h1 @ W["l.attn.v.weight"].T + W["l.attn.v.bias"]
    assert np.allclose(O.self_attention(sh, W, "l.", h1), v1 @ W["l.attn.out.weight"].T + W["l.attn.out.bias"], atol=1e-12)
    # softmax rows sum to one and are invariant to a per-row shift.
    s = rng.normal(size=(5, 9)) * 4
    P = O.softmax_rows(s)
    assert np.allclose(P.sum(-1), 1, atol=1e-14)
    assert np.allclose(O.softmax_rows(s + 100.0), P, atol=1e-14)


def test_attention_matches_torch_sdpa():
    H, dh, T = 3, 64, 41
    d = H * dh
    rng = np.random.default_rng(10)
    h = rng.normal(size=(T, d))
    W = _attn_weights(d, rng)
    sh = S.small_shape(d_model=d, n_heads=H)
    q, k, v = (torch.tensor(h @ W[f"l.attn.{n}.weight"].T + W[f"l.attn.{n}.bias"]).view(T, H, dh).transpose(0, 1) for n in "qkv")
    o = F.scaled_dot_product_attention(q[None], k[None], v[None])[0].transpose(0, 1).reshape(T, d).numpy()
    ref = o @ W["l.attn.out.weight"].T + W["l.attn.out.bias"]
    assert np.allclose(O.self_attention(sh, W, "l.", h), ref, atol=1e-12)


# ------------------------------------------------------------------------ CTC
def test_ctc_collapse_golden():
    for row in _rows("ctc_cases.txt"):
        lhs, rhs = row.split("->")
        ids = [int(v) for v in lhs.split()]
        want = [int(v) for v in rhs.split()]
        assert O.ctc_collapse(ids, 0) == want, row


def test_argmax_lowest_index_on_ties():
    z = np.array([[1.0, 3.0, 3.0, 0.0], [2.0, 2.0, 2.0, 2.0], [-1.0, -5.0, -1.0, -2.0]])
    assert list(O.argmax_lowest(z)) == [1, 0, 0]


def test_ctc_greedy_valid_frames_only():
    z = np.zeros((6, 4))
    for t, a in enumerate([1, 1, 0, 2, 3, 3]):
        z[t, a] = 1.0
    assert O.ctc_greedy(z, 6) == [1, 2, 3]
    assert O.ctc_greedy(z, 4) == [1, 2]
    assert O.ctc_greedy(z, 0) == []


# ----------------------------------------------------------------- input recipe
def test_pcm_recipe_is_normalised_and_seeded():
    x = S.synth_pcm(16000, 0)
    assert x.dtype == np.float32 and x.shape == (16000,)
    assert abs(float(x.astype(np.float64).mean())) < 1e-6
    assert abs(float(x.astype(np.float64).var()) - 1.0) < 1e-5
    assert np.array_equal(x, S.synth_pcm(16000, 0))
    assert not np.array_equal(x, S.synth_pcm(16000, 1))
    w = S.workload("c1")
    short = w.calls[1][0][0]
    assert np.all(short[59200:] == 0) and O.num_frames(59200) == 184


def test_manifest_and_blob_roundtrip():
    sh = S.small_shape()
    W = S.init_weights(sh, 0)
    blob = S.pack_blob(sh, W)
    assert blob.size == sum(int(np.prod(s)) for _, s in S.weight_manifest(sh))
    off = 0
    for name, shp in S.weight_manifest(sh):
        n = int(np.prod(shp))
        assert np.array_equal(blob[off:off + n].reshape(shp), W[name])
        off += n


# ---------------------------------------------- whole model vs an independent one
def _hf_model(shape):
    transformers = pytest.importorskip("transformers")
    cfg = transformers.Wav2Vec2Config(
        hidden_size=shape.d_model, num_hidden_layers=shape.n_layers, num_attention_heads=shape.n_heads,
        intermediate_size=shape.d_ffn, vocab_size=shape.vocab, feat_extract_norm=shape.conv_norm,
        do_stable_layer_norm=shape.stable_layer_norm, conv_bias=shape.conv_bias,
        num_conv_pos_embeddings=128, num_conv_pos_embedding_groups=16,
        hidden_act="gelu_pytorch_tanh" if shape.gelu_tanh else "gelu",
        feat_extract_activation="gelu_pytorch_tanh" if shape.gelu_tanh else "gelu",
        layer_norm_eps=shape.ln_eps, hidden_dropout=0.0, attention_dropout=0.0, activation_dropout=0.0,
        feat_proj_dropout=0.0, final_dropout=0.0, layerdrop=0.0, apply_spec_augment=False)
    return transformers.Wav2Vec2ForCTC(cfg).double().eval()


def _load_hf(model, shape, W):
    sd = {}
    fe = "wav2vec2.feature_extractor.conv_layers."
    for i in range(7):
        sd[f"{fe}{i}.conv.weight"] = W[f"conv{i}.weight"]
        if shape.conv_bias:
            sd[f"{fe}{i}.conv.bias"] = W[f"conv{i}.bias"]
        if shape.conv_norm == "layer" or i == 0:
            sd[f"{fe}{i}.layer_norm.weight"] = W[f"conv{i}.norm.weight"]
            sd[f"{fe}{i}.layer_norm.bias"] = W[f"conv{i}.norm.bias"]
    fp = "wav2vec2.feature_projection."
    sd[fp + "layer_norm.weight"], sd[fp + "layer_norm.bias"] = W["fp.norm.weight"], W["fp.norm.bias"]
    sd[fp + "projection.weight"], sd[fp + "projection.bias"] = W["fp.proj.weight"], W["fp.proj.bias"]
    pc = "wav2vec2.encoder.pos_conv_embed.conv."
    wv = np.asarray(W["pos_conv.weight"], dtype=np.float64)
    # weight_norm over dim 2: weight = g * v / ||v||, the norm taken over dims (0, 1)
    sd[pc + "parametrizations.weight.original1"] = wv
    sd[pc + "parametrizations.weight.original0"] = np.sqrt((wv ** 2).sum(axis=(0, 1), keepdims=True))
    sd[pc + "bias"] = W["pos_conv.bias"]
    sd["wav2vec2.encoder.layer_norm.weight"], sd["wav2vec2.encoder.layer_norm.bias"] = W["enc.norm.weight"], W["enc.norm.bias"]
    for l in range(shape.n_layers):
        p, q = f"layers.{l}.", f"wav2vec2.encoder.layers.{l}."
        for a, b in (("q", "q_proj"), ("k", "k_proj"), ("v", "v_proj"), ("out", "out_proj")):
            sd[f"{q}attention.{b}.weight"] = W[f"{p}attn.{a}.weight"]
            sd[f"{q}attention.{b}.bias"] = W[f"{p}attn.{a}.bias"]
        sd[q + "layer_norm.weight"], sd[q + "layer_norm.bias"] = W[p + "attn_norm.weight"], W[p + "attn_norm.bias"]
        sd[q + "feed_forward.intermediate_dense.weight"] = W[p + "ffn.in.weight"]
        sd[q + "feed_forward.intermediate_dense.bias"] = W[p + "ffn.in.bias"]
        sd[q + "feed_forward.output_dense.weight"] = W[p + "ffn.out.weight"]
        sd[q + "feed_forward.output_dense.bias"] = W[p + "ffn.out.bias"]
        sd[q + "final_layer_norm.weight"], sd[q + "final_layer_norm.bias"] = W[p + "ffn_norm.weight"], W[p + "ffn_norm.bias"]
    sd["lm_head.weight"], sd["lm_head.bias"] = W["lm_head.weight"], W["lm_head.bias"]
    sd = {k: torch.tensor(np.asarray(v, dtype=np.float64)) for k, v in sd.items()}
    missing, unexpected = model.load_state_dict(sd, strict=False)
    assert not unexpected, unexpected
    assert set(missing) <= {"wav2vec2.masked_spec_embed"}, missing


@pytest.mark.parametrize("layout", ["group_post", "group_post_tanh", "layer_stable", "layer_stable_tanh"])
def test_whole_model_matches_transformers(layout):
    group = layout.startswith("group")
    shape = S.small_shape(conv_norm="group" if group else "layer", stable=not group, conv_bias=not group,
                          gelu_tanh=layout.endswith("tanh"), d_model=128, n_layers=2, n_heads=2, d_ffn=256, vocab=40)
    W = S.init_weights(shape, seed=11, affine_noise=True)
    W64 = O.to_f64(W)
    model = _hf_model(shape)
    _load_hf(model, shape, W)
    pcm = S.synth_pcm(6000, 12)
    with torch.no_grad():
        ref = model(torch.tensor(pcm.astype(np.float64))[None]).logits[0].numpy()
    got = O.forward(shape, W64, pcm)
    assert got.shape == ref.shape == (O.num_frames(6000), 40)
    assert np.abs(got - ref).max() < 1e-9 * max(1.0, np.abs(ref).max())
