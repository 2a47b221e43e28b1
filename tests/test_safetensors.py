"""Checkpoint loader (host only, no GPU): a single-file safetensors checkpoint
with the checkpoint's module names, mixed dtypes and a weight-normalised
positional conv packs into exactly the weight blob w2v_create expects; the
weight-norm fold matches its definition g * v / ||v||; malformed files, missing
tensors and wrong shapes are refused with the tensor named."""
import json
import os
import struct

import numpy as np
import pytest

from speech_encoder_b200 import w2v as B
from synth import inputs as S


def _ckpt_name(m):
    """The checkpoint module path of a manifest name (the interface of the
    loader, restated here independently)."""
    p = m.split(".")
    if p[0].startswith("conv"):
        i = p[0][4:]
        if p[1] == "norm":
            return f"feature_extractor.conv_layers.{i}.layer_norm.{p[2]}"
        return f"feature_extractor.conv_layers.{i}.conv.{p[1]}"
    if p[0] == "fp":
        return {"norm": "feature_projection.layer_norm", "proj": "feature_projection.projection"}[p[1]] + "." + p[2]
    if p[0] == "pos_conv":
        return "encoder.pos_conv_embed.conv." + p[1]
    if p[0] == "enc":
        return "encoder.layer_norm." + p[2]
    if p[0] == "layers":
        l, rest = p[1], p[2:]
        pre = f"encoder.layers.{l}."
        if rest[0] == "attn":
            return pre + f"attention.{rest[1]}_proj.{rest[2]}"
        if rest[0] == "attn_norm":
            return pre + "layer_norm." + rest[1]
        if rest[0] == "ffn":
            return pre + {"in": "feed_forward.intermediate_dense", "out": "feed_forward.output_dense"}[rest[1]] + \
                "." + rest[2]
        if rest[0] == "ffn_norm":
            return pre + "final_layer_norm." + rest[1]
    if p[0] == "lm_head":
        return m
    raise KeyError(m)


def _bf16_bits(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)  # round to nearest even


def _bits_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def write_safetensors(path, tensors, metadata=None, pad_header=True):
    """tensors: name -> (dtype str, numpy array in that dtype's storage)."""
    header, blobs, off = {}, [], 0
    for name, (dt, arr) in tensors.items():
        raw = np.ascontiguousarray(arr).tobytes()
        header[name] = {"dtype": dt, "shape": list(arr.shape), "data_offsets": [off, off + len(raw)]}
        blobs.append(raw)
        off += len(raw)
    if metadata is not None:
        header["__metadata__"] = metadata
    h = json.dumps(header).encode()
    if pad_header:
        h += b" " * ((8 - len(h) % 8) % 8)
    with open(path, "wb") as f:
        f.write(struct.pack("<Q", len(h)))
        f.write(h)
        for b in blobs:
            f.write(b)


def _fixture(cfg, prefix="wav2vec2.", wn="weight_g", seed=7):
    """A checkpoint dict of every manifest tensor with random values, plus the
    blob the loader must produce from it."""
    rng = np.random.default_rng(seed)
    man = B.w2v_weight_manifest(cfg)
    total = B.w2v_weight_count(cfg)
    want = np.zeros(total, dtype=np.float32)
    tensors = {}
    for k, (name, shape, off) in enumerate(man):
        cnt = int(np.prod(shape))
        x = rng.standard_normal(shape).astype(np.float32)
        ck = _ckpt_name(name)
        ck = ck if name.startswith("lm_head") else prefix + ck
        if name == "pos_conv.weight" and wn:
            g = (1.0 + rng.random((1, 1, shape[2]))).astype(np.float32)  # weight norm kept along the taps
            v = x
            base = ck[:-len("weight")]
            gname, vname = (base + "weight_g", base + "weight_v") if wn == "weight_g" else \
                (base + "parametrizations.weight.original0", base + "parametrizations.weight.original1")
            tensors[gname] = ("F32", g)
            tensors[vname] = ("F16", v.astype(np.float16))
            want_v16 = v.astype(np.float16).astype(np.float64)
            norm16 = np.sqrt((want_v16 ** 2).sum(axis=(0, 1), keepdims=True))
            want[off:off + cnt] = (g.astype(np.float64) * want_v16 / norm16).astype(np.float32).ravel()
            continue
        kind = k % 3
        if kind == 0:
            tensors[ck] = ("F32", x)
            want[off:off + cnt] = x.ravel()
        elif kind == 1:
            h = x.astype(np.float16)
            tensors[ck] = ("F16", h)
            want[off:off + cnt] = h.astype(np.float32).ravel()
        else:
            bits = _bf16_bits(x)
            tensors[ck] = ("BF16", bits)
            want[off:off + cnt] = _bits_to_f32(bits).ravel()
    return tensors, want, man


@pytest.fixture(scope="module")
def cfg():
    B.lib()
    return B.make_config(S.small_shape(), 48000, 1)


@pytest.mark.parametrize("prefix,wn,layout", [("wav2vec2.", "weight_g", "group_post"), ("", "param", "group_post"),
                                               ("wav2vec2.", "weight_g", "layer_stable")])
def test_pack_matches_the_manifest_blob(tmp_path, prefix, wn, layout):
    B.lib()
    kw = {} if layout == "group_post" else dict(conv_norm="layer", stable=True, conv_bias=True)
    cfg = B.make_config(S.small_shape(**kw), 48000, 1)
    tensors, want, man = _fixture(cfg, prefix=prefix, wn=wn)
    path = tmp_path / "model.safetensors"
    write_safetensors(path, tensors, metadata={"format": "pt"})
    got = B.w2v_pack_safetensors(str(path), cfg)
    pos = [(o, int(np.prod(s))) for n, s, o in man if n == "pos_conv.weight"][0]
    mask = np.ones_like(want, dtype=bool)
    mask[pos[0]:pos[0] + pos[1]] = False
    assert np.array_equal(got[mask], want[mask])
    np.testing.assert_allclose(got[~mask], want[~mask], rtol=2e-7, atol=1e-9)


def test_weight_norm_fold_definition(cfg, tmp_path):
    # every tap's slice of the folded weight has Frobenius norm g[k]
    tensors, _, man = _fixture(cfg)
    path = tmp_path / "m.safetensors"
    write_safetensors(path, tensors)
    got = B.w2v_pack_safetensors(str(path), cfg)
    name, shape, off = [e for e in man if e[0] == "pos_conv.weight"][0]
    w = got[off:off + int(np.prod(shape))].reshape(shape).astype(np.float64)
    g = [t for n, t in tensors.items() if n.endswith("weight_g")][0][1].reshape(-1)
    np.testing.assert_allclose(np.sqrt((w ** 2).sum(axis=(0, 1))), g, rtol=1e-6)


def test_manifest_names_and_prefolded_weight_are_accepted(cfg, tmp_path):
    man = B.w2v_weight_manifest(cfg)
    rng = np.random.default_rng(1)
    want = np.zeros(B.w2v_weight_count(cfg), dtype=np.float32)
    tensors = {}
    for name, shape, off in man:
        x = rng.standard_normal(shape).astype(np.float32)
        tensors[name] = ("F32", x)  # the manifest's own names, pos_conv already folded
        want[off:off + x.size] = x.ravel()
    path = tmp_path / "m.safetensors"
    write_safetensors(path, tensors, pad_header=False)
    assert np.array_equal(B.w2v_pack_safetensors(str(path), cfg), want)


def test_missing_tensor_wrong_shape_and_bad_files_are_refused(cfg, tmp_path):
    tensors, _, _ = _fixture(cfg)
    path = tmp_path / "m.safetensors"
    t2 = dict(tensors)
    gone = "wav2vec2.encoder.layers.0.feed_forward.output_dense.bias"
    del t2[gone]
    write_safetensors(path, t2)
    with pytest.raises(B.W2VError) as ei:
        B.w2v_pack_safetensors(str(path), cfg)
    assert ei.value.code == B.W2V_EINVAL and "layers.0.ffn.out.bias" in str(ei.value)

    t3 = dict(tensors)
    name = "wav2vec2.feature_projection.projection.weight"
    dt, a = t3[name]
    t3[name] = (dt, a[:, :-1].copy())
    write_safetensors(path, t3)
    with pytest.raises(B.W2VError) as ei:
        B.w2v_pack_safetensors(str(path), cfg)
    assert ei.value.code == B.W2V_ESHAPE and "feature_projection.projection.weight" in str(ei.value)

    write_safetensors(path, tensors)
    data = path.read_bytes()
    (tmp_path / "short.safetensors").write_bytes(data[:len(data) - 100])
    with pytest.raises(B.W2VError, match="past the end"):
        B.w2v_pack_safetensors(str(tmp_path / "short.safetensors"), cfg)
    (tmp_path / "junk.safetensors").write_bytes(struct.pack("<Q", 5) + b"{oops")
    with pytest.raises(B.W2VError, match="bad header"):
        B.w2v_pack_safetensors(str(tmp_path / "junk.safetensors"), cfg)
    with pytest.raises(B.W2VError, match="cannot open"):
        B.w2v_pack_safetensors(str(tmp_path / "absent.safetensors"), cfg)
    t4 = dict(tensors)
    t4["wav2vec2.encoder.layer_norm.weight"] = ("I32", np.zeros(t4["wav2vec2.encoder.layer_norm.weight"][1].shape,
                                                                dtype=np.int32))
    write_safetensors(path, t4)
    with pytest.raises(B.W2VError, match="unsupported dtype"):
        B.w2v_pack_safetensors(str(path), cfg)


@pytest.mark.parametrize("layout", ["group_post", "layer_stable"])
def test_loader_on_a_transformers_checkpoint_reproduces_its_logits(tmp_path, layout):
    # An independent pin of the name map and the weight-norm fold: a randomly
    # initialised transformers Wav2Vec2ForCTC (its own parameter names, its
    # positional conv under weight normalisation, g perturbed away from ||v||)
    # saved as safetensors, packed by the loader, run through the oracle,
    # gives the module's own logits.
    torch = pytest.importorskip("torch")
    from oracle import w2v_oracle as O
    from test_oracle_pins import _hf_model
    group = layout.startswith("group")
    shape = S.small_shape(conv_norm="group" if group else "layer", stable=not group, conv_bias=not group)
    torch.manual_seed(3)
    model = _hf_model(shape)
    sd = model.state_dict()
    gk = [k for k in sd if k.endswith("parametrizations.weight.original0") or k.endswith("weight_g")]
    assert len(gk) == 1
    with torch.no_grad():
        sd[gk[0]].mul_(1.0 + 0.5 * torch.rand_like(sd[gk[0]]))
        for k, v in sd.items():  # make biases and norm affines non-trivial too
            if k.endswith("bias") or "layer_norm" in k:
                v.add_(0.1 * torch.randn_like(v))
    model.load_state_dict(sd)
    tensors = {k: ("F32", v.float().numpy()) for k, v in sd.items()}
    path = tmp_path / "model.safetensors"
    write_safetensors(path, tensors)
    B.lib()
    cfg = B.make_config(shape, 48000, 1)
    blob = B.w2v_pack_safetensors(str(path), cfg)
    W = {name: blob[off:off + int(np.prod(shp))].reshape(shp) for name, shp, off in B.w2v_weight_manifest(cfg)}
    pcm = S.synth_pcm(6000, 12)
    with torch.no_grad():
        ref = model(torch.tensor(pcm.astype(np.float64))[None]).logits[0].numpy()
    got = O.forward(shape, O.to_f64(W), pcm)
    # the checkpoint went through fp32: agreement to fp32 rounding of the weights
    assert np.abs(got - ref).max() < 1e-4 * max(1.0, np.abs(ref).max())
