"""The varlen batched forward (w2v_forward_varlen / w2v_ctc_greedy_varlen):
clips of different lengths in one launch set, each processed at its own true
length.  Every clip's logits are compared with the fp64 oracle run on that
clip alone (same bar as the other whole-model tests), and the packed decode
with the oracle's decode of the same logits."""
import numpy as np
import pytest
import torch

from oracle import w2v_oracle as O
from speech_encoder_b200 import w2v as B
from synth import inputs as S

import w2v_testutil as U

pytestmark = pytest.mark.gpu


def _check_clips(model, shape, clips_np, what, seed=0, affine_noise=False):
    clips = [torch.from_numpy(c).cuda() for c in clips_np]
    logits, frames = model.forward_varlen(clips)
    model.sync()
    assert frames == [O.num_frames(len(c)) for c in clips_np]
    assert logits.shape == (sum(frames), shape.vocab)
    got = logits.cpu().numpy()
    off = 0
    for i, (c, T) in enumerate(zip(clips_np, frames)):
        ref = U.oracle_logits(shape, c, seed=seed, affine_noise=affine_noise)
        print(what, i, len(c), U.compare_logits(got[off:off + T], ref, f"{what} clip {i} (n={len(c)})"))
        off += T
    toks = model.ctc_greedy_varlen(logits, frames)
    off = 0
    for i, T in enumerate(frames):
        want = O.ctc_greedy(got[off:off + T], T, shape.blank_id)
        assert toks[i].cpu().tolist() == want, (what, i)
        off += T
    return got, frames


@pytest.mark.parametrize("layout", ["group_post", "layer_stable"])
def test_small_model_varlen_matches_oracle_per_clip(layout):
    kw = dict(conv_norm="group", stable=False) if layout == "group_post" else \
        dict(conv_norm="layer", stable=True, conv_bias=True)
    shape = S.small_shape(**kw)
    model = U.make_model(shape, max_samples=48000, max_batch=6, seed=3, affine_noise=True)
    # lengths: a 1-frame clip, one exactly 128 frames, ragged others
    lens = [41234, 400, 16000, 40960 + 400 - 320 + 1, 23456, 47999]
    clips = [S.synth_pcm(n, 60 + i) for i, n in enumerate(lens)]
    assert O.num_frames(lens[3]) == 128
    got, frames = _check_clips(model, shape, clips, layout, seed=3, affine_noise=True)
    # the same clips one by one through the fixed-length entry point agree too
    off = 0
    for c, T in zip(clips, frames):
        one = model.forward(torch.from_numpy(c[None]).cuda())
        model.sync()
        np.testing.assert_allclose(one[0].cpu().numpy(), got[off:off + T], atol=2e-2, rtol=0)
        off += T
    # a second call with a different set (other bucket) reuses the model
    _check_clips(model, shape, clips[:2][::-1], layout + " second", seed=3, affine_noise=True)
    model.close()


def test_c4_true_length_clips_in_one_varlen_call():
    w = S.workload("c4")
    model = U.make_model(w.model, 320000, 8)
    clips = [p[0] for p, _ in w.calls]
    clips_t = [torch.from_numpy(c).cuda() for c in clips]
    logits, frames = model.forward_varlen(clips_t)
    model.sync()
    got = logits.cpu().numpy()
    off = 0
    for i, T in enumerate(frames):
        print("c4 varlen", i, len(clips[i]),
              U.compare_logits(got[off:off + T], U.oracle_workload_clip("c4", i, 0), f"c4 varlen clip {i}"))
        off += T
    model.close()


def test_varlen_rejects_bad_arguments():
    shape = S.small_shape()
    m = U.make_model(shape, 20000, 2)
    pcm = torch.zeros(40000, device="cuda")
    lg = torch.zeros(200, shape.vocab, device="cuda")
    L = B.lib()
    arr3, _ = B._int_array([16000, 16000, 16000])
    arr_short, _ = B._int_array([16000, 399])
    arr_long, _ = B._int_array([20001])
    assert L.w2v_forward_varlen(m.handle, pcm.data_ptr(), arr3, 3, lg.data_ptr(), None) == B.W2V_ESHAPE
    assert L.w2v_forward_varlen(m.handle, pcm.data_ptr(), arr_short, 2, lg.data_ptr(), None) == B.W2V_ESHAPE
    assert L.w2v_forward_varlen(m.handle, pcm.data_ptr(), arr_long, 1, lg.data_ptr(), None) == B.W2V_ESHAPE
    assert L.w2v_forward_varlen(m.handle, pcm.data_ptr() + 4, arr3, 1, lg.data_ptr(), None) == B.W2V_EINVAL
    assert L.w2v_forward_varlen(m.handle, pcm.data_ptr(), None, 1, lg.data_ptr(), None) == B.W2V_EINVAL
    m.sync()
    m.close()
