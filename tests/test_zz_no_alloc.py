"""The allocation-free greedy CTC entry point (w2v_ctc_greedy_static).

It serves callers that may not allocate device memory while decoding (for
example work queued from a real-time audio callback, or a host application
that owns all GPU memory).  It must give exactly the tokens of w2v_ctc_greedy,
including on a second call right after the first, whose inputs differ: the
shared scratch array keeps the previous call's ids and must not leak them.
This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from speech_encoder_b200 import w2v as B
from synth import inputs as S

pytestmark = pytest.mark.gpu


def _logits(seed, batch, T, V):
    rng = np.random.default_rng(seed)
    z = rng.normal(size=(batch, T, V)).astype(np.float32)
    ids = rng.integers(0, min(V, 5), size=(batch, T))
    z[np.arange(batch)[:, None], np.arange(T)[None], ids] += 4.0
    z[:, ::13, 2] = z[:, ::13, 3] = 40.0  # exact ties: the lower index must win
    return torch.from_numpy(z).cuda()


def _decode_existing(model, lg, batch, T, t_valid):
    tok = torch.full((batch, max(t_valid, 1)), -7, dtype=torch.int32, device="cuda")
    nt = torch.full((batch,), -7, dtype=torch.int32, device="cuda")
    B.w2v_ctc_greedy(model.handle, lg, batch, T, t_valid, tok, nt)
    return tok, nt


def _decode_static(lg, batch, T, V, t_valid, blank=0):
    tok = torch.full((batch, max(t_valid, 1)), -7, dtype=torch.int32, device="cuda")
    nt = torch.full((batch,), -7, dtype=torch.int32, device="cuda")
    rc = B.w2v_ctc_greedy_static(lg, batch, T, V, t_valid, blank, tok, nt)
    assert rc == B.W2V_OK, rc
    return tok, nt


def _same(a, b):
    ta, na = a
    tb, nb = b
    torch.cuda.synchronize()
    assert torch.equal(na, nb)
    for i in range(na.shape[0]):
        n = int(na[i])
        assert torch.equal(ta[i, :n], tb[i, :n])


def test_static_ctc_matches_existing_entry_point_on_two_calls_in_a_row():
    V = 32
    shape = S.small_shape(vocab=V)
    model = B.Model(shape, S.pack_blob(shape, S.init_weights(shape, 0)), max_samples=320000, max_batch=4)
    # first call: 4 clips x 999 frames, all frames decoded
    lg1 = _logits(1, 4, 999, V)
    _same(_decode_static(lg1, 4, 999, V, 999), _decode_existing(model, lg1, 4, 999, 999))
    # second call right after: fewer, shorter rows and a partial valid range,
    # so stale ids from the first call would show up if they were read
    lg2 = _logits(2, 2, 799, V)
    _same(_decode_static(lg2, 2, 799, V, 184), _decode_existing(model, lg2, 2, 799, 184))
    model.sync()
    model.close()


def test_static_ctc_allocates_nothing_after_its_first_call():
    # After the first call on a device has loaded the library's array, a call
    # changes the device's free memory by nothing: the scratch is the fixed
    # array, not an allocation.  Also covers a blank id other than 0 (against
    # the existing entry point of a model whose blank id is 5) and an empty
    # valid range (every count 0).
    V = 32
    shape = S.small_shape(vocab=V).with_(blank_id=5)
    model = B.Model(shape, S.pack_blob(shape, S.init_weights(shape, 0)), max_samples=320000, max_batch=4)
    lg = _logits(3, 3, 640, V)
    out_a = _decode_static(lg, 3, 640, V, 640, blank=5)  # first call: loads the array if not yet loaded
    torch.cuda.synchronize()
    tok = torch.full((3, 640), -7, dtype=torch.int32, device="cuda")
    nt = torch.full((3,), -7, dtype=torch.int32, device="cuda")
    tok0 = torch.full((3, 1), -7, dtype=torch.int32, device="cuda")
    nt0 = torch.full((3,), -7, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    assert B.w2v_ctc_greedy_static(lg, 3, 640, V, 640, 5, tok, nt) == B.W2V_OK
    assert B.w2v_ctc_greedy_static(lg, 3, 640, V, 0, 5, tok0, nt0) == B.W2V_OK
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, (free_before, free_after)
    _same((tok, nt), out_a)
    _same((tok, nt), _decode_existing(model, lg, 3, 640, 640))
    assert nt0.cpu().tolist() == [0, 0, 0]
    model.sync()
    model.close()


def test_static_ctc_rejects_sizes_beyond_its_array():
    lg = torch.zeros(16, dtype=torch.float32, device="cuda")
    tok = torch.zeros(16, dtype=torch.int32, device="cuda")
    nt = torch.zeros(16, dtype=torch.int32, device="cuda")
    too_many = (1 << 20) // 1000 + 1
    assert B.w2v_ctc_greedy_static(lg, too_many, 1000, 32, 10, 0, tok, nt) == B.W2V_ESHAPE
    assert B.w2v_ctc_greedy_static(lg, 1, 10, 32, 11, 0, tok, nt) == B.W2V_ESHAPE
    assert B.w2v_ctc_greedy_static(lg, 1, 10, 32, 5, 32, tok, nt) == B.W2V_EINVAL
    torch.cuda.synchronize()
