"""Data-parallel transcription of independent clips, one process per GPU.

The forward pass of one clip does not shard (its GEMMs and attention are too
small to split), so several GPUs serve a set of independent clips: each rank
transcribes a share of the clips on its own model replica, with no collective
on the data path, and one gather brings the token sequences to rank 0.

Shares are chosen longest-first (LPT): clips sorted by length, longest first,
each given to the rank with the fewest samples so far.  The busiest rank then
carries at most 4/3 of the optimal makespan, and for the throughput batches of
equal-length clips the shares differ by at most one clip.

Every rank makes the same collective call whatever happened locally: a clip
that fails on one rank is reported to rank 0 through the gather, and every
rank raises after it, so that no rank is left waiting in a collective.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import numpy as np


class ShardError(RuntimeError):
    """A clip failed on some rank; raised on every rank after the gather."""


def lpt_partition(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Clip indices per rank, in the order each rank processes them.

    Longest first (ties: lower clip index first); each clip goes to the rank
    with the smallest total length so far (ties: lower rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    load = [0] * world
    shares: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        shares[r].append(i)
        load[r] += int(lengths[i])
    return shares


def run_sharded(lengths: Sequence[int], decode: Callable[[int], np.ndarray], rank: int, world: int,
                group=None) -> Optional[List[np.ndarray]]:
    """Decodes this rank's share of the clips with decode(i) -> int32 tokens,
    then gathers every clip's tokens to rank 0 in clip order.

    Returns the list on rank 0 and None elsewhere.  With world == 1 no
    process group is needed.  Raises ShardError on every rank if any clip
    failed anywhere (after the gather)."""
    share = lpt_partition(lengths, world)[rank]
    mine = {}
    err = None
    for i in share:
        try:
            mine[i] = np.asarray(decode(i), dtype=np.int32)
        except Exception as ex:  # reported through the gather, raised below
            err = f"rank {rank} clip {i}: {type(ex).__name__}: {ex}"
            break
    payload = (mine, err)
    if world == 1:
        gathered = [payload]
    else:
        import torch.distributed as dist
        gathered = [None] * world if rank == 0 else None
        dist.gather_object(payload, gathered, dst=0, group=group)
        # rank 0 tells everyone whether any clip failed (one more collective,
        # made by every rank)
        flag = [None]
        if rank == 0:
            errs = [g[1] for g in gathered if g[1] is not None]
            flag = ["; ".join(errs) if errs else ""]
        dist.broadcast_object_list(flag, src=0, group=group)
        if flag[0]:
            raise ShardError(flag[0])
    if world == 1 and err is not None:
        raise ShardError(err)
    if rank != 0:
        return None
    out: List[Optional[np.ndarray]] = [None] * len(lengths)
    for mine_r, _ in gathered:
        for i, tok in mine_r.items():
            out[i] = tok
    missing = [i for i, t in enumerate(out) if t is None]
    if missing:
        raise ShardError(f"clips never decoded: {missing}")
    return out  # type: ignore[return-value]


def transcribe_clips(model, clips: Sequence[np.ndarray], rank: int, world: int, group=None):
    """Greedy-CTC token sequences of independent clips (float32 PCM arrays of
    any lengths >= 400 samples, already normalised) on this rank's model
    replica (a speech_encoder_b200.w2v.Model on this rank's GPU), gathered
    to rank 0 in clip order."""
    from speech_encoder_b200 import w2v as B

    def decode(i: int) -> np.ndarray:
        pcm = np.ascontiguousarray(clips[i], dtype=np.float32)[None]
        T = B.w2v_num_frames(pcm.shape[1])
        tok = np.empty((1, T), dtype=np.int32)
        nt = np.empty((1,), dtype=np.int32)
        B.w2v_transcribe(model.handle, pcm, T, tok, nt)
        return tok[0, :int(nt[0])].copy()

    return run_sharded([len(c) for c in clips], decode, rank, world, group)
