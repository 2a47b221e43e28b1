"""Clip sharding across ranks (host logic of the multi-GPU path), run as two
gloo processes on the CPU: every clip decoded exactly once, rank 0 receives
the token sequences in clip order, shares balanced longest-first, and a clip
that fails on one rank raises on every rank without leaving a collective
hanging."""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch.multiprocessing as mp

from speech_encoder_b200.shard import ShardError, lpt_partition, run_sharded


def test_lpt_partition_is_balanced_and_complete():
    rng = np.random.default_rng(4)
    lengths = rng.integers(32000, 320001, size=8)  # the true-length clip mix
    for world in (1, 2, 3, 4, 8):
        shares = lpt_partition(lengths, world)
        flat = sorted(i for s in shares for i in s)
        assert flat == list(range(len(lengths)))
        loads = [sum(int(lengths[i]) for i in s) for s in shares]
        # Graham's bound for longest-first: makespan <= (4/3 - 1/(3m)) OPT,
        # and OPT >= max(total / m, longest clip)
        opt_lb = max(sum(int(x) for x in lengths) / world, int(lengths.max()))
        assert max(loads) <= (4 / 3 - 1 / (3 * world)) * opt_lb + 1e-6
        for s in shares:  # each rank takes its clips longest first
            assert [int(lengths[i]) for i in s] == sorted((int(lengths[i]) for i in s), reverse=True)


def test_lpt_partition_equal_lengths_round_robin():
    shares = lpt_partition([160000] * 16, 4)  # the batch of 16 ten-second clips
    assert shares == [[0, 4, 8, 12], [1, 5, 9, 13], [2, 6, 10, 14], [3, 7, 11, 15]]
    assert lpt_partition([], 2) == [[], []]
    with pytest.raises(ValueError):
        lpt_partition([1, 2], 0)


def _fake_tokens(i):
    return np.arange(i % 5, dtype=np.int32) + 10 * i


def _worker(rank, world, port, lengths, fail_clip, outdir):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    seen = []

    def decode(i):
        seen.append(i)
        if i == fail_clip:
            raise RuntimeError("injected failure")
        return _fake_tokens(i)

    status = "ok"
    try:
        out = run_sharded(lengths, decode, rank, world)
        if rank == 0:
            assert len(out) == len(lengths)
            for i, t in enumerate(out):
                assert np.array_equal(t, _fake_tokens(i))
        else:
            assert out is None
    except ShardError as ex:
        status = f"shard-error: {ex}"
    np.save(os.path.join(outdir, f"seen{rank}.npy"), np.array(seen, dtype=np.int64))
    with open(os.path.join(outdir, f"status{rank}.txt"), "w") as f:
        f.write(status)
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spawn(lengths, fail_clip):
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), lengths, fail_clip, d), nprocs=world,
                           join=True, start_method="spawn")
        seen = [np.load(os.path.join(d, f"seen{r}.npy")).tolist() for r in range(world)]
        status = [open(os.path.join(d, f"status{r}.txt")).read() for r in range(world)]
    return seen, status


def test_two_gloo_ranks_decode_every_clip_once_and_gather_in_order():
    lengths = [int(x) for x in np.random.default_rng(4).integers(32000, 320001, size=8)]
    seen, status = _spawn(lengths, fail_clip=-1)
    assert status == ["ok", "ok"]
    shares = lpt_partition(lengths, 2)
    assert seen == shares
    assert sorted(seen[0] + seen[1]) == list(range(8))


def test_failure_on_one_rank_raises_on_every_rank():
    lengths = [160000] * 6
    fail = lpt_partition(lengths, 2)[1][1]  # the second clip of rank 1
    seen, status = _spawn(lengths, fail_clip=fail)
    assert all(s.startswith("shard-error") and f"clip {fail}" in s for s in status), status
    assert seen[1][-1] == fail  # rank 1 stopped at the failing clip
