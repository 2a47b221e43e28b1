"""A host model of the attention kernel's mbarrier protocol
(speech_encoder_b200/csrc/k_attention.cu), run under random schedules.

The actors of one CTA are modelled the way the kernel runs them: the TMA
producer (Q once, then K/V tiles into a 3-stage ring), the MMA thread (scores
up to two tiles ahead into three TMEM buffers, P V products in order, completed
products confirmed strictly in order), 16 softmax warps (four per TMEM lane
quarter, a quarter barrier per tile, an occasional accumulator rescale, the
P_{j-2} guard before publishing P_j), an in-order tensor core whose commits
arrive only when every earlier operation has run, and asynchronous TMA
completions.  The barriers follow the hardware's parity rule: a wait for the
phase with parity P passes when the barrier's current phase parity differs
from P.

Each run checks that every actor finishes (no deadlock), that every parity
test aims at the phase it means (a barrier two phases on would make it pass
or fail wrongly), and that no buffer is overwritten early: a score buffer
before all warps read its S and before the P V that reads its P ran, a K/V
stage before its S and P V ran, the accumulator while a rescale reads it.
A negative control replaces the ordered confirmation with the direct parity
test of the product three tiles back, the form that timed out on the GPU, and
must be caught."""
import random

import pytest

KV = 3       # K/V stages and score buffers
WARPS = 16   # softmax warps, four per lane quarter


class ProtocolError(AssertionError):
    pass


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending < 0:
            raise ProtocolError(f"{self.name}: too many arrivals")
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def test(self, parity, want_phase, who):
        passed = (self.phase & 1) != parity
        if self.phase > want_phase + 1 or passed != (self.phase > want_phase):
            raise ProtocolError(f"{who}: parity test on {self.name} for phase {want_phase}, barrier at {self.phase}")
        return passed


def run(nkv, seed, ordered_confirm=True, move_prob=0.2, max_steps=200000):
    rng = random.Random(seed)
    q_full = Bar("q_full", 1)
    kv_full = [Bar(f"kv_full{i}", 1) for i in range(KV)]
    kv_empty = [Bar(f"kv_empty{i}", 1) for i in range(KV)]
    s_full = [Bar(f"s_full{i}", 1) for i in range(KV)]
    p_full = [Bar(f"p_full{i}", WARPS) for i in range(2)]
    pv_done = [Bar(f"pv_done{i}", 1) for i in range(2)]
    tensor, tma = [], []
    s_loaded, p_written, s_ran, pv_ran, kv_landed = {}, {}, set(), set(), set()
    quarter = [dict() for _ in range(4)]

    def wait(bar, phase, who):
        while not bar.test(phase & 1, phase, who):
            yield

    def producer():
        tma.append(("q", q_full, None))
        for j in range(nkv):
            st = j % KV
            if j >= KV:
                yield from wait(kv_empty[st], j // KV - 1, "producer")
                if (j - KV) not in s_ran or (j - KV) not in pv_ran:
                    raise ProtocolError(f"K/V stage {st} refilled before tile {j - KV} was used")
            tma.append(("kv", kv_full[st], j))
            yield

    def mma():
        def issue_s(i):
            tensor.append(("S", i))
            tensor.append(("commit", s_full[i % KV]))

        def issue_pv(j):
            tensor.append(("PV", j))
            tensor.append(("commit", pv_done[j & 1]))
            tensor.append(("commit", kv_empty[j % KV]))

        yield from wait(q_full, 0, "mma q")
        yield from wait(kv_full[0], 0, "mma kv0")
        issue_s(0)
        if nkv > 1:
            yield from wait(kv_full[1], 0, "mma kv1")
            issue_s(1)
        next_s = 2 if nkv > 1 else 1
        pv_seen = 0
        for j in range(nkv):
            have_p = False
            while True:
                if ordered_confirm:
                    while pv_seen < j and pv_done[pv_seen & 1].test((pv_seen >> 1) & 1, pv_seen >> 1, "mma pv"):
                        pv_seen += 1
                    buffer_free = next_s < 3 or pv_seen >= next_s - 2
                else:
                    m = next_s - 3
                    buffer_free = next_s < 3 or (next_s < nkv and pv_done[m & 1].test((m >> 1) & 1, m >> 1, "mma gate"))
                if next_s < nkv and next_s <= j + 2 and buffer_free and \
                        kv_full[next_s % KV].test((next_s // KV) & 1, next_s // KV, "mma kv"):
                    issue_s(next_s)
                    next_s += 1
                if not have_p:
                    have_p = p_full[j & 1].test((j >> 1) & 1, j >> 1, "mma p")
                if have_p and (not ordered_confirm or j < 2 or pv_seen >= j - 1):
                    break
                yield
            issue_pv(j)
            yield

    def warp(w):
        q = w % 4
        for j in range(nkv):
            yield from wait(s_full[j % KV], j // KV, f"warp {w} S")
            s_loaded.setdefault(j, set()).add(w)
            yield
            quarter[q][j] = quarter[q].get(j, 0) + 1
            while quarter[q][j] < 4:
                yield
            if j > 0 and rng.random() < move_prob:
                yield from wait(pv_done[(j - 1) & 1], (j - 1) >> 1, f"warp {w} rescale")
                if (j - 1) not in pv_ran or j in pv_ran:
                    raise ProtocolError("rescale races a P V product")
            yield
            if j >= 2:
                yield from wait(pv_done[j & 1], (j - 2) >> 1, f"warp {w} P guard")
            p_written.setdefault(j, set()).add(w)
            p_full[j & 1].arrive()
            yield
        last = nkv - 1
        yield from wait(pv_done[last & 1], last >> 1, f"warp {w} final")
        if last not in pv_ran:
            raise ProtocolError("accumulator read before the last P V ran")

    actors = {"producer": producer(), "mma": mma()}
    for w in range(WARPS):
        actors[f"warp{w}"] = warp(w)
    done = set()
    for _ in range(max_steps):
        choices = [k for k in actors if k not in done] + (["tensor"] if tensor else []) + (["tma"] if tma else [])
        if not choices:
            return
        k = rng.choice(choices)
        if k == "tensor":
            op = tensor.pop(0)
            if op[0] == "S":
                i = op[1]
                if i not in kv_landed:
                    raise ProtocolError(f"S{i} before its K tile landed")
                if i >= KV and (s_loaded.get(i - KV, set()) != set(range(WARPS)) or (i - KV) not in pv_ran):
                    raise ProtocolError(f"S{i} overwrites buffer {i % KV} too early")
                s_ran.add(i)
            elif op[0] == "PV":
                if p_written.get(op[1], set()) != set(range(WARPS)):
                    raise ProtocolError(f"P{op[1]} V before every warp wrote P")
                pv_ran.add(op[1])
            else:
                op[1].arrive()
        elif k == "tma":
            kind, bar, j = tma.pop(rng.randrange(len(tma)))
            if kind == "kv":
                kv_landed.add(j)
            bar.arrive()
        else:
            try:
                next(actors[k])
            except StopIteration:
                done.add(k)
    raise ProtocolError("no progress: deadlock")


@pytest.mark.parametrize("nkv", list(range(1, 10)))
def test_attention_protocol_holds_under_random_schedules(nkv):
    for seed in range(150):
        run(nkv, seed * 7919 + nkv)


def test_protocol_model_catches_the_unordered_buffer_gate():
    caught = 0
    for nkv in (6, 7, 8, 9):
        for seed in range(300):
            try:
                run(nkv, seed * 7919 + nkv, ordered_confirm=False)
            except ProtocolError:
                caught += 1
    assert caught > 0
