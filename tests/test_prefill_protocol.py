"""Model check of the tcgen05 head-expanded prefill's mbarrier protocol (prefill_tc.cu), on CPU.

One unit per CTA pair (a head and a tile of 256 queries over n_steps 128-token steps).  Roles: the
K/Q producer (a K ring of NK page slots), the V producer (a ring of NV step slots), the QK^T issuer,
the PV issuer, and the softmax warps of both CTAs (16 arrivals on the counted barriers).  S and P
are double-buffered in tensor memory, so the softmax of step i writes P(i) once PV(i-2) is done,
and waits for PV(i-1) first only when it rescales O.  A rescale is decided per warp (its rows),
the same in the two warps that share a lane quadrant.

Each role is a coroutine yielding its waits with the kernel's slot and parity arithmetic; barriers
follow the hardware's phase rule.  Every slot and buffer carries the step that wrote it, and
consumers assert they read their own step.  Random interleavings must neither deadlock nor alias;
planted mistakes must do one or the other."""
import random

import pytest

NK, NV = 4, 2
SOFTMAX_ARRIVALS = 16      # 8 softmax warps x 2 CTAs


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


def rescales(quad, i, seed):
    """Steps at which the rows of lane quadrant `quad` rescale O (data-driven in the kernel)."""
    return i > 0 and random.Random(seed * 131 + quad * 17 + i).random() < 0.3


def simulate(n_steps, seed, k_parity_flip=False, skip_pfull=False, skip_pv_wait=False, skip_rescale_wait=False):
    rnd = random.Random(seed)
    bars = {}

    def bar(name, count=1):
        return bars.setdefault(name, Bar(count))

    for i in range(NK):
        bar(("KFULL", i)), bar(("KEMPTY", i))
    for i in range(NV):
        bar(("VFULL", i)), bar(("VEMPTY", i))
    bar("QFULL")
    for i in range(2):
        bar(("SFULL", i)), bar(("SFREE", i), SOFTMAX_ARRIVALS), bar(("PVDONE", i))
        bar(("PFULL", i), SOFTMAX_ARRIVALS)
    k_slots, v_slots, s_buf, p_buf = [None] * NK, [None] * NV, [None, None], [None, None]
    state = {"Q": False, "pv_done": -1}

    def k_producer():
        state["Q"] = True
        bar("QFULL").arrive()
        for i in range(n_steps):
            slot = i % NK
            yield ("KEMPTY", slot), ((i // NK) & 1) ^ (0 if k_parity_flip else 1)
            k_slots[slot] = i
            bar(("KFULL", slot)).arrive()

    def v_producer():
        for i in range(n_steps):
            slot = i % NV
            yield ("VEMPTY", slot), ((i // NV) & 1) ^ 1
            v_slots[slot] = i
            bar(("VFULL", slot)).arrive()

    def qk_issuer():
        yield "QFULL", 0
        assert state["Q"]
        for i in range(n_steps):
            sb, slot = i & 1, i % NK
            if i >= 2:
                yield ("SFREE", sb), ((i - 2) >> 1) & 1
            yield ("KFULL", slot), (i // NK) & 1
            assert k_slots[slot] == i, ("K", k_slots[slot], i)
            s_buf[sb] = i
            bar(("KEMPTY", slot)).arrive()
            bar(("SFULL", sb)).arrive()

    def pv_issuer():
        for i in range(n_steps):
            slot = i % NV
            if not skip_pfull:
                yield ("PFULL", i & 1), (i >> 1) & 1
            yield ("VFULL", slot), (i // NV) & 1
            assert v_slots[slot] == i, ("V", v_slots[slot], i)
            assert p_buf[i & 1] == i, ("P", p_buf[i & 1], i)
            state["pv_done"] = i
            bar(("VEMPTY", slot)).arrive()
            bar(("PVDONE", i & 1)).arrive()

    def softmax_warp(quad):
        for i in range(n_steps):
            sb = i & 1
            yield ("SFULL", sb), (i >> 1) & 1
            assert s_buf[sb] == i, ("S", s_buf[sb], i)
            bar(("SFREE", sb)).arrive()
            rescale = rescales(quad, i, seed)
            if rescale and not skip_rescale_wait:
                yield ("PVDONE", (i - 1) & 1), ((i - 1) >> 1) & 1
            elif i >= 2 and not skip_pv_wait:
                yield ("PVDONE", i & 1), ((i - 2) >> 1) & 1
            if rescale:
                assert state["pv_done"] >= i - 1, ("rescale", state["pv_done"], i)
            p_buf[i & 1] = i
            bar(("PFULL", i & 1)).arrive()
        if n_steps:
            yield ("PVDONE", (n_steps - 1) & 1), ((n_steps - 1) >> 1) & 1
            assert state["pv_done"] == n_steps - 1

    roles = [k_producer(), v_producer(), qk_issuer(), pv_issuer()] + \
        [softmax_warp(w % 4) for w in range(SOFTMAX_ARRIVALS)]
    pending = {}
    for r, co in enumerate(roles):
        try:
            pending[r] = next(co)
        except StopIteration:
            pass
    while pending:
        ready = [r for r, (name, parity) in pending.items() if bars[name].passed(parity)]
        if not ready:
            return "deadlock"
        r = rnd.choice(ready)
        try:
            pending[r] = next(roles[r])
        except StopIteration:
            del pending[r]
    return "ok"


def _cases(n, seed0):
    rnd = random.Random(seed0)
    for s in range(n):
        yield rnd.randint(1, 12), seed0 + s


def test_protocol_has_no_deadlock_or_aliasing():
    for n_steps, seed in _cases(300, 5000):
        assert simulate(n_steps, seed) == "ok", (n_steps, seed)


# a wrong producer parity deadlocks; a PV that does not wait for P reads a P the softmax has not
# written; writing P(i) before PV(i-2) is done lets PV(i-2) read P(i); rescaling O before PV(i-1)
# is done races with it
@pytest.mark.parametrize("mistake", [dict(k_parity_flip=True), dict(skip_pfull=True), dict(skip_pv_wait=True),
                                     dict(skip_rescale_wait=True)])
def test_planted_mistakes_are_caught(mistake):
    outcomes = set()
    for n_steps, seed in _cases(60, 6000):
        try:
            outcomes.add(simulate(max(n_steps, 5), seed, **mistake))
        except AssertionError:
            outcomes.add("alias")
    assert outcomes & {"deadlock", "alias"}, outcomes
