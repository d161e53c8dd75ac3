"""Model check of the tcgen05 absorbed decode's mbarrier protocol (decode_tc.cu), on CPU.

Each role of the kernel (the two K producers, the second of which also loads Q, the V producer, the QK^T and PV issuers and the 16
softmax warps of a CTA pair) is a coroutine that yields the barrier waits it performs, in the
kernel's order, with the kernel's slot and parity arithmetic.  mbarriers follow the hardware's
phase rule: a wait on parity P returns once the phase of that parity has completed, so a fresh
barrier passes a wait on parity 1.  Every ring slot and buffer carries the generation its producer
wrote, and every consumer asserts it reads the one it expects.  Random interleavings of the roles
over random work-item lists must neither deadlock nor alias; planted mistakes must do one or the
other, which shows the model can fail."""
import random

import pytest

NK, NV = 3, 2              # K ring: three slots (one step); V ring: one slot per page of a step
K_SPLIT = 2                # K slots [0, K_SPLIT) come from the first producer, the rest from the second
SOFTMAX_ARRIVALS = 16      # 8 softmax warps x 2 CTAs arrive on the counted barriers


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


def rescales(g):
    """Steps whose softmax rescales O (a CTA-uniform decision in the kernel; here a fixed pattern)."""
    return g % 5 == 3


def ragged(n, steps, pg):
    """Whether page pg of the last step of item n is a request's ragged last page (a fixed pattern;
    the kernel decides it from the item's end)."""
    return (n % 3 == 1 and pg == 1) or (n % 3 == 2 and pg == 0 and steps % 2 == 0)


def simulate(items, seed, k_parity_flip=False, skip_qempty=False, skip_pv_wait=False, skip_rescale_wait=False,
             skip_tail_wait=False):
    """Runs the roles over work items (token steps per item) in a random order; returns "ok",
    "deadlock", or raises AssertionError on a generation mismatch."""
    rnd = random.Random(seed)
    bars = {}

    def bar(name, count=1):
        return bars.setdefault(name, Bar(count))

    for i in range(NK):
        bar(("KFULL", i)), bar(("KEMPTY", i))
    for i in range(NV):
        bar(("VFULL", i)), bar(("VEMPTY", i))
    bar("QFULL"), bar("QEMPTY")
    for i in range(2):
        bar(("SFULL", i)), bar(("SFREE", i), SOFTMAX_ARRIVALS), bar(("PVDONE", i))
    bar(("PFULL", 0), SOFTMAX_ARRIVALS), bar(("PFULL", 1), SOFTMAX_ARRIVALS), bar("OFREE", SOFTMAX_ARRIVALS)
    bar("VTAIL")
    k_slots, v_slots, s_buf, p_buf = [None] * NK, [None] * NV, [None, None], [None, None]
    state = {"Q": None, "O": None, "pv_done": -1}

    def k_producer(j0, j1):
        g = 0
        for n, steps in enumerate(items):
            if j1 == NK:
                if n > 0:
                    yield "QEMPTY", (n - 1) & 1
                state["Q"] = n
                bar("QFULL").arrive()
            for _ in range(steps):
                for j in range(j0, j1):
                    parity = (g & 1) ^ (0 if k_parity_flip else 1)
                    yield ("KEMPTY", j), parity
                    k_slots[j] = (g, j)
                    bar(("KFULL", j)).arrive()
                g += 1

    def v_producer():
        g = 0
        for n, steps in enumerate(items):
            for i in range(steps):
                for pg in range(NV):
                    yield ("VEMPTY", pg), (g & 1) ^ 1
                    if i == steps - 1 and ragged(n, steps, pg):
                        # the copy lands on the CTA's own barrier; VFULL's phase carries no bytes, and
                        # the tile is complete (stale rows zeroed) only at the tail barrier
                        v_slots[pg] = "partial"
                        bar(("VFULL", pg)).arrive()
                        yield None, None                 # the copy and the zeroing take a while
                        v_slots[pg] = (g, pg)
                        bar("VTAIL").arrive()
                    else:
                        v_slots[pg] = (g, pg)
                        bar(("VFULL", pg)).arrive()
                g += 1

    def qk_issuer():
        g = 0
        for n, steps in enumerate(items):
            yield "QFULL", n & 1
            for i in range(steps):
                sb = g & 1
                if g >= 2:
                    yield ("SFREE", sb), ((g - 2) >> 1) & 1
                for j in range(NK):
                    yield ("KFULL", j), g & 1
                    assert k_slots[j] == (g, j), ("K", k_slots[j], (g, j))
                    assert state["Q"] == n, ("Q", state["Q"], n)
                    bar(("KEMPTY", j)).arrive()
                if i == steps - 1 and not skip_qempty:
                    bar("QEMPTY").arrive()
                s_buf[sb] = g
                bar(("SFULL", sb)).arrive()
                g += 1

    def pv_issuer():
        g = 0
        nt = 0
        for n, steps in enumerate(items):
            for i in range(steps):
                yield ("PFULL", g & 1), (g >> 1) & 1
                if i == 0 and n > 0:
                    yield "OFREE", (n - 1) & 1
                assert p_buf[g & 1] == g, ("P", p_buf[g & 1], g)
                for pg in range(NV):
                    yield ("VFULL", pg), g & 1
                    if i == steps - 1 and ragged(n, steps, pg):
                        if not skip_tail_wait:
                            yield "VTAIL", nt & 1
                        nt += 1
                    assert v_slots[pg] == (g, pg), ("V", v_slots[pg], (g, pg))
                    bar(("VEMPTY", pg)).arrive()
                state["O"] = n
                state["pv_done"] = g
                bar(("PVDONE", g & 1)).arrive()
                g += 1

    def softmax_warp():
        g = 0
        for n, steps in enumerate(items):
            for i in range(steps):
                sb = g & 1
                yield ("SFULL", sb), (g >> 1) & 1
                assert s_buf[sb] == g, ("S", s_buf[sb], g)
                bar(("SFREE", sb)).arrive()
                # P is double-buffered: P(g) needs PV(g-2) done; a rescale of O needs PV(g-1) done
                rescale = i > 0 and rescales(g)
                if rescale and not skip_rescale_wait:
                    yield ("PVDONE", (g - 1) & 1), ((g - 1) >> 1) & 1
                elif g >= 2 and not skip_pv_wait:
                    yield ("PVDONE", g & 1), ((g - 2) >> 1) & 1
                if rescale:
                    assert state["pv_done"] >= g - 1, ("rescale", state["pv_done"], g)
                p_buf[g & 1] = g
                bar(("PFULL", g & 1)).arrive()
                g += 1
            yield ("PVDONE", (g - 1) & 1), ((g - 1) >> 1) & 1
            assert state["O"] == n, ("O", state["O"], n)
            bar("OFREE").arrive()

    roles = [k_producer(0, K_SPLIT), k_producer(K_SPLIT, NK), v_producer(), qk_issuer(), pv_issuer()] + \
        [softmax_warp() for _ in range(SOFTMAX_ARRIVALS)]
    pending = {}
    for r, co in enumerate(roles):
        try:
            pending[r] = next(co)
        except StopIteration:
            pass
    while pending:
        ready = [r for r, (name, parity) in pending.items() if name is None or bars[name].passed(parity)]
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
        yield [rnd.randint(1, 6) for _ in range(rnd.randint(1, 4))], seed0 + s


def test_protocol_has_no_deadlock_or_aliasing():
    for items, seed in _cases(300, 1000):
        assert simulate(items, seed) == "ok", (items, seed)


def test_single_step_items_back_to_back():
    # items of one step exercise the Q and O hand-over on every step
    for seed in range(50):
        assert simulate([1] * 6, seed) == "ok"


# a wrong producer parity and a missing QEMPTY commit deadlock; writing P(g) before PV(g-2) is done
# lets PV(g-2) read P(g); rescaling O before PV(g-1) is done races with it; reading a ragged V tile
# before its tail barrier sees its stale rows
@pytest.mark.parametrize("mistake", [dict(k_parity_flip=True), dict(skip_qempty=True), dict(skip_pv_wait=True),
                                     dict(skip_rescale_wait=True), dict(skip_tail_wait=True)])
def test_planted_mistakes_are_caught(mistake):
    outcomes = set()
    for items, seed in _cases(50, 2000):
        try:
            outcomes.add(simulate(items, seed, **mistake))
        except AssertionError:
            outcomes.add("alias")
    assert outcomes & {"deadlock", "alias"}, outcomes
