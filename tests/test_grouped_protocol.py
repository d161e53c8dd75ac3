"""Model check of the grouped (GQA-path) decode's mbarrier pipeline (decode_grouped.cu), on CPU.

One CTA streams the pages of its chunk through STAGES shared-memory stages.  Thread 0 (which also
belongs to warp 0) issues the tensor copies of a page into stage i % STAGES with completion on the
stage's `full` barrier (one arrival carrying the bytes); each of the four warps waits on `full`,
reads the page, zeroes its own rows past the chunk's end when the page is the ragged last one,
and arrives on the stage's `empty` barrier (four arrivals); thread 0 then waits on `empty` and
issues page i + STAGES into the stage.  The copies land asynchronously, at any later time.

Each role is a coroutine that yields the waits it performs, with the kernel's stage and parity
arithmetic; barriers follow the hardware's phase rule (a wait on parity P returns once the phase of
that parity has completed, so a fresh barrier passes a wait on parity 1).  Every stage carries the
page its last completed copy wrote; a warp asserts it reads the page it expects and that no copy
into the stage is still in flight while it reads.  Random interleavings over random chunk lengths
must neither deadlock nor alias; planted mistakes must do one or the other."""
import random

import pytest

STAGES, WARPS = 2, 4


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


def simulate(n_pages, seed, full_parity_flip=False, skip_empty_wait=False, empty_count=WARPS,
             refill_early=False):
    """Runs the warps and the in-flight copies in a random order; returns "ok", "deadlock", or
    raises AssertionError when a warp reads a stage holding another page or one still being written."""
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(STAGES)]
    empty = [Bar(empty_count) for _ in range(STAGES)]
    stage_page = [None] * STAGES        # page whose copy last landed in the stage
    in_flight = [0] * STAGES            # copies issued into the stage that have not landed
    copies = []                         # pending copy completions: (stage, page)

    def issue(i):
        st = i % STAGES
        in_flight[st] += 1
        copies.append((st, i))

    def copy_engine():
        # lands one pending copy (any of them) each time it is scheduled; idle while none is pending
        while True:
            yield "copies", None
            st, page = copies.pop(rnd.randrange(len(copies)))
            stage_page[st] = page
            in_flight[st] -= 1
            full[st].arrive()

    def warp(w):
        if w == 0:   # thread 0: the prologue issues the first STAGES pages
            for i in range(min(STAGES, n_pages)):
                issue(i)
        for i in range(n_pages):
            st = i % STAGES
            parity = ((i // STAGES) & 1) ^ (1 if full_parity_flip else 0)
            yield ("full", st), parity
            assert stage_page[st] == i, ("stage", st, "holds", stage_page[st], "expected", i)
            assert in_flight[st] == 0, ("stage", st, "is being overwritten while page", i, "is read")
            yield None, None   # the warp computes on the stage (and zeroes its stale rows)
            assert stage_page[st] == i and in_flight[st] == 0, ("stage", st, "changed during page", i)
            empty[st].arrive()
            if w == 0 and i + STAGES < n_pages:
                if refill_early:     # a refill that does not wait for the other warps
                    issue(i + STAGES)
                    continue
                if not skip_empty_wait:
                    yield ("empty", st), (i // STAGES) & 1
                issue(i + STAGES)

    bars = {("full", s): full[s] for s in range(STAGES)}
    bars.update({("empty", s): empty[s] for s in range(STAGES)})
    roles = [warp(w) for w in range(WARPS)] + [copy_engine()]
    pending = {}
    for r, co in enumerate(roles):
        try:
            pending[r] = next(co)
        except StopIteration:
            pass

    def ready(name, parity):
        if name is None:
            return True
        if name == "copies":
            return bool(copies)
        return bars[name].passed(parity)

    engine = len(roles) - 1
    while set(pending) - {engine}:
        runnable = [r for r, (name, parity) in pending.items() if ready(name, parity)]
        if not runnable:
            return "deadlock"
        r = rnd.choice(runnable)
        try:
            pending[r] = next(roles[r])
        except StopIteration:
            del pending[r]
    return "ok"


def _cases(n, seed0):
    rnd = random.Random(seed0)
    for s in range(n):
        yield rnd.randint(1, 9), seed0 + s


def test_pipeline_has_no_deadlock_or_aliasing():
    for n_pages, seed in _cases(400, 3000):
        assert simulate(n_pages, seed) == "ok", (n_pages, seed)


def test_single_page_and_exact_multiples_of_the_stage_count():
    for n_pages in (1, STAGES, 2 * STAGES, 3 * STAGES + 1):
        for seed in range(40):
            assert simulate(n_pages, seed) == "ok", (n_pages, seed)


# a wrong full-barrier parity and an empty barrier that expects more arrivals than warps deadlock;
# refilling a stage without waiting for every warp to release it lets a copy overwrite a page
# that a warp is still reading
@pytest.mark.parametrize("mistake", [dict(full_parity_flip=True), dict(empty_count=WARPS + 1),
                                     dict(skip_empty_wait=True), dict(refill_early=True)])
def test_planted_mistakes_are_caught(mistake):
    outcomes = set()
    for n_pages, seed in _cases(60, 4000):
        try:
            outcomes.add(simulate(max(n_pages, 2 * STAGES + 1), seed, **mistake))
        except AssertionError:
            outcomes.add("alias")
    assert outcomes & {"deadlock", "alias"}, outcomes
