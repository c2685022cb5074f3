"""Model check of the attention kernel's shared-memory stage ring (host logic, no GPU).

Block i of a CTA goes to stage i % NST and is consumed by slot i % SLOTS; the producer
issues loads in order but loads complete in any order; mbarrier parity waits succeed iff
(completed phases) % 2 != parity. The kernel relies on NST being a multiple of SLOTS
(static_assert in the attention kernel): then a consumer can never pass its wait before
its block has landed. A ring of 6 stages for 4 slots breaks this, which this test shows.
"""
import random


def _run(nst, slots, n, seed):
    rnd = random.Random(seed)
    full_done, empty_done = [0] * nst, [0] * nst
    holds = [None] * nst
    issued, loading = 0, []
    nxt = list(range(slots))
    busy = {}
    for _ in range(200000):
        acts = []
        if issued < n:
            st, k = issued % nst, issued // nst
            if k == 0 or empty_done[st] % 2 != ((k - 1) & 1):
                acts.append(("issue", None))
        acts += [("land", b) for b in loading]
        for s in range(slots):
            if s in busy:
                acts.append(("release", s))
            elif nxt[s] < n:
                i = nxt[s]
                if full_done[i % nst] % 2 != ((i // nst) & 1):
                    acts.append(("start", s))
        if not acts:
            return "deadlock" if any(v < n for v in nxt) else None
        kind, arg = rnd.choice(acts)
        if kind == "issue":
            loading.append(issued)
            issued += 1
        elif kind == "land":
            loading.remove(arg)
            holds[arg % nst] = arg
            full_done[arg % nst] += 1
        elif kind == "start":
            i = nxt[arg]
            if holds[i % nst] != i:
                return "slot %d started block %d before it landed" % (arg, i)
            busy[arg] = i
        else:
            i = busy.pop(arg)
            empty_done[i % nst] += 1
            nxt[arg] += slots
    return "no progress"


def test_ring_used_by_the_kernel_is_sound():
    # (stages, slots) of the kernel shapes: four slots with 8 (three CTAs per SM) or 4/12
    # stages (the tensor-core consumer), three slots with 6 stages (four CTAs per SM)
    for nst, slots in ((8, 4), (12, 4), (4, 4), (6, 3)):
        for seed in range(1500):
            assert _run(nst, slots, 48, seed) is None, (nst, slots, seed)


def test_ring_that_is_not_a_multiple_of_the_slots_is_unsound():
    assert any(_run(6, 4, 48, seed) for seed in range(200))
    assert any(_run(8, 3, 48, seed) for seed in range(200))
