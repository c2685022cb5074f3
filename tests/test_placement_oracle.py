"""Pins for the placement oracle (oracle/placement.py): a hand-worked example, the
window invariant and id bookkeeping after every operation, conservation of every logical
block's contents through plan execution, the independence of a plan's moves, and the
degenerate budgets."""
import random

import numpy as np
import pytest

from oracle.placement import HBM, HOST, RecencyPlacement, execute_plan


def test_hand_worked_example():
    # T=16, budget 4 blocks, 5 HBM ids, 16 host ids; derived by hand from the policy.
    P = RecencyPlacement(max_rows=4, max_blocks=8, T=16, hbm_ids=5, host_ids=16, budget=4)
    p = P.add(40)  # W = 4; nb = 3 -> all HBM, ids 0, 1, 2
    assert p == {"moves": [], "entries": [(0, 0, HBM, 0), (0, 1, HBM, 1), (0, 2, HBM, 2)],
                 "seq_lens": [40]}
    p = P.add(17)  # W = 2; row 0 demotes block 0 (HBM 0 -> host 0); row 1 gets HBM 0, 3
    assert p == {"moves": [(HBM, 0, HOST, 0)],
                 "entries": [(0, 0, HOST, 0), (1, 0, HBM, 0), (1, 1, HBM, 3)],
                 "seq_lens": [40, 17]}
    plans = [P.step() for _ in range(15)]
    for k, p in enumerate(plans, start=1):
        assert p["seq_lens"] == [40 + k, 17 + k]
        if k not in (8, 15):
            assert p["moves"] == [] and p["entries"] == []
    # step 8: row 0 reaches 48 tokens -> block 3 in HBM 4, block 1 (HBM 1) -> host 1
    assert plans[7]["moves"] == [(HBM, 1, HOST, 1)]
    assert plans[7]["entries"] == [(0, 1, HOST, 1), (0, 3, HBM, 4)]
    # step 15: row 1 reaches 32 tokens -> block 2 in HBM 1, block 0 (HBM 0) -> host 2
    assert plans[14]["moves"] == [(HBM, 0, HOST, 2)]
    assert plans[14]["entries"] == [(1, 0, HOST, 2), (1, 2, HBM, 1)]
    # remove row 0: row 1 takes its place; W = 4 -> promote block 0 (host 2 -> HBM 0)
    p = P.remove(0)
    assert p == {"moves": [(HOST, 2, HBM, 0)],
                 "entries": [(0, 0, HBM, 0), (0, 1, HBM, 3), (0, 2, HBM, 1)],
                 "seq_lens": [32]}
    bt, tm, sl = P.tables()
    assert sl.tolist() == [32, -1, -1, -1]
    assert bt[0, :3].tolist() == [0, 3, 1] and tm[0, :3].tolist() == [HBM] * 3


def check_invariants(P: RecencyPlacement, hbm_ids: int, host_ids: int):
    W = P.window()
    used = [set(), set()]
    hbm_total = 0
    for L, row in zip(P.lens, P.blocks):
        nb = L // P.T + 1
        assert len(row) == nb
        hot = min(W, nb)
        assert [t for t, _ in row] == [HOST] * (nb - hot) + [HBM] * hot
        for t, i in row:
            assert i not in used[t]
            used[t].add(i)
        hbm_total += hot
    assert hbm_total <= P.budget
    assert used[HBM] | P.free[HBM] == set(range(hbm_ids)) and not (used[HBM] & P.free[HBM])
    assert used[HOST] | P.free[HOST] == set(range(host_ids)) and not (used[HOST] & P.free[HOST])


def check_plan_independent(plan):
    src = [(st, si) for st, si, _, _ in plan["moves"]]
    dst = [(dt, di) for _, _, dt, di in plan["moves"]]
    assert len(set(src)) == len(src) and len(set(dst)) == len(dst)
    assert not (set(src) & set(dst))
    assert all(st != dt for st, _, dt, _ in plan["moves"])
    keys = [(r, j) for r, j, _, _ in plan["entries"]]
    assert keys == sorted(set(keys))


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("budget", [0, 3, 7, 20, 400])
def test_random_runs_conserve_contents(layout, budget):
    """Every logical block keeps its contents through every plan; tags stand for data."""
    T, L, max_rows, max_blocks = 4, 2, 5, 40
    hbm_ids, host_ids = budget + max_rows + 1, 5 * 40
    rng = random.Random(budget * 7 + layout)
    P = RecencyPlacement(max_rows, max_blocks, T, hbm_ids, host_ids, budget)
    shape = lambda n: (L, n, 1) if layout == 0 else (n, L, 1)
    tiers = [np.full(shape(hbm_ids), -1, np.int64), np.full(shape(host_ids), -1, np.int64)]
    bt = np.full((max_rows, max_blocks), -1, np.int32)
    tm = np.zeros((max_rows, max_blocks), np.uint8)
    sl = np.full((max_rows,), -1, np.int32)
    seq_ids = []          # row -> sequence identity
    next_seq = [0]

    def tag(seq, j, layer):
        return (seq * 1000 + j) * 10 + layer

    def write_block(r, j):
        t, i = int(tm[r, j]), int(bt[r, j])
        for layer in range(L):
            if layout == 0:
                tiers[t][layer, i, 0] = tag(seq_ids[r], j, layer)
            else:
                tiers[t][i, layer, 0] = tag(seq_ids[r], j, layer)

    def read_block(r, j, layer):
        t, i = int(tm[r, j]), int(bt[r, j])
        return tiers[t][layer, i, 0] if layout == 0 else tiers[t][i, layer, 0]

    moved_any = False
    for op in range(300):
        choice = rng.random()
        if P.n() == 0 or (choice < 0.15 and P.n() < max_rows):
            length = rng.randrange(0, 60)
            plan = P.add(length)
            execute_plan(plan, tiers, layout, bt, tm, sl)
            seq_ids.append(next_seq[0]); next_seq[0] += 1
            for j in range(length // T + 1):  # the caller fills the new sequence (prefill)
                write_block(P.n() - 1, j)
        elif choice < 0.25:
            r = rng.randrange(P.n())
            plan = P.remove(r)
            execute_plan(plan, tiers, layout, bt, tm, sl)
            last = len(seq_ids) - 1
            seq_ids[r] = seq_ids[last]
            seq_ids.pop()
        else:
            if any((Lr + 1) // T + 1 > max_blocks for Lr in P.lens):
                r = max(range(P.n()), key=lambda k: P.lens[k])
                plan = P.remove(r)
                execute_plan(plan, tiers, layout, bt, tm, sl)
                seq_ids[r] = seq_ids[-1]
                seq_ids.pop()
            else:
                old_nb = [Lr // T + 1 for Lr in P.lens]
                plan = P.step()
                execute_plan(plan, tiers, layout, bt, tm, sl)
                for r, Lr in enumerate(P.lens):  # the decode step writes the new tail block
                    if Lr // T + 1 > old_nb[r]:
                        write_block(r, Lr // T)
        moved_any |= bool(plan["moves"])
        check_plan_independent(plan)
        check_invariants(P, hbm_ids, host_ids)
        # the executed device tables equal the manager's snapshot on every active row
        sbt, stm, ssl = P.tables()
        for r in range(P.n()):
            nb = P.lens[r] // T + 1
            assert (bt[r, :nb] == sbt[r, :nb]).all() and (tm[r, :nb] == stm[r, :nb]).all()
            assert sl[r] == ssl[r]
            for j in range(nb):
                for layer in range(L):
                    assert read_block(r, j, layer) == tag(seq_ids[r], j, layer)
    if budget in (0, 400):
        assert not moved_any  # nothing ever in HBM / everything fits: no block ever moves
    else:
        assert moved_any


def test_budget_zero_is_all_host_and_large_budget_all_hbm():
    P = RecencyPlacement(3, 20, 16, hbm_ids=1, host_ids=100, budget=0)
    P.add(100); P.add(5)
    assert all(t == HOST for row in P.blocks for t, _ in row)
    P2 = RecencyPlacement(3, 20, 16, hbm_ids=100, host_ids=1, budget=99)
    P2.add(100); P2.add(5)
    assert all(t == HBM for row in P2.blocks for t, _ in row)
    for _ in range(40):
        assert P2.step()["moves"] == []


def test_window_is_budget_over_rows():
    P = RecencyPlacement(8, 64, 16, hbm_ids=40, host_ids=400, budget=30)
    for k in range(1, 7):
        P.add(16 * 20)
        assert P.window() == 30 // k
        assert all(sum(t == HBM for t, _ in row) == min(30 // k, len(row)) for row in P.blocks)
