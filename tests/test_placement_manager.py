"""The library's block manager (dkv_bm_*, host-side C++) against the placement oracle:
identical plans (moves in order, entries, cached-token counts) and identical table
snapshots after every operation of seeded random runs, integer for integer. Plans live
in ordinary host memory here (DKV_PLAN_HOST), so no device is needed."""
import random

import numpy as np
import pytest

import kv_cache_offload_b200 as dkv
from oracle.placement import CapacityError, RecencyPlacement


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_offload_b200.build import build
    build()


def _mk(max_rows, max_blocks, T, hbm_ids, host_ids, budget):
    bm = dkv.BlockManager(max_rows, max_blocks, hbm_ids, host_ids, budget, block_tokens=T,
                          plan_memory=dkv.DKV_PLAN_HOST)
    ref = RecencyPlacement(max_rows, max_blocks, T, hbm_ids, host_ids, budget)
    return bm, ref


def _same_state(bm, ref):
    bt, tm, sl = bm.tables()
    rbt, rtm, rsl = ref.tables()
    np.testing.assert_array_equal(bt, rbt)
    np.testing.assert_array_equal(tm, rtm)
    np.testing.assert_array_equal(sl, rsl)
    assert bm.rows == ref.n() and bm.window == ref.window()


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("T,budget", [(16, 0), (16, 9), (4, 13), (4, 64), (1, 5)])
def test_manager_equals_oracle(seed, T, budget):
    rng = random.Random(seed * 101 + budget)
    max_rows, max_blocks = 6, 48
    hbm_ids, host_ids = budget + 1 + rng.randrange(0, 4), max_rows * max_blocks
    bm, ref = _mk(max_rows, max_blocks, T, hbm_ids, host_ids, budget)
    try:
        slots = []
        for op in range(250):
            c = rng.random()
            if ref.n() == 0 or (c < 0.12 and ref.n() < max_rows):
                length = rng.randrange(0, T * (max_blocks - 8))
                want = ref.add(length)
                row = bm.add(length)
                assert row == ref.n() - 1
            elif c < 0.2:
                r = rng.randrange(ref.n())
                last = ref.n() - 1
                want = ref.remove(r)
                moved = bm.remove(r)
                assert moved == (last if r != last else -1)
            else:
                if any((L + 1) // T + 1 > max_blocks for L in ref.lens):
                    with pytest.raises(dkv.DkvError) as e:
                        bm.step()
                    assert e.value.code == dkv.DKV_ERR_CAPACITY
                    with pytest.raises(CapacityError):
                        ref.step()
                    r = max(range(ref.n()), key=lambda k: ref.lens[k])
                    want = ref.remove(r)
                    bm.remove(r)
                else:
                    want = ref.step()
                    bm.step()
            slot, _, dev = bm.plan()
            assert dev is None
            slots.append(slot)
            assert bm.last_plan() == {k: [tuple(x) for x in v] if k != "seq_lens" else v
                                      for k, v in want.items()}
            _same_state(bm, ref)
        assert slots[:4] == [0, 1, 0, 1]  # plans alternate between the two buffers
    finally:
        bm.close()


def test_capacity_errors_leave_state_unchanged():
    bm, _ = _mk(3, 8, 16, hbm_ids=3, host_ids=2, budget=2)
    try:
        bm.add(16 * 2)                     # 3 blocks: W = 2 -> 2 HBM + 1 host
        snap, plan0 = bm.tables(), bm.last_plan()
        with pytest.raises(dkv.DkvError) as e:
            bm.add(16 * 2)                 # W = 1: 1 demotion + 2 cold blocks need 3 host ids, 1 free
        assert e.value.code == dkv.DKV_ERR_CAPACITY
        with pytest.raises(dkv.DkvError) as e:
            bm.add(16 * 8)                 # 9 blocks > max_blocks 8
        assert e.value.code == dkv.DKV_ERR_CAPACITY
        for a, b in zip(snap, bm.tables()):
            np.testing.assert_array_equal(a, b)
        assert bm.last_plan() == plan0 and bm.rows == 1 and bm.plan()[0] == 0
        with pytest.raises(dkv.DkvError) as e:
            bm.remove(5)
        assert e.value.code == dkv.DKV_ERR_ARG
        with pytest.raises(dkv.DkvError) as e:
            bm.add(-1)
        assert e.value.code == dkv.DKV_ERR_ARG
    finally:
        bm.close()


def test_bad_configs_rejected():
    for args in [(0, 4, 5, 5, 1), (2, 0, 5, 5, 1), (2, 4, 1, 5, 1), (2, 4, 5, 5, -1)]:
        with pytest.raises(dkv.DkvError) as e:
            dkv.BlockManager(*args, plan_memory=dkv.DKV_PLAN_HOST)
        assert e.value.code == dkv.DKV_ERR_ARG
