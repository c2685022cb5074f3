"""Adaptive placement on the device: the block manager's plans applied by dkv_apply_plan and
by multi-layer decode graphs, against the oracle's own copy of the pool driven by the
placement oracle.

A serving loop of 3 sequences over 2 layers decodes ~40 tokens while the recency window
moves blocks between the tiers (demotions as tails fill, promotions after a sequence
leaves, a late arrival shrinking the window again). Every step's outputs match the fp64
oracle; at the end the device tables equal the oracle's, every prefilled token is
bit-identical wherever its block now lives, and every decoded token is within one bf16 ulp.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as WL

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_offload_b200 as dkv
    import dkv_testlib as TL
    from oracle import dkv_oracle as O
    from oracle.placement import RecencyPlacement, execute_plan
else:
    dkv = TL = O = None


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_offload_b200.build import build
    build()


def _bits(t):
    return WL.bf16_bits(t)


class Loop:
    """Device side (pool, manager, device tables, graphs) and oracle side (tiers, tables,
    placement model) of one serving loop."""

    def __init__(self, layout, D, G, L=2, Hkv=2, T=16, hidden=256, max_rows=4, max_blocks=14,
                 budget=5):
        self.layout, self.D, self.G, self.L, self.Hkv, self.T = layout, D, G, L, Hkv, T
        self.hidden, self.Hq, self.theta = hidden, Hkv * G, 5e5
        self.max_rows, self.max_blocks = max_rows, max_blocks
        self.hbm_ids, self.host_ids = budget + max_rows + 1, max_rows * max_blocks + 8
        shape = lambda P: ((L, P, 2, Hkv, T, D) if layout == 0 else (P, L, 2, Hkv, T, D))
        self.hbm = torch.zeros(int(np.prod(shape(self.hbm_ids))), dtype=torch.bfloat16, device="cuda")
        self.pool = dkv.dkv_pool_create(L, Hkv, D, self.hbm_ids, self.host_ids, block_tokens=T, layout=layout,
                                        hbm_base=self.hbm)
        self.host = dkv.host_tier_tensor(self.pool)
        self.host.zero_()
        self.bm = dkv.BlockManager(max_rows, max_blocks, self.hbm_ids, self.host_ids, budget, block_tokens=T)
        self.ref = RecencyPlacement(max_rows, max_blocks, T, self.hbm_ids, self.host_ids, budget)
        self.bt = torch.zeros((max_rows, max_blocks), dtype=torch.int32, device="cuda")
        self.tm = torch.zeros((max_rows, max_blocks), dtype=torch.uint8, device="cuda")
        self.sl = torch.zeros((max_rows,), dtype=torch.int32, device="cuda")
        self.otiers = [np.zeros(shape(self.hbm_ids), np.uint16), np.zeros(shape(self.host_ids), np.uint16)]
        self.obt = np.zeros((max_rows, max_blocks), np.int32)
        self.otm = np.zeros((max_rows, max_blocks), np.uint8)
        self.osl = np.zeros((max_rows,), np.int32)
        self.W = [WL.randn_bf16(((self.Hq + 2 * Hkv) * D, hidden), seed=11 + l, std=hidden ** -0.5)
                  for l in range(L)]
        self.Wd = [w.cuda() for w in self.W]
        self.prefill = []   # per row: number of prefilled tokens (bit-exact positions)
        self.graphs = []
        self.nstep = 0
        self.moves = 0

    # ------------------------------------------------------------ helpers
    def oview(self, tier, layer, phys):
        t = self.otiers[tier]
        return t[layer, phys] if self.layout == 0 else t[phys, layer]

    def check_plan(self, want):
        got = self.bm.last_plan()
        assert got == {k: [tuple(x) for x in v] if k != "seq_lens" else v for k, v in want.items()}
        self.moves += len(want["moves"])

    def apply_eager(self, want):
        self.check_plan(want)
        dkv.dkv_apply_plan(self.pool, self.bm.plan()[2], self.bt, self.tm, self.sl)
        execute_plan(want, self.otiers, self.layout, self.obt, self.otm, self.osl)

    def close(self):
        self.drop_graphs()
        self.bm.close()
        self.host = None
        dkv.dkv_pool_destroy(self.pool)

    def drop_graphs(self):
        for g in self.graphs:
            dkv.dkv_graph_destroy(g)
        self.graphs = []

    def build_graphs(self):
        self.drop_graphs()
        B = self.ref.n()
        self.x = [torch.empty((B, self.hidden), dtype=torch.bfloat16, device="cuda") for _ in range(self.L)]
        self.out = [torch.empty((B, self.Hq * self.D), dtype=torch.bfloat16, device="cuda") for _ in range(self.L)]
        nws = dkv.dkv_decode_workspace_bytes(self.pool, B, self.max_blocks, self.Hq, self.hidden)
        self.ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        layers = [(l, self.x[l], self.Wd[l], self.out[l]) for l in range(self.L)]
        for slot in (0, 1):
            plan_dev = self.bm.plan(slot)[2]
            self.graphs.append(dkv.dkv_decode_graph_create(self.pool, plan_dev, layers, self.bt, self.sl, self.tm, B,
                                                           self.hidden, self.Hq, self.theta, self.ws))

    # ----------------------------------------------------------- operations
    def add(self, length, seed):
        want = self.ref.add(length)
        row = self.bm.add(length)
        self.apply_eager(want)
        k = WL.randn_bf16((self.L, 1, length, self.Hkv, self.D), seed=seed)
        v = WL.randn_bf16((self.L, 1, length, self.Hkv, self.D), seed=seed + 1)
        zero = torch.zeros((1,), dtype=torch.int32, device="cuda")
        for l in range(self.L):
            dkv.dkv_append_kv(self.pool, l, k[l].cuda(), v[l].cuda(), self.bt[row:row + 1], zero,
                              self.tm[row:row + 1])
        kb, vb = _bits(k), _bits(v)
        for t in range(length):
            j, s = divmod(t, self.T)
            tier, phys = self.ref.blocks[row][j]
            for l in range(self.L):
                blk = self.oview(tier, l, phys)
                blk[0, :, s] = kb[l, 0, t]
                blk[1, :, s] = vb[l, 0, t]
        self.prefill.append(length)

    def remove(self, row):
        want = self.ref.remove(row)
        moved = self.bm.remove(row)
        self.apply_eager(want)
        if moved >= 0:
            self.prefill[row] = self.prefill[moved]
        self.prefill.pop()

    def step_eager(self):
        want = self.ref.step()
        self.bm.step()
        self.apply_eager(want)

    def _oracle_decode(self, xs):
        B = self.ref.n()
        outs = []
        for l in range(self.L):
            res = O.decode_step(_bits(xs[l]), _bits(self.W[l]), self.otiers, self.obt[:B], self.osl[:B],
                                self.otm[:B], self.Hq, self.Hkv, self.D, self.T, self.theta, layer=l,
                                layout=self.layout)
            outs.append(res["out"])
            for b in range(B):
                j, s = divmod(int(self.osl[b]), self.T)
                blk = self.oview(int(self.otm[b, j]), l, int(self.obt[b, j]))
                blk[0, :, s] = res["k_hat"][b]
                blk[1, :, s] = res["v_hat"][b]
        return outs

    def _inputs(self):
        B = self.ref.n()
        xs = [WL.randn_bf16((B, self.hidden), seed=1000 + 10 * self.nstep + l) for l in range(self.L)]
        for l in range(self.L):
            self.x[l].copy_(xs[l])
        self.nstep += 1
        return xs

    def decode_eager(self):
        """A decode step with no placement change (right after add/remove), eager calls."""
        xs = self._inputs()
        for l in range(self.L):
            dkv.dkv_decode_step(self.pool, l, self.x[l], self.Wd[l], self.bt[: self.ref.n()], self.sl,
                                self.tm[: self.ref.n()], self.Hq, self.theta, self.out[l], self.ws)
        self._compare(xs)

    def step_graph(self):
        """step() on the host, then one graph replay: apply the plan, decode every layer."""
        want = self.ref.step()
        self.bm.step()
        self.check_plan(want)
        slot = self.bm.plan()[0]
        xs = self._inputs()
        dkv.dkv_graph_launch(self.graphs[slot])
        execute_plan(want, self.otiers, self.layout, self.obt, self.otm, self.osl)
        self._compare(xs)

    def _compare(self, xs):
        assert dkv.dkv_check(self.pool) == dkv.DKV_OK, dkv.dkv_last_error()
        refs = self._oracle_decode(xs)
        for l in range(self.L):
            TL.assert_out_close(self.out[l], refs[l].reshape(self.ref.n(), -1), "step %d layer %d" % (self.nstep, l))

    # ---------------------------------------------------------------- final
    def check_final(self):
        torch.cuda.synchronize()
        n = self.ref.n()
        rbt, rtm, rsl = self.ref.tables()
        bt, tm, sl = self.bt.cpu().numpy(), self.tm.cpu().numpy(), self.sl.cpu().numpy()
        assert (sl[:n] == rsl[:n]).all()
        for r in range(n):
            nb = int(rsl[r]) // self.T + 1
            assert (bt[r, :nb] == rbt[r, :nb]).all() and (tm[r, :nb] == rtm[r, :nb]).all()
        gt = [self.hbm.cpu().view(torch.int16).numpy().view(np.uint16).reshape(self.otiers[0].shape),
              self.host.numpy().view(np.uint16).reshape(self.otiers[1].shape).copy()]
        for r in range(n):
            for t in range(int(rsl[r])):
                j, s = divmod(t, self.T)
                tier, phys = int(rtm[r, j]), int(rbt[r, j])
                for l in range(self.L):
                    g = (gt[tier][l, phys] if self.layout == 0 else gt[tier][phys, l])[:, :, s]
                    o = self.oview(tier, l, phys)[:, :, s]
                    if t < self.prefill[r]:
                        assert np.array_equal(g, o), (r, t, l)
                    else:
                        gf, of = O.bf16_to_f64(g), O.bf16_to_f64(o)
                        ok = (np.abs(gf - of) <= TL._spacing(of)) | (np.abs(gf - of) <= 2e-5)
                        assert ok.all(), (r, t, l, gf[~ok][:3], of[~ok][:3])


@pytest.mark.parametrize("layout,D,G", [(0, 128, 4), (1, 64, 2)])
def test_adaptive_serving_loop(layout, D, G):
    lp = Loop(layout, D, G)
    try:
        for i, n in enumerate((40, 17, 70)):
            lp.add(n, seed=100 + 10 * i)
        assert lp.bm.window == 1
        lp.build_graphs()
        lp.decode_eager()
        for _ in range(12):
            lp.step_graph()
        lp.remove(1)                      # the window grows 1 -> 2: promotions
        assert lp.bm.window == 2
        lp.build_graphs()
        for _ in range(10):
            lp.step_graph()
        lp.step_eager()                   # count the last tokens, then a late arrival
        lp.add(33, seed=500)              # window shrinks 2 -> 1: demotions
        lp.build_graphs()
        lp.decode_eager()
        for _ in range(14):
            lp.step_graph()
        assert lp.moves >= 6
        lp.check_final()
    finally:
        lp.close()


def test_graph_equals_eager_bit_for_bit():
    lp = Loop(0, 128, 4)
    try:
        lp.add(50, seed=7)
        lp.add(21, seed=9)
        B = lp.ref.n()
        lp.build_graphs()
        xs = lp._inputs()
        for l in range(lp.L):
            dkv.dkv_decode_step(lp.pool, l, lp.x[l], lp.Wd[l], lp.bt[:B], lp.sl, lp.tm[:B], lp.Hq, lp.theta,
                                lp.out[l], lp.ws)
        eager = [o.clone() for o in lp.out]
        torch.cuda.synchronize()
        tiers_eager = (lp.hbm.clone(), lp.host.clone())
        g = dkv.dkv_decode_graph_create(lp.pool, None, [(l, lp.x[l], lp.Wd[l], lp.out[l]) for l in range(lp.L)],
                                        lp.bt, lp.sl, lp.tm, B, lp.hidden, lp.Hq, lp.theta, lp.ws)
        try:
            for o in lp.out:
                o.zero_()
            dkv.dkv_graph_launch(g)
            torch.cuda.synchronize()
        finally:
            dkv.dkv_graph_destroy(g)
        for a, b in zip(eager, lp.out):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert torch.equal(tiers_eager[0].view(torch.int16), lp.hbm.view(torch.int16))
        assert torch.equal(tiers_eager[1], lp.host)
    finally:
        lp.close()


def test_apply_plan_rejects_bad_plans():
    lp = Loop(0, 64, 2, max_rows=2, max_blocks=6, budget=2)
    try:
        lp.add(20, seed=3)
        before = (lp.bt.clone(), lp.tm.clone(), lp.sl.clone())
        lp.bm.step()
        _, host, dev = lp.bm.plan()
        hdr = (ctypes.c_int32 * 8).from_address(host)
        good = hdr[3]
        hdr[3] = good + 1                          # header's max_blocks does not match the tables
        dkv.dkv_apply_plan(lp.pool, dev, lp.bt, lp.tm, lp.sl)
        assert dkv.dkv_check(lp.pool) == dkv.DKV_ERR_BAD_TABLE
        assert "plan-header-mismatch" in dkv.dkv_last_error()
        for a, b in zip(before, (lp.bt, lp.tm, lp.sl)):
            assert torch.equal(a, b)
        hdr[3] = good
        # an entry naming a physical id beyond the tier is skipped and flagged
        lp.bm.step()
        _, host, dev = lp.bm.plan()
        hdr = (ctypes.c_int32 * 8).from_address(host)
        move_cap = hdr[4]
        hdr[1] = 1                                 # one entry
        entry = (ctypes.c_int32 * 4).from_address(host + 32 + 16 * move_cap)
        entry[0], entry[1], entry[2], entry[3] = 0, 0, 0, lp.hbm_ids + 5
        hdr[0] = 0                                 # no moves
        dkv.dkv_apply_plan(lp.pool, dev, lp.bt, lp.tm, lp.sl)
        assert dkv.dkv_check(lp.pool) == dkv.DKV_ERR_BAD_TABLE
        assert int(lp.bt[0, 0]) == int(before[0][0, 0])
    finally:
        lp.close()


def test_manager_waits_for_the_device_to_release_a_plan_buffer():
    """Operation k rewrites plan buffer k mod 2 only after the device applied plan k-2;
    otherwise it times out and changes nothing."""
    lp = Loop(0, 64, 2, max_rows=2, max_blocks=6, budget=2)
    try:
        lp.bm.close()
        lp.bm = dkv.BlockManager(2, 6, lp.hbm_ids, lp.host_ids, 2, wait_ms=200)
        lp.bm.add(20)                                   # plan 0 -> buffer 0
        dkv.dkv_apply_plan(lp.pool, lp.bm.plan()[2], lp.bt, lp.tm, lp.sl)
        lp.bm.step()                                    # plan 1 -> buffer 1, not applied yet
        lp.bm.step()                                    # plan 2 -> buffer 0 (waits for plan 0: applied)
        snap = lp.bm.tables()
        with pytest.raises(dkv.DkvError) as e:
            lp.bm.step()                                # buffer 1 still holds plan 1
        assert e.value.code == dkv.DKV_ERR_TIMEOUT
        for a, b in zip(snap, lp.bm.tables()):
            assert np.array_equal(a, b)
        for slot in (1, 0):                             # apply plans 1 and 2, in order
            dkv.dkv_apply_plan(lp.pool, lp.bm.plan(slot)[2], lp.bt, lp.tm, lp.sl)
        lp.bm.step()                                    # now proceeds
        dkv.dkv_apply_plan(lp.pool, lp.bm.plan()[2], lp.bt, lp.tm, lp.sl)
        assert dkv.dkv_check(lp.pool) == dkv.DKV_OK
        bt, tm, sl = lp.bm.tables()
        assert int(lp.sl[0]) == int(sl[0]) == 23
        assert torch.equal(lp.bt[0, :2].cpu(), torch.from_numpy(bt[0, :2]))
    finally:
        lp.close()
