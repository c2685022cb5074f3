"""Recency-window placement of paged KV blocks over the HBM and host tiers, and the plain
execution of a placement plan on the oracle's own copy of the tiers.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link this
module: only the tests, the package smoke check and the benchmark's CPU-baseline leg use
it. It shares no code with the library's block manager or its plan kernel.

Where the policy comes from. The DirectKV summary page ("长上下文 LLM 的零拷贝 KV Cache 卸载
（OSDI 2026）", section 局限与后续工作) names adaptive placement as the next step: hot KV
stays in HBM, cold KV is read directly from CPU memory, and no large staging buffer is
needed. The "KV Offload" wiki page (section CXL 作为 KV Offload 通道, its tier table) calls
the KV being decoded the hot KV of HBM and older, possibly reused KV the warm KV of CPU
DRAM. Neither page defines hotness further, so this module writes out the plainest
reading (every name below is ours):

* A sequence with `len` cached tokens covers nb(len) = len // T + 1 logical blocks (the
  last one holds the slot the next decoded token is written to).
* With n active sequences and an HBM budget of `budget` blocks, every sequence keeps its
  newest W = budget // n logical blocks in HBM (all of them if it has fewer) and the rest
  in the host tier. Decode attention reads every cached block of a sequence once per
  step, so access counts do not distinguish blocks; recency (the block being written is
  the newest) is the only signal, and it is the one the pages name.
* Physical ids are taken smallest-free-first in each tier.
* add(len): the window shrinks to budget // (n + 1). Rows 0..n-1, in order, move their
  oldest HBM blocks to the host tier until each holds at most the new window; then the
  new row n gets blocks j = 0..nb-1, in order, the newest min(W, nb) in HBM.
* remove(r): row r's blocks are freed; the last row, if it is not r, takes row r's place
  (its table row is rewritten, its data does not move); the window grows to
  budget // (n - 1), and rows 0..n-2, in order, bring their newest host blocks into HBM
  until each holds min(W, nb) HBM blocks.
* step(): every row, in order, counts the token the last decode step wrote (len += 1);
  when that opens a new logical block (len % T == 0) the block is allocated in HBM if
  W >= 1, else in the host tier; then the row's oldest HBM blocks move to the host tier
  until it holds at most W.

A plan (what one operation changes) is: the block moves in decision order
(src_tier, src_id, dst_tier, dst_id); the table entries the operation touched, once each
in ascending (row, block) order with their final (tier, id); and the cached-token count
of every active row. Executing a plan copies each moved block (every layer, K and V,
every kv head) and then writes the entries and counts. Within one plan no block is both
the source of a move and the destination of another, so the moves may run in any order.

Pinned by the CPU tests: a hand-worked example, the window invariant and id bookkeeping
after every operation of random runs, conservation of every logical block's contents
through the moves (content tags carried through plan execution), and the degenerate
budgets (everything in HBM; nothing in HBM, so never a move).
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np

HBM, HOST = 0, 1


class CapacityError(RuntimeError):
    pass


class RecencyPlacement:
    def __init__(self, max_rows: int, max_blocks: int, T: int, hbm_ids: int, host_ids: int,
                 budget: int):
        self.max_rows, self.max_blocks, self.T = max_rows, max_blocks, T
        self.budget = budget
        self.free = [set(range(hbm_ids)), set(range(host_ids))]
        self.lens: List[int] = []
        self.blocks: List[List[Tuple[int, int]]] = []   # per row: [(tier, id)] for j < nb
        self._moves: List[Tuple[int, int, int, int]] = []
        self._dirty = set()

    # ---------------------------------------------------------------- helpers
    def n(self) -> int:
        return len(self.lens)

    def window(self) -> int:
        return self.budget // self.n() if self.n() else 0

    def nb(self, length: int) -> int:
        return length // self.T + 1

    def _take(self, tier: int) -> int:
        if not self.free[tier]:
            raise CapacityError("tier %d is full" % tier)
        i = min(self.free[tier])
        self.free[tier].remove(i)
        return i

    def _hbm_count(self, r: int) -> int:
        return sum(1 for t, _ in self.blocks[r] if t == HBM)

    def _demote_oldest(self, r: int) -> None:
        j = next(k for k, (t, _) in enumerate(self.blocks[r]) if t == HBM)
        old = self.blocks[r][j][1]
        new = self._take(HOST)
        self.free[HBM].add(old)
        self.blocks[r][j] = (HOST, new)
        self._moves.append((HBM, old, HOST, new))
        self._dirty.add((r, j))

    def _promote_newest(self, r: int) -> None:
        j = max(k for k, (t, _) in enumerate(self.blocks[r]) if t == HOST)
        old = self.blocks[r][j][1]
        new = self._take(HBM)
        self.free[HOST].add(old)
        self.blocks[r][j] = (HBM, new)
        self._moves.append((HOST, old, HBM, new))
        self._dirty.add((r, j))

    def _begin(self) -> None:
        self._moves, self._dirty = [], set()

    def _plan(self) -> Dict:
        entries = [(r, j, self.blocks[r][j][0], self.blocks[r][j][1])
                   for (r, j) in sorted(self._dirty)]
        return {"moves": list(self._moves), "entries": entries, "seq_lens": list(self.lens)}

    # ------------------------------------------------------------- operations
    def add(self, length: int) -> Dict:
        if self.n() >= self.max_rows or self.nb(length) > self.max_blocks or length < 0:
            raise CapacityError("no room for the sequence")
        self._begin()
        W = self.budget // (self.n() + 1)
        for r in range(self.n()):
            while self._hbm_count(r) > W:
                self._demote_oldest(r)
        nb = self.nb(length)
        hot = min(W, nb)
        row = []
        for j in range(nb):
            row.append((HBM, self._take(HBM)) if j >= nb - hot else (HOST, self._take(HOST)))
        self.lens.append(length)
        self.blocks.append(row)
        r = self.n() - 1
        self._dirty.update((r, j) for j in range(nb))
        return self._plan()

    def remove(self, r: int) -> Dict:
        if not 0 <= r < self.n():
            raise IndexError(r)
        self._begin()
        for t, i in self.blocks[r]:
            self.free[t].add(i)
        last = self.n() - 1
        if r != last:
            self.lens[r], self.blocks[r] = self.lens[last], self.blocks[last]
            self._dirty.update((r, j) for j in range(len(self.blocks[r])))
        self.lens.pop()
        self.blocks.pop()
        W = self.window()
        for s in range(self.n()):
            while self._hbm_count(s) < min(W, len(self.blocks[s])):
                self._promote_newest(s)
        return self._plan()

    def step(self) -> Dict:
        if any(self.nb(L + 1) > self.max_blocks for L in self.lens):
            raise CapacityError("a sequence outgrows its table row")
        self._begin()
        W = self.window()
        for r in range(self.n()):
            self.lens[r] += 1
            if self.lens[r] % self.T == 0:
                tier = HBM if W >= 1 else HOST
                self.blocks[r].append((tier, self._take(tier)))
                self._dirty.add((r, len(self.blocks[r]) - 1))
            while self._hbm_count(r) > W:
                self._demote_oldest(r)
        return self._plan()

    # ---------------------------------------------------------------- tables
    def tables(self):
        """Host snapshot: block_table int32 [max_rows][max_blocks] (-1 unused), tier_map
        uint8 (0 unused), seq_lens int32 [max_rows] (-1 for inactive rows)."""
        bt = np.full((self.max_rows, self.max_blocks), -1, dtype=np.int32)
        tm = np.zeros((self.max_rows, self.max_blocks), dtype=np.uint8)
        sl = np.full((self.max_rows,), -1, dtype=np.int32)
        for r in range(self.n()):
            sl[r] = self.lens[r]
            for j, (t, i) in enumerate(self.blocks[r]):
                bt[r, j], tm[r, j] = i, t
        return bt, tm, sl


def execute_plan(plan: Dict, tiers: Sequence[np.ndarray], layout: int, block_table: np.ndarray,
                 tier_map: np.ndarray, seq_lens: np.ndarray) -> None:
    """Apply a plan in place to the oracle's copy of the pool and of the device tables.

    tiers: [hbm, host] arrays shaped [L][P][2][Hkv][T][D] (layout 0, layer-first) or
    [P][L][2][Hkv][T][D] (layout 1, page-first). A move copies one physical block of every
    layer; the moves are independent, so they are applied one after another.
    """
    for st, si, dt, di in plan["moves"]:
        if layout == 0:
            tiers[dt][:, di] = tiers[st][:, si]
        else:
            tiers[dt][di] = tiers[st][si]
    for r, j, t, i in plan["entries"]:
        block_table[r, j] = i
        tier_map[r, j] = t
    for r, L in enumerate(plan["seq_lens"]):
        seq_lens[r] = L
