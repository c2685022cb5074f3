"""Test-side plumbing: place seeded workloads into a libdkv pool, run the CUDA path through
the C ABI, run the fp64 oracle on the same bytes, and compare.

Tolerances (fixed by the attention output bar and derived for the cache write):
  * attention output: max |gpu - ref| <= 3e-2 and mean |gpu - ref| <= 3e-3, plus an
    internal relative-rms bar ||gpu - ref|| / ||ref|| <= 1e-2 (outputs shrink like
    1/sqrt(context), so the absolute bars alone say little at long contexts);
  * new cache contents: the GPU's bf16 value is RNE(ref) or one of its two bf16 neighbours
    (|gpu - RNE(ref)| <= one bf16 spacing at RNE(ref)). Near zero the bf16 spacing falls
    below the fp32 error of the H-term dot product itself (bf16 x bf16 products are exact
    in fp32; each of the H - 1 additions errs by <= 2^-24 |partial sum|, and with partial
    sums growing like a random walk of steps of rms size p_rms the accumulated error is
    about 2^-24 p_rms H / sqrt(2)). There |gpu - ref| <= spacing(ref)/2 + tau is accepted,
    tau = 8 * 2^-24 * p_rms * H / sqrt(2) per row (doubled for a RoPE-rotated pair);
  * everything else in both tiers: bit-exact (unchanged).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

import kv_cache_offload_b200 as dkv
import workloads as WL
from oracle import dkv_oracle as O


@dataclasses.dataclass
class PoolCtx:
    pool: int
    hbm: torch.Tensor = dataclasses.field(repr=False)    # device tier (pool's hbm_base)
    host: torch.Tensor = dataclasses.field(repr=False)   # CPU alias of the pinned host tier
    table: torch.Tensor = dataclasses.field(repr=False)
    tier_map: torch.Tensor = dataclasses.field(repr=False)
    seq_lens: torch.Tensor = dataclasses.field(repr=False)
    inp: WL.DecodeInputs = dataclasses.field(repr=False)

    def close(self):
        self.host = None  # the alias must not outlive the pinned memory
        if self.pool:
            dkv.dkv_pool_destroy(self.pool)
            self.pool = 0


def make_pool(inp: WL.DecodeInputs, host_flags: int = 0) -> PoolCtx:
    cfg, lay = inp.cfg, inp.layout
    hbm = inp.hbm.cuda() if inp.hbm.numel() else torch.empty(0, dtype=torch.bfloat16, device="cuda")
    pool = dkv.dkv_pool_create(cfg.layers, cfg.Hkv, cfg.D, lay.hbm_blocks, lay.host_blocks,
                               block_tokens=cfg.T, layout=inp.pool_layout, host_flags=host_flags,
                               hbm_base=hbm if hbm.numel() else None)
    host = dkv.host_tier_tensor(pool)
    if inp.host.numel():
        host.copy_(inp.host.reshape(-1).view(torch.int16))
    return PoolCtx(pool, hbm, host, lay.block_table.cuda(), lay.tier_map.cuda(),
                   torch.tensor(lay.seq_lens, dtype=torch.int32, device="cuda"), inp)


def run_step(ctx: PoolCtx, layer: int = 0, attn_splits: int = 0, proj_splits: int = 0):
    cfg = ctx.inp.cfg
    dkv.dkv_pool_set_tuning(ctx.pool, attn_splits=attn_splits, proj_splits=proj_splits)
    x, W = ctx.inp.x.cuda(), ctx.inp.W.cuda()
    out = torch.empty((cfg.B, cfg.Hq * cfg.D), dtype=torch.bfloat16, device="cuda")
    nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    dkv.dkv_decode_step(ctx.pool, layer, x, W, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.Hq,
                        cfg.theta, out, ws)
    rc = dkv.dkv_check(ctx.pool)
    assert rc == dkv.DKV_OK, dkv.dkv_last_error()
    return out


def oracle_step(inp: WL.DecodeInputs, layer: int = 0, batch=None, heads=None):
    cfg, lay = inp.cfg, inp.layout
    return O.decode_step(WL.bf16_bits(inp.x), WL.bf16_bits(inp.W),
                         [WL.bf16_bits(inp.hbm), WL.bf16_bits(inp.host)],
                         lay.block_table.numpy(), lay.seq_lens, lay.tier_map.numpy(), cfg.Hq,
                         cfg.Hkv, cfg.D, cfg.T, cfg.theta, layer=layer, layout=inp.pool_layout,
                         batch=batch, heads=heads)


def out_errors(out_gpu: torch.Tensor, ref: np.ndarray):
    cfg_shape = ref.shape
    got = out_gpu.float().cpu().double().numpy().reshape(cfg_shape)
    mask = ~np.isnan(ref)
    d = np.abs(got[mask] - ref[mask])
    rel = float(np.linalg.norm(got[mask] - ref[mask]) / max(np.linalg.norm(ref[mask]), 1e-300))
    return float(d.max()), float(d.mean()), rel


def assert_out_close(out_gpu, ref, what=""):
    mx, mean, rel = out_errors(out_gpu, ref)
    assert mx <= 3e-2 and mean <= 3e-3 and rel <= 1e-2, \
        "%s: max %.3g mean %.3g rel-rms %.3g" % (what, mx, mean, rel)
    return mx, mean, rel


def _slot_index(inp: WL.DecodeInputs, layer: int, b: int, kv: int, g: int):
    """(tier, index tuple into the tier tensor) of the new token's D-row for (b, kv, g)."""
    lay, T = inp.layout, inp.cfg.T
    pos = lay.seq_lens[b]
    j, slot = divmod(pos, T)
    tier = int(lay.tier_map[b, j])
    phys = int(lay.block_table[b, j])
    if inp.pool_layout == 0:
        return tier, (layer, phys, kv, g, slot)
    return tier, (phys, layer, kv, g, slot)


def _spacing(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 2.0 ** -133)))
    return np.exp2(np.maximum(e - 7, -133))


def bf16_within_one_ulp(gpu_bits: np.ndarray, ref: np.ndarray, tau=0.0) -> np.ndarray:
    g = O.bf16_to_f64(gpu_bits)
    r = O.bf16_to_f64(O.f64_to_bf16_rne(ref))
    ok = np.abs(g - r) <= _spacing(r)
    ok |= np.abs(g - ref) <= 0.5 * _spacing(ref) + tau
    return ok


def accumulation_tau(W_rows: np.ndarray, xb: np.ndarray) -> np.ndarray:
    """Per-row fp32 accumulation allowance 8 * 2^-24 * p_rms * H / sqrt(2)."""
    H = xb.shape[0]
    p_rms = np.sqrt(np.mean((W_rows * xb[None, :]) ** 2, axis=1))
    return 8.0 * 2.0 ** -24 * p_rms * H / np.sqrt(2.0)


def check_cache(ctx: PoolCtx, ores, layer: int = 0, full_compare: bool = True):
    """New K/V rows within one bf16 ulp of the oracle; every other element unchanged."""
    inp, cfg = ctx.inp, ctx.inp.cfg
    torch.cuda.synchronize()
    tiers_after = [ctx.hbm.cpu().view(torch.int16).numpy().view(np.uint16).reshape(inp.hbm.shape),
                   ctx.host.numpy().view(np.uint16).reshape(inp.host.shape).copy()]
    tiers_before = [WL.bf16_bits(inp.hbm), WL.bf16_bits(inp.host)]
    # exact k_rot / v in fp64 for the 1-ulp check (only the key/value rows of W)
    D = cfg.D
    Wkv = O.bf16_to_f64(WL.bf16_bits(inp.W)[cfg.Hq * D:])
    half = D // 2
    for b in range(cfg.B):
        xb = O.bf16_to_f64(WL.bf16_bits(inp.x)[b])
        kv_rows = Wkv @ xb
        k = kv_rows[: cfg.Hkv * D].reshape(cfg.Hkv, D)
        v = kv_rows[cfg.Hkv * D:].reshape(cfg.Hkv, D)
        tau = accumulation_tau(Wkv, xb)
        tk = tau[: cfg.Hkv * D].reshape(cfg.Hkv, D)
        tk = 2.0 * np.maximum(tk, np.concatenate([tk[:, half:], tk[:, :half]], axis=1))
        tv = tau[cfg.Hkv * D:].reshape(cfg.Hkv, D)
        k_rot = O.rope_rotate_half(k, inp.layout.seq_lens[b], cfg.theta)
        for g in range(cfg.Hkv):
            for kv, ref, tt in ((0, k_rot[g], tk[g]), (1, v[g], tv[g])):
                tier, idx = _slot_index(inp, layer, b, kv, g)
                got = tiers_after[tier][idx]
                ok = bf16_within_one_ulp(got, ref, tt)
                assert ok.all(), "cache b=%d g=%d kv=%d: %d bad (e.g. got %r want %r)" % (
                    b, g, kv, int((~ok).sum()), O.bf16_to_f64(got[~ok][:3]), ref[~ok][:3])
                # restore so the remaining comparison is whole-array
                tiers_after[tier][idx] = tiers_before[tier][idx]
    if full_compare:
        for t in (0, 1):
            assert np.array_equal(tiers_after[t], tiers_before[t]), "tier %d changed outside the new slots" % t
