"""The DKV_DEBUG build (libdkv_debug.so): the same kernels with a device-side range check on
every block, slot and workspace index they compute. Run in a child process with
DKV_LIBRARY=debug (a process loads one of the two libraries), over decode steps of both
layouts, both tiers, every attention shape and both group sizes, block copies (both
methods), token appends, layout permutation and placement plans: every check must pass
(dkv_check == DKV_OK) and every result must still match the fp64 oracle or be bit-exact."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

pytestmark = pytest.mark.gpu


def test_debug_build_range_checks_pass_on_every_path():
    from kv_cache_offload_b200.build import build
    build()
    env = dict(os.environ, DKV_LIBRARY="debug", PYTHONPATH=os.pathsep.join([ROOT, HERE]))
    r = subprocess.run([sys.executable, os.path.abspath(__file__)], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "debug build: all cases passed" in r.stdout


def _cases():
    import kv_cache_offload_b200 as dkv
    import dkv_testlib as TL
    import workloads as WL
    from oracle import dkv_oracle as O
    assert dkv.binding.LIB_PATH.endswith("libdkv_debug.so")
    torch.cuda.set_device(0)
    n = 0
    # decode: layouts, tiers, shapes, group sizes
    for layout in (0, 1):
        for (Hq, Hkv, D, variants) in ((8, 2, 128, (5, 1, 6)), (16, 2, 128, (5, 1, 6)), (8, 2, 64, (5, 1))):
            cfg = WL.small_config(B=3, Hq=Hq, Hkv=Hkv, D=D, H=256, ctx_range=(1, 400), host_prob=0.5)
            inp = WL.make_decode_inputs(cfg, seed=40 + n, pool_layout=layout)
            ctx = TL.make_pool(inp)
            try:
                ref = TL.oracle_step(inp, layer=1)["out"]
                for v in variants:
                    for splits in (0, 1):
                        dkv.dkv_pool_set_tuning(ctx.pool, attn_splits=splits, attn_variant=v)
                        x, W = inp.x.cuda(), inp.W.cuda()
                        out = torch.empty((cfg.B, cfg.Hq * cfg.D), dtype=torch.bfloat16, device="cuda")
                        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
                        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
                        dkv.dkv_decode_step(ctx.pool, 1, x, W, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.Hq,
                                            cfg.theta, out, ws)
                        rc = dkv.dkv_check(ctx.pool)
                        assert rc == dkv.DKV_OK, (layout, Hq, D, v, splits, rc, dkv.dkv_last_error())
                        TL.assert_out_close(out, ref, "debug build variant %d" % v)
                        n += 1
                TL.check_cache(ctx, TL.oracle_step(inp, layer=1), layer=1, full_compare=True)
            finally:
                ctx.close()
    # block copies, both methods and directions
    cfg = WL.small_config(B=3, layers=2, ctx_range=(40, 200), host_prob=0.5)
    inp = WL.make_decode_inputs(cfg, seed=7)
    ctx = TL.make_pool(inp)
    try:
        k = min(inp.layout.hbm_blocks, inp.layout.host_blocks, 9)
        src = torch.arange(k, dtype=torch.int32)
        dst = torch.arange(k, dtype=torch.int32).flip(0).contiguous()
        for method, dev in ((dkv.DKV_COPY_DMA, lambda t: t), (dkv.DKV_COPY_KERNEL, lambda t: t.cuda())):
            dkv.dkv_copy_blocks(ctx.pool, 1, 0, dev(src), dev(dst), method)
            dkv.dkv_copy_blocks(ctx.pool, 0, 1, dev(dst), dev(src), method)
            assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK, dkv.dkv_last_error()
            n += 1
        hb = WL.bf16_bits(inp.host)
        got = ctx.host.numpy().view(np.uint16).reshape(hb.shape)
        assert np.array_equal(got[:, :k], hb[:, :k])  # host -> HBM -> host round trip
        # token appends into both tiers
        B, nt = cfg.B, 3
        kk = torch.randn((B, nt, cfg.Hkv, cfg.D), device="cuda").to(torch.bfloat16)
        vv = torch.randn((B, nt, cfg.Hkv, cfg.D), device="cuda").to(torch.bfloat16)
        lens = torch.clamp(ctx.seq_lens - nt, min=0).to(torch.int32)
        dkv.dkv_append_kv(ctx.pool, 0, kk, vv, ctx.table, lens, ctx.tier_map)
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK, dkv.dkv_last_error()
        n += 1
        # layout permutation of either tier
        for tier in (0, 1):
            _, _, nbytes = dkv.dkv_pool_tier_ptr(ctx.pool, tier)
            out = torch.empty(nbytes // 2, dtype=torch.int16, device="cuda")
            dkv.dkv_convert_layout(ctx.pool, tier, out)
            assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK, dkv.dkv_last_error()
            n += 1
    finally:
        ctx.close()
    # placement plans applied on the device
    L, Bm, T = 2, 4, 16
    pool = dkv.dkv_pool_create(L, 2, 64, 64, 64)
    try:
        bm = dkv.BlockManager(Bm, 20, 64, 64, 24)
        bt = torch.zeros((Bm, 20), dtype=torch.int32, device="cuda")
        tm = torch.zeros((Bm, 20), dtype=torch.uint8, device="cuda")
        sl = torch.zeros((Bm,), dtype=torch.int32, device="cuda")
        for c in (100, 60, 150):
            bm.add(c)
            dkv.dkv_apply_plan(pool, bm.plan()[2], bt, tm, sl)
        for _ in range(20):
            bm.step()
            dkv.dkv_apply_plan(pool, bm.plan()[2], bt, tm, sl)
        assert dkv.dkv_check(pool) == dkv.DKV_OK, dkv.dkv_last_error()
        n += 1
        bm.close()
    finally:
        dkv.dkv_pool_destroy(pool)
    print("debug build: all cases passed (%d)" % n)


if __name__ == "__main__":
    _cases()
