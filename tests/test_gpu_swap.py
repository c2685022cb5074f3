"""Block copies between tiers (swap-in / swap-out) and the staged-swap decode baseline:
copying the host-tier blocks into HBM first and attending over HBM must give exactly the
zero-copy result (same arithmetic, different load path)."""
import numpy as np
import pytest
import torch

import workloads as WL
from oracle import dkv_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_offload_b200 as dkv
    import dkv_testlib as TL
else:
    dkv = TL = None


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_offload_b200.build import build
    build()


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("method", ["DMA", "KERNEL"])
def test_copy_blocks_both_directions_bit_exact(layout, method):
    cfg = WL.small_config(B=4, layers=3, ctx_range=(40, 300), host_prob=0.5)
    inp = WL.make_decode_inputs(cfg, seed=9, pool_layout=layout)
    ctx = TL.make_pool(inp)
    try:
        m = getattr(dkv, "DKV_COPY_" + method)
        n = min(inp.layout.hbm_blocks, inp.layout.host_blocks, 37)
        g = torch.Generator().manual_seed(1)
        src = torch.randperm(inp.layout.host_blocks, generator=g)[:n].to(torch.int32)
        dst = torch.randperm(inp.layout.hbm_blocks, generator=g)[:n].to(torch.int32)
        dev = (lambda t: t.cuda()) if method == "KERNEL" else (lambda t: t)
        dkv.dkv_copy_blocks(ctx.pool, 1, 0, dev(src), dev(dst), m)   # host -> HBM
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
        hbm = WL.bf16_bits(inp.hbm).copy()
        host = WL.bf16_bits(inp.host)
        for s, d in zip(src.tolist(), dst.tolist()):
            if layout == 0:
                hbm[:, d] = host[:, s]
            else:
                hbm[d] = host[s]
        got = ctx.hbm.cpu().view(torch.int16).numpy().view(np.uint16).reshape(hbm.shape)
        assert np.array_equal(got, hbm)
        # and back: HBM -> host into other slots
        src2 = dst[:5].clone()
        dst2 = torch.arange(5, dtype=torch.int32)
        dkv.dkv_copy_blocks(ctx.pool, 0, 1, dev(src2), dev(dst2), m)
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
        hostx = host.copy()
        for s, d in zip(src2.tolist(), dst2.tolist()):
            if layout == 0:
                hostx[:, d] = hbm[:, s]
            else:
                hostx[d] = hbm[s]
        assert np.array_equal(ctx.host.numpy().view(np.uint16).reshape(hostx.shape), hostx)
    finally:
        ctx.close()


@pytest.mark.parametrize("method", ["DMA", "KERNEL"])
def test_staged_swap_decode_equals_zero_copy(method):
    cfg = WL.small_config(B=3, ctx_range=(100, 600), host_prob=0.7, layers=1)
    inp = WL.make_decode_inputs(cfg, seed=4)
    lay = inp.layout
    # zero-copy reference
    ctx = TL.make_pool(inp)
    try:
        zc = TL.run_step(ctx, layer=0)
    finally:
        ctx.close()
    # staged: an HBM tier with room for every host block, host blocks swapped in first
    nh, ns = lay.hbm_blocks, lay.host_blocks
    hbm = torch.empty((cfg.layers, nh + ns) + tuple(inp.hbm.shape[2:]), dtype=torch.bfloat16)
    hbm[:, :nh] = inp.hbm
    hbm_d = hbm.cuda()
    pool = dkv.dkv_pool_create(cfg.layers, cfg.Hkv, cfg.D, nh + ns, ns, hbm_base=hbm_d)
    try:
        dkv.host_tier_tensor(pool).copy_(inp.host.reshape(-1).view(torch.int16))
        src = torch.arange(ns, dtype=torch.int32)
        dst = torch.arange(nh, nh + ns, dtype=torch.int32)
        dev = (lambda t: t.cuda()) if method == "KERNEL" else (lambda t: t)
        dkv.dkv_copy_blocks(pool, 1, 0, dev(src), dev(dst), getattr(dkv, "DKV_COPY_" + method))
        table = lay.block_table.clone()
        table[lay.tier_map == 1] += nh
        table[lay.block_table < 0] = -1
        tmap = torch.zeros_like(lay.tier_map)
        out = torch.empty_like(zc)
        nws = dkv.dkv_decode_workspace_bytes(pool, cfg.B, lay.max_blocks, cfg.Hq, cfg.H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        lens = torch.tensor(lay.seq_lens, dtype=torch.int32, device="cuda")
        dkv.dkv_decode_step(pool, 0, inp.x.cuda(), inp.W.cuda(), table.cuda(), lens, tmap.cuda(), cfg.Hq,
                            cfg.theta, out, ws)
        assert dkv.dkv_check(pool) == dkv.DKV_OK
        assert torch.equal(out, zc)
        # against the fp64 oracle: on the original two-tier inputs, and walking the staged
        # tables over the oracle's own copy of the staged HBM tier (host blocks appended)
        TL.assert_out_close(out, TL.oracle_step(inp)["out"], "staged vs oracle")
        staged = np.concatenate([WL.bf16_bits(inp.hbm), WL.bf16_bits(inp.host)], axis=1)
        ref = O.decode_step(WL.bf16_bits(inp.x), WL.bf16_bits(inp.W), [staged, WL.bf16_bits(inp.host)],
                            table.numpy(), lay.seq_lens, tmap.numpy(), cfg.Hq, cfg.Hkv, cfg.D, cfg.T,
                            cfg.theta)["out"]
        TL.assert_out_close(out, ref, "staged vs oracle on the staged tables")
    finally:
        dkv.dkv_pool_destroy(pool)
