"""dkv_decode_step_static — the decode step for callers that cannot allocate device memory
(a serving loop whose device memory is reserved up front by its own allocator, a loop that
cannot take cudaMalloc's implicit synchronisation, a plain C host without a device
allocator). It takes its workspace from a fixed 16 MiB array inside the library instead of
a caller buffer. This file is collected last so a stop-at-first-failure run has already
run every other test; it also passes alone in a fresh process (the first call on the
device performs the one-time address lookup).
"""
import pytest
import torch

import workloads as WL

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


def test_static_workspace_step_matches_workspace_step_twice():
    cfg = WL.small_config(B=5, ctx_range=(1, 300), host_prob=0.5, layers=2)
    inp = WL.make_decode_inputs(cfg, seed=3)
    ctx = TL.make_pool(inp)
    try:
        x, W = inp.x.cuda(), inp.W.cuda()
        ref = TL.run_step(ctx, layer=1)
        outs = [torch.full_like(ref, float("nan")) for _ in range(2)]
        for i, out in enumerate(outs):  # two calls in a row share (and reuse) the static array
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info()[0]
            dkv.dkv_decode_step_static(ctx.pool, 1, x, W, ctx.table, ctx.seq_lens, ctx.tier_map,
                                       cfg.Hq, cfg.theta, out)
            torch.cuda.synchronize()
            free1 = torch.cuda.mem_get_info()[0]
            assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
            # same kernels, split count and workspace layout as the caller-workspace step:
            # the same bits
            assert torch.equal(out, ref)
            if i == 1:  # the first call may commit the array (lazy module loading); later ones nothing
                assert free1 == free0, "device memory changed across a static-workspace call"
        TL.assert_out_close(outs[1], TL.oracle_step(inp, layer=1)["out"], "static workspace vs oracle")
    finally:
        ctx.close()


def test_static_workspace_rejects_oversized_shapes():
    cfg = WL.small_config(B=2, ctx_range=(10, 20), layers=1)
    inp = WL.make_decode_inputs(cfg)
    ctx = TL.make_pool(inp)
    try:
        cap = dkv.dkv_decode_static_workspace_capacity()
        assert cap == 16 << 20
        # many splits per (sequence, kv head) make the partial-state area exceed the array
        dkv.dkv_pool_set_tuning(ctx.pool, attn_splits=4096)
        big_blocks = 8192
        table = torch.zeros((cfg.B, big_blocks), dtype=torch.int32, device="cuda")
        tmap = torch.zeros((cfg.B, big_blocks), dtype=torch.uint8, device="cuda")
        need = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, big_blocks, cfg.Hq, cfg.H)
        assert need > cap
        out = torch.empty((cfg.B, cfg.Hq * cfg.D), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(dkv.DkvError) as e:
            dkv.dkv_decode_step_static(ctx.pool, 0, inp.x.cuda(), inp.W.cuda(), table, ctx.seq_lens, tmap,
                                       cfg.Hq, cfg.theta, out)
        assert e.value.code == dkv.DKV_ERR_CAPACITY
    finally:
        ctx.close()


def test_static_workspace_unsupported_shape_has_the_same_code():
    # a batch of 33 is beyond the step's limit: both entry points say DKV_ERR_UNSUPPORTED
    cfg = WL.small_config(B=2, ctx_range=(10, 20), layers=1)
    inp = WL.make_decode_inputs(cfg)
    ctx = TL.make_pool(inp)
    try:
        B = 33
        x = torch.zeros((B, cfg.H), dtype=torch.bfloat16, device="cuda")
        table = torch.zeros((B, 4), dtype=torch.int32, device="cuda")
        tmap = torch.zeros((B, 4), dtype=torch.uint8, device="cuda")
        lens = torch.zeros((B,), dtype=torch.int32, device="cuda")
        out = torch.empty((B, cfg.Hq * cfg.D), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        with pytest.raises(dkv.DkvError) as e1:
            dkv.dkv_decode_step(ctx.pool, 0, x, inp.W.cuda(), table, lens, tmap, cfg.Hq, cfg.theta, out, ws)
        with pytest.raises(dkv.DkvError) as e2:
            dkv.dkv_decode_step_static(ctx.pool, 0, x, inp.W.cuda(), table, lens, tmap, cfg.Hq, cfg.theta, out)
        assert e1.value.code == e2.value.code == dkv.DKV_ERR_UNSUPPORTED
    finally:
        ctx.close()
