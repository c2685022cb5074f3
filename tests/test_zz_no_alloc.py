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


def _close(a: torch.Tensor, b: torch.Tensor):
    # same bars as the oracle comparisons: max-abs 3e-2, mean-abs 3e-3, rel-rms 1e-2
    d = (a.float() - b.float()).abs()
    rel = (a.float() - b.float()).norm() / b.float().norm().clamp_min(1e-30)
    assert d.max().item() <= 3e-2 and d.mean().item() <= 3e-3 and rel.item() <= 1e-2


def test_static_workspace_step_matches_workspace_step_twice():
    cfg = WL.small_config(B=5, ctx_range=(1, 300), host_prob=0.5, layers=2)
    inp = WL.make_decode_inputs(cfg, seed=3)
    ctx = TL.make_pool(inp)
    try:
        x, W = inp.x.cuda(), inp.W.cuda()
        ref = TL.run_step(ctx, layer=1)
        for _ in range(2):  # two calls in a row share (and reuse) the static array
            out = torch.full_like(ref, float("nan"))
            dkv.dkv_decode_step_static(ctx.pool, 1, x, W, ctx.table, ctx.seq_lens, ctx.tier_map,
                                       cfg.Hq, cfg.theta, out)
            assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
            _close(out, ref)
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
