"""Parity of the CUDA decode step (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import workloads as WL

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_offload_b200 as dkv
    import dkv_testlib as TL
else:  # collected on CPU-only hosts, never run
    dkv = TL = None


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_offload_b200.build import build
    build()


def _run_and_check(cfg, seed=0, layout=0, layer=None, attn_splits=0, seq_lens=None, host_flags=0):
    inp = WL.make_decode_inputs(cfg, seed=seed, pool_layout=layout, seq_lens=seq_lens)
    layer = cfg.layers - 1 if layer is None else layer
    ctx = TL.make_pool(inp, host_flags=host_flags)
    try:
        out = TL.run_step(ctx, layer=layer, attn_splits=attn_splits)
        ores = TL.oracle_step(inp, layer=layer)
        errs = TL.assert_out_close(out, ores["out"], cfg.name)
        TL.check_cache(ctx, ores, layer=layer)
        return out, ores, errs
    finally:
        ctx.close()


def test_tiny_config_all_host():
    _run_and_check(WL.CONFIGS["tiny"])


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 2, 128), (8, 8, 128), (4, 2, 128), (16, 2, 128),
                                      (8, 2, 64), (8, 8, 64), (4, 2, 64), (16, 2, 64)])
def test_group_sizes_and_head_dims(Hq, Hkv, D):
    cfg = WL.small_config(Hq=Hq, Hkv=Hkv, D=D, H=256 if D == 64 else 384)
    _run_and_check(cfg)


@pytest.mark.parametrize("layout", [0, 1])
def test_ragged_lengths_both_tiers_both_layouts(layout):
    cfg = WL.small_config(B=7, layers=3)
    _run_and_check(cfg, layout=layout, layer=1, seq_lens=[0, 1, 15, 16, 17, 100, 257])


@pytest.mark.parametrize("cs", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("B", [3, 13, 32])
def test_projection_cluster_sizes(cs, B):
    """Every cluster size of the projection's split-K reduction (its gather of the partial
    columns is compiled per size), with batches below, between and at multiples of it
    (B < CS leaves ranks that finish no column)."""
    cfg = WL.small_config(B=B, H=512, ctx_range=(1, 64))
    inp = WL.make_decode_inputs(cfg, seed=cs)
    ctx = TL.make_pool(inp)
    try:
        out = TL.run_step(ctx, layer=1, proj_splits=cs)
        ores = TL.oracle_step(inp, layer=1)
        TL.assert_out_close(out, ores["out"], cfg.name)
        TL.check_cache(ctx, ores, layer=1)
    finally:
        ctx.close()


@pytest.mark.parametrize("splits", [1, 2, 5, 64])
def test_split_counts(splits):
    cfg = WL.small_config(B=2, ctx_range=(300, 400))
    _run_and_check(cfg, attn_splits=splits)


def test_split_invariance_close():
    cfg = WL.small_config(B=2, ctx_range=(500, 700), host_prob=0.3)
    o1, _, _ = _run_and_check(cfg, attn_splits=1)
    o2, _, _ = _run_and_check(cfg, attn_splits=13)
    d = (o1.float() - o2.float()).abs().max().item()
    assert d <= 2 * 2.0 ** -8 * max(o1.float().abs().max().item(), 1e-3)


def test_batch_32_and_write_combined_host():
    cfg = WL.small_config(B=32, H=256, Hq=8, Hkv=8, D=64, ctx_range=(1, 90), layers=1)
    _run_and_check(cfg, host_flags=dkv.DKV_HOST_WRITE_COMBINED)


def test_step_is_repeatable():
    cfg = WL.small_config(B=3)
    inp = WL.make_decode_inputs(cfg)
    ctx = TL.make_pool(inp)
    try:
        a = TL.run_step(ctx, layer=1)
        b = TL.run_step(ctx, layer=1)
        # every reduction has a fixed order: the step is bit-for-bit repeatable
        assert torch.equal(a, b)
    finally:
        ctx.close()


def test_automatic_attention_variant():
    """The automatic shape and split count (148 SMs). Splits: G = 4 and the one-CTA G = 8
    shape take the most that fit in one wave of CTA slots (two for G = 4 above 64
    (sequence, kv head) units), the three-CTA G = 8 shape the most within 2.33 waves (0.86
    of a wave where that would exceed 64 splits), other group sizes about 2.9 waves. Shape:
    variant 5 for G = 4 while its splits keep >= 39 table blocks each, for G = 8 while they
    keep >= 6 and number at most 64 (>= 40 blocks when cut under a wave), else (and for
    other group sizes) variant 1; an explicit tuning value is taken as is."""
    pool = dkv.dkv_pool_create(1, 8, 128, 4, 1, block_tokens=16)
    try:
        assert dkv.dkv_decode_attn_variant(pool, 16, 2050, 32) == 5
        assert dkv.dkv_decode_attn_splits(pool, 16, 2050, 32) == 9     # two waves of 592 slots
        assert dkv.dkv_decode_attn_variant(pool, 4, 2050, 32) == 5     # 18 splits of 113 blocks
        assert dkv.dkv_decode_attn_splits(pool, 4, 2050, 32) == 18     # one wave
        assert dkv.dkv_decode_attn_variant(pool, 1, 513, 32) == 1      # 74 splits of 6 blocks
        assert dkv.dkv_decode_attn_splits(pool, 1, 513, 32) == 55      # one wave of 444 slots
        assert dkv.dkv_decode_attn_variant(pool, 8, 2050, 32) == 5     # 9 splits of 227
        assert dkv.dkv_decode_attn_variant(pool, 16, 2050, 64) == 5    # G = 8, long contexts
        assert dkv.dkv_decode_attn_splits(pool, 16, 2050, 64) == 8     # within 2.33 waves of 444
        assert dkv.dkv_decode_attn_variant(pool, 8, 130, 64) == 5      # G = 8: 20 splits of 6
        assert dkv.dkv_decode_attn_variant(pool, 4, 130, 64) == 1      # G = 8: 40 splits of 3
        assert dkv.dkv_decode_attn_variant(pool, 1, 2050, 64) == 5     # G = 8, one sequence:
        assert dkv.dkv_decode_attn_splits(pool, 1, 2050, 64) == 47     # 0.86 wave, 43 blocks each
        assert dkv.dkv_decode_attn_variant(pool, 1, 513, 64) == 1      # 10 blocks per split: the
        assert dkv.dkv_decode_attn_splits(pool, 1, 513, 64) == 18      # one-CTA shape, one wave
        assert dkv.dkv_decode_attn_variant(pool, 16, 2050, 16) == 1    # G = 2: not measured
        dkv.dkv_pool_set_tuning(pool, attn_variant=7)
        assert dkv.dkv_decode_attn_variant(pool, 16, 2050, 32) == 7
    finally:
        dkv.dkv_pool_destroy(pool)


@pytest.mark.parametrize("Hq", [8, 16, 32, 64])
def test_automatic_split_count_respects_its_wave_bound(Hq):
    """Over many batch sizes and table widths (8 kv heads, so G = 1, 2, 4, 8): the automatic
    split count is at least 1, at most the table width, and its grid fits the documented
    number of waves of the chosen shape's CTA slots whenever the width allows it."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    per_sm = {(4, 1): 3, (4, 5): 4, (8, 1): 1, (8, 5): 3}
    pool = dkv.dkv_pool_create(1, 8, 128, 4, 1, block_tokens=16)
    try:
        G = Hq // 8
        for B in (1, 2, 3, 5, 8, 13, 16, 24, 32):
            for blocks in (1, 2, 7, 33, 130, 513, 2050, 8193):
                S = dkv.dkv_decode_attn_splits(pool, B, blocks, Hq)
                v = dkv.dkv_decode_attn_variant(pool, B, blocks, Hq)
                assert 1 <= S <= blocks, (B, blocks, Hq, S)
                units = B * 8
                if G not in (4, 8):
                    continue
                slots = sms * per_sm[(G, v)]
                if G == 4 or v == 1:
                    waves = 2 if (G == 4 and units > 64) else 1
                else:
                    waves = 2.33 if 233 * slots // (100 * units) <= 64 else 0.86
                assert units * S <= max(units, waves * slots), (B, blocks, Hq, v, S)
                if S < blocks:  # not capped by the table: the most splits within the bound
                    assert units * (S + 1) > waves * slots, (B, blocks, Hq, v, S)
    finally:
        dkv.dkv_pool_destroy(pool)


def test_bad_table_entries_are_flagged_not_fatal():
    cfg = WL.small_config(B=2, ctx_range=(40, 60), host_prob=0.5)
    inp = WL.make_decode_inputs(cfg)
    ctx = TL.make_pool(inp)
    try:
        x, W = inp.x.cuda(), inp.W.cuda()
        out = torch.empty((cfg.B, cfg.Hq * cfg.D), dtype=torch.bfloat16, device="cuda")
        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        for mutate in ("tier", "block", "ctx"):
            table, tmap, lens = ctx.table.clone(), ctx.tier_map.clone(), ctx.seq_lens.clone()
            if mutate == "tier":
                tmap[0, 1] = 7
            elif mutate == "block":
                table[1, 0] = 1 << 30
            else:
                lens[0] = table.shape[1] * cfg.T + 5
            dkv.dkv_decode_step(ctx.pool, 1, x, W, table, lens, tmap, cfg.Hq, cfg.theta, out, ws)
            assert dkv.dkv_check(ctx.pool) == dkv.DKV_ERR_BAD_TABLE, mutate
        # the pool is still usable and clean afterwards
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
    finally:
        ctx.close()


@pytest.mark.parametrize("variant", [5, 1, 6])
def test_bounded_wait_gives_up_and_the_pool_stays_usable(variant):
    # a stage that is never loaded (the test hook withholds the first block of CTA (0, 0, 0)):
    # its consumer's bounded wait gives up after 2 ms, the kernel returns, dkv_check reports
    # DKV_ERR_TIMEOUT; the other sequence's output is unaffected and the next step is exact
    cfg = WL.small_config(B=2, Hq=8, Hkv=2, ctx_range=(600, 800), host_prob=0.3, layers=1)
    inp = WL.make_decode_inputs(cfg, seed=12)
    ctx = TL.make_pool(inp)
    try:
        x, W = inp.x.cuda(), inp.W.cuda()
        out = torch.empty((cfg.B, cfg.Hq * cfg.D), dtype=torch.bfloat16, device="cuda")
        dkv.dkv_pool_set_tuning(ctx.pool, attn_splits=1, attn_variant=variant, wait_limit_us=2000,
                                test_withhold_block=1)
        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        dkv.dkv_decode_step(ctx.pool, 0, x, W, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.Hq, cfg.theta, out, ws)
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_ERR_TIMEOUT
        assert "timed out" in dkv.dkv_last_error()
        TL.assert_out_close(out, TL.oracle_step(inp, batch=[1])["out"], "sequence 1 beside a timed-out CTA")
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK  # the status word was cleared
        good = TL.run_step(ctx)  # default tuning again (run_step asserts DKV_OK)
        TL.assert_out_close(good, TL.oracle_step(inp)["out"], "step after the timeout")
    finally:
        ctx.close()


def test_argument_errors():
    cfg = WL.small_config(B=2)
    inp = WL.make_decode_inputs(cfg)
    ctx = TL.make_pool(inp)
    try:
        with pytest.raises(dkv.DkvError):
            dkv.dkv_decode_workspace_bytes(ctx.pool, 33, ctx.table.shape[1], cfg.Hq, cfg.H)
        with pytest.raises(dkv.DkvError):
            dkv.dkv_decode_workspace_bytes(ctx.pool, 2, ctx.table.shape[1], 6, cfg.H)  # G = 3
        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, 2, ctx.table.shape[1], cfg.Hq, cfg.H)
        ws = torch.empty(nws - 256, dtype=torch.uint8, device="cuda")
        out = torch.empty((2, cfg.Hq * cfg.D), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(dkv.DkvError):
            dkv.dkv_decode_step(ctx.pool, 0, inp.x.cuda(), inp.W.cuda(), ctx.table, ctx.seq_lens,
                                ctx.tier_map, cfg.Hq, cfg.theta, out, ws)
        for bad in (dict(proj_splits=9), dict(proj_splits=-1), dict(attn_splits=-1), dict(attn_variant=2)):
            with pytest.raises(dkv.DkvError):
                dkv.dkv_pool_set_tuning(ctx.pool, **bad)
    finally:
        ctx.close()


def test_append_kv_places_tokens_bit_exact():
    cfg = WL.small_config(B=3, ctx_range=(5, 40), layers=2)
    inp = WL.make_decode_inputs(cfg)
    ctx = TL.make_pool(inp)
    try:
        n = 9
        lens = [max(0, c - n) for c in inp.layout.seq_lens]  # positions that exist in the table
        k = WL.randn_bf16((cfg.B, n, cfg.Hkv, cfg.D), 77)
        v = WL.randn_bf16((cfg.B, n, cfg.Hkv, cfg.D), 78)
        lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
        dkv.dkv_append_kv(ctx.pool, 1, k.cuda(), v.cuda(), ctx.table, lens_d, ctx.tier_map)
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
        exp = [WL.bf16_bits(inp.hbm).copy(), WL.bf16_bits(inp.host).copy()]
        kb, vb = WL.bf16_bits(k), WL.bf16_bits(v)
        for b in range(cfg.B):
            for t in range(n):
                pos = lens[b] + t
                j, slot = divmod(pos, cfg.T)
                tier = int(inp.layout.tier_map[b, j]); phys = int(inp.layout.block_table[b, j])
                exp[tier][1, phys, 0, :, slot] = kb[b, t]
                exp[tier][1, phys, 1, :, slot] = vb[b, t]
        got = [ctx.hbm.cpu().view(torch.int16).numpy().view(np.uint16).reshape(inp.hbm.shape),
               ctx.host.numpy().view(np.uint16).reshape(inp.host.shape)]
        assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1])
    finally:
        ctx.close()


@pytest.mark.parametrize("src_tier", [0, 1])
def test_layout_conversion_bit_exact(src_tier):
    from oracle import dkv_oracle as O
    cfg = WL.small_config(B=4, layers=5, ctx_range=(30, 200), host_prob=0.5)
    for layout in (0, 1):
        inp = WL.make_decode_inputs(cfg, pool_layout=layout)
        ctx = TL.make_pool(inp)
        try:
            src = (inp.hbm, inp.host)[src_tier]
            dst = torch.empty(src.numel(), dtype=torch.bfloat16, device="cuda")
            dkv.dkv_convert_layout(ctx.pool, src_tier, dst)
            torch.cuda.synchronize()
            bits = WL.bf16_bits(src)
            exp = O.layer_first_to_page_first(bits) if layout == 0 else O.page_first_to_layer_first(bits)
            got = dst.cpu().view(torch.int16).numpy().view(np.uint16).reshape(exp.shape)
            assert np.array_equal(got, exp)
            # and back again with the raw-buffer entry point
            back = torch.empty_like(dst)
            chunk = 2 * cfg.Hkv * cfg.T * cfg.D * 2
            nblk = src.shape[1] if layout == 0 else src.shape[0]
            dkv.dkv_permute_layout(dst, back, 1 - layout, cfg.layers, nblk, chunk)
            torch.cuda.synchronize()
            assert np.array_equal(back.cpu().view(torch.int16).numpy().view(np.uint16), bits.reshape(-1))
        finally:
            ctx.close()


def test_staged_calls_match_fused_step():
    # project; attend(out=None); combine  ==  project; attend(out)  ==  dkv_decode_step
    cfg = WL.small_config(B=4, ctx_range=(100, 400), host_prob=0.4)
    inp = WL.make_decode_inputs(cfg, seed=5)
    ctx = TL.make_pool(inp)
    try:
        fused = TL.run_step(ctx, layer=1)
        x, W = inp.x.cuda(), inp.W.cuda()
        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        staged = torch.empty_like(fused)
        dkv.dkv_decode_project(ctx.pool, 1, x, W, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.Hq, cfg.theta, ws)
        dkv.dkv_decode_attend(ctx.pool, 1, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.H, cfg.Hq, ws)
        dkv.dkv_decode_combine(ctx.pool, cfg.B, ctx.table.shape[1], cfg.H, cfg.Hq, staged, ws)
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
        assert torch.equal(staged, fused)
    finally:
        ctx.close()


@pytest.mark.parametrize("variant", [1, 5, 6, 7])
@pytest.mark.parametrize("splits", [1, 0])  # one split: long CTAs that wrap the stage ring
@pytest.mark.parametrize("D", [64, 128])
def test_attention_kernel_variants(variant, splits, D):
    cfg = WL.small_config(B=3, Hq=8, Hkv=2, D=D, H=256, ctx_range=(300, 700), host_prob=0.5)
    inp = WL.make_decode_inputs(cfg, seed=11)
    ctx = TL.make_pool(inp)
    try:
        base = TL.run_step(ctx, layer=1)
        dkv.dkv_pool_set_tuning(ctx.pool, attn_splits=splits, attn_variant=variant,
                                attn_lsu_hbm=variant % 2)
        x, W = inp.x.cuda(), inp.W.cuda()
        out = torch.empty_like(base)
        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        dkv.dkv_decode_step(ctx.pool, 1, x, W, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.Hq, cfg.theta, out, ws)
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
        TL.assert_out_close(out, TL.oracle_step(inp, layer=1)["out"], "variant %d" % variant)
        # same splits, same reduction order per (slot, head): the variants agree closely
        assert (out.float() - base.float()).abs().max().item() <= 2 ** -6
    finally:
        ctx.close()


@pytest.mark.parametrize("variant", [1, 5, 6])
@pytest.mark.parametrize("splits", [1, 0])
@pytest.mark.parametrize("D", [64, 128])
def test_attention_kernel_variants_group_of_8(variant, splits, D):
    # G = 8 (the 70B shape): two consumer warps of four heads per block in the CUDA-core
    # shapes; every shape against the oracle, and against each other
    cfg = WL.small_config(B=3, Hq=16, Hkv=2, D=D, H=256, ctx_range=(300, 700), host_prob=0.5)
    inp = WL.make_decode_inputs(cfg, seed=13)
    ctx = TL.make_pool(inp)
    try:
        base = TL.run_step(ctx, layer=1)
        dkv.dkv_pool_set_tuning(ctx.pool, attn_splits=splits, attn_variant=variant)
        x, W = inp.x.cuda(), inp.W.cuda()
        out = torch.empty_like(base)
        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        dkv.dkv_decode_step(ctx.pool, 1, x, W, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.Hq, cfg.theta, out, ws)
        assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
        TL.assert_out_close(out, TL.oracle_step(inp, layer=1)["out"], "G=8 variant %d" % variant)
        assert (out.float() - base.float()).abs().max().item() <= 2 ** -6
    finally:
        ctx.close()


@pytest.mark.parametrize("D,Hq", [(128, 8), (64, 16)])
def test_unwritten_tail_slots_are_ignored(D, Hq):
    """Slots past a sequence's last cached token may hold any bits (here NaN in both tiers):
    the outputs must not see them."""
    cfg = WL.small_config(B=4, Hq=Hq, Hkv=2, D=D, H=256, ctx_range=(33, 300), host_prob=0.5)
    inp = WL.make_decode_inputs(cfg, seed=23)
    lay, T = inp.layout, cfg.T
    tiers = [inp.hbm.view(torch.int16), inp.host.view(torch.int16)]
    for b in range(cfg.B):
        c = lay.seq_lens[b]
        for pos in range(c + 1, (c // T + 1) * T):   # after the new token's slot
            j, slot = divmod(pos, T)
            t, phys = int(lay.tier_map[b, j]), int(lay.block_table[b, j])
            tiers[t][0, phys, :, :, slot, :] = 0x7FC0   # bf16 quiet NaN
        j = (c - 1) // T                                 # and the cached tail's own spare slots
        t, phys = int(lay.tier_map[b, j]), int(lay.block_table[b, j])
        for slot in range(c - j * T, T):
            if j * T + slot != c:
                tiers[t][0, phys, :, :, slot, :] = 0x7FC0
    ctx = TL.make_pool(inp)
    try:
        out = TL.run_step(ctx, layer=0)
        assert torch.isfinite(out.float()).all()
        TL.assert_out_close(out, TL.oracle_step(inp, layer=0)["out"], "NaN in unwritten slots")
    finally:
        ctx.close()


def test_serial_launch_matches_overlapped_launch():
    """Programmatic dependent launch only moves kernel starts: outputs are bit-identical
    with the kernels launched one after another, and with the overlap kept inside a step."""
    cfg = WL.small_config(B=5, Hq=16, Hkv=2, D=128, H=512, ctx_range=(100, 900), host_prob=0.3)
    inp = WL.make_decode_inputs(cfg, seed=31)
    ctx = TL.make_pool(inp)
    try:
        a = TL.run_step(ctx, layer=1)
        x, W = inp.x.cuda(), inp.W.cuda()
        nws = dkv.dkv_decode_workspace_bytes(ctx.pool, cfg.B, ctx.table.shape[1], cfg.Hq, cfg.H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        for mode in (1, 2, 3, 0):
            dkv.dkv_pool_set_tuning(ctx.pool, serial_launch=mode)
            b = torch.empty_like(a)
            for _ in range(3):  # back to back on one stream, as a serving loop runs them
                dkv.dkv_decode_step(ctx.pool, 1, x, W, ctx.table, ctx.seq_lens, ctx.tier_map, cfg.Hq, cfg.theta,
                                    b, ws)
            assert dkv.dkv_check(ctx.pool) == dkv.DKV_OK
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), mode
        with pytest.raises(dkv.DkvError):
            dkv.dkv_pool_set_tuning(ctx.pool, serial_launch=4)
    finally:
        ctx.close()


@pytest.mark.parametrize("layout", [0, 1])
def test_empty_context_returns_the_new_value_exactly(layout):
    """With no cached tokens the softmax has one term: every q head of a group outputs the
    new value v_hat of its kv head, bit for bit (the value the step wrote into the cache)."""
    cfg = WL.small_config(B=4, Hq=8, Hkv=2, D=128, H=256, host_prob=0.5)
    inp = WL.make_decode_inputs(cfg, seed=41, pool_layout=layout, seq_lens=[0, 37, 0, 16])
    ctx = TL.make_pool(inp)
    try:
        out = TL.run_step(ctx, layer=1).view(torch.int16).cpu().reshape(cfg.B, cfg.Hq, cfg.D)
        torch.cuda.synchronize()
        tiers = [ctx.hbm.cpu().view(torch.int16).reshape(inp.hbm.shape),
                 ctx.host.clone().reshape(inp.host.shape)]
        lay, G = inp.layout, cfg.Hq // cfg.Hkv
        for b in (0, 2):
            t, phys = int(lay.tier_map[b, 0]), int(lay.block_table[b, 0])
            for h in range(cfg.Hq):
                g = h // G
                vhat = tiers[t][1, phys, 1, g, 0] if layout == 0 else tiers[t][phys, 1, 1, g, 0]
                assert torch.equal(out[b, h], vhat), (b, h)
        TL.assert_out_close(out.view(torch.bfloat16).reshape(cfg.B, -1).cuda(),
                            TL.oracle_step(inp, layer=1)["out"], "empty contexts")
    finally:
        ctx.close()
