"""Full-size parity in the benchmark's launch configuration (default tuning): the 8B-shaped
layer with the cache in HBM (B=16, 32768 cached tokens), the 8B layer with 4096 recent
tokens in HBM and older blocks in the host tier (B=4, 131072 tokens), the 70B-shaped
layer with 80% host blocks (B=32, 8192..65536 tokens) and the same layer with every block
in HBM (the group-of-8 shape on HBM). The oracle computes sampled (sequence, q head)
outputs one by one — random ones, plus the longest sequence and the one whose last cached
block holds the fewest tokens (most of that block masked) — every new cache row is checked
to one bf16 ulp and the rest of both tiers must be unchanged."""
import numpy as np
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


def _samples(cfg, seq_lens, n=6, seed=0):
    g = torch.Generator().manual_seed(seed)
    bs = torch.randperm(cfg.B, generator=g)[: min(n, cfg.B)].tolist()
    # the longest sequence, and the one whose cached tail block holds the fewest tokens
    longest = max(range(cfg.B), key=lambda b: seq_lens[b])
    tails = [b for b in range(cfg.B) if seq_lens[b] % cfg.T]
    partial = min(tails, key=lambda b: seq_lens[b] % cfg.T) if tails else longest
    bs += [longest, partial]
    # spread the sampled heads over different kv-head groups (the last q head of a group
    # for the two added sequences)
    hs = [(b * 7 + 3) % cfg.Hq for b in bs[:-2]] + [cfg.Hq - 1, cfg.G - 1]
    return bs, hs


@pytest.mark.parametrize("name", ["8b_hbm", "8b_mixed", "70b_mixed", "70b_hbm"])
def test_full_size_sampled(name):
    cfg = WL.CONFIGS[name]
    inp = WL.make_decode_inputs(cfg, seed=0)
    ctx = TL.make_pool(inp)
    try:
        out = TL.run_step(ctx, layer=0)  # default tuning = the benchmark's launch configuration
        bs, hs = _samples(cfg, inp.layout.seq_lens)
        got = out.float().cpu().double().numpy().reshape(cfg.B, cfg.Hq, cfg.D)
        errs = []
        for b, h in zip(bs, hs):
            ref = TL.oracle_step(inp, layer=0, batch=[b], heads=[h])["out"][b, h]
            e = np.abs(got[b, h] - ref)
            assert e.max() <= 3e-2 and e.mean() <= 3e-3, (name, b, h, e.max(), e.mean())
            assert np.linalg.norm(got[b, h] - ref) <= 1e-2 * np.linalg.norm(ref), (name, b, h)
            errs.append(e.max())
        TL.check_cache(ctx, None, layer=0, full_compare=True)
    finally:
        ctx.close()
