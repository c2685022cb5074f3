"""Seeded synthetic workloads for the zero-copy decode step and the zero-copy GEMM study.

This module only draws random inputs and lays out block tables; it holds none of the
method's arithmetic (no projection, RoPE, softmax or GEMM). It is the one piece shared
by the CUDA path's tests/bench and the fp64 oracle: both sides receive the very same
tensors produced here.

Shapes follow the Llama-shaped layers the DirectKV summary evaluates on ("长上下文 LLM 的
零拷贝 KV Cache 卸载（OSDI 2026）", 实验与结果: multiple models, long contexts), stated as five
concrete configurations:

  tiny      B=1,  H=256,  Hq=4,  Hkv=2, D=64,  theta=1e4, ctx=512, all blocks in the host tier
  8b_hbm    B=16, H=4096, Hq=32, Hkv=8, D=128, theta=5e5, ctx=32768 each, all blocks in HBM
  8b_mixed  B=4,  same layer, ctx=131072 each, the most recent 4096 tokens (256 blocks) and
            the tail block in HBM, older blocks in the host tier, physical ids permuted
  70b_mixed B=32, H=8192, Hq=64, Hkv=8, D=128, theta=5e5, ctx ~ U{8192..65536}, each
            logical block host-resident with probability 0.8, physical ids permuted
  70b_hbm   the 70b_mixed layer and lengths with every block in HBM (an added case for
            the group-size-8 attention against the HBM roofline)
  gemm      M=N=K=10240 bf16, A in HBM, B in the host tier, entries ~ U(-1, 1)

Seeding: one CPU ``torch.Generator`` per tensor, seeded ``seed + index`` with the index
order x=0, Wqkv=1, K=2, V=3, tables=4, tiers=5, lengths=6. Normal draws are fp32 in
chunks of 2**24 elements, scaled in fp32, then rounded to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

T_BLOCK = 16          # tokens per KV block
_CHUNK = 1 << 24      # elements per generator draw

SEED_X, SEED_W, SEED_K, SEED_V, SEED_TABLE, SEED_TIER, SEED_LEN = range(7)


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    Hq: int
    Hkv: int
    D: int
    theta: float
    ctx: Optional[int]            # fixed context per sequence, or None for a drawn mix
    ctx_range: Optional[tuple] = None
    tier_policy: str = "hbm"      # "hbm" | "host" | "recent_hbm" | "bernoulli"
    recent_hbm_tokens: int = 0
    host_prob: float = 0.0
    permute: bool = False
    layers: int = 1
    T: int = T_BLOCK

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def rows(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.D


CONFIGS = {
    "tiny": DecodeConfig("tiny", B=1, H=256, Hq=4, Hkv=2, D=64, theta=1e4, ctx=512,
                         tier_policy="host"),
    "8b_hbm": DecodeConfig("8b_hbm", B=16, H=4096, Hq=32, Hkv=8, D=128, theta=5e5,
                           ctx=32768, tier_policy="hbm"),
    "8b_mixed": DecodeConfig("8b_mixed", B=4, H=4096, Hq=32, Hkv=8, D=128, theta=5e5,
                             ctx=131072, tier_policy="recent_hbm", recent_hbm_tokens=4096,
                             permute=True),
    "70b_mixed": DecodeConfig("70b_mixed", B=32, H=8192, Hq=64, Hkv=8, D=128, theta=5e5,
                              ctx=None, ctx_range=(8192, 65536), tier_policy="bernoulli",
                              host_prob=0.8, permute=True),
    # the same 70B-shaped layer with every block in HBM: the group size 8 attention
    # against the HBM roofline (an added measurement case, not one of the five above)
    "70b_hbm": DecodeConfig("70b_hbm", B=32, H=8192, Hq=64, Hkv=8, D=128, theta=5e5,
                            ctx=None, ctx_range=(8192, 65536), tier_policy="hbm", permute=True),
}


@dataclasses.dataclass(frozen=True)
class GemmConfig:
    name: str
    M: int
    N: int
    K: int


GEMM_CONFIGS = {"gemm": GemmConfig("gemm", 10240, 10240, 10240)}


def small_config(name="small", B=3, H=384, Hq=8, Hkv=2, D=128, theta=5e5, ctx=None,
                 ctx_range=(1, 200), tier_policy="bernoulli", host_prob=0.5,
                 permute=True, layers=2, recent_hbm_tokens=0) -> DecodeConfig:
    """A reduced configuration for parity tests: several tiles, ragged tails, both tiers."""
    return DecodeConfig(name, B=B, H=H, Hq=Hq, Hkv=Hkv, D=D, theta=theta, ctx=ctx,
                        ctx_range=ctx_range, tier_policy=tier_policy, host_prob=host_prob,
                        permute=permute, layers=layers, recent_hbm_tokens=recent_hbm_tokens)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, seed: int, std: float = 1.0, gen: Optional[torch.Generator] = None,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """N(0, std^2) draws as bf16, drawn in fp32 chunks of 2**24 from a seeded generator."""
    g = gen if gen is not None else _gen(seed)
    n = math.prod(shape)
    res = out if out is not None else torch.empty(shape, dtype=torch.bfloat16)
    flat = res.view(-1)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        v = torch.randn(e - s, generator=g, dtype=torch.float32)
        if std != 1.0:
            v.mul_(std)
        flat[s:e].copy_(v)
    return res


def uniform_bf16(shape, seed: int, lo=-1.0, hi=1.0) -> torch.Tensor:
    g = _gen(seed)
    n = math.prod(shape)
    res = torch.empty(shape, dtype=torch.bfloat16)
    flat = res.view(-1)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        v = torch.rand(e - s, generator=g, dtype=torch.float32)
        v.mul_(hi - lo).add_(lo)
        flat[s:e].copy_(v)
    return res


def seq_lengths(cfg: DecodeConfig, seed: int = 0) -> List[int]:
    if cfg.ctx is not None:
        return [cfg.ctx] * cfg.B
    lo, hi = cfg.ctx_range
    g = _gen(seed + SEED_LEN)
    return [int(v) for v in torch.randint(lo, hi + 1, (cfg.B,), generator=g)]


@dataclasses.dataclass
class BlockLayout:
    """Logical -> (tier, physical block) map for one batch, plus tier sizes."""
    seq_lens: List[int]
    nblk: List[int]              # logical blocks per sequence incl. the new token's slot
    max_blocks: int
    block_table: torch.Tensor    # int32 [B, max_blocks]; unused entries -1
    tier_map: torch.Tensor       # uint8 [B, max_blocks]; 0 = HBM, 1 = host
    hbm_blocks: int
    host_blocks: int


def block_layout(cfg: DecodeConfig, seed: int = 0, seq_lens: Optional[List[int]] = None) -> BlockLayout:
    """Place every logical block (cached blocks plus the block holding slot ctx) in a tier.

    The table covers ceil((ctx+1)/T) logical blocks per sequence so the new token's slot
    exists. Physical ids are sequential (b-major) or a seeded permutation within each tier.
    """
    lens = list(seq_lens) if seq_lens is not None else seq_lengths(cfg, seed)
    T = cfg.T
    nblk = [(c + 1 + T - 1) // T for c in lens]
    maxb = max(nblk)
    tiers = []
    if cfg.tier_policy == "bernoulli":
        total = sum(nblk)
        r = torch.rand(total, generator=_gen(seed + SEED_TIER))
        flat = (r < cfg.host_prob).to(torch.uint8)
    off = 0
    for b, n in enumerate(nblk):
        if cfg.tier_policy == "hbm":
            t = torch.zeros(n, dtype=torch.uint8)
        elif cfg.tier_policy == "host":
            t = torch.ones(n, dtype=torch.uint8)
        elif cfg.tier_policy == "recent_hbm":
            # blocks holding the most recent `recent_hbm_tokens` cached tokens, and the
            # tail block that receives the new token, stay in HBM; older ones in host
            n_cached_full = lens[b] // T
            first_hbm = max(0, n_cached_full - cfg.recent_hbm_tokens // T)
            t = torch.ones(n, dtype=torch.uint8)
            t[first_hbm:] = 0
        elif cfg.tier_policy == "bernoulli":
            t = flat[off:off + n].clone()
        else:
            raise ValueError(cfg.tier_policy)
        off += n
        tiers.append(t)
    counts = [sum(int((t == k).sum()) for t in tiers) for k in (0, 1)]
    if cfg.permute:
        g = _gen(seed + SEED_TABLE)
        ids = [torch.randperm(counts[0], generator=g), torch.randperm(counts[1], generator=g)]
    else:
        ids = [torch.arange(counts[0]), torch.arange(counts[1])]
    nxt = [0, 0]
    table = torch.full((cfg.B, maxb), -1, dtype=torch.int32)
    tmap = torch.zeros((cfg.B, maxb), dtype=torch.uint8)
    for b, t in enumerate(tiers):
        for k in (0, 1):
            sel = (t == k).nonzero().flatten()
            cnt = sel.numel()
            table[b, sel] = ids[k][nxt[k]:nxt[k] + cnt].to(torch.int32)
            nxt[k] += cnt
        tmap[b, :len(t)] = t
    return BlockLayout(lens, nblk, maxb, table, tmap, counts[0], counts[1])


def pool_shape(cfg: DecodeConfig, blocks: int, layout: int = 0):
    """Tier shape: layer-first [L][P][2][Hkv][T][D] (layout 0) or page-first [P][L][...]."""
    if layout == 0:
        return (cfg.layers, blocks, 2, cfg.Hkv, cfg.T, cfg.D)
    return (blocks, cfg.layers, 2, cfg.Hkv, cfg.T, cfg.D)


def fill_pool(cfg: DecodeConfig, hbm_blocks: int, host_blocks: int, seed: int = 0,
              layout: int = 0, hbm_out: Optional[torch.Tensor] = None,
              host_out: Optional[torch.Tensor] = None):
    """K ~ N(0,1) from generator seed+2 and V ~ N(0,1) from seed+3, HBM tier then host tier.

    Draw order within a tier follows its layout with the K/V axis removed. Returns the two
    tier tensors (bf16, CPU unless `*_out` buffers are given).
    """
    gk, gv = _gen(seed + SEED_K), _gen(seed + SEED_V)
    res = []
    for blocks, out in ((hbm_blocks, hbm_out), (host_blocks, host_out)):
        shp = pool_shape(cfg, blocks, layout)
        t = out if out is not None else torch.empty(shp, dtype=torch.bfloat16)
        assert tuple(t.shape) == shp
        kv_axis = 2
        for kv, g in ((0, gk), (1, gv)):
            view = t.select(kv_axis, kv)
            tmp = randn_bf16(tuple(view.shape), 0, gen=g)
            view.copy_(tmp)
            del tmp
        res.append(t)
    return res[0], res[1]


@dataclasses.dataclass
class DecodeInputs:
    cfg: DecodeConfig
    x: torch.Tensor          # bf16 [B, H]
    W: torch.Tensor          # bf16 [rows, H]
    layout: BlockLayout
    hbm: torch.Tensor        # bf16 tier
    host: torch.Tensor       # bf16 tier
    pool_layout: int = 0


def make_decode_inputs(cfg: DecodeConfig, seed: int = 0, pool_layout: int = 0,
                       seq_lens: Optional[List[int]] = None) -> DecodeInputs:
    x = randn_bf16((cfg.B, cfg.H), seed + SEED_X)
    W = randn_bf16((cfg.rows, cfg.H), seed + SEED_W, std=1.0 / math.sqrt(cfg.H))
    lay = block_layout(cfg, seed, seq_lens)
    hbm, host = fill_pool(cfg, lay.hbm_blocks, lay.host_blocks, seed, pool_layout)
    return DecodeInputs(cfg, x, W, lay, hbm, host, pool_layout)


def make_gemm_inputs(cfg: GemmConfig, seed: int = 0):
    """A [M, K] and B stored column-major ([N, K] row-major, K contiguous), ~U(-1, 1)."""
    A = uniform_bf16((cfg.M, cfg.K), seed + 0)
    Bt = uniform_bf16((cfg.N, cfg.K), seed + 1)
    return A, Bt


def gemm_sample_pairs(M: int, N: int, count: int = 4096, seed: int = 0):
    g = _gen(seed)
    i = torch.randint(0, M, (count,), generator=g)
    j = torch.randint(0, N, (count,), generator=g)
    return i, j


def bf16_bits(t: torch.Tensor):
    """Raw bf16 bit patterns as a numpy uint16 array (a view when possible)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
