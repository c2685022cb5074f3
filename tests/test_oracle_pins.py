"""Pins for the fp64 oracle: each check ties it to something other than itself.

Brute-force re-derivations on tiny inputs (pure-Python loops, exact rationals), closed
forms, invariants the mathematics fixes, and the figures the pages print for the GEMM
study. A plausible slip in the oracle (dropped term, wrong sign, wrong head mapping,
transposed operand, double rounding) fails at least one of these.
"""
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import dkv_oracle as O
import workloads as WL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- bf16

def _bits_of(x: float) -> int:
    return int(O.f64_to_bf16_rne(np.array([x]))[0])


def test_bf16_rne_hand_cases():
    # exactly representable values keep their pattern
    assert _bits_of(1.0) == 0x3F80
    assert _bits_of(-2.5) == 0xC020
    assert _bits_of(0.0) == 0x0000
    assert _bits_of(-0.0) == 0x8000
    # tie between 1.0 (even) and 1 + 2^-7 (odd) -> 1.0
    assert _bits_of(1.0 + 2.0 ** -8) == 0x3F80
    # tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even) -> 1 + 2^-6
    assert _bits_of(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above a tie rounds up
    assert _bits_of(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    # no double rounding through fp32: 1 + 2^-8 + 2^-40 is above the tie
    assert _bits_of(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    # overflow and the largest finite value
    assert _bits_of(float.fromhex("0x1.fep127")) == 0x7F7F
    assert _bits_of(2.0 ** 128 * 0.999999) == 0x7F80
    assert _bits_of(-1e300) == 0xFF80
    # subnormals: 2^-133 is the smallest; half of it ties to zero, 1.5x rounds to 2x
    assert _bits_of(2.0 ** -133) == 0x0001
    assert _bits_of(2.0 ** -134) == 0x0000
    assert _bits_of(1.5 * 2.0 ** -133) == 0x0002


def test_bf16_rne_matches_library_on_fp32_values():
    # for inputs exactly representable in fp32, torch's fp32 -> bf16 cast (RNE) is the
    # same rounding problem, so it must agree bit for bit
    g = torch.Generator().manual_seed(1)
    x = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-140, 120, (200000,), generator=g).float())
    x = torch.cat([x, torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.0e38, -3.3e38, 1e-40])])
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f64_to_bf16_rne(x.double().numpy())
    assert np.array_equal(ref, got)


def test_bf16_to_f64_exact():
    bits = np.array([0x3F80, 0xC020, 0x0001, 0x7F7F, 0x8000], dtype=np.uint16)
    v = O.bf16_to_f64(bits)
    assert v[0] == 1.0 and v[1] == -2.5 and v[2] == 2.0 ** -133
    assert v[3] == float.fromhex("0x1.fep127") and math.copysign(1, v[4]) < 0


# ----------------------------------------------------------------------- projection

def test_projection_brute_force():
    rng = random.Random(3)
    R, H = 7, 5
    W = [[rng.uniform(-1, 1) for _ in range(H)] for _ in range(R)]
    x = [rng.uniform(-1, 1) for _ in range(H)]
    ref = [sum(Fraction(W[r][c]) * Fraction(x[c]) for c in range(H)) for r in range(R)]
    got = O.qkv_projection(np.array(W), np.array(x))
    for r in range(R):
        assert abs(got[r] - float(ref[r])) < 1e-15


def test_split_qkv_row_order():
    # one-hot rows: row r of W selects x[r], so q/k/v must be consecutive row ranges
    Hq, Hkv, D = 4, 2, 3
    rows = (Hq + 2 * Hkv) * D
    W = np.eye(rows)
    x = np.arange(rows, dtype=np.float64)
    q, k, v = O.split_qkv(O.qkv_projection(W, x), Hq, Hkv, D)
    assert q[2, 1] == 2 * D + 1
    assert k[1, 0] == Hq * D + D
    assert v[0, 2] == (Hq + Hkv) * D + 2


# ----------------------------------------------------------------------------- RoPE

def test_rope_position_zero_is_identity():
    v = np.random.default_rng(0).normal(size=(3, 64))
    assert np.array_equal(O.rope_rotate_half(v, 0, 1e4), v)


def test_rope_d2_closed_form():
    # D = 2 has one pair with frequency theta^0 = 1: a plain rotation by `pos` radians
    x0, x1, pos = 0.3, -1.7, 5
    y = O.rope_rotate_half(np.array([x0, x1]), pos, 1e4)
    assert abs(y[0] - (x0 * math.cos(pos) - x1 * math.sin(pos))) < 1e-15
    assert abs(y[1] - (x1 * math.cos(pos) + x0 * math.sin(pos))) < 1e-15


def test_rope_frequency_ladder():
    # D = 4, theta = 100: pair 0 turns by pos, pair 1 (dims 1 and 3) by pos * 100^(-1/2)
    pos = 3
    y = O.rope_rotate_half(np.array([0.0, 1.0, 0.0, 0.0]), pos, 100.0)
    a = pos * 0.1
    assert abs(y[1] - math.cos(a)) < 1e-15 and abs(y[3] - math.sin(a)) < 1e-15
    assert y[0] == 0.0 and y[2] == 0.0


def test_rope_preserves_pair_norms_and_relative_position():
    rng = np.random.default_rng(1)
    D = 128
    q, k = rng.normal(size=D), rng.normal(size=D)
    th = 5e5
    y = O.rope_rotate_half(q, 131072, th)
    h = D // 2
    assert np.allclose(y[:h] ** 2 + y[h:] ** 2, q[:h] ** 2 + q[h:] ** 2, rtol=1e-12)
    for m, n, d in [(7, 3, 11), (1000, 10, 517), (65536, 0, 3)]:
        a = O.rope_rotate_half(q, m, th) @ O.rope_rotate_half(k, n, th)
        b = O.rope_rotate_half(q, m + d, th) @ O.rope_rotate_half(k, n + d, th)
        assert abs(a - b) < 1e-9 * (1 + abs(a))


# ------------------------------------------------------------------------ attention

def _tiny_inputs(ctx_list, Hq=4, Hkv=2, D=8, H=12, T=4, host_prob=0.5, seed=0, layers=2, layout=0):
    cfg = WL.DecodeConfig("t", B=len(ctx_list), H=H, Hq=Hq, Hkv=Hkv, D=D, theta=1e4, ctx=None,
                          ctx_range=(0, 1), tier_policy="bernoulli", host_prob=host_prob,
                          permute=True, layers=layers, T=T)
    inp = WL.make_decode_inputs(cfg, seed=seed, pool_layout=layout, seq_lens=ctx_list)
    return cfg, inp


def _run_oracle(cfg, inp, layer=1, **kw):
    lay = inp.layout
    tiers = [WL.bf16_bits(inp.hbm), WL.bf16_bits(inp.host)]
    return O.decode_step(WL.bf16_bits(inp.x), WL.bf16_bits(inp.W), tiers,
                         lay.block_table.numpy(), lay.seq_lens, lay.tier_map.numpy(),
                         cfg.Hq, cfg.Hkv, cfg.D, cfg.T, cfg.theta, layer=layer,
                         layout=inp.pool_layout, **kw)


def _brute_force(cfg, inp, layer=1):
    """Independent dense attention: walk the table token by token in pure Python."""
    lay = inp.layout
    x = inp.x.float().double().numpy()
    W = inp.W.float().double().numpy()
    tiers = [inp.hbm.float().double().numpy(), inp.host.float().double().numpy()]
    D, T, G = cfg.D, cfg.T, cfg.Hq // cfg.Hkv
    out = np.zeros((cfg.B, cfg.Hq, D))
    for b in range(cfg.B):
        ctx = lay.seq_lens[b]
        proj = [sum(W[r, c] * x[b, c] for c in range(cfg.H)) for r in range(cfg.rows)]

        def rope(v):
            h = D // 2
            r = [0.0] * D
            for i in range(h):
                ang = ctx / (cfg.theta ** (2 * i / D))
                r[i] = v[i] * math.cos(ang) - v[i + h] * math.sin(ang)
                r[i + h] = v[i + h] * math.cos(ang) + v[i] * math.sin(ang)
            return r

        def rnd(v):  # bf16 RNE (pinned on its own above)
            return float(O.bf16_to_f64(O.f64_to_bf16_rne(np.array([v])))[0])

        for h in range(cfg.Hq):
            g = h // G
            q = rope(proj[h * D:(h + 1) * D])
            kn = [rnd(t) for t in rope(proj[cfg.Hq * D + g * D: cfg.Hq * D + (g + 1) * D])]
            vn = [rnd(t) for t in proj[(cfg.Hq + cfg.Hkv) * D + g * D:(cfg.Hq + cfg.Hkv) * D + (g + 1) * D]]
            keys, vals = [], []
            for t in range(ctx):
                j, s = divmod(t, T)
                tier = int(lay.tier_map[b, j])
                p = int(lay.block_table[b, j])
                arr = tiers[tier]
                if inp.pool_layout == 0:
                    keys.append(arr[layer, p, 0, g, s])
                    vals.append(arr[layer, p, 1, g, s])
                else:
                    keys.append(arr[p, layer, 0, g, s])
                    vals.append(arr[p, layer, 1, g, s])
            keys.append(np.array(kn))
            vals.append(np.array(vn))
            w = [math.exp(sum(q[d] * kk[d] for d in range(D)) / math.sqrt(D)) for kk in keys]
            z = sum(w)
            for d in range(D):
                out[b, h, d] = sum(w[t] * vals[t][d] for t in range(len(keys))) / z
    return out


@pytest.mark.parametrize("layout", [0, 1])
def test_attention_matches_brute_force(layout):
    cfg, inp = _tiny_inputs([0, 1, 5, 9, 16], layout=layout)
    got = _run_oracle(cfg, inp)["out"]
    ref = _brute_force(cfg, inp)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(2)
    q = rng.normal(size=64) * 4
    K = rng.normal(size=(300, 64))
    _, p = O.softmax_attention(q, K, rng.normal(size=(300, 64)))
    assert abs(p.sum() - 1.0) < 1e-12 and np.all(p >= 0)


def test_one_token_context_returns_new_value():
    cfg, inp = _tiny_inputs([0, 0, 0], Hq=8, Hkv=2)
    r = _run_oracle(cfg, inp)
    G = cfg.Hq // cfg.Hkv
    for b in range(cfg.B):
        for h in range(cfg.Hq):
            assert np.array_equal(r["out"][b, h], O.bf16_to_f64(r["v_hat"][b, h // G]))


def test_identical_keys_give_mean_of_values():
    cfg, inp = _tiny_inputs([3, 17, 33])
    D = cfg.D
    # zero the key rows of Wqkv and every cached key: all scores equal
    inp.W[cfg.Hq * D:(cfg.Hq + cfg.Hkv) * D] = 0
    inp.hbm[:, :, 0] = 0
    inp.host[:, :, 0] = 0
    r = _run_oracle(cfg, inp)
    G = cfg.Hq // cfg.Hkv
    tiers = [WL.bf16_bits(inp.hbm), WL.bf16_bits(inp.host)]
    for b, ctx in enumerate(inp.layout.seq_lens):
        for h in range(cfg.Hq):
            g = h // G
            _, Vc = O.gather_sequence(tiers, 0, 1, inp.layout.block_table[b].numpy(),
                                      inp.layout.tier_map[b].numpy(), ctx, g, cfg.T)
            allv = np.concatenate([Vc, O.bf16_to_f64(r["v_hat"][b, g])[None]])
            assert np.allclose(r["out"][b, h], allv.mean(axis=0), atol=1e-14)


def test_gqa_mapping_uses_h_div_g():
    # poison the cached values of kv head 1 only: q heads 0..G-1 must not change
    cfg, inp = _tiny_inputs([9, 20], Hq=6, Hkv=3)
    base = _run_oracle(cfg, inp)["out"]
    inp.hbm[:, :, 1, 1] = 100.0
    inp.host[:, :, 1, 1] = 100.0
    r = _run_oracle(cfg, inp)["out"]
    G = cfg.Hq // cfg.Hkv
    for h in range(cfg.Hq):
        same = np.array_equal(base[:, h], r[:, h])
        assert same == (h // G != 1)


def test_invariant_under_block_permutation_and_tier_moves():
    cfg, inp = _tiny_inputs([13, 30, 7], host_prob=0.5)
    base = _run_oracle(cfg, inp)
    lay = inp.layout
    # move every block to a fresh physical id in the other tier, copying its data
    nb_total = int((lay.block_table >= 0).sum())
    L = cfg.layers
    new_h = torch.zeros((L, nb_total) + tuple(inp.hbm.shape[2:]), dtype=torch.bfloat16)
    new_s = torch.zeros_like(new_h)
    perm = torch.randperm(nb_total, generator=torch.Generator().manual_seed(9))
    table = lay.block_table.clone()
    tmap = lay.tier_map.clone()
    n = 0
    for b in range(cfg.B):
        for j in range(lay.nblk[b]):
            old_t, old_p = int(lay.tier_map[b, j]), int(lay.block_table[b, j])
            src = (inp.hbm, inp.host)[old_t][:, old_p]
            new_t = 1 - old_t
            new_p = int(perm[n]); n += 1
            (new_h, new_s)[new_t][:, new_p] = src
            table[b, j] = new_p
            tmap[b, j] = new_t
    r = O.decode_step(WL.bf16_bits(inp.x), WL.bf16_bits(inp.W), [WL.bf16_bits(new_h), WL.bf16_bits(new_s)],
                      table.numpy(), lay.seq_lens, tmap.numpy(), cfg.Hq, cfg.Hkv, cfg.D, cfg.T,
                      cfg.theta, layer=1)
    assert np.array_equal(r["out"], base["out"])
    assert np.array_equal(r["k_hat"], base["k_hat"])


def test_subset_selection_matches_full():
    cfg, inp = _tiny_inputs([11, 40, 2])
    full = _run_oracle(cfg, inp)["out"]
    part = _run_oracle(cfg, inp, batch=[1], heads=[3])["out"]
    assert np.array_equal(part[1, 3], full[1, 3])
    assert np.isnan(part[0]).all()


def test_new_cache_contents_are_rounded_projection():
    cfg, inp = _tiny_inputs([5, 6])
    r = _run_oracle(cfg, inp)
    x = inp.x.double().numpy()
    W = inp.W.double().numpy()
    D = cfg.D
    for b in range(cfg.B):
        v = W[(cfg.Hq + cfg.Hkv) * D:] @ x[b]
        assert np.array_equal(r["v_hat"][b].reshape(-1), O.f64_to_bf16_rne(v))


# ----------------------------------------------------------------------- layout

def test_layout_permutation_round_trip_and_mapping():
    rng = np.random.default_rng(4)
    pool = rng.integers(0, 65535, size=(3, 5, 2, 2, 4, 8), dtype=np.uint16)
    pf = O.layer_first_to_page_first(pool)
    assert pf.shape == (5, 3, 2, 2, 4, 8)
    assert np.array_equal(O.page_first_to_layer_first(pf), pool)
    L, P, C = 3, 5, 2 * 2 * 4 * 8
    flat_src, flat_dst = pool.reshape(-1), pf.reshape(-1)
    for _ in range(200):
        l, p, c = rng.integers(L), rng.integers(P), rng.integers(C)
        assert flat_dst[(p * L + l) * C + c] == flat_src[(l * P + p) * C + c]


# ------------------------------------------------------------------------- GEMM

def test_gemm_entries_exact_on_integers():
    rng = np.random.default_rng(5)
    M, N, K = 9, 7, 33
    A = rng.integers(-8, 9, size=(M, K))
    B = rng.integers(-8, 9, size=(K, N))
    a_bits = O.f64_to_bf16_rne(A.astype(np.float64))
    bt_bits = O.f64_to_bf16_rne(B.T.astype(np.float64))
    rows, cols = np.array([0, 3, 8, 8]), np.array([6, 0, 2, 6])
    got = O.gemm_entries(a_bits, bt_bits, rows, cols)
    for n, (i, j) in enumerate(zip(rows, cols)):
        assert got[n] == sum(int(A[i, k]) * int(B[k, j]) for k in range(K))
    # a transposed operand would read B[j, k] instead: make sure that differs here
    assert any(got[n] != sum(int(A[i, k]) * int(B[j % K, k % N]) for k in range(K))
               for n, (i, j) in enumerate(zip(rows, cols)))


def test_gemm_entries_rational_reference():
    A, Bt = WL.uniform_bf16((4, 257), 11), WL.uniform_bf16((3, 257), 12)
    a_bits, b_bits = WL.bf16_bits(A), WL.bf16_bits(Bt)
    rows, cols = np.array([0, 3, 1]), np.array([2, 0, 1])
    got = O.gemm_entries(a_bits, b_bits, rows, cols)
    Af, Bf = A.double().numpy(), Bt.double().numpy()
    for n, (i, j) in enumerate(zip(rows, cols)):
        exact = sum(Fraction(float(Af[i, k])) * Fraction(float(Bf[j, k])) for k in range(257))
        assert abs(got[n] - float(exact)) <= 1e-14 * float(sum(abs(Fraction(float(Af[i, k])) * Fraction(float(Bf[j, k]))) for k in range(257)))


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    return vals


def test_naive_zero_copy_traffic_matches_published_figure():
    g = _golden("directkv_fig2a_gemm.txt")
    n = int(g["matrix_dim"])
    b_bytes = O.cpu_aware_host_bytes(n, n, n)
    # the "200 MB" swap buffer holds exactly one bf16 B operand: 200 MiB
    assert b_bytes == int(g["swap_buffer_MB"]) * 2 ** 20
    # 33.5 GB of B traffic = B re-read once per 64-row M tile (160 times), no reuse
    naive = O.naive_zero_copy_host_bytes(n, n, n, BM=64)
    assert naive == 160 * b_bytes
    assert abs(naive / 1e9 - g["naive_B_traffic_GB"]) < 0.1
    # other tile heights do not reproduce the figure
    for bm in (32, 128, 256):
        assert abs(O.naive_zero_copy_host_bytes(n, n, n, BM=bm) / 1e9 - g["naive_B_traffic_GB"]) > 5
    assert round(g["naive_ms"] / g["swap_ms"]) == g["slowdown"]


def test_gemm_abs_bound_exact_on_integers():
    # sum_k |A[i,k] B[k,j]| written out over integers (exact in fp64), mixed signs, so a
    # bound that keeps a sign, drops a factor or reads the wrong row/column differs
    rng = np.random.default_rng(8)
    M, N, K = 6, 5, 41
    A = rng.integers(-9, 10, size=(M, K))
    B = rng.integers(-9, 10, size=(K, N))
    a_bits = O.f64_to_bf16_rne(A.astype(np.float64))
    bt_bits = O.f64_to_bf16_rne(B.T.astype(np.float64))
    rows, cols = np.array([0, 5, 2, 2, 4]), np.array([4, 0, 3, 1, 4])
    got = O.gemm_abs_bound(a_bits, bt_bits, rows, cols)
    for n, (i, j) in enumerate(zip(rows, cols)):
        want = sum(abs(int(A[i, k]) * int(B[k, j])) for k in range(K))
        assert got[n] == want
        # the triangle inequality: the bound is never below |C_ij|
        assert got[n] >= abs(sum(int(A[i, k]) * int(B[k, j]) for k in range(K)))
    # with every product non-negative the bound is the entry itself
    Ap, Bp = np.abs(A), np.abs(B)
    gp = O.gemm_abs_bound(O.f64_to_bf16_rne(Ap.astype(np.float64)), O.f64_to_bf16_rne(Bp.T.astype(np.float64)),
                          rows, cols)
    ep = O.gemm_entries(O.f64_to_bf16_rne(Ap.astype(np.float64)), O.f64_to_bf16_rne(Bp.T.astype(np.float64)),
                        rows, cols)
    assert np.array_equal(gp, ep)
