"""fp64 CPU oracle for the zero-copy decode step, the block-layout permutation and the
zero-copy GEMM study.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link this
module: only the tests, the package smoke check and the benchmark's CPU-baseline leg use
it. It shares no code with the CUDA path (no kernels, headers, constants or helpers);
its inputs are the raw bf16 bit patterns and integer tables the seeded generators make.

What it computes, and where each step comes from:

* DirectKV changes where the key/value bytes come from (CPU-resident KV read in place by
  the attention kernel, no staging buffer) but not the arithmetic of the step; the
  summary page "长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", section 核心方法, fuses
  the QKV projection with attention and keeps the new K/V on chip. So the result the
  method must reach is plain decode attention:

    1. qkv = Wqkv . x_b, no norm, no bias; rows ordered [q heads][k heads][v heads],
       D rows per head (reading: nn.Linear row order; the pages give no layout).
    2. rotate-half RoPE on q and k at position pos = ctx_b with inv_i = theta^(-2i/D)
       (reading: the pages never name a RoPE variant).
    3. the new key/value as stored in the cache: k_hat = bf16_rne(k_rot),
       v_hat = bf16_rne(v) (the single cache write of the fused step).
    4. keys/values 0..ctx_b-1 gathered through block_table/tier_map from the two tiers
       (paged KV blocks, "KV Offload" wiki page, section Swap-out / Swap-in), then
       k_hat/v_hat appended as key ctx_b.
    5. q head h attends kv head h // G (reading: grouped-query mapping); scores
       q.k / sqrt(D); softmax with max subtraction; o_h = sum_t p_t v_t; no output
       projection.

* The block-layout permutation layer-first [L][P][2][Hkv][T][D] <-> page-first
  [P][L][2][Hkv][T][D] is Strata's layout decoupling ("「KV Cache 内存层级」系列总纲",
  §2.4 Strata). It is a pure index permutation, checked bit for bit.

* The zero-copy GEMM study (same series page, §一 / §2.1, DirectKV Fig. 2(a)):
  C = A . B with fp64 accumulation, evaluated on sampled entries; and the host-link byte
  model of a naive zero-copy GEMM, where every M-tile re-reads all of B.

Every function here is pinned by the CPU tests (brute force, closed forms and invariants);
no part is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

# ----------------------------------------------------------------------------- bf16


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact bf16 -> fp64: a bf16 value is the top half of an IEEE binary32 pattern."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (ties to even), returned as uint16 bits.

    bf16 keeps 8 significant bits (1 implicit + 7 stored) and fp32's exponent range.
    With x = m * 2^e, 0.5 <= |m| < 1, the spacing of bf16 values around x is 2^(e-8)
    for normal numbers, and 2^-133 in the subnormal range (exponent floor -126 - 7).
    Rounding x / spacing to an integer with ties-to-even and scaling back gives the
    nearest representable value; it is exactly representable in fp32, so its binary32
    pattern's top 16 bits are the bf16 pattern. Overflow beyond the largest finite bf16
    goes to infinity, as round-to-nearest requires.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    finite = np.isfinite(x)
    xf = np.where(finite, x, 0.0)
    m, e = np.frexp(xf)
    spacing_exp = np.maximum(e - 8, -133)
    scaled = np.ldexp(xf, -spacing_exp)
    r = np.ldexp(np.rint(scaled), spacing_exp)
    max_bf16 = float.fromhex("0x1.fep127")
    # halfway between max finite and the next power (2^128) rounds to infinity
    r = np.where(np.abs(r) > max_bf16, np.copysign(np.inf, xf), r)
    out[...] = np.where(finite, r, x)
    f32 = out.astype(np.float32)
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------- projection


def qkv_projection(W: np.ndarray, xb: np.ndarray) -> np.ndarray:
    """qkv[r] = sum_c W[r, c] * x[c] in fp64 (matrix-vector product, library matmul)."""
    return np.asarray(W, dtype=np.float64) @ np.asarray(xb, dtype=np.float64)


def split_qkv(qkv: np.ndarray, Hq: int, Hkv: int, D: int):
    q = qkv[: Hq * D].reshape(Hq, D)
    k = qkv[Hq * D: (Hq + Hkv) * D].reshape(Hkv, D)
    v = qkv[(Hq + Hkv) * D: (Hq + 2 * Hkv) * D].reshape(Hkv, D)
    return q, k, v


# ----------------------------------------------------------------------------- RoPE


def rope_rotate_half(vec: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotate pairs (i, i + D/2) by angle pos * theta^(-2i/D), all in fp64.

    y[i]       = x[i] cos a_i - x[i + D/2] sin a_i
    y[i + D/2] = x[i + D/2] cos a_i + x[i] sin a_i
    Works on the last axis of `vec`.
    """
    vec = np.asarray(vec, dtype=np.float64)
    D = vec.shape[-1]
    half = D // 2
    i = np.arange(half, dtype=np.float64)
    inv = np.power(float(theta), -2.0 * i / D)
    ang = float(pos) * inv
    c, s = np.cos(ang), np.sin(ang)
    a, b = vec[..., :half], vec[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


# ------------------------------------------------------------------- paged KV gather


def chunk_view(tier: np.ndarray, layout: int, layer: int, phys: np.ndarray, kv: int, g: int):
    """[n, T, D] bf16 chunks of kv head g for physical blocks `phys` of one tier.

    layout 0 = layer-first [L][P][2][Hkv][T][D]; 1 = page-first [P][L][2][Hkv][T][D].
    """
    if layout == 0:
        return tier[layer, phys, kv, g]
    return tier[phys, layer, kv, g]


def gather_sequence(tiers: Sequence[np.ndarray], layout: int, layer: int,
                    table_row: np.ndarray, tier_row: np.ndarray, ctx: int, g: int,
                    T: int) -> Tuple[np.ndarray, np.ndarray]:
    """Keys/values 0..ctx-1 of kv head g, in logical order, as fp64 [ctx, D].

    Logical block j lives in tier tier_row[j] at physical index table_row[j].
    """
    nb = (ctx + T - 1) // T
    D = tiers[0].shape[-1] if tiers[0].size else tiers[1].shape[-1]
    K = np.empty((nb, T, D), dtype=np.float64)
    V = np.empty((nb, T, D), dtype=np.float64)
    tr = np.asarray(tier_row[:nb])
    ids = np.asarray(table_row[:nb]).astype(np.int64)
    for t in (0, 1):
        sel = np.nonzero(tr == t)[0]
        if sel.size == 0:
            continue
        K[sel] = bf16_to_f64(chunk_view(tiers[t], layout, layer, ids[sel], 0, g))
        V[sel] = bf16_to_f64(chunk_view(tiers[t], layout, layer, ids[sel], 1, g))
    return K.reshape(nb * T, D)[:ctx], V.reshape(nb * T, D)[:ctx]


# ------------------------------------------------------------------------ attention


def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """One query over keys K [n, D] / values V [n, D]: softmax(K q / sqrt(D)) . V.

    Returns (output [D], probabilities [n]). Max subtraction keeps exp in range.
    """
    D = q.shape[-1]
    s = (K @ q) / math.sqrt(D)
    m = np.max(s)
    e = np.exp(s - m)
    p = e / np.sum(e)
    return p @ V, p


def decode_step(x_bits: np.ndarray, W_bits: np.ndarray, tiers: Sequence[np.ndarray],
                block_table: np.ndarray, seq_lens: Sequence[int], tier_map: np.ndarray,
                Hq: int, Hkv: int, D: int, T: int, theta: float, layer: int = 0,
                layout: int = 0, batch: Optional[Iterable[int]] = None,
                heads: Optional[Iterable[int]] = None) -> Dict[str, np.ndarray]:
    """The full decode step for every (or the selected) sequence and q head.

    Returns fp64 `out` [B, Hq, D] (NaN where not computed), the expected new cache
    contents `k_hat`/`v_hat` as bf16 bits [B, Hkv, D], and `q_rot` fp64 [B, Hq, D].
    """
    B = x_bits.shape[0]
    G = Hq // Hkv
    bsel = list(range(B)) if batch is None else list(batch)
    hsel = list(range(Hq)) if heads is None else list(heads)
    W = bf16_to_f64(W_bits)
    out = np.full((B, Hq, D), np.nan)
    q_rot_all = np.full((B, Hq, D), np.nan)
    k_hat = np.zeros((B, Hkv, D), dtype=np.uint16)
    v_hat = np.zeros((B, Hkv, D), dtype=np.uint16)
    for b in bsel:
        ctx = int(seq_lens[b])
        xb = bf16_to_f64(x_bits[b])
        q, k, v = split_qkv(qkv_projection(W, xb), Hq, Hkv, D)
        q_rot = rope_rotate_half(q, ctx, theta)
        k_rot = rope_rotate_half(k, ctx, theta)
        k_hat[b] = f64_to_bf16_rne(k_rot)
        v_hat[b] = f64_to_bf16_rne(v)
        q_rot_all[b] = q_rot
        groups = sorted({h // G for h in hsel})
        for g in groups:
            Kc, Vc = gather_sequence(tiers, layout, layer, block_table[b], tier_map[b], ctx, g, T)
            Kf = np.concatenate([Kc, bf16_to_f64(k_hat[b, g])[None]], axis=0)
            Vf = np.concatenate([Vc, bf16_to_f64(v_hat[b, g])[None]], axis=0)
            for h in hsel:
                if h // G != g:
                    continue
                out[b, h], _ = softmax_attention(q_rot[h], Kf, Vf)
    return {"out": out, "k_hat": k_hat, "v_hat": v_hat, "q_rot": q_rot_all}


# ------------------------------------------------------------------- layout permute


def layer_first_to_page_first(pool: np.ndarray) -> np.ndarray:
    """[L][P][2][Hkv][T][D] -> [P][L][2][Hkv][T][D]: element (l,p,...) moves to (p,l,...)."""
    L, P = pool.shape[0], pool.shape[1]
    out = np.empty((P, L) + pool.shape[2:], dtype=pool.dtype)
    for l in range(L):
        out[:, l] = pool[l]
    return out


def page_first_to_layer_first(pool: np.ndarray) -> np.ndarray:
    P, L = pool.shape[0], pool.shape[1]
    out = np.empty((L, P) + pool.shape[2:], dtype=pool.dtype)
    for p in range(P):
        out[:, p] = pool[p]
    return out


# ------------------------------------------------------------------------- GEMM study


def gemm_entries(A_bits: np.ndarray, Bt_bits: np.ndarray, rows: np.ndarray,
                 cols: np.ndarray) -> np.ndarray:
    """C[i, j] = sum_k A[i, k] * B[k, j] in fp64 for the sampled (i, j) pairs.

    B is held column-major: Bt[j, k] = B[k, j].
    """
    out = np.empty(len(rows), dtype=np.float64)
    for n, (i, j) in enumerate(zip(rows, cols)):
        out[n] = float(np.dot(bf16_to_f64(A_bits[int(i)]), bf16_to_f64(Bt_bits[int(j)])))
    return out


def gemm_abs_bound(A_bits: np.ndarray, Bt_bits: np.ndarray, rows, cols) -> np.ndarray:
    """sum_k |A[i, k] B[k, j]| for each sampled pair (scale for the fp32 error bound)."""
    out = np.empty(len(rows), dtype=np.float64)
    for n, (i, j) in enumerate(zip(rows, cols)):
        out[n] = float(np.dot(np.abs(bf16_to_f64(A_bits[int(i)])),
                              np.abs(bf16_to_f64(Bt_bits[int(j)]))))
    return out


def naive_zero_copy_host_bytes(M: int, N: int, K: int, BM: int, elem_bytes: int = 2) -> int:
    """Host-link bytes of a zero-copy GEMM whose every M-tile re-reads the whole of B
    from host memory with no cache reuse: ceil(M/BM) * |B|."""
    return ((M + BM - 1) // BM) * K * N * elem_bytes


def cpu_aware_host_bytes(M: int, N: int, K: int, elem_bytes: int = 2) -> int:
    """Host-link bytes when each B tile crosses the link exactly once: |B|."""
    return K * N * elem_bytes
