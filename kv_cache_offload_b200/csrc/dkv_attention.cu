// Split-K GQA decode attention over a two-tier paged KV cache, and the split combine.
//
// DirectKV ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", 核心方法) lets the attention
// kernel read CPU-resident KV in place and hides the slow fetches behind compute with a
// warp-level producer/consumer pipeline. This kernel is that pipeline on sm_100a:
//
//  * one CTA per (split s, kv head g, sequence b) walks a contiguous range of logical
//    blocks; the KV of kv head g is read once for all G = Hq/Hkv query heads;
//  * one producer warp fills an NST-stage shared-memory ring, one stage per block
//    (K rows [T][D] then V rows [T][D]):
//      - HBM-tier block: bulk copies (TMA engine) of the chunks, issued by the lanes;
//      - host-tier block: all 32 lanes issue 16-byte cp.async loads straight from the
//        mapped pinned host memory (coalesced 512-byte warp requests), no staging buffer;
//    both complete on the stage's mbarrier, so the consumers see one kind of stage;
//  * SL consumer "slots" (warps; three in the default shape, four otherwise) take blocks
//    round robin, each keeping its own online-softmax state (running max m, running sum
//    l, accumulator) in registers; the slots merge at the end and the CTA writes one
//    partial state (m, l, acc[D]) per q head to the workspace; the last split CTA of a
//    (sequence, kv head) merges the splits.
//
// Scores are in the log2 domain: q arrives pre-scaled by log2(e)/sqrt(D), so p = 2^(s - m).
// Two consumer implementations:
//  * CUDA cores (the default = variant 5: three slots, a 6-stage ring, four CTAs per SM;
//    variant 1: four slots, an 8-stage ring, three CTAs per SM; at G = 8 a slot is two
//    warps of four heads each): packed fp32x2 FMAs. A decode query group is G <= 8 rows, G flops per KV byte: an HBM-bound
//    product, not a dense contraction, and the tensor cores are kept for the projection.
//  * tensor cores (opt-in, variants 6 and 7): per block, S = Q.K^T and O^T += V^T.P^T as
//    m16n8k16 bf16 mma.sync with fp32 accumulation. The G query rows of a kv head are padded to the
//    16-row tile, and the spare rows carry the bf16 low parts: q = q_hi + q_lo (rows
//    0..G-1 and 8..8+G-1) and p = p_hi + p_lo (separate columns), so the products keep
//    about 16 significant bits of the fp32 q and p. A decode step is HBM-bound at G
//    flops per KV byte; on the tensor cores ~800 issued instructions per block become
//    ~100, and this consumer measured faster on B200. But padding the query rows to the
//    tensor-core tile is exactly the reshaping of an HBM-bound product into a GEMM that
//    this design otherwise avoids, so it stays opt-in. Its stages use the TMA 128-byte
//    swizzle, so ldmatrix is conflict-free.
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include <utility>

#include "dkv_internal.h"
#include "dkv_umma.cuh"

namespace dkv {

constexpr int kSlots = 4;
constexpr int kT = 16;

template <int D, int HPW, int WPB, int NST, int SL = kSlots>
struct AttnCfg {
  static constexpr int G = HPW * WPB;
  static constexpr int NCW = SL * WPB;  // consumer warps
  static constexpr int THREADS = (NCW + 1) * 32;
  static constexpr int STAGE_ELEMS = 2 * kT * D;
  static constexpr int STAGE_BYTES = STAGE_ELEMS * 2;
  static constexpr int DPL = D / 32;   // value dims per lane in P.V
  static constexpr int QCH = D / 64;   // 16-byte key chunks per lane per token in Q.K
  static constexpr int NV = HPW * 4;   // partial scores per lane (heads x 4 tokens)
  static constexpr int LOGH = HPW == 8 ? 3 : (HPW == 4 ? 2 : (HPW == 2 ? 1 : 0));
  static constexpr int LOWMASK = (1 << (3 - LOGH)) - 1;  // dg bits shared by one head
  static constexpr int NR = NV >= 8 ? NV / 8 : 1;        // scores per lane after reduction
  static constexpr int OFF_P = NST * STAGE_BYTES;
  static constexpr int OFF_ALPHA = OFF_P + NCW * kT * HPW * 8;
  static constexpr int OFF_FLAGS = OFF_ALPHA + NCW * HPW * 4;
  static constexpr int OFF_BARS = (OFF_FLAGS + NST * 4 + 7) / 8 * 8;
  static constexpr int SMEM = OFF_BARS + 2 * NST * 8;
  static constexpr int MERGE_BYTES = NCW * HPW * D * 4 + NCW * HPW * 8;
  static_assert(MERGE_BYTES <= NST * STAGE_BYTES, "merge area must fit in the stage ring");
  // Block i uses stage i % NST and consumer slot i % SL. Stage loads complete out of
  // order, and a parity wait is only sound if the stage's barrier is at most one phase
  // behind the waiter; that holds when every stage belongs to a single slot.
  static_assert(NST % SL == 0, "each stage must belong to exactly one consumer slot");
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One warp merges the n partial states of one (sequence, q head) -- entries base,
// base + stride, ... -- with the new token's term and writes the D bf16 outputs:
// M = max(s_new, m_s), L = 2^(s_new-M) + sum l_s 2^(m_s-M),
// o_d = (v_d 2^(s_new-M) + sum acc_s[d] 2^(m_s-M)) / L.
// Lane s (mod 32) holds the weight of entry s; L is summed over a fixed shuffle tree and
// o over the entries in index order, so the result does not depend on which CTA merges
// and the fused and the standalone combine produce identical bits. The accumulator loads
// of four entries for all of a lane's D/32 dims are in flight together.
template <int D, int UM, int UA>
__device__ __forceinline__ void combine_head_warp(const float2* __restrict__ ml, const float* __restrict__ acc,
                                                  int n, int64_t base, int stride, float sn,
                                                  const float* __restrict__ vn, uint16_t* __restrict__ out,
                                                  int lane) {
  constexpr int DL = D / 32;
  // UM: (m, l) loads a lane has in flight together; UA: splits whose accumulator loads are
  // in flight together (the caller's register budget sets both). The partial states sit in
  // L2 (written by the other split CTAs moments ago): every round of loads costs a full L2
  // round trip, so the loads of a round are issued before any is used. The arithmetic
  // order is fixed (lane l takes splits l, l + 32, ... in increasing order, then a
  // butterfly; the accumulators in split order), so the fused and the standalone combine
  // give identical bits.
  float M = sn;
  if constexpr (UM == 1) {  // one load at a time (the tightest register budget)
    for (int s = lane; s < n; s += 32) M = fmaxf(M, __ldcg(ml + base + (int64_t)s * stride).x);
  } else {
    for (int s0 = lane; s0 < n; s0 += 32 * UM) {
      float x[UM];
#pragma unroll
      for (int u = 0; u < UM; ++u) {
        const int s = s0 + 32 * u;
        x[u] = s < n ? __ldcg(ml + base + (int64_t)s * stride).x : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < UM; ++u) M = fmaxf(M, x[u]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float wn = exp2f(sn - M);  // M >= s_new is finite; an empty state (m = -inf) weighs 0
  float Lp = 0.f;
  if constexpr (UM == 1) {
    for (int s = lane; s < n; s += 32) {
      const float2 m = __ldcg(ml + base + (int64_t)s * stride);
      Lp = fmaf(m.y, exp2f(m.x - M), Lp);
    }
  } else {
    for (int s0 = lane; s0 < n; s0 += 32 * UM) {
      float2 x[UM];
#pragma unroll
      for (int u = 0; u < UM; ++u) {
        const int s = s0 + 32 * u;
        x[u] = s < n ? __ldcg(ml + base + (int64_t)s * stride) : make_float2(-INFINITY, 0.f);
      }
#pragma unroll
      for (int u = 0; u < UM; ++u)
        if (s0 + 32 * u < n) Lp = fmaf(x[u].y, exp2f(x[u].x - M), Lp);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Lp += __shfl_xor_sync(0xffffffffu, Lp, o);
  const float L = wn + Lp;
  float A[DL];
#pragma unroll
  for (int k = 0; k < DL; ++k) A[k] = wn * vn[lane + 32 * k];
  for (int s0 = 0; s0 < n; s0 += 32) {
    const int cnt = min(32, n - s0);
    float wmine = 0.f;
    if (lane < cnt) wmine = exp2f(__ldcg(ml + base + (int64_t)(s0 + lane) * stride).x - M);
    int t = 0;
    if constexpr (UA > 4) {
      for (; t + UA <= cnt; t += UA) {
        float a[UA][DL];
#pragma unroll
        for (int u = 0; u < UA; ++u)
#pragma unroll
          for (int k = 0; k < DL; ++k)
            a[u][k] = __ldcg(acc + (base + (int64_t)(s0 + t + u) * stride) * D + lane + 32 * k);
#pragma unroll
        for (int u = 0; u < UA; ++u) {
          const float w = __shfl_sync(0xffffffffu, wmine, t + u);
#pragma unroll
          for (int k = 0; k < DL; ++k) A[k] = fmaf(a[u][k], w, A[k]);
        }
      }
    }
    for (; t + 4 <= cnt; t += 4) {
      float a[4][DL];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int k = 0; k < DL; ++k)
          a[u][k] = __ldcg(acc + (base + (int64_t)(s0 + t + u) * stride) * D + lane + 32 * k);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = __shfl_sync(0xffffffffu, wmine, t + u);
#pragma unroll
        for (int k = 0; k < DL; ++k) A[k] = fmaf(a[u][k], w, A[k]);
      }
    }
    for (; t < cnt; ++t) {
      const float w = __shfl_sync(0xffffffffu, wmine, t);
#pragma unroll
      for (int k = 0; k < DL; ++k)
        A[k] = fmaf(__ldcg(acc + (base + (int64_t)(s0 + t) * stride) * D + lane + 32 * k), w, A[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < DL; ++k) out[lane + 32 * k] = f32_to_bf16_bits(A[k] / L);
}

// The new token's score s_new = q . k_hat (log2 domain: q is pre-scaled), computed by one
// full warp in a fixed order (lane l sums dims l, l+32, ...; then a butterfly), so the
// fused and the standalone combine produce identical bits.
__device__ __forceinline__ float new_token_score(const float* __restrict__ q, const float* __restrict__ k, int D,
                                                 int lane) {
  float s = 0.f;
  for (int d = lane; d < D; d += 32) s = fmaf(q[d], k[d], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// One level of a warp reduce-scatter: lanes with `up` keep the upper half of the N live
// values, their partner (lane ^ mask) the lower half; each adds the partner's copy.
template <int N>
__device__ __forceinline__ void rs_level(float* v, bool up, int mask) {
  if constexpr (N >= 2) {
#pragma unroll
    for (int x = 0; x < N / 2; ++x) {
      const float send = up ? v[x] : v[x + N / 2];
      const float keep = up ? v[x + N / 2] : v[x];
      v[x] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
    }
  } else {
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
  }
}

// ------------------------------------------------------------- slot merge + combine
// The consumer slots have left their state in shared memory: acc [NCW*HPW][D] fp32 at the
// base, then (m, l) per (warp, head). Merge the SL slots per q head, write this
// split's partial state, and, when the launch fuses the combine, let the last split CTA of
// (b, g) merge all S partial states in split order with the new token's term.
template <int D, int HPW, int WPB, int SL = kSlots>
__device__ __forceinline__ void attn_merge_combine(const AttnParams& p, uint8_t* smem, int b, int g, int s,
                                                   int warp, int lane) {
  constexpr int G = HPW * WPB;
  constexpr int NCW = SL * WPB;
  const PoolView& pool = p.pool;
  const float* macc = reinterpret_cast<const float*>(smem);
  const float2* mml = reinterpret_cast<const float2*>(smem + NCW * HPW * D * 4);
  for (int o = threadIdx.x; o < G * D; o += NCW * 32) {
    const int hh = o / D, d = o % D;
    const int wq = hh / HPW, h = hh % HPW;
    float M = -INFINITY;
#pragma unroll
    for (int sl = 0; sl < SL; ++sl) M = fmaxf(M, mml[(sl * WPB + wq) * HPW + h].x);
    float A = 0.f, Ls = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int sl = 0; sl < SL; ++sl) {
        const float2 ml = mml[(sl * WPB + wq) * HPW + h];
        const float w = fast_exp2(ml.x - M);
        A = fmaf(macc[((sl * WPB + wq) * HPW + h) * D + d], w, A);
        Ls = fmaf(ml.y, w, Ls);
      }
    }
    const int64_t base = ((int64_t)b * p.Hq + g * G + hh) * p.S + s;
    if (!DKV_DEBUG_RANGE(pool.status, base, base + 1, (int64_t)gridDim.z * p.Hq * p.S)) continue;
    p.part_acc[base * D + d] = A;
    if (d == 0) p.part_ml[base] = make_float2(M, Ls);
  }

  // fused combine: the last split CTA of (b, g) to finish merges all S partial states
  // (in split order, so the result does not depend on which CTA finishes last)
  if (p.out) {
    __shared__ int s_last;
    __threadfence();
    named_bar_sync(1, NCW * 32);
    if (threadIdx.x == 0) s_last = atomicAdd(p.cnt + (int64_t)b * pool.Hkv + g, 1) == p.S - 1;
    named_bar_sync(1, NCW * 32);
    if (s_last) {  // one warp per q head of the group
      __threadfence();
      const float* kn = p.knew + ((int64_t)b * pool.Hkv + g) * D;
      for (int hh = warp; hh < G; hh += NCW) {
        const int hg = g * G + hh;
        if (!DKV_DEBUG_RANGE(pool.status, (int64_t)b * p.Hq + hg, (int64_t)b * p.Hq + hg + 1,
                             (int64_t)gridDim.z * p.Hq))
          continue;
        const float sn = new_token_score(p.qs + ((int64_t)b * p.Hq + hg) * D, kn, D, lane);
        // the three-CTAs-per-SM G = 8 shape (two slots of two warps) runs at its full
        // register budget: its merge keeps one (m, l) load and four splits in flight, the
        // other shapes eight of each
        constexpr bool tight = HPW * WPB == 8 && WPB == 2 && SL == 2;
        combine_head_warp<D, tight ? 1 : 8, tight ? 4 : 8>(p.part_ml, p.part_acc, p.S, ((int64_t)b * p.Hq + hg) * p.S, 1, sn,
                             p.vnew + ((int64_t)b * pool.Hkv + g) * D, p.out + ((int64_t)b * p.Hq + hg) * D, lane);
      }
      if (threadIdx.x == 0) p.cnt[(int64_t)b * pool.Hkv + g] = 0;
    }
  }
}

// ------------------------------------------------------------------- producer warp
// Fills the NST-stage ring for blocks j0..j1-1 of (b, g). A stage holds the K rows then the
// V rows of one block, in one of two layouts:
//   packed (SW = false): row r of K at byte r*2D, of V at (T + r)*2D; HBM blocks arrive by
//     two bulk copies (one per chunk);
//   swizzled (SW = true): per chunk, D/64 boxes of [T rows][128 bytes] (dims 64h..64h+63),
//     the 16-byte piece c of row r stored at piece c ^ (r mod 8) (the TMA 128-byte
//     swizzle; the stage is 1024-byte aligned); HBM blocks arrive by 2*D/64 TMA tensor
//     copies through `tmap` (the HBM tier as [rows][D]).
// Host-tier blocks (and HBM blocks when bit 0 of p.lsu_hbm is set) arrive by 16-byte
// cp.async from all 32 lanes into the same layout; with bit 1 set, host blocks of the packed
// layout arrive by bulk copies from the mapped host memory instead. Table entries are fetched 32 blocks at a time (lane l holds
// block base + l) and broadcast by shuffle, so no dependent global load sits on the
// per-block path.
template <int D, int NST, bool SW>
__device__ __forceinline__ void attn_produce(const AttnParams& p, const CUtensorMap* tmap, uint8_t* stages,
                                             int* flags, uint64_t* full, uint64_t* empty, int b, int g, int ctx,
                                             int j0, int j1, int lane) {
  constexpr int DATA_BYTES = 2 * kT * D * 2;
  constexpr int CHUNK = kT * D * 2;  // bytes of the K (or V) rows of one block
  const PoolView& pool = p.pool;
  const int n_local = j1 - j0;
  const int64_t rowbase = (int64_t)b * p.max_blocks;
  // chunk address of (phys, K) = kbase[tier] + phys * pstride; the V chunk is kvoff further
  // (both layouts are linear in the physical id)
  const int64_t TD = (int64_t)kT * D;
  const int64_t pstride = (pool.layout == DKV_LAYOUT_LAYER_FIRST ? 2LL : 2LL * pool.L) * pool.Hkv * TD;
  const int64_t kvoff = (int64_t)pool.Hkv * TD;
  const uint16_t* kbase0 = pool.tier[0] + chunk_offset(pool, 0, p.layer, 0, 0, g);
  const uint16_t* kbase1 = pool.tier[1] + chunk_offset(pool, 1, p.layer, 0, 0, g);
  int pf_tier = 0, pf_phys = 0;
  int issued = 0;
  const uint64_t kv_policy = l2_policy_evict_first();  // cached KV is read once per step
  // test hook (bounded-wait test): the first CTA never loads nor signals its first block
  const int withheld = (p.withhold && blockIdx.x == 0 && g == 0 && b == 0) ? 0 : -1;
  for (int i = 0; i < n_local; ++i) {
    if ((i & 31) == 0) {
      const int j = j0 + i + lane;
      if (j < j1) {
        pf_tier = __ldcg(p.tier_map + rowbase + j);  // L2: tables may be rewritten between launches
        pf_phys = __ldcg(p.table + rowbase + j);
      }
    }
    const int st = i % NST;
    const int k = i / NST;
    if (k > 0 && !mbar_wait_bounded(&empty[st], (k - 1) & 1, pool.status, p.wait_ns)) break;
    if (i == withheld) {
      issued = i + 1;
      continue;
    }
    const int j = j0 + i;
    const int tier = __shfl_sync(0xffffffffu, pf_tier, i & 31);
    const int64_t phys = __shfl_sync(0xffffffffu, pf_phys, i & 31);
    const int ntok = min(kT, ctx - j * kT);
    bool valid = true;
    if (tier > 1) {
      valid = false;
      if (lane == 0) flag_error(pool.status, kErrBadTier);
    } else if (phys < 0 || phys >= tier_blocks(pool, tier)) {
      valid = false;
      if (lane == 0) flag_error(pool.status, kErrBadBlock);
    }
    uint8_t* dst = stages + st * DATA_BYTES;
    const uint16_t* kp = (tier ? kbase1 : kbase0) + phys * pstride;
    const uint16_t* vp = kp + kvoff;
    if (valid) {  // the K and V chunks lie inside the tier (DKV_DEBUG build)
      const int64_t ko = kp - tier_base(pool, tier), vo = vp - tier_base(pool, tier);
      valid = DKV_DEBUG_RANGE(pool.status, ko, ko + TD, tier_elems(pool, tier)) &&
              DKV_DEBUG_RANGE(pool.status, vo, vo + TD, tier_elems(pool, tier));
    }
    if (lane == 0) flags[st] = valid ? ntok : -1;
    if (!valid) {
      mbar_arrive(&full[st]);
      if (lane == 0) mbar_arrive(&full[st]);
      issued = i + 1;
      continue;
    }
    // bulk copies (TMA engine) for HBM blocks, and for host blocks when asked (the swizzled
    // stage layout takes HBM tensor-map copies only)
    if ((tier == DKV_TIER_HBM && !(p.lsu_hbm & 1)) || (!SW && tier == DKV_TIER_HOST && (p.lsu_hbm & 2))) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[st], DATA_BYTES);
        mbar_arrive(&full[st]);
        if constexpr (SW) {
          const int row = (int)((kp - pool.tier[0]) / D);  // row of the [rows][D] tier view
#pragma unroll
          for (int kv = 0; kv < 2; ++kv)
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_2d(dst + kv * CHUNK + h * kT * 128, tmap, 64 * h, row + kv * (int)(kvoff / D), &full[st]);
        } else {
          bulk_g2s_hint(dst, kp, CHUNK, &full[st], kv_policy);
          bulk_g2s_hint(dst + CHUNK, vp, CHUNK, &full[st], kv_policy);
        }
      } else {
        mbar_arrive(&full[st]);
      }
    } else {
      constexpr int RP = 2 * D / 16;       // 16-byte pieces per row
      constexpr int PIECES = 2 * kT * RP;  // per stage
#pragma unroll
      for (int c = 0; c < PIECES / 32; ++c) {
        const int idx = c * 32 + lane;
        const int kv = idx / (kT * RP), r = (idx / RP) % kT, q = idx % RP;
        const int off = SW ? kv * CHUNK + (q >> 3) * kT * 128 + r * 128 + (((q & 7) ^ (r & 7)) << 4)
                           : kv * CHUNK + r * 2 * D + q * 16;
        cp_async16(dst + off, (kv ? vp : kp) + r * D + q * 8);
      }
      cp_async_arrive_noinc(&full[st]);
      if (lane == 0) mbar_arrive(&full[st]);
    }
    issued = i + 1;
  }
  cp_async_wait_all();
  // Never leave with a bulk copy still writing this CTA's shared memory: the last NST
  // issued loads are the only ones that can be in flight; their stage barrier is at the
  // load's phase or past it, so the parity wait is exact (bounded, 100 ms).
  for (int j = issued > NST ? issued - NST : 0; j < issued; ++j)
    if (j != withheld)
      mbar_wait_bounded(&full[j % NST], (j / NST) & 1, pool.status, p.wait_ns < 100000000ull ? p.wait_ns : 100000000ull);
}

// Longest sequences first. CTAs start in grid order, so the z index of the grid is mapped
// to sequences by decreasing cached length (ties by index): the CTAs of the longest
// sequences take the first slots and the short ones fill in behind them, so a ragged batch
// finishes together (a uniform batch keeps its order). Warp 0 ranks the B <= 32 lengths.
__device__ __forceinline__ int longest_first_sequence(const AttnParams& p, int* s_b, int warp, int lane) {
  if (warp == 0) {
    const int nB = (int)gridDim.z;
    const int len = lane < nB ? __ldcg(p.seq_lens + lane) : INT32_MIN;
    int rank = 0;
    for (int j = 0; j < nB; ++j) {
      const int lj = __shfl_sync(0xffffffffu, len, j);
      rank += (lj > len) || (lj == len && j < lane);
    }
    const unsigned m = __ballot_sync(0xffffffffu, lane < nB && rank == (int)blockIdx.z);
    if (lane == 0) *s_b = m ? __ffs(m) - 1 : (int)blockIdx.z;
  }
  __syncthreads();
  return *s_b;
}

template <int D, int HPW, int WPB, int NST, int MINB, int SL>
__global__ void __launch_bounds__(AttnCfg<D, HPW, WPB, NST, SL>::THREADS, MINB)
    attn_splitk_kernel(const AttnParams p) {
  using C = AttnCfg<D, HPW, WPB, NST, SL>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* stages = reinterpret_cast<uint16_t*>(smem);
  float2* pbuf = reinterpret_cast<float2*>(smem + C::OFF_P);
  float* alph = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  int* flags = reinterpret_cast<int*>(smem + C::OFF_FLAGS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  uint64_t* empty = full + NST;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_b;
  const int s = blockIdx.x, g = blockIdx.y, b = longest_first_sequence(p, &s_b, warp, lane);
  const PoolView& pool = p.pool;
  // Behind this step's projection (p.early_kv) only the consumers wait for it, before q;
  // the producer streams the cached blocks at once (see attn_mma_kernel for why that is
  // safe). Behind anything else every thread waits first.
  if (!p.early_kv) griddep_wait();
  if (p.signal_next && threadIdx.x == 0) griddep_launch_dependents();

  // cached tokens of this sequence, clamped to what the table can hold
  int ctx = __ldcg(p.seq_lens + b);
  if (ctx < 0 || ctx / kT + 1 > p.max_blocks) {
    if (threadIdx.x == 0 && s == 0 && g == 0) flag_error(pool.status, kErrCtxTooLong);
    ctx = ctx < 0 ? 0 : min(ctx, p.max_blocks * kT);
  }
  const int nb = (ctx + kT - 1) / kT;
  const int j0 = (int)((int64_t)nb * s / p.S);
  const int j1 = (int)((int64_t)nb * (s + 1) / p.S);
  const int n_local = j1 - j0;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 33);   // 32 producer lanes + 1 flag publish
      mbar_init(&empty[i], WPB); // lane 0 of each warp of the consuming slot
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == C::NCW) {
    attn_produce<D, NST, false>(p, nullptr, smem, flags, full, empty, b, g, ctx, j0, j1, lane);
    return;  // consumers below sync only among themselves (named barrier 1)
  }

  // -------------------------------------------------------------------- consumers
  const int slot = warp / WPB, hq = warp % WPB;
  const int tg = lane >> 3, dg = lane & 7;
  griddep_wait();  // q, k_hat, v_hat and the counters are the projection's
  const int hbase = g * C::G + hq * HPW;  // first global q head of this warp

  // q of this lane's key dims in registers, as (even, odd) dim pairs for the packed
  // fp32x2 FMA
  float2 q2[HPW][C::QCH][4];
#pragma unroll
  for (int h = 0; h < HPW; ++h)
#pragma unroll
    for (int hh = 0; hh < C::QCH; ++hh) {
      const float4* src = reinterpret_cast<const float4*>(
          p.qs + ((int64_t)b * p.Hq + hbase + h) * D + (dg + 8 * hh) * 8);
      const float4 a = src[0], c = src[1];
      q2[h][hh][0] = make_float2(a.x, a.y);
      q2[h][hh][1] = make_float2(a.z, a.w);
      q2[h][hh][2] = make_float2(c.x, c.y);
      q2[h][hh][3] = make_float2(c.z, c.w);
    }

  constexpr int NP = C::DPL / 2;  // value-dim pairs per lane
  float2 acc2[HPW][NP];
#pragma unroll
  for (int h = 0; h < HPW; ++h)
#pragma unroll
    for (int e = 0; e < NP; ++e) acc2[h][e] = make_float2(0.f, 0.f);
  float m_run = -INFINITY, l_run = 0.f;  // state of head h_lane (lane-group uniform m)
  const int h_lane = dg >> (3 - C::LOGH);
  const bool head_leader = tg == 0 && (dg & C::LOWMASK) == 0;
  float2* pb = pbuf + warp * kT * HPW;   // (p, p) per (token, head)
  float* al = alph + warp * HPW;

  for (int i = slot; i < n_local; i += SL) {
    const int st = i % NST;
    if (!mbar_wait_bounded(&full[st], (i / NST) & 1, pool.status, p.wait_ns)) break;
    const int ntok = flags[st];
    if (ntok > 0) {
      const uint16_t* Ks = stages + st * C::STAGE_ELEMS;
      const uint16_t* Vs = Ks + kT * D;
      // ---- partial scores: lane (tg, dg) covers tokens tg + 4 i4 and 16-byte key
      // chunks dg + 8 hh (eight lanes read one 128-byte row segment: no bank conflicts);
      // even and odd dims accumulate in the two halves of a packed pair
      float2 v2[C::NV];
#pragma unroll
      for (int x = 0; x < C::NV; ++x) v2[x] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const int t = tg + 4 * i4;
#pragma unroll
        for (int hh = 0; hh < C::QCH; ++hh) {
          const uint4 w = *reinterpret_cast<const uint4*>(Ks + t * D + (dg + 8 * hh) * 8);
          const float2 k0 = make_float2(bf16lo(w.x), bf16hi(w.x));
          const float2 k1 = make_float2(bf16lo(w.y), bf16hi(w.y));
          const float2 k2 = make_float2(bf16lo(w.z), bf16hi(w.z));
          const float2 k3 = make_float2(bf16lo(w.w), bf16hi(w.w));
#pragma unroll
          for (int h = 0; h < HPW; ++h) {
            float2 a = v2[h * 4 + i4];
            a = __ffma2_rn(q2[h][hh][0], k0, a);
            a = __ffma2_rn(q2[h][hh][1], k1, a);
            a = __ffma2_rn(q2[h][hh][2], k2, a);
            a = __ffma2_rn(q2[h][hh][3], k3, a);
            v2[h * 4 + i4] = a;
          }
        }
      }
      float v[C::NV];
#pragma unroll
      for (int x = 0; x < C::NV; ++x) v[x] = v2[x].x + v2[x].y;
      // ---- reduce-scatter over the 8 dg lanes (masks 4, 2, 1): value index h*4+i4
      rs_level<C::NV>(v, (dg & 4) != 0, 4);
      rs_level<(C::NV >= 2 ? C::NV / 2 : 1)>(v, (dg & 2) != 0, 2);
      rs_level<(C::NV >= 4 ? C::NV / 4 : 1)>(v, (dg & 1) != 0, 1);
      // lane now holds NR full scores of head h_lane
      float sv[C::NR];
      int tk[C::NR];
      float bmax = -INFINITY;
#pragma unroll
      for (int r = 0; r < C::NR; ++r) {
        const int idx = C::NV >= 8 ? dg * C::NR + r : (dg >> 1);
        tk[r] = tg + 4 * (idx & 3);
        sv[r] = tk[r] < ntok ? v[r] : -INFINITY;
        bmax = fmaxf(bmax, sv[r]);
      }
#pragma unroll
      for (int mask = 1; mask <= C::LOWMASK; mask <<= 1)
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, mask));
      bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 8));
      bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 16));
      const float m_new = fmaxf(m_run, bmax);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = fast_exp2(m_run - m_use);
      float psum = 0.f;
#pragma unroll
      for (int r = 0; r < C::NR; ++r) {
        const float pr = fast_exp2(sv[r] - m_use);
        if (C::NV >= 8 || (dg & 1) == 0) {
          pb[tk[r] * HPW + h_lane] = make_float2(pr, pr);
          psum += pr;
        }
      }
      l_run = l_run * alpha + psum;
      m_run = m_new;
      if (head_leader) al[h_lane] = alpha;
      __syncwarp();
      // ---- P.V: lane owns value dims [lane*DPL, lane*DPL + DPL) as packed pairs
if (__any_sync(0xffffffffu, alpha != 1.f))  // lazy rescale: multiplying by 1 is exact
#pragma unroll
      for (int h = 0; h < HPW; ++h) {
        const float a = al[h];
        const float2 a2 = make_float2(a, a);
#pragma unroll
        for (int e = 0; e < NP; ++e) acc2[h][e] = __fmul2_rn(acc2[h][e], a2);
      }
      const int d0 = lane * C::DPL;
      auto pv_token = [&](int t) {
        float2 vf[NP];
        if constexpr (NP == 2) {
          const uint2 w = *reinterpret_cast<const uint2*>(Vs + t * D + d0);
          vf[0] = make_float2(bf16lo(w.x), bf16hi(w.x));
          vf[1] = make_float2(bf16lo(w.y), bf16hi(w.y));
        } else {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(Vs + t * D + d0);
          vf[0] = make_float2(bf16lo(w), bf16hi(w));
        }
        float2 pp[HPW];
        if constexpr (HPW >= 2) {
#pragma unroll
          for (int h2 = 0; h2 < HPW; h2 += 2) {
            const float4 q4 = *reinterpret_cast<const float4*>(pb + t * HPW + h2);
            pp[h2] = make_float2(q4.x, q4.y);
            pp[h2 + 1] = make_float2(q4.z, q4.w);
          }
        } else {
          pp[0] = pb[t];
        }
#pragma unroll
        for (int h = 0; h < HPW; ++h)
#pragma unroll
          for (int e = 0; e < NP; ++e) acc2[h][e] = __ffma2_rn(pp[h], vf[e], acc2[h][e]);
      };
      if (ntok == kT) {  // full block: no per-token tests
#pragma unroll
        for (int t = 0; t < kT; ++t) pv_token(t);
      } else {
#pragma unroll
        for (int t = 0; t < kT; ++t)
          if (t < ntok) pv_token(t);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---- per-warp totals of l, then merge the SL slots through shared memory
  float l_tot = l_run;
#pragma unroll
  for (int mask = 1; mask <= C::LOWMASK; mask <<= 1) l_tot += __shfl_xor_sync(0xffffffffu, l_tot, mask);
  l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 8);
  l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 16);

  named_bar_sync(1, C::NCW * 32);  // every slot is done reading the stage ring
  float* macc = reinterpret_cast<float*>(smem);
  float2* mml = reinterpret_cast<float2*>(smem + C::NCW * HPW * D * 4);
#pragma unroll
  for (int h = 0; h < HPW; ++h)
#pragma unroll
    for (int e = 0; e < NP; ++e)
      *reinterpret_cast<float2*>(macc + (warp * HPW + h) * D + lane * C::DPL + 2 * e) = acc2[h][e];
  if (head_leader) mml[warp * HPW + h_lane] = make_float2(m_run, l_tot);
  named_bar_sync(1, C::NCW * 32);

  attn_merge_combine<D, HPW, WPB, SL>(p, smem, b, g, s, warp, lane);
}

// ------------------------------------------------------------ tensor-core consumer

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

// c (16x8 fp32) += a (16x16 bf16, row) . b (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (x, y) -> bf16 pairs hi = rn(x, y) and lo = rn((x, y) - hi); the low half holds x.
__device__ __forceinline__ void split_bf16x2(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// One consumer warp per slot, all G query heads of kv head g. Fragment layouts are those
// of mma.m16n8k16 (lane = 4*grp + qd):
//   S tile (rows = q rows, cols = 8 tokens): A = q rows (hi part of head h in row h, lo part
//   in row 8 + h), B = K rows via ldmatrix; the lane gets S_hi and S_lo of head grp for
//   tokens 2qd, 2qd+1 in c0..c3 and adds them in place.
//   O^T tile (rows = 16 value dims, cols = 8): A = V^T via ldmatrix.trans, B = P^T, whose
//   fragment is exactly what the lane holds after the softmax (head grp, tokens 2qd, 2qd+1,
//   2qd+8, 2qd+9). Columns: G = 8 uses two tiles (p_hi, p_lo); G <= 4 puts p_hi of head c
//   in column c and p_lo in column 4 + c (taken from lane ^ 16).
template <int D, int G, int NST, int MINB>
__global__ void __launch_bounds__((kSlots + 1) * 32, MINB)
    attn_mma_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmap) {
  constexpr int STAGE = 2 * kT * D * 2;  // swizzled K and V rows of one block
  constexpr int CHUNK = kT * D * 2;
  constexpr int NCW = kSlots;
  constexpr int KS = D / 16;
  constexpr int NTP = G == 8 ? 2 : 1;
  constexpr int OFF_FLAGS = NST * STAGE;
  constexpr int OFF_BARS = (OFF_FLAGS + NST * 4 + 7) / 8 * 8;
  static_assert(NST % kSlots == 0, "each stage must belong to exactly one consumer slot");
  static_assert(NCW * G * D * 4 + NCW * G * 8 <= NST * STAGE, "merge area must fit in the stage ring");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  extern __shared__ __align__(128) uint8_t smem_raw[];
  // the 128-byte swizzle is a function of address bits 4..9: stages start 1024-byte aligned
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int* flags = reinterpret_cast<int*>(smem + OFF_FLAGS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BARS);
  uint64_t* empty = full + NST;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_b;
  const int s = blockIdx.x, g = blockIdx.y, b = longest_first_sequence(p, &s_b, warp, lane);
  const PoolView& pool = p.pool;
  // Launched with programmatic dependent launch behind the projection of the same step
  // (p.early_kv): q, the new token's k/v and the split counters come from it, so the
  // consumers wait for it (griddep_wait) before touching them. The tables, the positions
  // and the cached blocks were finished by the kernels before it (the projection signals
  // only after its own wait), and the one cache slot it writes is masked here, so the
  // producer starts at once; tables and positions are read through L2. Launched behind
  // anything else, every thread waits first.
  if (!p.early_kv) griddep_wait();
  if (p.signal_next && threadIdx.x == 0) griddep_launch_dependents();

  int ctx = __ldcg(p.seq_lens + b);
  if (ctx < 0 || ctx / kT + 1 > p.max_blocks) {
    if (threadIdx.x == 0 && s == 0 && g == 0) flag_error(pool.status, kErrCtxTooLong);
    ctx = ctx < 0 ? 0 : min(ctx, p.max_blocks * kT);
  }
  const int nb = (ctx + kT - 1) / kT;
  const int j0 = (int)((int64_t)nb * s / p.S);
  const int j1 = (int)((int64_t)nb * (s + 1) / p.S);
  const int n_local = j1 - j0;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 33);  // 32 producer lanes + 1 flag publish
      mbar_init(&empty[i], 1);  // lane 0 of the consuming warp
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == NCW) {
    attn_produce<D, NST, true>(p, &tmap, smem, flags, full, empty, b, g, ctx, j0, j1, lane);
    return;
  }

  const int slot = warp;
  const int grp = lane >> 2, qd = lane & 3;
  constexpr unsigned FULL = 0xffffffffu;
  griddep_wait();  // q, k_hat, v_hat and the counters are the projection's

  // q of head grp as A fragments: rows grp (hi) and grp + 8 (lo), dims 16ks + 2qd + {0,1,8,9}
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) qa[ks][0] = qa[ks][1] = qa[ks][2] = qa[ks][3] = 0u;
  if (grp < G) {
    const float* q = p.qs + ((int64_t)b * p.Hq + g * G + grp) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const float2 x0 = *reinterpret_cast<const float2*>(q + 16 * ks + 2 * qd);
      const float2 x1 = *reinterpret_cast<const float2*>(q + 16 * ks + 2 * qd + 8);
      split_bf16x2(x0.x, x0.y, qa[ks][0], qa[ks][1]);
      split_bf16x2(x1.x, x1.y, qa[ks][2], qa[ks][3]);
    }
  }

  float o[KS][NTP][4];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt)
#pragma unroll
    for (int nt = 0; nt < NTP; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // head grp (rows >= G carry zeros)

  const uint32_t sbase = smem_u32(smem);
  // ldmatrix row addresses in the swizzled stage (piece c of row r at c ^ (r & 7)):
  //   K (non-trans): row = token lane&7 (+8 nt), pieces of dims 32*k2 + 8*(lane>>3);
  //   V (trans):     row = token 8*(lane>>4) + (lane&7), pieces of dims 16*mt + 8*((lane>>3)&1)
  const int r7 = lane & 7;
  const uint32_t krow = r7 * 128;
  const uint32_t kx0 = (((lane >> 3) ^ r7) << 4), kx1 = (((4 + (lane >> 3)) ^ r7) << 4);
  const uint32_t vrow = CHUNK + (8 * (lane >> 4) + r7) * 128;
  const int vb = (lane >> 3) & 1;
  // the heads whose rescale factor applies to this lane's two O^T columns
  const int hc0 = G == 8 ? 2 * qd : (2 * qd) & 3;
  const int hc1 = G == 8 ? 2 * qd + 1 : (2 * qd + 1) & 3;

  for (int i = slot; i < n_local; i += kSlots) {
    const int st = i % NST;
    // warp-uniform: a give-up on any lane ends the loop for the whole warp
    if (!__all_sync(FULL, mbar_wait_bounded(&full[st], (i / NST) & 1, pool.status, p.wait_ns))) break;
    const int ntok = flags[st];
    if (ntok > 0) {
      const uint32_t kb = sbase + st * STAGE;
      if (ntok < kT) {
        // a sequence's last block: zero the V rows past its last token (p = 0 there, and
        // unwritten slots may hold any bits)
        uint8_t* vst = smem + st * STAGE + CHUNK;
        for (int x = lane; x < (kT - ntok) * (2 * D / 16); x += 32) {
          const int r = ntok + x / (2 * D / 16), c = x % (2 * D / 16);
          *reinterpret_cast<uint4*>(vst + (c >> 3) * kT * 128 + r * 128 + (c & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      // ---- S = Q . K^T for tokens 0..7 (nt = 0) and 8..15 (nt = 1)
      float sacc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < KS / 2; ++k2) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kb + (k2 >> 1) * kT * 128 + nt * 1024 + krow + ((k2 & 1) ? kx1 : kx0), r0, r1, r2, r3);
          mma_bf16_16816(sacc[nt], qa[2 * k2], r0, r1);
          mma_bf16_16816(sacc[nt], qa[2 * k2 + 1], r2, r3);
        }
      }
      // tokens 2qd, 2qd+1, 8+2qd, 9+2qd of head grp: hi row + lo row
      float sc[4] = {sacc[0][0] + sacc[0][2], sacc[0][1] + sacc[0][3], sacc[1][0] + sacc[1][2],
                     sacc[1][1] + sacc[1][3]};
      if (ntok < kT) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((e >> 1) * 8 + 2 * qd + (e & 1) >= ntok) sc[e] = -INFINITY;
      }
      float bm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, 1));
      bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, 2));
      const float m_new = fmaxf(m_run, bm);
      // rescale only when some head's running max grew (multiplying by 1 is exact)
      if (__any_sync(FULL, m_new > m_run)) {
        const float alpha = m_new > m_run ? fast_exp2(m_run - m_new) : 1.f;
        l_run *= alpha;
        const float a0 = __shfl_sync(FULL, alpha, hc0 * 4), a1 = __shfl_sync(FULL, alpha, hc1 * 4);
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
          for (int nt = 0; nt < NTP; ++nt) {
            o[mt][nt][0] *= a0;
            o[mt][nt][1] *= a1;
            o[mt][nt][2] *= a0;
            o[mt][nt][3] *= a1;
          }
      }
      m_run = m_new;
      const float mu = m_new == -INFINITY ? 0.f : m_new;
      float pr[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pr[e] = fast_exp2(sc[e] - mu);
      l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);
      uint32_t ph0, pl0, ph1, pl1;
      split_bf16x2(pr[0], pr[1], ph0, pl0);  // tokens 2qd, 2qd+1   (B rows 0..7)
      split_bf16x2(pr[2], pr[3], ph1, pl1);  // tokens 2qd+8, 2qd+9 (B rows 8..15)
      uint32_t b0 = ph0, b1 = ph1;
      if constexpr (G < 8) {
        const uint32_t x0 = __shfl_xor_sync(FULL, pl0, 16), x1 = __shfl_xor_sync(FULL, pl1, 16);
        if (grp >= 4) {
          b0 = x0;
          b1 = x1;
        }
      }
      // ---- O^T += V^T . P^T, 16 value dims per tile
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        uint32_t a[4];
        ldsm_x4_t(kb + vrow + (mt >> 2) * kT * 128 + ((((2 * (mt & 3) + vb) ^ r7)) << 4), a[0], a[1], a[2], a[3]);
        mma_bf16_16816(o[mt][0], a, b0, b1);
        if constexpr (G == 8) mma_bf16_16816(o[mt][1], a, pl0, pl1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---- l of head grp over the four token lanes; O = hi columns + lo columns
  l_run += __shfl_xor_sync(FULL, l_run, 1);
  l_run += __shfl_xor_sync(FULL, l_run, 2);
  named_bar_sync(1, NCW * 32);  // every slot is done reading the stage ring
  float* macc = reinterpret_cast<float*>(smem);
  float2* mml = reinterpret_cast<float2*>(smem + NCW * G * D * 4);
#pragma unroll
  for (int mt = 0; mt < KS; ++mt) {
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (G == 8)
        v[e] = o[mt][0][e] + o[mt][NTP - 1][e];
      else
        v[e] = o[mt][0][e] + __shfl_xor_sync(FULL, o[mt][0][e], 2);
    }
    if (G == 8 || qd < 2) {
      const int h0 = 2 * qd, h1 = 2 * qd + 1;
      const int dl = 16 * mt + grp, dh = dl + 8;
      if (h0 < G) {
        macc[(warp * G + h0) * D + dl] = v[0];
        macc[(warp * G + h0) * D + dh] = v[2];
      }
      if (h1 < G) {
        macc[(warp * G + h1) * D + dl] = v[1];
        macc[(warp * G + h1) * D + dh] = v[3];
      }
    }
  }
  if (qd == 0 && grp < G) mml[warp * G + grp] = make_float2(m_run, l_run);
  named_bar_sync(1, NCW * 32);
  attn_merge_combine<D, G, 1>(p, smem, b, g, s, warp, lane);
}

// ----------------------------------------------------------------------- combine

// out[b][h] = (sum_s acc_s 2^(m_s-M) + v_new 2^(s_new-M)) / (sum_s l_s 2^(m_s-M) + 2^(s_new-M))
// over the S split partials and the new token's (score s_new, value v_hat); bf16 RNE.
// The standalone combine (after attend(out = nullptr)): one warp per (q head, sequence),
// the same merge as the fused combine.
template <int D>
__global__ void __launch_bounds__(32) combine_kernel(int Hq, int Hkv, int S, const float2* __restrict__ ml,
                                                     const float* __restrict__ acc, const float* __restrict__ qs,
                                                     const float* __restrict__ knew, const float* __restrict__ vnew,
                                                     uint16_t* __restrict__ out) {
  const int hg = blockIdx.x, b = blockIdx.y, lane = threadIdx.x;
  const int g = hg / (Hq / Hkv);
  const float sn = new_token_score(qs + ((int64_t)b * Hq + hg) * D, knew + ((int64_t)b * Hkv + g) * D, D, lane);
  combine_head_warp<D, 8, 16>(ml, acc, S, ((int64_t)b * Hq + hg) * S, 1, sn, vnew + ((int64_t)b * Hkv + g) * D,
                       out + ((int64_t)b * Hq + hg) * D, lane);
}

// ---------------------------------------------------------------------- launchers

// Launch with programmatic stream serialization: the kernel may be scheduled while the
// projection ahead of it finishes; it waits for it (griddep_wait) before reading anything.
template <typename... KArgs, typename... Args>
static int launch_pdl(void (*fn)(KArgs...), dim3 grid, int threads, int smem, cudaStream_t st, bool pdl,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1] = {};
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cuda_check(cudaLaunchKernelEx(&cfg, fn, std::forward<Args>(args)...), "attention launch");
}

template <int D, int HPW, int WPB, int NST, int MINB, int SL = kSlots>
static int launch_attn_t(const AttnParams& p, int B, int Hkv, cudaStream_t st) {
  using C = AttnCfg<D, HPW, WPB, NST, SL>;
  auto* fn = attn_splitk_kernel<D, HPW, WPB, NST, MINB, SL>;
  constexpr int smem = C::SMEM;
  static bool attr_done = false;  // per instantiation
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_check(e, "attention: set smem attribute");
    attr_done = true;
  }
  return launch_pdl(fn, dim3(p.S, Hkv, B), C::THREADS, smem, st, p.pdl != 0, p);
}

template <int D, int G, int NST, int MINB>
static int launch_attn_mma(const AttnParams& p, int B, int Hkv, cudaStream_t st) {
  constexpr int smem = 1024 + (NST * 2 * kT * D * 2 + NST * 4 + 7) / 8 * 8 + 2 * NST * 8;
  auto* fn = attn_mma_kernel<D, G, NST, MINB>;
  // the HBM tier as a [rows][D] bf16 array, boxes of [T rows][64 dims], 128-byte swizzle
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  const PoolView& v = p.pool;
  if (v.blocks[0] > 0) {
    const uint64_t rows = (uint64_t)v.blocks[0] * v.L * 2 * v.Hkv * v.T;
    if (rows > (uint64_t)INT32_MAX) return set_error(DKV_ERR_UNSUPPORTED, "attention: HBM tier too large for TMA rows");
    int rc = encode_bf16_2d(&tmap, v.tier[0], rows, (uint64_t)D, (uint32_t)kT);
    if (rc) return rc;
  }
  static bool attr_done = false;  // per instantiation
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_check(e, "attention: set smem attribute");
    attr_done = true;
  }
  return launch_pdl(fn, dim3(p.S, Hkv, B), (kSlots + 1) * 32, smem, st, p.pdl != 0, p, tmap);
}

// Kernel per (D, G) and variant:
//   0 automatic = 5 (the tensor cores are reserved for the projection)
//   5: CUDA cores, q in registers, three consumer slots with two stages each (6-stage
//      ring), four CTAs per SM: 16 warps of 128 registers fill the register file, and
//      four producers per SM stream HBM faster than three (G = 8: the variant-1 shape)
//   1: CUDA cores, q in registers, four slots, 8-stage ring, three CTAs per SM (G = 8: two
//      warps per block, one CTA per SM)
//   2: CUDA cores, q in shared memory, 4-stage ring (one stage per consumer slot), four
//      CTAs per SM (G <= 4)
//   6: tensor cores, 4-stage ring, four CTAs per SM (G = 8: 12 stages, two CTAs per SM)
//   7: tensor cores, 8-stage ring, three CTAs per SM (G <= 4)
// (Rings must be a multiple of the consumer slots.)
template <int D>
static int launch_attn_d(const AttnParams& p, int B, int Hkv, int G, int variant, cudaStream_t st) {
  if (variant == 7 && G <= 4) {
    switch (G) {
      case 1: return launch_attn_mma<D, 1, 8, 3>(p, B, Hkv, st);
      case 2: return launch_attn_mma<D, 2, 8, 3>(p, B, Hkv, st);
      case 4: return launch_attn_mma<D, 4, 8, 3>(p, B, Hkv, st);
    }
  }
  if (variant == 6 || variant == 7) {
    switch (G) {
      case 1: return launch_attn_mma<D, 1, 4, 4>(p, B, Hkv, st);
      case 2: return launch_attn_mma<D, 2, 4, 4>(p, B, Hkv, st);
      case 4: return launch_attn_mma<D, 4, 4, 4>(p, B, Hkv, st);
      case 8: return launch_attn_mma<D, 8, 12, 2>(p, B, Hkv, st);
    }
    return set_error(DKV_ERR_UNSUPPORTED, "attention: unsupported G=%d", G);
  }
  if (variant == 5 || variant == 0) {
    switch (G) {
      case 1: return launch_attn_t<D, 1, 1, 6, 4, 3>(p, B, Hkv, st);
      case 2: return launch_attn_t<D, 2, 1, 6, 4, 3>(p, B, Hkv, st);
      case 4: return launch_attn_t<D, 4, 1, 6, 4, 3>(p, B, Hkv, st);
      case 8: return launch_attn_t<D, 4, 2, 4, 3, 2>(p, B, Hkv, st);
    }
  }
  switch (G) {
    case 1: return launch_attn_t<D, 1, 1, 8, 3>(p, B, Hkv, st);
    case 2: return launch_attn_t<D, 2, 1, 8, 3>(p, B, Hkv, st);
    case 4: return launch_attn_t<D, 4, 1, 8, 3>(p, B, Hkv, st);
    case 8: return launch_attn_t<D, 4, 2, 8, 1>(p, B, Hkv, st);
  }
  return set_error(DKV_ERR_UNSUPPORTED, "attention: unsupported G=%d", G);
}

int attention_ctas_per_sm(int G, int variant) {
  if (variant == 6) return G == 8 ? 2 : 4;
  if (variant == 7) return G == 8 ? 2 : 3;
  if (variant == 5 || variant == 0) return G == 8 ? 3 : 4;
  return G == 8 ? 1 : 3;
}

int launch_attention(const AttnParams& p, int B, int Hkv, int D, int G, int variant, cudaStream_t st) {
  if (D == 128) return launch_attn_d<128>(p, B, Hkv, G, variant, st);
  if (D == 64) return launch_attn_d<64>(p, B, Hkv, G, variant, st);
  return set_error(DKV_ERR_UNSUPPORTED, "attention: unsupported D=%d", D);
}

int launch_combine(int B, int Hq, int Hkv, int D, int S, const float2* ml, const float* acc,
                   const float* qs, const float* knew, const float* vnew, uint16_t* out, cudaStream_t st) {
  dim3 grid(Hq, B);
  if (D == 128)
    combine_kernel<128><<<grid, 32, 0, st>>>(Hq, Hkv, S, ml, acc, qs, knew, vnew, out);
  else
    combine_kernel<64><<<grid, 32, 0, st>>>(Hq, Hkv, S, ml, acc, qs, knew, vnew, out);
  return cuda_check(cudaGetLastError(), "combine launch");
}

}  // namespace dkv
