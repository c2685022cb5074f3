// Split-K GQA decode attention over a two-tier paged KV cache, and the split combine.
//
// DirectKV ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", 核心方法) lets the attention
// kernel read CPU-resident KV in place and hides the slow fetches behind compute with a
// warp-level producer/consumer pipeline. This kernel is that pipeline on sm_100a:
//
//  * one CTA per (split s, kv head g, sequence b) walks a contiguous range of logical
//    blocks; the KV of kv head g is read once for all G = Hq/Hkv query heads;
//  * one producer warp fills an NST-stage shared-memory ring, one stage per block
//    (K chunk [T][D] then V chunk [T][D], both contiguous in the pool):
//      - HBM-tier block: one lane issues two bulk copies (TMA engine) of the chunks;
//      - host-tier block: all 32 lanes issue 16-byte cp.async loads straight from the
//        mapped pinned host memory (coalesced 512-byte warp requests), no staging buffer;
//    both complete on the stage's mbarrier, so the consumers see one kind of stage;
//  * four consumer "slots" (WPB warps each; heads split across the WPB warps) take
//    blocks round robin, each keeping its own online-softmax state (running max m,
//    running sum l, accumulator acc) in registers; the slots merge at the end and the CTA
//    writes one partial state (m, l, acc[D]) per q head to the workspace.
//
// Scores are computed in the log2 domain: q arrives pre-scaled by log2(e)/sqrt(D), so
// p = 2^(s - m). Arithmetic is fp32 on CUDA cores (a decode query is a handful of rows:
// G flops per byte of KV, HBM-bound, not a tensor-core contraction).
#include <math.h>

#include "dkv_internal.h"

namespace dkv {

constexpr int kSlots = 4;
constexpr int kT = 16;

template <int D, int HPW, int WPB, int NST>
struct AttnCfg {
  static constexpr int G = HPW * WPB;
  static constexpr int NCW = kSlots * WPB;  // consumer warps
  static constexpr int THREADS = (NCW + 1) * 32;
  static constexpr int STAGE_ELEMS = 2 * kT * D;
  static constexpr int STAGE_BYTES = STAGE_ELEMS * 2;
  static constexpr int DPL = D / 32;   // value dims per lane in P.V
  static constexpr int QCH = D / 64;   // 16-byte key chunks per lane per token in Q.K
  static constexpr int NV = HPW * 4;   // partial scores per lane (heads x 4 tokens)
  static constexpr int LOGH = HPW == 4 ? 2 : (HPW == 2 ? 1 : 0);
  static constexpr int LOWMASK = (1 << (3 - LOGH)) - 1;  // dg bits shared by one head
  static constexpr int NR = NV >= 8 ? NV / 8 : 1;        // scores per lane after reduction
  static constexpr int OFF_P = NST * STAGE_BYTES;
  static constexpr int OFF_ALPHA = OFF_P + NCW * kT * HPW * 8;
  static constexpr int OFF_FLAGS = OFF_ALPHA + NCW * HPW * 4;
  static constexpr int OFF_BARS = (OFF_FLAGS + NST * 4 + 7) / 8 * 8;
  static constexpr int SMEM = OFF_BARS + 2 * NST * 8;
  static constexpr int MERGE_BYTES = NCW * HPW * D * 4 + NCW * HPW * 8;
  static_assert(MERGE_BYTES <= NST * STAGE_BYTES, "merge area must fit in the stage ring");
  // Block i uses stage i % NST and consumer slot i % kSlots. Stage loads complete out of
  // order, and a parity wait is only sound if the stage's barrier is at most one phase
  // behind the waiter; that holds when every stage belongs to a single slot.
  static_assert(NST % kSlots == 0, "each stage must belong to exactly one consumer slot");
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Merge the S split states of one (b, q head) output element with the new token's term:
// M = max(s_new, m_s), L = 2^(s_new-M) + sum l_s 2^(m_s-M),
// o = (v_new 2^(s_new-M) + sum acc_s 2^(m_s-M)) / L. Splits are read in index order.
__device__ __forceinline__ float combine_value(const float2* __restrict__ ml, const float* __restrict__ acc,
                                               int S, int64_t base, int D, int d, float sn, float vn) {
  float M = sn;
  for (int s = 0; s < S; ++s) M = fmaxf(M, __ldcg(ml + base + s).x);
  const float wn = exp2f(sn - M);
  float L = wn;
  float A = wn * vn;
  for (int s = 0; s < S; ++s) {
    const float2 m = __ldcg(ml + base + s);
    if (m.x != -INFINITY) {
      const float w = exp2f(m.x - M);
      L = fmaf(m.y, w, L);
      A = fmaf(__ldcg(acc + (base + s) * D + d), w, A);
    }
  }
  return A / L;
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

// QS: keep q in shared memory instead of registers (fewer registers, more CTAs per SM).
template <int D, int HPW, int WPB, int NST, int MINB, bool QS>
__global__ void __launch_bounds__(AttnCfg<D, HPW, WPB, NST>::THREADS, MINB)
    attn_splitk_kernel(const AttnParams p) {
  using C = AttnCfg<D, HPW, WPB, NST>;
  constexpr int OFF_Q = (C::SMEM + 15) / 16 * 16;  // q area (QS only): [G][QCH][2][8][4] fp32
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* stages = reinterpret_cast<uint16_t*>(smem);
  float2* pbuf = reinterpret_cast<float2*>(smem + C::OFF_P);
  float* alph = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  int* flags = reinterpret_cast<int*>(smem + C::OFF_FLAGS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  uint64_t* empty = full + NST;

  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PoolView& pool = p.pool;

  // cached tokens of this sequence, clamped to what the table can hold
  int ctx = p.seq_lens[b];
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
    // ------------------------------------------------------------------ producer
    // Table entries are fetched 32 blocks at a time (lane l holds block base + l) and
    // broadcast by shuffle, so no dependent global load sits on the per-block path.
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
    for (int i = 0; i < n_local; ++i) {
      if ((i & 31) == 0) {
        const int j = j0 + i + lane;
        if (j < j1) {
          pf_tier = p.tier_map[rowbase + j];
          pf_phys = p.table[rowbase + j];
        }
      }
      const int st = i % NST;
      const int k = i / NST;
      if (k > 0 && !mbar_wait_bounded(&empty[st], (k - 1) & 1, pool.status)) break;
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
      uint16_t* dst = stages + st * C::STAGE_ELEMS;
      if (lane == 0) flags[st] = valid ? ntok : -1;
      if (!valid) {
        mbar_arrive(&full[st]);
        if (lane == 0) mbar_arrive(&full[st]);
        issued = i + 1;
        continue;
      }
      const uint16_t* kp = (tier ? kbase1 : kbase0) + phys * pstride;
      const uint16_t* vp = kp + kvoff;
      if (tier == DKV_TIER_HBM && !p.lsu_hbm) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
          mbar_arrive(&full[st]);
          bulk_g2s(dst, kp, C::STAGE_BYTES / 2, &full[st]);
          bulk_g2s(dst + kT * D, vp, C::STAGE_BYTES / 2, &full[st]);
        } else {
          mbar_arrive(&full[st]);
        }
      } else {
        constexpr int PIECES = C::STAGE_BYTES / 16;  // 16-byte pieces per stage
        constexpr int HALF = PIECES / 2;
#pragma unroll
        for (int c = 0; c < PIECES / 32; ++c) {
          const int idx = c * 32 + lane;
          const uint16_t* src = idx < HALF ? kp + idx * 8 : vp + (idx - HALF) * 8;
          cp_async16(dst + idx * 8, src);
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
      mbar_wait_bounded(&full[j % NST], (j / NST) & 1, pool.status, 100000000ull);
    return;  // consumers below sync only among themselves (named barrier 1)
  }

  // -------------------------------------------------------------------- consumers
  const int slot = warp / WPB, hq = warp % WPB;
  const int tg = lane >> 3, dg = lane & 7;
  const int hbase = g * C::G + hq * HPW;  // first global q head of this warp

  // q of this lane's key dims, as (even, odd) dim pairs for the packed fp32x2 FMA: in
  // registers, or (QS) in shared memory laid out [head][hh][half][dg][4] so that the eight
  // dg lanes read 128 contiguous bytes.
  float2 q2[QS ? 1 : HPW][QS ? 1 : C::QCH][4];
  float* qsm = reinterpret_cast<float*>(smem + OFF_Q);
  if constexpr (QS) {
    for (int e = threadIdx.x; e < C::G * D; e += C::NCW * 32) {
      const int h = e / D, d = e % D, c = d / 8, w = d % 8;
      qsm[(((h * C::QCH + c / 8) * 2 + w / 4) * 8 + c % 8) * 4 + w % 4] =
          p.qs[((int64_t)b * p.Hq + g * C::G + h) * D + d];
    }
    named_bar_sync(1, C::NCW * 32);
  } else {
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

  for (int i = slot; i < n_local; i += kSlots) {
    const int st = i % NST;
    if (!mbar_wait_bounded(&full[st], (i / NST) & 1, pool.status)) break;
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
      if constexpr (QS) {
#pragma unroll
        for (int hh = 0; hh < C::QCH; ++hh) {
          float2 kk[4][4];
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const uint4 w = *reinterpret_cast<const uint4*>(Ks + (tg + 4 * i4) * D + (dg + 8 * hh) * 8);
            kk[i4][0] = make_float2(bf16lo(w.x), bf16hi(w.x));
            kk[i4][1] = make_float2(bf16lo(w.y), bf16hi(w.y));
            kk[i4][2] = make_float2(bf16lo(w.z), bf16hi(w.z));
            kk[i4][3] = make_float2(bf16lo(w.w), bf16hi(w.w));
          }
#pragma unroll
          for (int h = 0; h < HPW; ++h) {
            const float4* qp = reinterpret_cast<const float4*>(qsm) + (((hq * HPW + h) * C::QCH + hh) * 2) * 8 + dg;
            const float4 qa = qp[0], qb = qp[8];
            const float2 q0 = make_float2(qa.x, qa.y), q1 = make_float2(qa.z, qa.w);
            const float2 q2b = make_float2(qb.x, qb.y), q3 = make_float2(qb.z, qb.w);
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
              float2 a = v2[h * 4 + i4];
              a = __ffma2_rn(q0, kk[i4][0], a);
              a = __ffma2_rn(q1, kk[i4][1], a);
              a = __ffma2_rn(q2b, kk[i4][2], a);
              a = __ffma2_rn(q3, kk[i4][3], a);
              v2[h * 4 + i4] = a;
            }
          }
        }
      } else {
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

  // ---- per-warp totals of l, then merge the four slots through shared memory
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

  for (int o = threadIdx.x; o < C::G * D; o += C::NCW * 32) {
    const int hh = o / D, d = o % D;
    const int wq = hh / HPW, h = hh % HPW;
    float M = -INFINITY;
#pragma unroll
    for (int sl = 0; sl < kSlots; ++sl) M = fmaxf(M, mml[(sl * WPB + wq) * HPW + h].x);
    float A = 0.f, Ls = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int sl = 0; sl < kSlots; ++sl) {
        const float2 ml = mml[(sl * WPB + wq) * HPW + h];
        const float w = fast_exp2(ml.x - M);
        A = fmaf(macc[((sl * WPB + wq) * HPW + h) * D + d], w, A);
        Ls = fmaf(ml.y, w, Ls);
      }
    }
    const int64_t base = ((int64_t)b * p.Hq + g * C::G + hh) * p.S + s;
    p.part_acc[base * D + d] = A;
    if (d == 0) p.part_ml[base] = make_float2(M, Ls);
  }

  // ---- fused combine: the last split CTA of (b, g) to finish merges all S partial states
  // (in split order, so the result does not depend on which CTA finishes last)
  if (p.out) {
    __shared__ int s_last;
    __shared__ float s_new[8];
    __threadfence();
    named_bar_sync(1, C::NCW * 32);
    if (threadIdx.x == 0) s_last = atomicAdd(p.cnt + (int64_t)b * pool.Hkv + g, 1) == p.S - 1;
    named_bar_sync(1, C::NCW * 32);
    if (s_last) {
      __threadfence();
      const float* kn = p.knew + ((int64_t)b * pool.Hkv + g) * D;
      for (int hh = warp; hh < C::G; hh += C::NCW) {
        const float sc = new_token_score(p.qs + ((int64_t)b * p.Hq + g * C::G + hh) * D, kn, D, lane);
        if (lane == 0) s_new[hh] = sc;
      }
      named_bar_sync(1, C::NCW * 32);
      for (int o = threadIdx.x; o < C::G * D; o += C::NCW * 32) {
        const int hh = o / D, d = o % D;
        const int hg = g * C::G + hh;
        const float r = combine_value(p.part_ml, p.part_acc, p.S, ((int64_t)b * p.Hq + hg) * p.S, D, d,
                                      s_new[hh], p.vnew[((int64_t)b * pool.Hkv + g) * D + d]);
        p.out[((int64_t)b * p.Hq + hg) * D + d] = f32_to_bf16_bits(r);
      }
      if (threadIdx.x == 0) p.cnt[(int64_t)b * pool.Hkv + g] = 0;
    }
  }
}

// ----------------------------------------------------------------------- combine

// out[b][h] = (sum_s acc_s 2^(m_s-M) + v_new 2^(s_new-M)) / (sum_s l_s 2^(m_s-M) + 2^(s_new-M))
// over the S split partials and the new token's (score s_new, value v_hat); bf16 RNE.
template <int D>
__global__ void __launch_bounds__(D) combine_kernel(int Hq, int Hkv, int S,
                                                    const float2* __restrict__ ml,
                                                    const float* __restrict__ acc,
                                                    const float* __restrict__ qs,
                                                    const float* __restrict__ knew,
                                                    const float* __restrict__ vnew,
                                                    uint16_t* __restrict__ out) {
  const int hg = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int g = hg / (Hq / Hkv);
  __shared__ float s_new;
  if (d < 32) {
    const float sc = new_token_score(qs + ((int64_t)b * Hq + hg) * D, knew + ((int64_t)b * Hkv + g) * D, D, d);
    if (d == 0) s_new = sc;
  }
  __syncthreads();
  const float r = combine_value(ml, acc, S, ((int64_t)b * Hq + hg) * S, D, d, s_new,
                                vnew[((int64_t)b * Hkv + g) * D + d]);
  out[((int64_t)b * Hq + hg) * D + d] = f32_to_bf16_bits(r);
}

// ---------------------------------------------------------------------- launchers

template <int D, int HPW, int WPB, int NST, int MINB, bool QS = false>
static int launch_attn_t(const AttnParams& p, int B, int Hkv, cudaStream_t st) {
  using C = AttnCfg<D, HPW, WPB, NST>;
  auto* fn = attn_splitk_kernel<D, HPW, WPB, NST, MINB, QS>;
  constexpr int smem = QS ? (C::SMEM + 15) / 16 * 16 + C::G * D * 4 : C::SMEM;
  static bool attr_done = false;  // per instantiation
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_check(e, "attention: set smem attribute");
    attr_done = true;
  }
  dim3 grid(p.S, Hkv, B);
  fn<<<grid, C::THREADS, smem, st>>>(p);
  return cuda_check(cudaGetLastError(), "attention launch");
}

// Kernel shape per (D, G) and variant (G = 4 only; other G have one shape):
//   0 automatic = 1: q in registers, 8-stage ring, three CTAs per SM
//   2: 12-stage ring, two CTAs per SM        3: two warps per block (G/2 heads each)
//   5: q in shared memory, 8-stage ring, three CTAs per SM
// (Rings must be a multiple of the four consumer slots; see AttnCfg.)
template <int D>
static int launch_attn_d(const AttnParams& p, int B, int Hkv, int G, int variant, cudaStream_t st) {
  switch (G) {
    case 1: return launch_attn_t<D, 1, 1, 8, 3>(p, B, Hkv, st);
    case 2: return launch_attn_t<D, 2, 1, 8, 3>(p, B, Hkv, st);
    case 4:
      switch (variant) {
        case 1: return launch_attn_t<D, 4, 1, 8, 3>(p, B, Hkv, st);
        case 2: return launch_attn_t<D, 4, 1, 12, 2>(p, B, Hkv, st);
        case 3: return launch_attn_t<D, 2, 2, 8, 2>(p, B, Hkv, st);
        case 5: return launch_attn_t<D, 4, 1, 8, 3, true>(p, B, Hkv, st);
        default: return launch_attn_t<D, 4, 1, 8, 3>(p, B, Hkv, st);
      }
    case 8: return launch_attn_t<D, 4, 2, 8, 1>(p, B, Hkv, st);
  }
  return set_error(DKV_ERR_UNSUPPORTED, "attention: unsupported G=%d", G);
}

int attention_ctas_per_sm(int G, int variant) {
  (void)G;
  return variant == 2 || variant == 3 ? 2 : 3;
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
    combine_kernel<128><<<grid, 128, 0, st>>>(Hq, Hkv, S, ml, acc, qs, knew, vnew, out);
  else
    combine_kernel<64><<<grid, 64, 0, st>>>(Hq, Hkv, S, ml, acc, qs, knew, vnew, out);
  return cuda_check(cudaGetLastError(), "combine launch");
}

}  // namespace dkv
