// The decode step: projection stage (QKV GEMM, RoPE, single cache write, new-token
// partial), attention stage, combine stage; workspace layout and the C entry points.
//
// DirectKV ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", 核心方法) fuses KV generation
// (the QKV projection) with attention so that the new K/V are consumed on chip and never
// written out and read back. Here the projection's epilogue owns one kv-head group
// (its G query heads plus the group's key and value rows), so it has everything the new
// token's attention term needs: it rotates q and k, writes bf16 k_hat/v_hat to the cache
// exactly once, and emits the new token's softmax partial (score q.k_hat, value v_hat),
// which the combine stage folds in. The attention stage then reads only cached blocks.
#include <math.h>

#include "dkv_internal.h"

namespace dkv {

struct ProjParams {
  PoolView pool;
  int layer;
  const uint16_t* x;
  const uint16_t* W;
  const int32_t* table;
  const int32_t* seq_lens;
  const uint8_t* tier_map;
  int max_blocks;
  int B, H, Hq, Hkv, D, SP;
  double theta;
  float qscale;   // log2(e) / sqrt(D)
  float* acc;     // [B][rows] fp32, zeroed before the launch
  int* cnt;       // [Hkv] arrival counters, zeroed before the launch
  float* qs;      // [B][Hq][D]
  float* snew;    // [B][Hq]
  float* vnew;    // [B][Hkv][D]
};

// First W row of piece `pc` of group g: pieces 0..G-1 are q heads g*G.., G is k_g, G+1 v_g.
__device__ __forceinline__ int piece_row(int pc, int g, int G, int Hq, int Hkv, int D) {
  if (pc < G) return (g * G + pc) * D;
  if (pc == G) return (Hq + g) * D;
  return (Hq + Hkv + g) * D;
}

// Epilogue for kv-head group g, run by the CTA that completes the group's reduction:
// RoPE, q scaling, the single bf16 cache write of k_hat / v_hat, and the new token's
// score s_new = q_scaled . k_hat for each of the G heads.
__device__ void proj_group_epilogue(const ProjParams& p, int g, float* sm) {
  const int D = p.D, G = p.Hq / p.Hkv, half = D / 2;
  const int rows = (p.Hq + 2 * p.Hkv) * D;
  float2* cs = reinterpret_cast<float2*>(sm);  // [D/2] (cos, sin)
  float* qsm = sm + D;                          // [G][D]
  float* ksm = qsm + G * D;                     // [D]
  const int tid = threadIdx.x, nth = blockDim.x;
  for (int b = 0; b < p.B; ++b) {
    const int pos = p.seq_lens[b];
    for (int i = tid; i < half; i += nth) {
      const double inv = pow(p.theta, -2.0 * (double)i / (double)D);
      double sn, cn;
      sincos((double)pos * inv, &sn, &cn);
      cs[i] = make_float2((float)cn, (float)sn);
    }
    // where the new token's K/V go
    const int64_t jb = pos >= 0 ? (int64_t)pos / p.pool.T : -1;
    const int slot = pos >= 0 ? pos % p.pool.T : 0;
    int tier = -1;
    int64_t phys = -1;
    if (jb >= 0 && jb < p.max_blocks) {
      tier = p.tier_map[(int64_t)b * p.max_blocks + jb];
      phys = p.table[(int64_t)b * p.max_blocks + jb];
    }
    bool ok = true;
    if (jb < 0 || jb >= p.max_blocks) {
      ok = false;
      if (tid == 0) flag_error(p.pool.status, kErrCtxTooLong);
    } else if (tier > 1) {
      ok = false;
      if (tid == 0) flag_error(p.pool.status, kErrBadTier);
    } else if (phys < 0 || phys >= tier_blocks(p.pool, tier)) {
      ok = false;
      if (tid == 0) flag_error(p.pool.status, kErrBadBlock);
    }
    uint16_t* kdst = ok ? tier_base(p.pool, tier) + chunk_offset(p.pool, tier, p.layer, phys, 0, g) + (int64_t)slot * D : nullptr;
    uint16_t* vdst = ok ? tier_base(p.pool, tier) + chunk_offset(p.pool, tier, p.layer, phys, 1, g) + (int64_t)slot * D : nullptr;
    __syncthreads();
    const float* a = p.acc + (int64_t)b * rows;
    for (int it = tid; it < (G + 1) * half; it += nth) {
      const int pc = it / half, i = it % half;
      const int r0 = piece_row(pc, g, G, p.Hq, p.Hkv, D) + i;
      const float x0 = __ldcg(a + r0), x1 = __ldcg(a + r0 + half);
      const float2 c = cs[i];
      const float y0 = x0 * c.x - x1 * c.y;
      const float y1 = x1 * c.x + x0 * c.y;
      if (pc < G) {
        const float q0 = y0 * p.qscale, q1 = y1 * p.qscale;
        qsm[pc * D + i] = q0;
        qsm[pc * D + i + half] = q1;
        float* qd = p.qs + ((int64_t)b * p.Hq + g * G + pc) * D;
        qd[i] = q0;
        qd[i + half] = q1;
      } else {
        const uint16_t k0 = f32_to_bf16_bits(y0), k1 = f32_to_bf16_bits(y1);
        ksm[i] = __uint_as_float((uint32_t)k0 << 16);
        ksm[i + half] = __uint_as_float((uint32_t)k1 << 16);
        if (kdst) {
          kdst[i] = k0;
          kdst[i + half] = k1;
        }
      }
    }
    for (int d = tid; d < D; d += nth) {
      const float vv = __ldcg(a + piece_row(G + 1, g, G, p.Hq, p.Hkv, D) + d);
      const uint16_t vb = f32_to_bf16_bits(vv);
      p.vnew[((int64_t)b * p.Hkv + g) * D + d] = __uint_as_float((uint32_t)vb << 16);
      if (vdst) vdst[d] = vb;
    }
    __syncthreads();
    // s_new for each head of the group: one warp per head
    const int warp = tid >> 5, lane = tid & 31;
    for (int h = warp; h < G; h += nth / 32) {
      float sacc = 0.f;
      for (int d = lane; d < D; d += 32) sacc = fmaf(qsm[h * D + d], ksm[d], sacc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
      if (lane == 0) p.snew[(int64_t)b * p.Hq + g * G + h] = sacc;
    }
    __syncthreads();
  }
}

// Projection, CUDA-core form: CTA (k-split ks, group g) multiplies the group's
// (G+2)*D rows of W by x over its slice of the hidden dimension and adds the partial
// sums into acc with fp32 reductions; the last CTA of a group runs the epilogue.
constexpr int kProjThreads = 256;

__global__ void __launch_bounds__(kProjThreads) proj_cudacore_kernel(const ProjParams p) {
  extern __shared__ __align__(16) float psm[];
  const int ks = blockIdx.x, g = blockIdx.y;
  const int D = p.D, G = p.Hq / p.Hkv, H = p.H;
  const int rows = (p.Hq + 2 * p.Hkv) * D;
  const int KR = H / p.SP, k0 = ks * KR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* xs = psm;  // [B][KR]
  for (int i = tid; i < p.B * KR; i += kProjThreads) {
    const int b = i / KR, k = i % KR;
    xs[i] = __uint_as_float((uint32_t)p.x[(int64_t)b * H + k0 + k] << 16);
  }
  __syncthreads();
  const int nrows = (G + 2) * D;
  for (int lr = warp; lr < nrows; lr += kProjThreads / 32) {
    const int grow = piece_row(lr / D, g, G, p.Hq, p.Hkv, D) + lr % D;
    float part[32];
#pragma unroll
    for (int b = 0; b < 32; ++b) part[b] = 0.f;
    const uint16_t* wr = p.W + (int64_t)grow * H + k0;
    for (int kk = lane * 8; kk < KR; kk += 256) {
      const uint4 w = __ldcs(reinterpret_cast<const uint4*>(wr + kk));
      const float wf[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                           bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
      for (int b = 0; b < 32; ++b) {
        if (b < p.B) {
          const float4 xa = *reinterpret_cast<const float4*>(xs + b * KR + kk);
          const float4 xb = *reinterpret_cast<const float4*>(xs + b * KR + kk + 4);
          float s = part[b];
          s = fmaf(wf[0], xa.x, s); s = fmaf(wf[1], xa.y, s); s = fmaf(wf[2], xa.z, s);
          s = fmaf(wf[3], xa.w, s); s = fmaf(wf[4], xb.x, s); s = fmaf(wf[5], xb.y, s);
          s = fmaf(wf[6], xb.z, s); s = fmaf(wf[7], xb.w, s);
          part[b] = s;
        }
      }
    }
    // reduce-scatter 32 batch slots over 32 lanes: lane l ends with batch l's total
#pragma unroll
    for (int lvl = 0; lvl < 5; ++lvl) {
      const int mask = 16 >> lvl;
      const int n = 32 >> lvl;
      const bool up = (lane & mask) != 0;
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        if (x < n / 2) {
          const float send = up ? part[x] : part[x + n / 2];
          const float keep = up ? part[x + n / 2] : part[x];
          part[x] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
        }
      }
    }
    if (lane < p.B) atomicAdd(p.acc + (int64_t)lane * rows + grow, part[0]);
  }
  __threadfence();
  __syncthreads();
  __shared__ int last;
  if (tid == 0) last = atomicAdd(p.cnt + g, 1) == p.SP - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  proj_group_epilogue(p, g, psm);
}

// ----------------------------------------------------------------- workspace

static int pick_proj_splits(const dkv_pool* pool, int Hkv, int H) {
  if (pool->tuning.proj_splits > 0) return pool->tuning.proj_splits;
  int want = (2 * pool->num_sms + Hkv - 1) / Hkv;
  int sp = want;
  if (sp > H / 64) sp = H / 64;
  while (sp > 1 && H % (sp * 64) != 0) --sp;
  return sp < 1 ? 1 : sp;
}

static int pick_attn_splits(const dkv_pool* pool, int B, int Hkv, int max_blocks) {
  int s = pool->tuning.attn_splits;
  if (s <= 0) {
    const int target = pool->num_sms * 4;
    const int units = B * Hkv;
    s = (target + units - 1) / units;
  }
  if (s > max_blocks) s = max_blocks;
  return s < 1 ? 1 : s;
}

int decode_ws_layout(const dkv_pool* pool, int B, int max_blocks, int Hq, int hidden, DecodeWs* w) {
  const int Hkv = pool->cfg.num_kv_heads, D = pool->cfg.head_dim;
  if (B < 1 || B > 32) return set_error(DKV_ERR_UNSUPPORTED, "decode: batch must be 1..32 (got %d)", B);
  if (max_blocks < 1) return set_error(DKV_ERR_ARG, "decode: max_blocks must be >= 1");
  if (hidden < 64 || hidden % 64) return set_error(DKV_ERR_UNSUPPORTED, "decode: hidden must be a positive multiple of 64");
  if (Hq < Hkv || Hq % Hkv) return set_error(DKV_ERR_ARG, "decode: num_q_heads must be a multiple of num_kv_heads");
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(DKV_ERR_UNSUPPORTED, "decode: Hq/Hkv must be 1, 2, 4 or 8 (got %d)", G);
  w->B = B; w->Hq = Hq; w->Hkv = Hkv; w->D = D; w->G = G;
  w->rows = (Hq + 2 * Hkv) * D;
  w->max_blocks = max_blocks;
  w->hidden = hidden;
  w->S = pick_attn_splits(pool, B, Hkv, max_blocks);
  w->proj_splits = pick_proj_splits(pool, Hkv, hidden);
  size_t o = 0;
  w->off_proj_acc = o; o = align_up(o + (size_t)B * w->rows * 4, 256);
  w->off_proj_cnt = o; o = align_up(o + (size_t)Hkv * 4, 256);
  w->off_qs = o;       o = align_up(o + (size_t)B * Hq * D * 4, 256);
  w->off_snew = o;     o = align_up(o + (size_t)B * Hq * 4, 256);
  w->off_vnew = o;     o = align_up(o + (size_t)B * Hkv * D * 4, 256);
  w->off_ml = o;       o = align_up(o + (size_t)B * Hq * w->S * 8, 256);
  w->off_acc = o;      o = align_up(o + (size_t)B * Hq * w->S * D * 4, 256);
  w->total = o;
  return DKV_OK;
}

static int check_common(const dkv_pool* p, int layer, void* ws, size_t ws_bytes, const DecodeWs& w) {
  if (layer < 0 || layer >= p->cfg.num_layers) return set_error(DKV_ERR_ARG, "decode: bad layer %d", layer);
  if (!ws) return set_error(DKV_ERR_ARG, "decode: null workspace");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return set_error(DKV_ERR_ARG, "decode: workspace must be 256-byte aligned");
  if (ws_bytes < w.total)
    return set_error(DKV_ERR_ARG, "decode: workspace too small (%zu < %zu)", ws_bytes, w.total);
  return DKV_OK;
}

}  // namespace dkv

using namespace dkv;

extern "C" {

size_t dkv_decode_workspace_bytes(const dkv_pool* pool, int B, int max_blocks, int num_q_heads, int hidden) {
  if (!pool) return 0;
  DecodeWs w;
  if (decode_ws_layout(pool, B, max_blocks, num_q_heads, hidden, &w)) return 0;
  return w.total;
}

int dkv_decode_attn_splits(const dkv_pool* pool, int B, int max_blocks, int num_q_heads) {
  if (!pool) return set_error(DKV_ERR_ARG, "null pool");
  DecodeWs w;
  int rc = decode_ws_layout(pool, B, max_blocks, num_q_heads, 64, &w);
  return rc ? rc : w.S;
}

int dkv_decode_project(dkv_pool* pool, int layer, const uint16_t* x, const uint16_t* Wqkv,
                       const int32_t* block_table, const int32_t* seq_lens, const uint8_t* tier_map, int B,
                       int max_blocks, int hidden, int num_q_heads, float rope_theta, void* workspace,
                       size_t ws_bytes, void* stream) {
  if (!pool || !x || !Wqkv || !block_table || !seq_lens || !tier_map)
    return set_error(DKV_ERR_ARG, "dkv_decode_project: null argument");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(Wqkv)) & 15)
    return set_error(DKV_ERR_ARG, "dkv_decode_project: x and Wqkv must be 16-byte aligned");
  if (!(rope_theta > 0.f)) return set_error(DKV_ERR_ARG, "dkv_decode_project: rope_theta must be > 0");
  DecodeWs w;
  int rc = decode_ws_layout(pool, B, max_blocks, num_q_heads, hidden, &w);
  if (rc) return rc;
  if ((rc = check_common(pool, layer, workspace, ws_bytes, w))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  rc = cuda_check(cudaMemsetAsync(ws + w.off_proj_acc, 0, w.off_qs - w.off_proj_acc, st), "projection: clear");
  if (rc) return rc;
  ProjParams p;
  p.pool = pool->view();
  p.layer = layer;
  p.x = x;
  p.W = Wqkv;
  p.table = block_table;
  p.seq_lens = seq_lens;
  p.tier_map = tier_map;
  p.max_blocks = max_blocks;
  p.B = B; p.H = hidden; p.Hq = num_q_heads; p.Hkv = w.Hkv; p.D = w.D; p.SP = w.proj_splits;
  p.theta = (double)rope_theta;
  p.qscale = (float)(1.4426950408889634 / sqrt((double)w.D));
  p.acc = reinterpret_cast<float*>(ws + w.off_proj_acc);
  p.cnt = reinterpret_cast<int*>(ws + w.off_proj_cnt);
  p.qs = reinterpret_cast<float*>(ws + w.off_qs);
  p.snew = reinterpret_cast<float*>(ws + w.off_snew);
  p.vnew = reinterpret_cast<float*>(ws + w.off_vnew);
  const int KR = hidden / w.proj_splits;
  size_t smem = (size_t)B * KR * 4;
  const size_t epi = (size_t)(w.D + w.G * w.D + w.D) * 4;
  if (smem < epi) smem = epi;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(proj_cudacore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    attr = true;
  }
  if (smem > 200 * 1024) return set_error(DKV_ERR_UNSUPPORTED, "projection: slice too large (raise proj_splits)");
  dim3 grid(w.proj_splits, w.Hkv);
  proj_cudacore_kernel<<<grid, kProjThreads, smem, st>>>(p);
  return cuda_check(cudaGetLastError(), "projection launch");
}

int dkv_decode_attend(dkv_pool* pool, int layer, const int32_t* block_table, const int32_t* seq_lens,
                      const uint8_t* tier_map, int B, int max_blocks, int hidden, int num_q_heads,
                      void* workspace, size_t ws_bytes, void* stream) {
  if (!pool || !block_table || !seq_lens || !tier_map)
    return set_error(DKV_ERR_ARG, "dkv_decode_attend: null argument");
  DecodeWs w;
  int rc = decode_ws_layout(pool, B, max_blocks, num_q_heads, hidden, &w);
  if (rc) return rc;
  if ((rc = check_common(pool, layer, workspace, ws_bytes, w))) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  AttnParams a;
  a.pool = pool->view();
  a.layer = layer;
  a.table = block_table;
  a.seq_lens = seq_lens;
  a.tier_map = tier_map;
  a.max_blocks = max_blocks;
  a.Hq = num_q_heads;
  a.S = w.S;
  a.qs = reinterpret_cast<const float*>(ws + w.off_qs);
  a.part_ml = reinterpret_cast<float2*>(ws + w.off_ml);
  a.part_acc = reinterpret_cast<float*>(ws + w.off_acc);
  return launch_attention(a, B, w.Hkv, w.D, w.G, (cudaStream_t)stream);
}

int dkv_decode_combine(dkv_pool* pool, int B, int max_blocks, int hidden, int num_q_heads, uint16_t* out,
                       void* workspace, size_t ws_bytes, void* stream) {
  if (!pool || !out) return set_error(DKV_ERR_ARG, "dkv_decode_combine: null argument");
  DecodeWs w;
  int rc = decode_ws_layout(pool, B, max_blocks, num_q_heads, hidden, &w);
  if (rc) return rc;
  if ((rc = check_common(pool, 0, workspace, ws_bytes, w))) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return launch_combine(B, num_q_heads, w.Hkv, w.D, w.S, reinterpret_cast<const float2*>(ws + w.off_ml),
                        reinterpret_cast<const float*>(ws + w.off_acc), reinterpret_cast<const float*>(ws + w.off_snew),
                        reinterpret_cast<const float*>(ws + w.off_vnew), out, (cudaStream_t)stream);
}

int dkv_decode_step(dkv_pool* pool, int layer, const uint16_t* x, const uint16_t* Wqkv, const int32_t* block_table,
                    const int32_t* seq_lens, const uint8_t* tier_map, int B, int max_blocks, int hidden,
                    int num_q_heads, float rope_theta, uint16_t* out, void* workspace, size_t ws_bytes,
                    void* stream) {
  if (!out) return set_error(DKV_ERR_ARG, "dkv_decode_step: null out");
  int rc = dkv_decode_project(pool, layer, x, Wqkv, block_table, seq_lens, tier_map, B, max_blocks, hidden,
                              num_q_heads, rope_theta, workspace, ws_bytes, stream);
  if (rc) return rc;
  rc = dkv_decode_attend(pool, layer, block_table, seq_lens, tier_map, B, max_blocks, hidden, num_q_heads,
                         workspace, ws_bytes, stream);
  if (rc) return rc;
  return dkv_decode_combine(pool, B, max_blocks, hidden, num_q_heads, out, workspace, ws_bytes, stream);
}

}  // extern "C"
