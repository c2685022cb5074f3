// QKV projection on the 5th-generation tensor cores, fused with RoPE, the single cache
// write of the new token's K/V, and the new token's attention term.
//
// DirectKV ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", 核心方法) fuses KV generation
// with attention so the new K/V are consumed on chip and written once. Here one thread-
// block cluster owns one kv-head group: the (G+2)*D rows of Wqkv holding the group's G
// query heads, its key head and its value head. Decode batches are small (B <= 32), so
// the product is computed "swap-AB": W rows are the M = 128 operand and the batch is the
// N operand (N = 16 or 32, zero-padded by TMA), accumulating fp32 in TMEM:
//
//   * the cluster's CS CTAs split the hidden (reduction) dimension; each CTA streams its
//     slice of the group's W rows once through an 8-stage TMA ring (128-byte swizzle),
//     one elected thread issues tcgen05.mma (M=128, N, K=16) per 16 columns;
//   * each CTA moves its partial [rows x N] accumulators TMEM -> shared memory; after a
//     cluster barrier, the CTA that owns batch column b sums the CS partials of that column
//     in rank order through distributed shared memory (a fixed order, so the result is
//     deterministic) and runs the epilogue for b: RoPE on q and k, q scaled by
//     log2(e)/sqrt(D), bf16 k_hat / v_hat written once into the cache slot, and the new
//     token's score s_new = q . k_hat for each of the G heads.
// The weight read is the whole cost (HBM-bound); the tensor cores only remove the
// CUDA-core FMA bound that B >= 16 would otherwise hit.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include "dkv_internal.h"
#include "dkv_umma.cuh"

namespace cg = cooperative_groups;

namespace dkv {

constexpr int kPThreads = 128;
constexpr int kPStages = 8;
constexpr int kWTile = 128 * 128;  // 128 rows x 64 bf16 (bytes)

struct ProjParams {
  PoolView pool;
  int layer;
  const int32_t* table;
  const int32_t* seq_lens;
  const uint8_t* tier_map;
  int max_blocks;
  int B, H, Hq, Hkv, D, G;
  int npieces, nt, ppt, Npad, CS, KB, tmem_cols;
  double theta;
  float qscale;
  float* qs;
  float* snew;
  float* vnew;
};

__device__ __forceinline__ int piece_row(const ProjParams& p, int g, int pc) {
  if (pc < p.G) return (g * p.G + pc) * p.D;
  if (pc == p.G) return (p.Hq + g) * p.D;
  return (p.Hq + p.Hkv + g) * p.D;
}

__global__ void __launch_bounds__(kPThreads, 1)
    proj_umma_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     const ProjParams p) {
  extern __shared__ uint8_t psmem_raw[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int g = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // 1024-byte aligned carve-up: ring | barriers | tmem slot
  const uint32_t base_u = smem_u32(psmem_raw);
  uint8_t* smem = psmem_raw + (((base_u + 1023u) & ~1023u) - base_u);
  const int xtile = p.Npad * 128;
  const int stage_bytes = kWTile + xtile;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPStages * stage_bytes);
  uint64_t* empty = full + kPStages;
  uint64_t* done = empty + kPStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  float* part = reinterpret_cast<float*>(smem);  // [nt][Npad][128], aliases the ring later
  float* fsum = reinterpret_cast<float*>(smem + kPStages * stage_bytes + 256);  // [npieces*D]
  float2* cs = reinterpret_cast<float2*>(fsum + p.npieces * p.D);              // [D/2]

  if (tid == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int kb0 = (int)((int64_t)p.KB * rank / p.CS);
  const int kb1 = (int)((int64_t)p.KB * (rank + 1) / p.CS);
  const int nsteps = (kb1 - kb0) * p.nt;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    for (int s = 0; s < nsteps; ++s) {
      const int st = s % kPStages, n = s / kPStages;
      if (n > 0 && !mbar_wait_bounded(&empty[st], (n - 1) & 1, p.pool.status)) break;
      const int kb = kb0 + s / p.nt, t = s % p.nt;
      uint8_t* wdst = smem + st * stage_bytes;
      int np = p.npieces - t * p.ppt;
      if (np > p.ppt) np = p.ppt;
      mbar_arrive_expect_tx(&full[st], (uint32_t)(np * p.D * 128 + xtile));
      for (int i = 0; i < np; ++i)
        tma_load_2d(wdst + i * p.D * 128, &tmW, kb * 64, piece_row(p, g, t * p.ppt + i), &full[st]);
      tma_load_2d(wdst + kWTile, &tmX, kb * 64, 0, &full[st]);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t idesc = umma_idesc_bf16_f32(128, p.Npad);
    for (int s = 0; s < nsteps; ++s) {
      const int st = s % kPStages;
      if (!mbar_wait_bounded(&full[st], (s / kPStages) & 1, p.pool.status)) break;
      tc_fence_after();
      const int kb = kb0 + s / p.nt, t = s % p.nt;
      const uint32_t a0 = smem_u32(smem + st * stage_bytes);
      const uint32_t b0 = a0 + kWTile;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_f16(tmem + t * p.Npad, umma_desc_k_sw128(a0 + kk * 32), umma_desc_k_sw128(b0 + kk * 32), idesc,
                 (kb > kb0 || kk > 0) ? 1u : 0u);
      umma_commit(&empty[st]);
    }
    umma_commit(done);
  }
  __syncwarp();

  // ------------------------------------------------ TMEM -> shared partial [t][n][row]
  mbar_wait_bounded(done, 0, p.pool.status);
  tc_fence_after();
  for (int t = 0; t < p.nt; ++t) {
    for (int c0 = 0; c0 < p.Npad; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(t * p.Npad + c0), v);
#pragma unroll
      for (int j = 0; j < 16; ++j) part[(t * p.Npad + c0 + j) * 128 + tid] = v[j];
    }
  }
  tc_fence_before();
  cluster.sync();  // every CTA's partial is in its shared memory

  // --------------------------------------- per-batch reduction over the cluster + epilogue
  const int D = p.D, G = p.G, half = D / 2;
  const int nrows = p.npieces * D;
  for (int b = rank; b < p.B; b += p.CS) {
    for (int lr = tid; lr < nrows; lr += kPThreads) {
      const int idx = ((lr >> 7) * p.Npad + b) * 128 + (lr & 127);
      float s = 0.f;
      for (int q = 0; q < p.CS; ++q) s += cluster.map_shared_rank(part, q)[idx];
      fsum[lr] = s;
    }
    const int pos = p.seq_lens[b];
    for (int i = tid; i < half; i += kPThreads) {
      const double inv = pow(p.theta, -2.0 * (double)i / (double)D);
      double sn, cn;
      sincos((double)pos * inv, &sn, &cn);
      cs[i] = make_float2((float)cn, (float)sn);
    }
    const int64_t jb = pos >= 0 ? (int64_t)pos / p.pool.T : -1;
    const int slot = pos >= 0 ? pos % p.pool.T : 0;
    int tier = -1;
    int64_t phys = -1;
    bool ok = jb >= 0 && jb < p.max_blocks;
    if (ok) {
      tier = p.tier_map[(int64_t)b * p.max_blocks + jb];
      phys = p.table[(int64_t)b * p.max_blocks + jb];
      if (tier > 1) {
        ok = false;
        if (tid == 0) flag_error(p.pool.status, kErrBadTier);
      } else if (phys < 0 || phys >= tier_blocks(p.pool, tier)) {
        ok = false;
        if (tid == 0) flag_error(p.pool.status, kErrBadBlock);
      }
    } else if (tid == 0) {
      flag_error(p.pool.status, kErrCtxTooLong);
    }
    uint16_t* kdst = ok ? tier_base(p.pool, tier) + chunk_offset(p.pool, tier, p.layer, phys, 0, g) + (int64_t)slot * D : nullptr;
    uint16_t* vdst = ok ? tier_base(p.pool, tier) + chunk_offset(p.pool, tier, p.layer, phys, 1, g) + (int64_t)slot * D : nullptr;
    __syncthreads();
    // q heads and the key head: rotate-half RoPE; q scaled for the log2-domain softmax
    for (int it = tid; it < (G + 1) * half; it += kPThreads) {
      const int pc = it / half, i = it % half;
      const float x0 = fsum[pc * D + i], x1 = fsum[pc * D + i + half];
      const float2 c = cs[i];
      const float y0 = x0 * c.x - x1 * c.y;
      const float y1 = x1 * c.x + x0 * c.y;
      if (pc < G) {
        const float q0 = y0 * p.qscale, q1 = y1 * p.qscale;
        fsum[pc * D + i] = q0;
        fsum[pc * D + i + half] = q1;
        float* qd = p.qs + ((int64_t)b * p.Hq + g * G + pc) * D;
        qd[i] = q0;
        qd[i + half] = q1;
      } else {
        const uint16_t k0 = f32_to_bf16_bits(y0), k1 = f32_to_bf16_bits(y1);
        fsum[pc * D + i] = __uint_as_float((uint32_t)k0 << 16);
        fsum[pc * D + i + half] = __uint_as_float((uint32_t)k1 << 16);
        if (kdst) {
          kdst[i] = k0;
          kdst[i + half] = k1;
        }
      }
    }
    for (int d = tid; d < D; d += kPThreads) {
      const uint16_t vb = f32_to_bf16_bits(fsum[(G + 1) * D + d]);
      p.vnew[((int64_t)b * p.Hkv + g) * D + d] = __uint_as_float((uint32_t)vb << 16);
      if (vdst) vdst[d] = vb;
    }
    __syncthreads();
    for (int h = warp; h < G; h += kPThreads / 32) {
      float sacc = 0.f;
      for (int d = lane; d < D; d += 32) sacc = fmaf(fsum[h * D + d], fsum[G * D + d], sacc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
      if (lane == 0) p.snew[(int64_t)b * p.Hq + g * G + h] = sacc;
    }
    __syncthreads();
  }
  cluster.sync();  // no CTA leaves while others may still read its partial
  if (warp == 0) tmem_dealloc(tmem, p.tmem_cols);
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] array, box [box_rows][64], 128B swizzle.
int encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return set_error(DKV_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(DKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DKV_OK;
}

static size_t proj_smem_bytes(int Npad, int npieces, int D) {
  return 1024 + (size_t)kPStages * (kWTile + Npad * 128) + 256 + (size_t)npieces * D * 4 + (size_t)D * 4;
}

int launch_projection(const ProjArgs& a, cudaStream_t st) {
  ProjParams p;
  memset(&p, 0, sizeof(p));
  p.pool = a.pool;
  p.layer = a.layer;
  p.table = a.table;
  p.seq_lens = a.seq_lens;
  p.tier_map = a.tier_map;
  p.max_blocks = a.max_blocks;
  p.B = a.B; p.H = a.H; p.Hq = a.Hq; p.Hkv = a.Hkv; p.D = a.D; p.G = a.Hq / a.Hkv;
  p.npieces = p.G + 2;
  p.ppt = 128 / a.D;
  p.nt = (p.npieces + p.ppt - 1) / p.ppt;
  p.Npad = a.B <= 16 ? 16 : 32;
  p.KB = a.H / 64;
  p.theta = a.theta;
  p.qscale = a.qscale;
  p.qs = a.qs;
  p.snew = a.snew;
  p.vnew = a.vnew;
  int cols = 32;
  while (cols < p.nt * p.Npad) cols <<= 1;
  p.tmem_cols = cols;
  if (cols > 512) return set_error(DKV_ERR_UNSUPPORTED, "projection: accumulators exceed TMEM");
  const size_t smem = proj_smem_bytes(p.Npad, p.npieces, p.D);
  // the partial-sum area aliases the stage ring
  if ((size_t)p.nt * p.Npad * 128 * 4 > (size_t)kPStages * (kWTile + p.Npad * 128))
    return set_error(DKV_ERR_UNSUPPORTED, "projection: group too large");

  CUtensorMap tmW, tmX;
  int rc = encode_bf16_2d(&tmW, a.W, (uint64_t)(a.Hq + 2 * a.Hkv) * a.D, a.H, (uint32_t)a.D);
  if (rc) return rc;
  rc = encode_bf16_2d(&tmX, a.x, (uint64_t)a.B, a.H, (uint32_t)p.Npad);
  if (rc) return rc;

  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(proj_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)proj_smem_bytes(32, 10, 128));
    if (e != cudaSuccess) return cuda_check(e, "projection: smem attribute");
    e = cudaFuncSetAttribute(proj_umma_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return cuda_check(e, "projection: cluster attribute");
    attr = true;
  }
  int CS = a.cluster > 0 ? a.cluster : 16;
  if (CS > p.KB) CS = p.KB;
  if (CS > 16) CS = 16;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1] = {};
  at[0].id = cudaLaunchAttributeClusterDimension;
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  // shrink the cluster until the device can co-schedule it
  for (;;) {
    at[0].val.clusterDim.x = CS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(CS, a.Hkv, 1);
    int nclusters = 0;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&nclusters, proj_umma_kernel, &cfg);
    if (e == cudaSuccess && nclusters >= 1) break;
    cudaGetLastError();
    if (CS == 1) return set_error(DKV_ERR_UNSUPPORTED, "projection: no cluster size fits");
    CS = CS > 8 ? 8 : CS / 2;
  }
  p.CS = CS;
  cudaError_t e = cudaLaunchKernelEx(&cfg, proj_umma_kernel, tmW, tmX, p);
  return cuda_check(e, "projection launch");
}

}  // namespace dkv
