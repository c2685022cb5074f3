// QKV projection on the 5th-generation tensor cores, fused with RoPE and the single
// cache write of the new token's K/V.
//
// DirectKV ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", 核心方法) fuses KV generation
// with attention so the new K/V are consumed on chip and written once. Decode batches are
// small (B <= 32), so the product qkv = Wqkv . x is computed "swap-AB": 128 rows of W are
// the M = 128 operand and the batch is the N operand (N = 16 or 32, zero-padded by TMA),
// accumulating fp32 in TMEM.
//
//  * Work unit: one 128-row tile of W = one head's D rows (D = 128) or two heads (D = 64).
//    Heads never straddle tiles, so every RoPE pair (i, i + D/2) lives in one tile.
//  * A cluster of CS CTAs owns one tile and splits the hidden (reduction) dimension; each
//    CTA streams its slice of the tile once through a TMA ring (128-byte swizzle, one
//    elected thread issues tcgen05.mma M=128, N, K=16 per 16 columns). Clusters are small
//    and CTAs light (two per SM), so the whole GPU streams W concurrently.
//  * While W streams, the otherwise idle warps look up, for every batch column b the CTA
//    will finish (b = r, r + CS, ... for cluster rank r), its position and cache-slot
//    addresses, and compute the RoPE (cos, sin) of each rotation pair at that position.
//  * Each CTA then copies its partial [128 x N] accumulator from TMEM into its own shared
//    memory; after one cluster barrier the CTA of rank r reads columns b = r, r + CS, ...
//    from all CS partials (distributed shared memory; independent loads, issued together)
//    and sums them in rank order (a fixed order: deterministic). It then finishes them:
//    q heads rotated and scaled by log2(e)/sqrt(D) for the log2-domain
//    softmax, the key head rotated and rounded to bf16 (k_hat), the value head rounded
//    (v_hat); k_hat and v_hat are written once into the cache slot and, as fp32, into the
//    workspace for the new token's attention term.
// Reading W is the whole cost (HBM-bound); the tensor cores only remove the CUDA-core FMA
// bound that B >= 16 would otherwise hit.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include "dkv_internal.h"
#include "dkv_umma.cuh"

namespace cg = cooperative_groups;

namespace dkv {

constexpr int kPThreads = 128;
constexpr int kWTile = 128 * 128;  // 128 rows x 64 bf16 (bytes)

struct ProjParams {
  PoolView pool;
  int layer;
  const int32_t* table;
  const int32_t* seq_lens;
  const uint8_t* tier_map;
  int max_blocks;
  int B, H, Hq, Hkv, D, G;
  int ppt, nt, Npad, CS, KB, nst;
  int slots;                           // batch columns a CTA finishes: ceil(B / CS)
  int pdl;                             // launched with programmatic dependent launch
  int off_part, off_rope, off_cols, off_bars;  // shared-memory carve-up (bytes)
  float qscale;
  float* qs;              // [B][Hq][D]
  float* knew;            // [B][Hkv][D]
  float* vnew;            // [B][Hkv][D]
  int* attn_cnt;          // [B][Hkv] split-arrival counters of the attention stage (reset here)
  double inv_freq[64];    // theta^(-2i/D), i < D/2, computed on the host in fp64
};

// Split cluster barrier: arrive (releasing this thread's prior memory operations) and wait
// (acquiring the other CTAs' released ones); every thread of every CTA takes both.
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Epilogue lookups done while W streams, one per batch column the CTA finishes: the
// position and the two cache-slot addresses (key, value) of kv head g (null where the
// table entry was rejected and flagged).
struct EpiCol {
  uint16_t* dst[2];
  int pos;
  int pad;
};

// Sum, for each column b = rank + CS * it (it < slots, b < B) this CTA finishes, row `row`
// of the CS partial accumulators part[b][128] held by the cluster's CTAs, in rank order,
// into colsum[it][row]. Columns go in groups of 8, each group's 8 x CS remote reads issued
// together.
template <int CS>
__device__ __forceinline__ void pull_columns(cg::cluster_group& cluster, float* part, float* colsum, int rank,
                                             int slots, int B, int row) {
  const float* peer[CS];
#pragma unroll
  for (int q = 0; q < CS; ++q) peer[q] = cluster.map_shared_rank(part, q);
  for (int it0 = 0; it0 < slots; it0 += 8) {
    float v[8][CS];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = rank + CS * (it0 + i);
      const bool ok = it0 + i < slots && b < B;
#pragma unroll
      for (int q = 0; q < CS; ++q) v[i][q] = ok ? peer[q][b * 128 + row] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float x = 0.f;
#pragma unroll
      for (int q = 0; q < CS; ++q) x += v[i][q];
      if (it0 + i < slots) colsum[(it0 + i) * 128 + row] = x;
    }
  }
}

// First W row of piece (head) `pc` of kv-head group g: pieces 0..G-1 are the group's q
// heads, G its key head, G+1 its value head.
__device__ __forceinline__ int piece_row(const ProjParams& p, int g, int pc) {
  if (pc < p.G) return (g * p.G + pc) * p.D;
  if (pc == p.G) return (p.Hq + g) * p.D;
  return (p.Hq + p.Hkv + g) * p.D;
}

__global__ void __launch_bounds__(kPThreads, 2)
    proj_umma_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     const ProjParams p) {
  extern __shared__ uint8_t psmem_raw[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tile = blockIdx.y;            // over (g, t)
  const int g = tile / p.nt, t = tile % p.nt;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // 1024-byte aligned carve-up: ring | partial accumulator | RoPE table | column lookups |
  // barriers | tmem slot
  const uint32_t base_u = smem_u32(psmem_raw);
  uint8_t* smem = psmem_raw + (((base_u + 1023u) & ~1023u) - base_u);
  const int xtile = p.Npad * 128;
  const int stage_bytes = kWTile + xtile;
  const int nst = p.nst;
  const int slots = p.slots;
  float* part = reinterpret_cast<float*>(smem + p.off_part);     // [B][128] this CTA's partial
  float2* rope = reinterpret_cast<float2*>(smem + p.off_rope);   // [slots][D/2] (cos, sin)
  EpiCol* cols = reinterpret_cast<EpiCol*>(smem + p.off_cols);   // [slots]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint64_t* empty = full + nst;
  uint64_t* done = empty + nst;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  // TMEM first: a second CTA is placed on this SM only once this one has given up its
  // allocation permit (tmem_alloc relinquishes it), so the allocation leads the prologue
  if (warp == 0) tmem_alloc(tmem_slot, 32);
  if (tid == 32) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int kb0 = (int)((int64_t)p.KB * rank / p.CS);
  const int kb1 = (int)((int64_t)p.KB * (rank + 1) / p.CS);
  const int nsteps = kb1 - kb0;
  int np = 2 + p.G - t * p.ppt;  // heads in this tile
  if (np > p.ppt) np = p.ppt;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    // W does not depend on the kernel ahead in the stream (weights are never written by
    // it): the first ring's W tiles are loaded, and the rest of this CTA's W slice is
    // prefetched into L2, before waiting for it; x and everything after come once it has
    // completed. (The attention streams its KV with an evict-first L2 policy, so a
    // projection launched early behind it keeps its prefetched W.)
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    const int pre = nsteps < nst ? nsteps : nst;
    for (int s = 0; s < pre; ++s) {
      uint8_t* wdst = smem + s * stage_bytes;
      mbar_arrive_expect_tx(&full[s], (uint32_t)(np * p.D * 128 + xtile));
      for (int i = 0; i < np; ++i)
        tma_load_2d(wdst + i * p.D * 128, &tmW, (kb0 + s) * 64, piece_row(p, g, t * p.ppt + i), &full[s]);
    }
    if (p.pdl)  // only worth its issue cost (~0.1 us each) when there is a kernel to overlap
      for (int s = pre; s < nsteps; ++s)
        for (int i = 0; i < np; ++i) tma_prefetch_l2_2d(&tmW, (kb0 + s) * 64, piece_row(p, g, t * p.ppt + i));
    griddep_wait();
    for (int s = 0; s < pre; ++s) tma_load_2d(smem + s * stage_bytes + kWTile, &tmX, (kb0 + s) * 64, 0, &full[s]);
    for (int s = pre; s < nsteps; ++s) {
      const int st = s % nst, n = s / nst;
      if (n > 0 && !mbar_wait_bounded(&empty[st], (n - 1) & 1, p.pool.status)) break;
      const int kb = kb0 + s;
      uint8_t* wdst = smem + st * stage_bytes;
      mbar_arrive_expect_tx(&full[st], (uint32_t)(np * p.D * 128 + xtile));
      for (int i = 0; i < np; ++i)
        tma_load_2d(wdst + i * p.D * 128, &tmW, kb * 64, piece_row(p, g, t * p.ppt + i), &full[st]);
      tma_load_2d(wdst + kWTile, &tmX, kb * 64, 0, &full[st]);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t idesc = umma_idesc_bf16_f32(128, p.Npad);
    for (int s = 0; s < nsteps; ++s) {
      const int st = s % nst;
      if (!mbar_wait_bounded(&full[st], (s / nst) & 1, p.pool.status)) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + st * stage_bytes);
      const uint32_t b0 = a0 + kWTile;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_f16(tmem, umma_desc_k_sw128(a0 + kk * 32), umma_desc_k_sw128(b0 + kk * 32), idesc,
                 (s > 0 || kk > 0) ? 1u : 0u);
      umma_commit(&empty[st]);
    }
    umma_commit(done);
  } else if (warp >= 2) {
    // ------------------------------------ epilogue tables, while W streams (warps 2, 3)
    // the tables and positions belong to the kernels ahead in the stream
    griddep_wait();
    if (tid == 64) griddep_launch_dependents();
    const int et = tid - 64;
    for (int it = et; it < slots; it += 64) {  // position and cache-slot addresses per column
      const int b = rank + p.CS * it;
      EpiCol c;
      c.dst[0] = c.dst[1] = nullptr;
      c.pos = 0;
      c.pad = 0;
      if (b < p.B) {
        const int pos = p.seq_lens[b];
        c.pos = pos;
        const int64_t jb = pos >= 0 ? (int64_t)pos / p.pool.T : -1;
        if (jb < 0 || jb >= p.max_blocks) {
          flag_error(p.pool.status, kErrCtxTooLong);
        } else {
          const int tier = p.tier_map[(int64_t)b * p.max_blocks + jb];
          const int64_t phys = p.table[(int64_t)b * p.max_blocks + jb];
          if (tier > 1) {
            flag_error(p.pool.status, kErrBadTier);
          } else if (phys < 0 || phys >= tier_blocks(p.pool, tier)) {
            flag_error(p.pool.status, kErrBadBlock);
          } else {
            const int64_t slot = (int64_t)(pos % p.pool.T) * p.D;
            const int64_t ok = chunk_offset(p.pool, tier, p.layer, phys, 0, g) + slot;
            const int64_t ov = chunk_offset(p.pool, tier, p.layer, phys, 1, g) + slot;
            const int64_t n = tier_elems(p.pool, tier);
            if (DKV_DEBUG_RANGE(p.pool.status, ok, ok + p.D, n) && DKV_DEBUG_RANGE(p.pool.status, ov, ov + p.D, n)) {
              c.dst[0] = tier_base(p.pool, tier) + ok;
              c.dst[1] = tier_base(p.pool, tier) + ov;
            }
          }
        }
      }
      cols[it] = c;
    }
    if (t * p.ppt <= p.G) {  // the tile holds q or key heads: RoPE (cos, sin) per column and pair
      // rotate-half RoPE: angle pos * theta^(-2i/D) reduced mod 2*pi in fp64, then a
      // single-precision sincos
      const int half = p.D / 2;
      for (int e = et; e < slots * half; e += 64) {
        const int it = e / half, pi = e % half;
        const int b = rank + p.CS * it;
        if (b >= p.B) continue;
        const double ang = (double)p.seq_lens[b] * p.inv_freq[pi];
        const double red = ang - rint(ang * 0.15915494309189535) * 6.283185307179586;
        float sn, cn;
        sincosf((float)red, &sn, &cn);
        rope[e] = make_float2(cn, sn);
      }
    }
  }
  __syncwarp();
  griddep_wait();

  // ------------------------------------ partial accumulator: TMEM -> own shared memory
  mbar_wait_bounded(done, 0, p.pool.status);
  tc_fence_after();
  for (int c0 = 0; c0 < p.Npad; c0 += 16) {
    float v[16];
    tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (c0 + j < p.B) part[(c0 + j) * 128 + tid] = v[j];
  }
  tc_fence_before();
  if (t == 0 && rank == 0 && tid < p.B && p.attn_cnt) p.attn_cnt[(int64_t)tid * p.Hkv + g] = 0;
  cluster.sync();  // every CTA's partial is in its shared memory
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 32);

  // ------------------------------------ column reduction (rank order) + epilogue
  // thread -> tile row (head row / D of the tile, dim d = row % D of that head), mapped so
  // that the two rows of a RoPE pair (d and d + D/2) sit in lanes l and l ^ 16 of one
  // warp: the pair exchange is a shuffle, with no block barrier per sequence
  const int D = p.D, half = D / 2, wph = D / 32;  // warps per head
  const int row = (warp / wph) * D + (warp % wph) * 16 + (lane & 15) + ((lane & 16) ? half : 0);
  const int pc = t * p.ppt + row / D;     // piece (head) index within the group
  const int d = row % D, pi = d % half;   // RoPE pair index
  const bool live = row / D < np;
  // column b is finished by cluster rank b mod CS: it reads row `row` of column b from the
  // CS partials (peers' shared memory) and sums them in rank order (deterministic). A
  // remote read costs about a microsecond of latency, so all of a thread's reads (up to 8
  // columns x CS ranks) are issued before the first sum; the sums go to the ring, free
  // once the MMAs have completed.
  float* colsum = reinterpret_cast<float*>(smem);  // [slots][128]
  switch (p.CS) {
    case 1: pull_columns<1>(cluster, part, colsum, rank, slots, p.B, row); break;
    case 2: pull_columns<2>(cluster, part, colsum, rank, slots, p.B, row); break;
    case 3: pull_columns<3>(cluster, part, colsum, rank, slots, p.B, row); break;
    case 4: pull_columns<4>(cluster, part, colsum, rank, slots, p.B, row); break;
    case 5: pull_columns<5>(cluster, part, colsum, rank, slots, p.B, row); break;
    case 6: pull_columns<6>(cluster, part, colsum, rank, slots, p.B, row); break;
    case 7: pull_columns<7>(cluster, part, colsum, rank, slots, p.B, row); break;
    default: pull_columns<8>(cluster, part, colsum, rank, slots, p.B, row); break;
  }
  cluster_arrive_release();  // done with the peers' shared memory

  for (int it = 0; it < slots; ++it) {
    const int b = rank + p.CS * it;
    if (b >= p.B) break;
    float x = colsum[it * 128 + row];  // written by this thread above
    const float xp = __shfl_xor_sync(0xffffffffu, x, 16);  // the pair's other row
    if (!live) continue;
    if (pc <= p.G) {
      const float2 cs = rope[it * half + pi];
      const float y = d < half ? x * cs.x - xp * cs.y : x * cs.x + xp * cs.y;
      if (pc < p.G) {
        p.qs[((int64_t)b * p.Hq + g * p.G + pc) * D + d] = y * p.qscale;
        continue;
      }
      x = y;  // the key head: rotated, stored below
    }
    const uint16_t hb = f32_to_bf16_bits(x);
    const int kv = pc == p.G ? 0 : 1;
    (kv ? p.vnew : p.knew)[((int64_t)b * p.Hkv + g) * D + d] = __uint_as_float((uint32_t)hb << 16);
    // the single cache write: slot pos mod T of logical block pos / T (bad entries were
    // flagged by the lookup and are skipped)
    uint16_t* dst = cols[it].dst[kv];
    if (dst) dst[d] = hb;
  }
  cluster_wait_acquire();  // no CTA leaves while a peer may still read its partial
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

// Shared memory per CTA: two CTAs share an SM (228 KB, 1 KB of it reserved per CTA).
constexpr int kProjSmemBudget = 113 * 1024;

// Carve-up of one CTA's shared memory for a ring of `nst` stages; returns the total
// (including the 1024-byte alignment slack).
static int proj_smem_layout(ProjParams* p, int nst) {
  const int stage = kWTile + p->Npad * 128;
  int o = nst * stage;
  p->off_part = o;
  o += p->B * 128 * 4;
  p->off_rope = o;
  o += p->slots * (p->D / 2) * 8;
  p->off_cols = o;
  o += p->slots * (int)sizeof(EpiCol);
  o = (o + 7) / 8 * 8;
  p->off_bars = o;
  o += (2 * nst + 1) * 8 + 8;
  return 1024 + o;
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
  p.ppt = 128 / a.D;
  p.nt = (p.G + 2 + p.ppt - 1) / p.ppt;
  p.Npad = a.B <= 16 ? 16 : 32;
  p.KB = a.H / 64;
  for (int i = 0; i < a.D / 2; ++i) p.inv_freq[i] = pow(a.theta, -2.0 * (double)i / (double)a.D);
  p.attn_cnt = a.attn_cnt;
  p.pdl = a.pdl;
  p.qscale = a.qscale;
  p.qs = a.qs;
  p.knew = a.knew;
  p.vnew = a.vnew;
  CUtensorMap tmW, tmX;
  int rc = encode_bf16_2d(&tmW, a.W, (uint64_t)(a.Hq + 2 * a.Hkv) * a.D, a.H, (uint32_t)a.D);
  if (rc) return rc;
  rc = encode_bf16_2d(&tmX, a.x, (uint64_t)a.B, a.H, (uint32_t)p.Npad);
  if (rc) return rc;

  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(proj_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kProjSmemBudget);
    if (e != cudaSuccess) return cuda_check(e, "projection: smem attribute");
    attr = true;
  }
  const int tiles = a.Hkv * p.nt;
  // each cluster splits one tile's reduction dimension; about 240 CTAs in total (one wave
  // at two CTAs per SM) measured best on B200 (launches back to back, W read from HBM):
  // clusters of 5 for the 8B-shaped layer (48 tiles, 16.4 us vs 16.6 at 4, 16.7 at 3 and
  // 22.5 at 6; with W in L2 12.3 vs 14.3 and 16.4) and of 3 for the 70B-shaped one (80
  // tiles, 36.0 us vs 39.5 at 2 and 45.4 at 4)
  int CS = a.cluster > 0 ? a.cluster : (240 + tiles / 2) / tiles;
  if (CS < 1) CS = 1;
  if (CS > 8) CS = 8;
  if (CS > p.KB) CS = p.KB;
  p.CS = CS;
  p.slots = (a.B + CS - 1) / CS;
  // the deepest ring (3..6 stages) that leaves room for the epilogue areas at two CTAs/SM
  int nst = 6;
  while (nst > 3 && proj_smem_layout(&p, nst) > kProjSmemBudget) --nst;
  const int smem = proj_smem_layout(&p, nst);
  if (smem > kProjSmemBudget) return set_error(DKV_ERR_UNSUPPORTED, "projection: shared memory (%d B)", smem);
  p.nst = nst;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[2] = {};
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CS;
  at[0].val.clusterDim.y = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(CS, tiles, 1);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = a.pdl ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, proj_umma_kernel, tmW, tmX, p);
  return cuda_check(e, "projection launch");
}

}  // namespace dkv
