// Zero-copy GEMM study: C = A . B with A (bf16, M x K) in HBM and B (bf16, stored
// column-major, i.e. Bt = B^T as N x K rows) in mapped pinned host memory, fp32 result.
//
// DirectKV's motivating experiment ("「KV Cache 内存层级」系列总纲", §一, Fig. 2(a) of the
// paper): the same 10240-square product takes 65 ms when B is swapped into a 200 MB GPU
// buffer first and 1122 ms when the GPU reads host memory directly ("naive zero-copy");
// naive zero-copy inflates B's traffic to 33.5 GB (§四). DirectKV's CPU-aware tiling (§2.1)
// swaps which operand stays resident: B tiles are fetched from host once, at the price of
// re-reading the HBM operand.
//
// One persistent tcgen05 kernel implements all variants; they differ in where B lives and
// in the order output tiles are visited (128 x 256 tiles, K in steps of 64):
//   * naive zero-copy  (DKV_GEMM_NAIVE_ZERO_COPY): row-major tile order. CTAs running at the
//     same time share an A row panel (L2-resident) but each needs a different B column
//     panel, so every M tile row re-reads B over the host link.
//   * CPU-aware        (DKV_GEMM_CPU_AWARE): B-panel-major order. Two fetcher warps per
//     CTA copy each 256-column B panel from host memory into a rotating HBM panel buffer
//     (kGPanelBufs buffers of [256][K]) exactly once, publishing per-panel readiness; the
//     M tiles of that panel then read B from the buffer in HBM, so each B element crosses
//     the host link once (the L2 alone does not keep repeated host reads off the link);
//     A is re-streamed from HBM once per column panel.
//   * staged swap      (DKV_GEMM_STAGED_SWAP): cudaMemcpyAsync of the whole B into a
//     device workspace, then the kernel on device-resident operands.
//   * device           (DKV_GEMM_DEVICE): both operands already in device memory.
//
// Roles per CTA (256 threads): warp 0 lane 0 loads A tiles with TMA (128-byte swizzle);
// warps 1-2 load B tiles with 16-byte cp.async (which can read host memory) and write them
// in the same 128-byte-swizzled K-major layout; warp 3 lane 0 issues tcgen05.mma
// (M=128, N=256, K=16) into a double-buffered TMEM accumulator; warps 4-7 move finished
// accumulators TMEM -> registers -> C.
#include <cudaTypedefs.h>
#include <string.h>

#include "dkv_internal.h"
#include "dkv_umma.cuh"

namespace dkv {

int encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

constexpr int kGBM = 128, kGBN = 256, kGBK = 64;
constexpr int kGStages = 4;
constexpr int kGThreads = 320;            // 8 pipeline warps + 2 fetcher warps
constexpr int kGPanelBufs = 4;             // CPU-aware mode: rotating HBM panel buffers
constexpr int kGRowGroups = kGBN / 8;      // fetch units per panel (8 rows each)
constexpr int kGATile = kGBM * kGBK * 2;   // 16 KB
constexpr int kGBTile = kGBN * kGBK * 2;   // 32 KB
constexpr int kGStage = kGATile + kGBTile; // 48 KB
constexpr int kGBProducers = 64;           // warps 1-2

struct GemmParams {
  const uint16_t* Bt;  // [N][K] (device-accessible; host alias for zero-copy variants)
  float* C;            // [M][N]
  int M, N, K;
  int MT, NT, KB;      // tiles and k-blocks
  int order;           // 0: row-major tiles (n fastest); 1: B-panel-major (m fastest)
  int* status;
  // CPU-aware mode (panel != nullptr): B column panels are copied host -> HBM once, up to
  // kGPanelBufs panels ahead, into rotating [256][K] buffers, and read from there.
  uint16_t* panel;     // [kGPanelBufs][256][K]
  int* ready;          // [NT] fetch units of panel n landed in its buffer (of kGRowGroups)
  int* consumed;       // [NT] epilogue warps (4 per tile) that finished a tile of panel n
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Spin (with a sleep back-off and a 4 s wall-clock bound) until *p >= want.
__device__ __forceinline__ bool wait_flag_ge(const int* p, int want, int* status) {
  if (ld_acquire(p) >= want) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(256);
    if (ld_acquire(p) >= want) return true;
    if (globaltimer_ns() - t0 > 4000000000ull) {
      flag_error(status, kErrTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void proxy_fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tile_coords(const GemmParams& p, int t, int& m, int& n) {
  if (p.order == 0) {
    m = t / p.NT;
    n = t % p.NT;
  } else {
    n = t / p.MT;
    m = t % p.MT;
  }
}

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_umma_kernel(const __grid_constant__ CUtensorMap tmA, const GemmParams p) {
  extern __shared__ uint8_t gsm_raw[];
  const uint32_t base_u = smem_u32(gsm_raw);
  uint8_t* smem = gsm_raw + (((base_u + 1023u) & ~1023u) - base_u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStage);
  uint64_t* empty = full + kGStages;
  uint64_t* tfull = empty + kGStages;   // [2]
  uint64_t* tempty = tfull + 2;         // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ int s_ok[2];  // uniform wait results for the B-producer / fetcher groups
  if (tid == 0) {
    s_ok[0] = s_ok[1] = 1;
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&full[i], 1 + kGBProducers);  // A producer + 64 B-producer threads
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = p.MT * p.NT;

  if (warp == 0) {
    // ------------------------------------------------------------- A producer (TMA)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        int m, n;
        tile_coords(p, t, m, n);
        for (int kb = 0; kb < p.KB; ++kb, ++it) {
          const int st = it % kGStages;
          const uint32_t k = it / kGStages;
          if (k > 0 && !mbar_wait_bounded(&empty[st], (k - 1) & 1, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[st], kGATile);
          tma_load_2d(smem + st * kGStage, &tmA, kb * kGBK, m * kGBM, &full[st]);
        }
      }
    }
  } else if (warp <= 2) {
    // --------------------------------------- B producers (cp.async, host or device)
    const int bt = tid - 32;  // 0..63
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      int m, n;
      tile_coords(p, t, m, n);
      const uint16_t* src0 = p.panel ? p.panel + (int64_t)(n % kGPanelBufs) * kGBN * p.K
                                     : p.Bt + (int64_t)n * kGBN * p.K;
      if (p.panel) {  // the whole column panel must have landed in its HBM buffer
        if (bt == 0 && !wait_flag_ge(p.ready + n, kGRowGroups, p.status)) s_ok[0] = 0;
        named_bar_sync(2, kGBProducers);
        if (!s_ok[0]) break;  // same value in every producer thread: leave together
      }
      for (int kb = 0; kb < p.KB; ++kb, ++it) {
        const int st = it % kGStages;
        const uint32_t k = it / kGStages;
        if (k > 0 && !mbar_wait_bounded(&empty[st], (k - 1) & 1, p.status)) {
          ok = false;
          break;
        }
        uint8_t* bdst = smem + st * kGStage + kGATile;
#pragma unroll 8
        for (int c = 0; c < (kGBN * 8) / kGBProducers; ++c) {
          const int idx = c * kGBProducers + bt;  // 16-byte chunk of the 256 x 128-byte tile
          const int r = idx >> 3, ch = idx & 7;
          cp_async16(bdst + r * 128 + ((ch ^ (r & 7)) << 4), src0 + (int64_t)r * p.K + kb * kGBK + ch * 8);
        }
        cp_async_arrive_noinc(&full[st]);
      }
    }
    cp_async_wait_all();
  } else if (warp == 3) {
    // ------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(kGBM, kGBN);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = local >> 1;
        if (use > 0 && !mbar_wait_bounded(&tempty[buf], (use - 1) & 1, p.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem + buf * kGBN;
        for (int kb = 0; kb < p.KB; ++kb, ++it) {
          const int st = it % kGStages;
          if (!mbar_wait_bounded(&full[st], (it / kGStages) & 1, p.status)) {
            ok = false;
            break;
          }
          proxy_fence_async_smem();  // B was written through the generic proxy (cp.async)
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + st * kGStage);
          const uint32_t b0 = a0 + kGATile;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(dt, umma_desc_k_sw128(a0 + kk * 32), umma_desc_k_sw128(b0 + kk * 32), idesc,
                     (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[st]);
        }
        umma_commit(&tfull[buf]);
      }
    }
  } else if (warp >= 8) {
    // ----------------------------------------- fetchers (CPU-aware mode, warps 8-9)
    // The fetchers of all CTAs walk the B column panels in order, in units of 8 whole rows
    // of Bt (8 x K contiguous bytes x 2: sequential reads of host memory); unit i of the
    // global sequence is copied by CTA i mod gridDim.x from host into the panel's HBM
    // buffer, so every B element crosses the host link exactly once. A panel is usable once
    // all of its units have landed (ready[q] == kGRowGroups). The fetchers run ahead of the
    // GEMM by up to kGPanelBufs panels: a buffer is refilled only after every tile of its
    // previous panel has been computed.
    if (p.panel) {
      const int ft = tid - 256, fw = ft >> 5;  // fetcher thread 0..63, warp 0..1
      const int seg = (p.K + 255) / 256;       // 512-byte segments per row (last may be partial)
      for (int i = blockIdx.x; i < p.NT * kGRowGroups; i += gridDim.x) {
        const int q = i / kGRowGroups, rg = i % kGRowGroups;
        if (q >= kGPanelBufs) {
          if (ft == 0 && !wait_flag_ge(p.consumed + (q - kGPanelBufs), 4 * p.MT, p.status)) s_ok[1] = 0;
          named_bar_sync(3, 64);
          if (!s_ok[1]) break;  // same value in every fetcher thread
        }
        // warp fw copies rows rg*8 + fw*4 .. +3, 512 bytes per warp instruction
        const int64_t row0 = (int64_t)q * kGBN + rg * 8 + fw * 4;
        const uint16_t* src0 = p.Bt + row0 * p.K + lane * 8;
        uint16_t* dst0 = p.panel + ((int64_t)(q % kGPanelBufs) * kGBN + rg * 8 + fw * 4) * p.K + lane * 8;
        const int total = 4 * seg;  // (row, segment) pairs of this warp
        for (int c0 = 0; c0 < total; c0 += 8) {
          uint4 v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int c = c0 + j;
            if (c < total && (c % seg) * 256 + lane * 8 < p.K)
              v[j] = __ldcs(reinterpret_cast<const uint4*>(src0 + (int64_t)(c / seg) * p.K + (c % seg) * 256));
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int c = c0 + j;
            if (c < total && (c % seg) * 256 + lane * 8 < p.K)
              *reinterpret_cast<uint4*>(dst0 + (int64_t)(c / seg) * p.K + (c % seg) * 256) = v[j];
          }
        }
        __threadfence();
        named_bar_sync(3, 64);
        if (ft == 0) red_release_add(p.ready + q, 1);
      }
    }
  } else {
    // ------------------------------------------------- epilogue (warps 4-7: TMEM lanes)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint32_t local = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
      int m, n;
      tile_coords(p, t, m, n);
      const int buf = local & 1;
      if (!mbar_wait_bounded(&tfull[buf], (local >> 1) & 1, p.status)) break;
      tc_fence_after();
      float* crow = p.C + (int64_t)(m * kGBM + row) * p.N + n * kGBN;
      for (int c0 = 0; c0 < kGBN; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kGBN + c0), v);
        float4* dst = reinterpret_cast<float4*>(crow + c0);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
        dst[2] = make_float4(v[8], v[9], v[10], v[11]);
        dst[3] = make_float4(v[12], v[13], v[14], v[15]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[buf]);
        if (p.consumed) atomicAdd(p.consumed + n, 1);  // this warp no longer needs panel n
      }
    }
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

static size_t gemm_smem_bytes() { return 1024 + (size_t)kGStages * kGStage + 256; }

static int launch_gemm_kernel(const uint16_t* A, const uint16_t* Bt, float* C, int M, int N, int K, int order,
                              int* status, uint16_t* panel, int* ready, int* consumed, cudaStream_t st) {
  CUtensorMap tmA;
  int rc = encode_bf16_2d(&tmA, A, (uint64_t)M, (uint64_t)K, kGBM);
  if (rc) return rc;
  static bool attr = false;
  static int sms = 148;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)gemm_smem_bytes());
    if (e != cudaSuccess) return cuda_check(e, "gemm: smem attribute");
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    attr = true;
  }
  GemmParams p;
  p.Bt = Bt;
  p.C = C;
  p.M = M; p.N = N; p.K = K;
  p.MT = M / kGBM; p.NT = N / kGBN; p.KB = K / kGBK;
  p.order = order;
  p.status = status;
  p.panel = panel;
  p.ready = ready;
  p.consumed = consumed;
  const int tiles = p.MT * p.NT;
  const int grid = tiles < sms ? tiles : sms;
  gemm_umma_kernel<<<grid, kGThreads, gemm_smem_bytes(), st>>>(tmA, p);
  return cuda_check(cudaGetLastError(), "gemm launch");
}

}  // namespace dkv

using namespace dkv;

extern "C" {

// Workspace: [status word | 256 B] [CPU-aware: ready flags, consumed counters, panel
// buffers] or [staged swap: the copy of B].
static size_t gemm_flags_bytes(int N, int K) {
  (void)K;
  return align_up((size_t)(N / kGBN) * 4 * 2, 256);
}

size_t dkv_gemm_workspace_bytes(int variant, int M, int N, int K) {
  (void)M;
  if (variant == DKV_GEMM_STAGED_SWAP) return 256 + align_up((size_t)N * K * 2, 256);
  if (variant == DKV_GEMM_CPU_AWARE) return 256 + gemm_flags_bytes(N, K) + (size_t)kGPanelBufs * kGBN * K * 2;
  return 256;  // status word
}

int dkv_gemm(int variant, const uint16_t* A, const uint16_t* Bt, float* C, int M, int N, int K, void* workspace,
             size_t ws_bytes, void* stream) {
  if (!A || !Bt || !C || !workspace) return set_error(DKV_ERR_ARG, "dkv_gemm: null argument");
  if (variant < DKV_GEMM_CPU_AWARE || variant > DKV_GEMM_DEVICE)
    return set_error(DKV_ERR_ARG, "dkv_gemm: unknown variant %d", variant);
  if (M <= 0 || N <= 0 || K <= 0 || M % kGBM || N % kGBN || K % kGBK)
    return set_error(DKV_ERR_UNSUPPORTED, "dkv_gemm: need M %% 128 == 0, N %% 256 == 0, K %% 64 == 0");
  if (ws_bytes < dkv_gemm_workspace_bytes(variant, M, N, K))
    return set_error(DKV_ERR_ARG, "dkv_gemm: workspace too small");
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(Bt) | reinterpret_cast<uintptr_t>(C) |
       reinterpret_cast<uintptr_t>(workspace)) & 255)
    return set_error(DKV_ERR_ARG, "dkv_gemm: pointers must be 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  int rc0 = cuda_check(cudaMemsetAsync(status, 0, sizeof(int), st), "dkv_gemm: clear status");
  if (rc0) return rc0;
  const uint16_t* b = Bt;
  int order = 0;
  uint16_t* panel = nullptr;
  int *ready = nullptr, *consumed = nullptr;
  if (variant == DKV_GEMM_CPU_AWARE) {
    order = 1;
    ready = reinterpret_cast<int*>(ws + 256);
    consumed = ready + (size_t)(N / kGBN);
    panel = reinterpret_cast<uint16_t*>(ws + 256 + gemm_flags_bytes(N, K));
    int rc = cuda_check(cudaMemsetAsync(ready, 0, gemm_flags_bytes(N, K), st), "dkv_gemm: clear flags");
    if (rc) return rc;
  }
  if (variant == DKV_GEMM_STAGED_SWAP) {
    uint16_t* staged = reinterpret_cast<uint16_t*>(ws + 256);
    int rc = cuda_check(cudaMemcpyAsync(staged, Bt, (size_t)N * K * 2, cudaMemcpyDefault, st), "dkv_gemm: swap-in copy");
    if (rc) return rc;
    b = staged;
  }
  return launch_gemm_kernel(A, b, C, M, N, K, order, status, panel, ready, consumed, st);
}

}  // extern "C"
