// Placement plans applied on the device, and the multi-layer decode step as one CUDA graph.
//
// A plan (format in dkv_placement.h) lists block moves between the tiers and the table
// entries they change. The apply kernel reads it where the block manager wrote it — pinned
// host memory mapped into the device address space — so the launch has fixed arguments
// and can be replayed inside a graph while the host writes the next plan. With zero-copy
// reads of the host tier every address of a decode step is fixed (the series page
// "「KV Cache 内存层级」系列总纲", §2.1 DirectKV and §五, names the dynamic addresses of
// staged copies as what keeps offload from CUDA-graph replay); the graph below holds the
// plan's application and every layer's decode step.
#include <stddef.h>

#include <new>

#include "dkv_internal.h"
#include "../../include/dkv_placement.h"

namespace dkv {

// One CTA per (move, layer) unit at a time: 2*Hkv*T*D bf16 (64 KiB at Hkv=8, D=128) in
// 16-byte pieces, four loads in flight per thread (the source may be host memory read over
// the host link). Then every thread takes table entries and cached-token counts.
// Plan words are read with ld.global.cv: the host rewrites the buffer between launches.
// The last CTA to finish (a counter in the pool's device scratch, reset by that CTA) sets
// the header's `applied` word in the plan buffer, which tells the block manager that the
// buffer may be rewritten.
__device__ __forceinline__ void apply_plan_body(const PoolView& pool, const uint8_t* plan, const int4 h0,
                                                const int4 h1, int4& s_move, int32_t* __restrict__ table,
                                                uint8_t* __restrict__ tier_map, int32_t* __restrict__ seq_lens,
                                                int max_rows, int max_blocks) {
  const int n_moves = h0.x, n_entries = h0.y, n_rows = h0.z;
  const int move_cap = h1.x, entry_cap = h1.y;
  const int4* moves = reinterpret_cast<const int4*>(plan + sizeof(dkv_plan_header));
  const int4* entries = moves + move_cap;
  const int32_t* lens = reinterpret_cast<const int32_t*>(entries + entry_cap);

  const int64_t chunk16 = (int64_t)2 * pool.Hkv * pool.T * pool.D / 8;
  const int64_t units = (int64_t)n_moves * pool.L;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int m = (int)(u / pool.L), layer = (int)(u % pool.L);
    __syncthreads();
    if (threadIdx.x == 0) s_move = __ldcv(moves + m);
    __syncthreads();
    const int4 mv = s_move;  // (src_tier, src_id, dst_tier, dst_id), uniform over the CTA
    if (mv.x < 0 || mv.x > 1 || mv.z < 0 || mv.z > 1 || mv.y < 0 || mv.y >= tier_blocks(pool, mv.x) ||
        mv.w < 0 || mv.w >= tier_blocks(pool, mv.z)) {
      if (threadIdx.x == 0 && layer == 0) flag_error(pool.status, kErrBadBlock);
      continue;
    }
    const int64_t so = chunk_offset(pool, mv.x, layer, mv.y, 0, 0), dof = chunk_offset(pool, mv.z, layer, mv.w, 0, 0);
    if (!DKV_DEBUG_RANGE(pool.status, so, so + chunk16 * 8, tier_elems(pool, mv.x)) ||
        !DKV_DEBUG_RANGE(pool.status, dof, dof + chunk16 * 8, tier_elems(pool, mv.z)))
      continue;
    const uint4* src = reinterpret_cast<const uint4*>(tier_base(pool, mv.x) + so);
    uint4* dst = reinterpret_cast<uint4*>(tier_base(pool, mv.z) + dof);
    int64_t c = threadIdx.x;
    for (; c + 3 * 256 < chunk16; c += 4 * 256) {
      const uint4 r0 = __ldcs(src + c), r1 = __ldcs(src + c + 256), r2 = __ldcs(src + c + 512),
                  r3 = __ldcs(src + c + 768);
      __stcs(dst + c, r0);
      __stcs(dst + c + 256, r1);
      __stcs(dst + c + 512, r2);
      __stcs(dst + c + 768, r3);
    }
    for (; c < chunk16; c += 256) __stcs(dst + c, __ldcs(src + c));
  }

  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = gt; i < n_entries; i += gs) {
    const int4 e = __ldcv(entries + i);  // (row, block, tier, id)
    if (e.x < 0 || e.x >= max_rows || e.y < 0 || e.y >= max_blocks || e.z < 0 || e.z > 1 || e.w < 0 ||
        e.w >= tier_blocks(pool, e.z)) {
      flag_error(pool.status, kErrBadBlock);
      continue;
    }
    const int64_t k = (int64_t)e.x * max_blocks + e.y;
    table[k] = e.w;
    tier_map[k] = (uint8_t)e.z;
  }
  for (int64_t i = gt; i < n_rows; i += gs) seq_lens[i] = __ldcv(lens + i);
}

__global__ void __launch_bounds__(256) apply_plan_kernel(PoolView pool, uint8_t* plan, int32_t* __restrict__ table,
                                                         uint8_t* __restrict__ tier_map,
                                                         int32_t* __restrict__ seq_lens, int max_rows,
                                                         int max_blocks, int* done_ctr) {
  __shared__ int4 s_hdr[2];
  __shared__ int4 s_move;
  if (threadIdx.x < 2) s_hdr[threadIdx.x] = __ldcv(reinterpret_cast<const int4*>(plan) + threadIdx.x);
  __syncthreads();
  const int4 h0 = s_hdr[0], h1 = s_hdr[1];
  const int64_t cap = (int64_t)max_rows * max_blocks;
  const bool ok = h0.w == max_blocks && h1.z == max_rows && h1.x == cap && h1.y == cap && h0.x >= 0 &&
                  h0.x <= h1.x && h0.y >= 0 && h0.y <= h1.y && h0.z >= 0 && h0.z <= max_rows;
  if (ok)
    apply_plan_body(pool, plan, h0, h1, s_move, table, tier_map, seq_lens, max_rows, max_blocks);
  else if (blockIdx.x == 0 && threadIdx.x == 0)
    flag_error(pool.status, kErrBadPlan);

  __syncthreads();  // every read of the plan by this CTA is done
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(done_ctr, 1) == (int)gridDim.x - 1) {
      *done_ctr = 0;  // the next launch (stream-ordered) starts from zero
      __threadfence_system();
      *reinterpret_cast<volatile int32_t*>(plan + offsetof(dkv_plan_header, applied)) = 1;
      __threadfence_system();
    }
  }
}

static int launch_apply_plan(const dkv_pool* p, const void* plan, int32_t* table, uint8_t* tier_map,
                             int32_t* seq_lens, int max_rows, int max_blocks, cudaStream_t st) {
  // Fixed grid (the plan's size is only known on the device): one CTA per SM.
  apply_plan_kernel<<<p->num_sms, 256, 0, st>>>(p->view(), static_cast<uint8_t*>(const_cast<void*>(plan)), table,
                                                tier_map, seq_lens, max_rows, max_blocks,
                                                p->d_status + kApplyCounterIdx);
  return cuda_check(cudaGetLastError(), "dkv_apply_plan kernel");
}

}  // namespace dkv

using namespace dkv;

struct dkv_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int device = 0;
};

extern "C" {

int dkv_apply_plan(dkv_pool* pool, const void* plan, int32_t* block_table, uint8_t* tier_map, int32_t* seq_lens,
                   int max_rows, int max_blocks, void* stream) {
  if (!pool || !plan || !block_table || !tier_map || !seq_lens)
    return set_error(DKV_ERR_ARG, "dkv_apply_plan: null argument");
  if (reinterpret_cast<uintptr_t>(plan) & 15) return set_error(DKV_ERR_ARG, "dkv_apply_plan: plan must be 16-byte aligned");
  if (!dkv_plan_bytes(max_rows, max_blocks)) return set_error(DKV_ERR_ARG, "dkv_apply_plan: bad table shape");
  return launch_apply_plan(pool, plan, block_table, tier_map, seq_lens, max_rows, max_blocks, (cudaStream_t)stream);
}

int dkv_decode_graph_create(dkv_pool* pool, const void* plan, int max_rows, const dkv_layer_io* layers, int n_layers,
                            int32_t* block_table, int32_t* seq_lens, uint8_t* tier_map, int B, int max_blocks,
                            int hidden, int num_q_heads, float rope_theta, void* workspace, size_t ws_bytes,
                            dkv_graph** out) {
  if (!pool || !layers || n_layers < 1 || !out || !block_table || !seq_lens || !tier_map)
    return set_error(DKV_ERR_ARG, "dkv_decode_graph_create: bad argument");
  *out = nullptr;
  if (plan && (B > max_rows || !dkv_plan_bytes(max_rows, max_blocks)))
    return set_error(DKV_ERR_ARG, "dkv_decode_graph_create: B must be <= max_rows");
  cudaStream_t cs;
  int rc = cuda_check(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking), "dkv_decode_graph_create: stream");
  if (rc) return rc;
  // Relaxed capture: the launch helpers may set kernel attributes on their first use.
  rc = cuda_check(cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed), "dkv_decode_graph_create: begin capture");
  if (rc) {
    cudaStreamDestroy(cs);
    return rc;
  }
  if (plan) rc = launch_apply_plan(pool, plan, block_table, tier_map, seq_lens, max_rows, max_blocks, cs);
  for (int i = 0; i < n_layers && !rc; ++i)
    rc = dkv_decode_step(pool, layers[i].layer, layers[i].x, layers[i].Wqkv, block_table, seq_lens, tier_map, B,
                         max_blocks, hidden, num_q_heads, rope_theta, layers[i].out, workspace, ws_bytes, cs);
  cudaGraph_t g = nullptr;
  const cudaError_t ee = cudaStreamEndCapture(cs, &g);
  cudaStreamDestroy(cs);
  if (!rc) rc = cuda_check(ee, "dkv_decode_graph_create: end capture");
  if (rc) {
    if (g) cudaGraphDestroy(g);
    return rc;
  }
  cudaGraphExec_t ex = nullptr;
  rc = cuda_check(cudaGraphInstantiate(&ex, g, 0), "dkv_decode_graph_create: instantiate");
  if (rc) {
    cudaGraphDestroy(g);
    return rc;
  }
  dkv_graph* gr = new (std::nothrow) dkv_graph;
  if (!gr) {
    cudaGraphExecDestroy(ex);
    cudaGraphDestroy(g);
    return set_error(DKV_ERR_OOM, "dkv_decode_graph_create: out of host memory");
  }
  gr->graph = g;
  gr->exec = ex;
  gr->device = pool->device;
  *out = gr;
  return DKV_OK;
}

int dkv_graph_launch(dkv_graph* g, void* stream) {
  if (!g) return set_error(DKV_ERR_ARG, "dkv_graph_launch: null graph");
  return cuda_check(cudaGraphLaunch(g->exec, (cudaStream_t)stream), "dkv_graph_launch");
}

int dkv_graph_destroy(dkv_graph* g) {
  if (!g) return DKV_OK;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
  return DKV_OK;
}

}  // extern "C"
