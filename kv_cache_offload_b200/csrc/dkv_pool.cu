// Two-tier paged KV block pool: creation, tier access, cache append, block-layout
// permutation, status checks. The host tier is pinned host memory mapped into the device
// address space, so kernels read and write it in place (DirectKV, "长上下文 LLM 的零拷贝
// KV Cache 卸载（OSDI 2026）", 核心方法: the attention kernel accesses CPU pinned memory
// directly, no staging buffer).
#include <stdio.h>
#include <string.h>

#include <new>

#include "dkv_internal.h"

namespace dkv {

static thread_local char g_last_error[512] = "";

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DKV_OK;
  return set_error(e == cudaErrorMemoryAllocation ? DKV_ERR_OOM : DKV_ERR_CUDA, "%s: %s (%d)",
                   what, cudaGetErrorString(e), (int)e);
}

// ------------------------------------------------------------------ append kernel

// Writes token t of sequence b (position seq_lens[b] + t) into its slot, 16 bytes per
// thread-item. Items are (b, t, g, kv, piece) with piece = 16-byte piece of a D row.
__global__ void append_kv_kernel(PoolView pool, int layer, const uint16_t* __restrict__ k,
                                 const uint16_t* __restrict__ v, int B, int n_tokens,
                                 const int32_t* __restrict__ table, int max_blocks,
                                 const int32_t* __restrict__ seq_lens,
                                 const uint8_t* __restrict__ tier_map) {
  const int pieces = pool.D / 8;
  const int64_t total = (int64_t)B * n_tokens * pool.Hkv * 2 * pieces;
  for (int64_t it = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; it < total;
       it += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = it;
    const int pc = (int)(r % pieces); r /= pieces;
    const int kv = (int)(r % 2); r /= 2;
    const int g = (int)(r % pool.Hkv); r /= pool.Hkv;
    const int t = (int)(r % n_tokens); r /= n_tokens;
    const int b = (int)r;
    const int64_t pos = (int64_t)seq_lens[b] + t;
    const int64_t j = pos / pool.T;
    const int slot = (int)(pos % pool.T);
    if (pos < 0 || j >= max_blocks) {
      flag_error(pool.status, kErrCtxTooLong);
      continue;
    }
    const int tier = tier_map[(int64_t)b * max_blocks + j];
    const int64_t phys = table[(int64_t)b * max_blocks + j];
    if (tier > 1) { flag_error(pool.status, kErrBadTier); continue; }
    if (phys < 0 || phys >= tier_blocks(pool, tier)) { flag_error(pool.status, kErrBadBlock); continue; }
    const uint16_t* src = (kv ? v : k) + (((int64_t)b * n_tokens + t) * pool.Hkv + g) * pool.D + pc * 8;
    const int64_t o = chunk_offset(pool, tier, layer, phys, kv, g) + (int64_t)slot * pool.D + pc * 8;
    if (!DKV_DEBUG_RANGE(pool.status, o, o + 8, tier_elems(pool, tier))) continue;
    uint16_t* dst = tier_base(pool, tier) + o;
    *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
  }
}

// ------------------------------------------------------------------ layout kernel

// dst[bb][a][c] = src[a][bb][c] for 16-byte items c < chunk16. One CTA per (a, bb) pair
// (grid-stride), each thread moving 4 items per round so that several 16-byte loads are
// in flight per thread when the source is host memory read over the host link.
__global__ void __launch_bounds__(256) permute_chunks_kernel(const uint4* __restrict__ src,
                                                             uint4* __restrict__ dst, int64_t A,
                                                             int64_t Bn, int64_t chunk16) {
  const int64_t pairs = A * Bn;
  for (int64_t pr = blockIdx.x; pr < pairs; pr += gridDim.x) {
    const int64_t a = pr / Bn, bb = pr % Bn;
    const uint4* s = src + pr * chunk16;
    uint4* d = dst + (bb * A + a) * chunk16;
    int64_t c = threadIdx.x;
    for (; c + 3 * 256 < chunk16; c += 4 * 256) {
      uint4 r0 = __ldcs(s + c), r1 = __ldcs(s + c + 256), r2 = __ldcs(s + c + 512),
            r3 = __ldcs(s + c + 768);
      __stcs(d + c, r0);
      __stcs(d + c + 256, r1);
      __stcs(d + c + 512, r2);
      __stcs(d + c + 768, r3);
    }
    for (; c < chunk16; c += 256) __stcs(d + c, __ldcs(s + c));
  }
}

// Block copy between tiers: item = (block i, layer l, 16-byte piece c); each thread moves
// four pieces per round so several loads are in flight when the source is host memory.
__global__ void __launch_bounds__(256) copy_blocks_kernel(PoolView pool, int src_tier, int dst_tier,
                                                          const int32_t* __restrict__ src_ids,
                                                          const int32_t* __restrict__ dst_ids, int n) {
  const int64_t pieces = (int64_t)2 * pool.Hkv * pool.T * pool.D / 8;  // 16-byte pieces per (block, layer)
  const int64_t per_block = pieces * pool.L;
  const int64_t total = per_block * n;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; base < total; base += 4 * stride) {
    uint4 v[4];
    uint4* dst[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dst[u] = nullptr;
      const int64_t it = base + u * stride;
      if (it >= total) continue;
      const int i = (int)(it / per_block);
      const int64_t r = it % per_block;
      const int l = (int)(r / pieces);
      const int64_t c = r % pieces;
      const int64_t s = src_ids[i], d = dst_ids[i];
      if (s < 0 || s >= tier_blocks(pool, src_tier) || d < 0 || d >= tier_blocks(pool, dst_tier)) {
        if (c == 0 && l == 0) flag_error(pool.status, kErrBadBlock);
        continue;
      }
      const int64_t so = chunk_offset(pool, src_tier, l, s, 0, 0) + c * 8;
      const int64_t dof = chunk_offset(pool, dst_tier, l, d, 0, 0) + c * 8;
      if (!DKV_DEBUG_RANGE(pool.status, so, so + 8, tier_elems(pool, src_tier)) ||
          !DKV_DEBUG_RANGE(pool.status, dof, dof + 8, tier_elems(pool, dst_tier)))
        continue;
      const uint4* src = reinterpret_cast<const uint4*>(tier_base(pool, src_tier) + so);
      dst[u] = reinterpret_cast<uint4*>(tier_base(pool, dst_tier) + dof);
      v[u] = __ldcs(src);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (dst[u]) __stcs(dst[u], v[u]);
  }
}

}  // namespace dkv

using namespace dkv;

extern "C" {

const char* dkv_last_error(void) { return g_last_error; }

const char* dkv_version(void) { return "dkv 0.1 (sm_100a)"; }

int dkv_pool_create(const dkv_pool_config* cfg, dkv_pool** out) {
  if (!cfg || !out) return set_error(DKV_ERR_ARG, "dkv_pool_create: null argument");
  *out = nullptr;
  const dkv_pool_config& c = *cfg;
  if (c.num_layers < 1 || c.num_kv_heads < 1 || c.hbm_blocks < 0 || c.host_blocks < 0 ||
      (c.layout != DKV_LAYOUT_LAYER_FIRST && c.layout != DKV_LAYOUT_PAGE_FIRST) ||
      (c.host_flags & ~(DKV_HOST_WRITE_COMBINED | DKV_HOST_NUMA_NEAREST)))
    return set_error(DKV_ERR_ARG, "dkv_pool_create: invalid geometry");
  if ((c.head_dim != 64 && c.head_dim != 128) || c.block_tokens != 16)
    return set_error(DKV_ERR_UNSUPPORTED, "dkv_pool_create: need head_dim 64|128, block_tokens 16");
  if (c.hbm_base && (reinterpret_cast<uintptr_t>(c.hbm_base) & 255))
    return set_error(DKV_ERR_ARG, "dkv_pool_create: hbm_base must be 256-byte aligned");
  int dev = 0;
  int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (rc) return rc;
  int major = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10) return set_error(DKV_ERR_UNSUPPORTED, "dkv_pool_create: needs an sm_100 device (got major %d)", major);

  dkv_pool* p = new (std::nothrow) dkv_pool();
  if (!p) return set_error(DKV_ERR_OOM, "dkv_pool_create: host allocation failed");
  p->cfg = c;
  p->device = dev;
  p->num_sms = sms;
  memset(&p->tuning, 0, sizeof(p->tuning));
  const size_t per_block = (size_t)c.num_layers * 2 * c.num_kv_heads * c.block_tokens * c.head_dim * 2;
  p->hbm_bytes = per_block * (size_t)c.hbm_blocks;
  p->host_bytes = per_block * (size_t)c.host_blocks;
  p->own_hbm = false;
  p->hbm = nullptr;
  p->host_h = p->host_d = nullptr;
  p->d_status = nullptr;

  cudaError_t e;
  if (p->hbm_bytes) {
    if (c.hbm_base) {
      p->hbm = static_cast<uint16_t*>(c.hbm_base);
    } else {
      e = cudaMalloc(&p->hbm, p->hbm_bytes);
      if (e != cudaSuccess) {
        cudaGetLastError();
        delete p;
        return set_error(DKV_ERR_OOM, "dkv_pool_create: cudaMalloc of %zu HBM-tier bytes failed: %s",
                         (size_t)per_block * c.hbm_blocks, cudaGetErrorString(e));
      }
      p->own_hbm = true;
    }
  }
  if (p->host_bytes) {
    unsigned flags = cudaHostAllocMapped | cudaHostAllocPortable;
    if (c.host_flags & DKV_HOST_WRITE_COMBINED) flags |= cudaHostAllocWriteCombined;
    void* h = nullptr;
    const int node = (c.host_flags & DKV_HOST_NUMA_NEAREST) ? gpu_numa_node(dev) : -1;
    const int arc = alloc_host_on_node(p->host_bytes, flags, node, &h);
    e = arc == DKV_OK ? cudaSuccess : (cudaError_t)arc;
    if (e != cudaSuccess) {
      cudaGetLastError();
      if (p->own_hbm) cudaFree(p->hbm);
      size_t hb = p->host_bytes;
      delete p;
      return set_error(DKV_ERR_OOM, "dkv_pool_create: pinned mapped host allocation of %zu bytes failed: %s",
                       hb, cudaGetErrorString(e));
    }
    void* d = nullptr;
    e = cudaHostGetDevicePointer(&d, h, 0);
    if (e != cudaSuccess) {
      cudaFreeHost(h);
      if (p->own_hbm) cudaFree(p->hbm);
      delete p;
      return cuda_check(e, "cudaHostGetDevicePointer");
    }
    p->host_h = static_cast<uint16_t*>(h);
    p->host_d = static_cast<uint16_t*>(d);
  }
  e = cudaMalloc(&p->d_status, kPoolScratchInts * sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, kPoolScratchInts * sizeof(int));
  if (e != cudaSuccess) {
    if (p->host_h) cudaFreeHost(p->host_h);
    if (p->own_hbm) cudaFree(p->hbm);
    delete p;
    return cuda_check(e, "dkv_pool_create: status word");
  }
  *out = p;
  return DKV_OK;
}

int dkv_pool_destroy(dkv_pool* p) {
  if (!p) return set_error(DKV_ERR_ARG, "dkv_pool_destroy: null pool");
  cudaDeviceSynchronize();
  if (p->d_status) cudaFree(p->d_status);
  if (p->host_h) cudaFreeHost(p->host_h);
  if (p->own_hbm && p->hbm) cudaFree(p->hbm);
  delete p;
  return DKV_OK;
}

int dkv_pool_tier_ptr(const dkv_pool* p, int tier, void** dev_ptr, void** host_ptr, size_t* bytes) {
  if (!p || (tier != DKV_TIER_HBM && tier != DKV_TIER_HOST))
    return set_error(DKV_ERR_ARG, "dkv_pool_tier_ptr: bad pool or tier");
  if (tier == DKV_TIER_HBM) {
    if (dev_ptr) *dev_ptr = p->hbm;
    if (host_ptr) *host_ptr = nullptr;
    if (bytes) *bytes = p->hbm_bytes;
  } else {
    if (dev_ptr) *dev_ptr = p->host_d;
    if (host_ptr) *host_ptr = p->host_h;
    if (bytes) *bytes = p->host_bytes;
  }
  return DKV_OK;
}

int dkv_pool_set_tuning(dkv_pool* p, const dkv_tuning* t) {
  if (!p) return set_error(DKV_ERR_ARG, "dkv_pool_set_tuning: null pool");
  if (t) {
    const int v = t->attn_variant;
    if (t->attn_splits < 0 || t->proj_splits < 0 || t->proj_splits > 8 || (v != 0 && v != 1 && v != 5 && v != 6 && v != 7) ||
        t->attn_lsu_hbm < 0 || t->attn_lsu_hbm > 3 || t->serial_launch < 0 || t->serial_launch > 3 ||
        t->wait_limit_us < 0 || t->test_withhold_block < 0 || t->test_withhold_block > 1)
      return set_error(DKV_ERR_ARG, "dkv_pool_set_tuning: value out of range");
    p->tuning = *t;
  } else {
    memset(&p->tuning, 0, sizeof(p->tuning));
  }
  return DKV_OK;
}

int dkv_append_kv(dkv_pool* p, int layer, const uint16_t* k, const uint16_t* v, int B, int n_tokens,
                  const int32_t* block_table, int max_blocks, const int32_t* seq_lens,
                  const uint8_t* tier_map, void* stream) {
  if (!p || !k || !v || !block_table || !seq_lens || !tier_map)
    return set_error(DKV_ERR_ARG, "dkv_append_kv: null argument");
  if (layer < 0 || layer >= p->cfg.num_layers || B < 0 || n_tokens < 0 || max_blocks < 1)
    return set_error(DKV_ERR_ARG, "dkv_append_kv: bad layer/B/n_tokens/max_blocks");
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15)
    return set_error(DKV_ERR_ARG, "dkv_append_kv: k and v must be 16-byte aligned");
  if (B == 0 || n_tokens == 0) return DKV_OK;
  const int64_t items = (int64_t)B * n_tokens * p->cfg.num_kv_heads * 2 * (p->cfg.head_dim / 8);
  int64_t blocks = (items + 255) / 256;
  const int64_t cap = (int64_t)p->num_sms * 16;
  if (blocks > cap) blocks = cap;
  append_kv_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      p->view(), layer, k, v, B, n_tokens, block_table, max_blocks, seq_lens, tier_map);
  return cuda_check(cudaGetLastError(), "dkv_append_kv launch");
}

int dkv_permute_layout(const void* src, void* dst, int src_layout, int num_layers, int64_t num_blocks,
                       int64_t chunk_bytes, void* stream) {
  if (!src || !dst) return set_error(DKV_ERR_ARG, "dkv_permute_layout: null pointer");
  if ((src_layout != DKV_LAYOUT_LAYER_FIRST && src_layout != DKV_LAYOUT_PAGE_FIRST) || num_layers < 1 ||
      num_blocks < 0 || chunk_bytes <= 0 || (chunk_bytes & 15))
    return set_error(DKV_ERR_ARG, "dkv_permute_layout: bad layout/sizes (chunk_bytes %% 16 == 0)");
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15)
    return set_error(DKV_ERR_ARG, "dkv_permute_layout: pointers must be 16-byte aligned");
  const uint8_t* s8 = static_cast<const uint8_t*>(src);
  const uint8_t* d8 = static_cast<const uint8_t*>(dst);
  const int64_t total = (int64_t)num_layers * num_blocks * chunk_bytes;
  if (total == 0) return DKV_OK;
  if (s8 < d8 + total && d8 < s8 + total)
    return set_error(DKV_ERR_ARG, "dkv_permute_layout: src and dst overlap");
  const int64_t A = src_layout == DKV_LAYOUT_LAYER_FIRST ? num_layers : num_blocks;
  const int64_t Bn = src_layout == DKV_LAYOUT_LAYER_FIRST ? num_blocks : num_layers;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = A * Bn;
  const int64_t cap = (int64_t)sms * 8;
  if (grid > cap) grid = cap;
  permute_chunks_kernel<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), A, Bn, chunk_bytes / 16);
  return cuda_check(cudaGetLastError(), "dkv_permute_layout launch");
}

int dkv_convert_layout(dkv_pool* p, int tier, void* dst, size_t dst_bytes, void* stream) {
  if (!p || !dst || (tier != DKV_TIER_HBM && tier != DKV_TIER_HOST))
    return set_error(DKV_ERR_ARG, "dkv_convert_layout: bad argument");
  const size_t bytes = tier == DKV_TIER_HBM ? p->hbm_bytes : p->host_bytes;
  if (dst_bytes < bytes) return set_error(DKV_ERR_ARG, "dkv_convert_layout: dst too small");
  if (bytes == 0) return DKV_OK;
  const void* src = tier == DKV_TIER_HBM ? (const void*)p->hbm : (const void*)p->host_d;
  const int64_t chunk = (int64_t)2 * p->cfg.num_kv_heads * p->cfg.block_tokens * p->cfg.head_dim * 2;
  const int64_t blocks = tier == DKV_TIER_HBM ? p->cfg.hbm_blocks : p->cfg.host_blocks;
  return dkv_permute_layout(src, dst, p->cfg.layout, p->cfg.num_layers, blocks, chunk, stream);
}

int dkv_copy_blocks(dkv_pool* p, int src_tier, int dst_tier, const int32_t* src_ids, const int32_t* dst_ids, int n,
                    int method, void* stream) {
  if (!p || (n > 0 && (!src_ids || !dst_ids)) || n < 0 || (src_tier != 0 && src_tier != 1) ||
      (dst_tier != 0 && dst_tier != 1) || (method != DKV_COPY_DMA && method != DKV_COPY_KERNEL))
    return set_error(DKV_ERR_ARG, "dkv_copy_blocks: bad argument");
  if (n == 0) return DKV_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const PoolView v = p->view();
  const size_t chunk = (size_t)2 * v.Hkv * v.T * v.D * 2;  // one block of one layer, bytes
  if (method == DKV_COPY_KERNEL) {
    const int64_t items = (int64_t)n * v.L * (chunk / 16);
    int64_t grid = (items + 255) / 256;
    const int64_t cap = (int64_t)p->num_sms * 8;
    if (grid > cap) grid = cap;
    copy_blocks_kernel<<<(unsigned)grid, 256, 0, st>>>(v, src_tier, dst_tier, src_ids, dst_ids, n);
    return cuda_check(cudaGetLastError(), "dkv_copy_blocks kernel");
  }
  for (int i = 0; i < n;) {
    const int64_t s0 = src_ids[i], d0 = dst_ids[i];
    if (s0 < 0 || s0 >= tier_blocks(v, src_tier) || d0 < 0 || d0 >= tier_blocks(v, dst_tier))
      return set_error(DKV_ERR_BAD_TABLE, "dkv_copy_blocks: block id out of range at %d", i);
    int run = 1;  // merge consecutive ids when a block's layers are contiguous (page-first or L == 1)
    if (v.layout == DKV_LAYOUT_PAGE_FIRST || v.L == 1)
      while (i + run < n && src_ids[i + run] == s0 + run && dst_ids[i + run] == d0 + run &&
             s0 + run < tier_blocks(v, src_tier) && d0 + run < tier_blocks(v, dst_tier))
        ++run;
    for (int l = 0; l < v.L; ++l) {
      const size_t bytes = chunk * ((v.layout == DKV_LAYOUT_PAGE_FIRST) ? (size_t)v.L * run : run);
      const uint16_t* src = tier_base(v, src_tier) + chunk_offset(v, src_tier, l, s0, 0, 0);
      uint16_t* dst = tier_base(v, dst_tier) + chunk_offset(v, dst_tier, l, d0, 0, 0);
      int rc = cuda_check(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, st), "dkv_copy_blocks: copy");
      if (rc) return rc;
      if (v.layout == DKV_LAYOUT_PAGE_FIRST) break;  // all layers in one copy
    }
    i += run;
  }
  return DKV_OK;
}

int dkv_host_alloc_mapped(size_t bytes, int host_flags, void** host_ptr, void** dev_ptr) {
  if (!host_ptr || !dev_ptr || bytes == 0 || (host_flags & ~DKV_HOST_WRITE_COMBINED))
    return set_error(DKV_ERR_ARG, "dkv_host_alloc_mapped: bad argument");
  unsigned flags = cudaHostAllocMapped | cudaHostAllocPortable;
  if (host_flags & DKV_HOST_WRITE_COMBINED) flags |= cudaHostAllocWriteCombined;
  void* h = nullptr;
  cudaError_t e = cudaHostAlloc(&h, bytes, flags);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return set_error(DKV_ERR_OOM, "dkv_host_alloc_mapped: %zu bytes: %s", bytes, cudaGetErrorString(e));
  }
  void* d = nullptr;
  e = cudaHostGetDevicePointer(&d, h, 0);
  if (e != cudaSuccess) {
    cudaFreeHost(h);
    return cuda_check(e, "dkv_host_alloc_mapped: cudaHostGetDevicePointer");
  }
  *host_ptr = h;
  *dev_ptr = d;
  return DKV_OK;
}

int dkv_host_free(void* host_ptr) {
  if (!host_ptr) return set_error(DKV_ERR_ARG, "dkv_host_free: null pointer");
  return cuda_check(cudaFreeHost(host_ptr), "dkv_host_free");
}

int dkv_check(dkv_pool* p, void* stream) {
  if (!p) return set_error(DKV_ERR_ARG, "dkv_check: null pool");
  int rc = cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "dkv_check: stream sync");
  if (rc) return rc;
  int word = 0;
  rc = cuda_check(cudaMemcpy(&word, p->d_status, sizeof(int), cudaMemcpyDeviceToHost), "dkv_check: read status");
  if (rc) return rc;
  if (!word) return DKV_OK;
  cudaMemset(p->d_status, 0, sizeof(int));
  if (word & kErrDebugBounds)
    return set_error(DKV_ERR_INTERNAL, "a debug-build range check failed in a kernel (status 0x%x)", word);
  if (word & kErrTimeout)
    return set_error(DKV_ERR_TIMEOUT, "device wait timed out (status 0x%x)", word);
  return set_error(DKV_ERR_BAD_TABLE, "device rejected table entries (status 0x%x:%s%s%s%s)", word,
                   (word & kErrBadTier) ? " bad-tier" : "", (word & kErrBadBlock) ? " bad-block-id" : "",
                   (word & kErrCtxTooLong) ? " context-exceeds-table" : "",
                   (word & kErrBadPlan) ? " plan-header-mismatch" : "");
}

}  // extern "C"
