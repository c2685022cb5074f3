// dkv_decode_step_static: the decode step for callers that cannot allocate device memory.
//
// dkv_decode_step needs a caller-provided workspace (the projection's q / new-token state
// and the attention's split partials). Some callers cannot allocate one: a serving loop
// whose device memory is entirely reserved up front by its own allocator (a cudaMalloc
// there fails or fragments that reservation), a latency-critical loop that cannot take
// cudaMalloc's implicit device synchronisation, or a plain C host that has no device
// allocator of its own. This entry point takes the workspace from a fixed-size array in
// the library's own device memory instead, so it allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// it (kDkvStaticWsBytes) until the process exits. In host code its name is only a host
// stand-in, never a device address, so its address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached. This file has no kernels,
// so under CUDA's lazy module loading (the default) its device memory is committed by that
// first lookup, i.e. by the first call on the device: a caller that reserves the rest of
// the device's memory up front makes one call before doing so.
#include <mutex>

#include "dkv_internal.h"

namespace dkv {

constexpr size_t kDkvStaticWsBytes = (size_t)16 << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_dkv_static_ws[kDkvStaticWsBytes];

static std::mutex g_static_mu;
static void* g_static_ptr[kMaxDevices] = {};

// Device address of the pool's device's array; looked up on the first call on each device.
// The pool's device must be the current one (the address is per device, and the kernels
// run on the current device).
static int static_ws_ptr(const dkv_pool* pool, void** out) {
  int dev = 0;
  int rc = cuda_check(cudaGetDevice(&dev), "dkv_decode_step_static: cudaGetDevice");
  if (rc) return rc;
  if (dev != pool->device)
    return set_error(DKV_ERR_ARG, "dkv_decode_step_static: the pool lives on device %d but device %d is current",
                     pool->device, dev);
  if (dev < 0 || dev >= kMaxDevices) return set_error(DKV_ERR_UNSUPPORTED, "dkv_decode_step_static: device %d", dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    rc = cuda_check(cudaGetSymbolAddress(&p, g_dkv_static_ws), "dkv_decode_step_static: cudaGetSymbolAddress");
    if (rc) return rc;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return DKV_OK;
}

}  // namespace dkv

using namespace dkv;

extern "C" {

size_t dkv_decode_static_workspace_capacity(void) { return kDkvStaticWsBytes; }

int dkv_decode_step_static(dkv_pool* pool, int layer, const uint16_t* x, const uint16_t* Wqkv,
                           const int32_t* block_table, const int32_t* seq_lens, const uint8_t* tier_map,
                           int B, int max_blocks, int hidden, int num_q_heads, float rope_theta,
                           uint16_t* out, void* stream) {
  if (!pool) return set_error(DKV_ERR_ARG, "dkv_decode_step_static: null pool");
  DecodeWs w;
  int rc = decode_ws_layout(pool, B, max_blocks, num_q_heads, hidden, &w);
  if (rc) return rc;  // the same code (and message) dkv_decode_step gives for this shape
  if (w.total > kDkvStaticWsBytes)
    return set_error(DKV_ERR_CAPACITY,
                     "dkv_decode_step_static: this shape needs %zu workspace bytes, more than the %zu-byte "
                     "static workspace; use dkv_decode_step with a caller workspace (or fewer attention splits)",
                     w.total, kDkvStaticWsBytes);
  void* ws = nullptr;
  rc = static_ws_ptr(pool, &ws);
  if (rc) return rc;
  return dkv_decode_step(pool, layer, x, Wqkv, block_table, seq_lens, tier_map, B, max_blocks, hidden,
                         num_q_heads, rope_theta, out, ws, kDkvStaticWsBytes, stream);
}

}  // extern "C"
