// Host-side internals shared by the libdkv translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dkv.h"
#include "dkv_common.cuh"

struct dkv_pool {
  dkv_pool_config cfg;
  int device;
  int num_sms;
  uint16_t* hbm;
  size_t hbm_bytes;
  bool own_hbm;
  uint16_t* host_h;   // host-side address of the host tier
  uint16_t* host_d;   // device alias of the host tier
  size_t host_bytes;
  int* d_status;      // device scratch: [0] status word, [32] plan-apply CTA counter
  dkv_tuning tuning;

  dkv::PoolView view() const {
    dkv::PoolView v;
    v.tier[0] = hbm;
    v.tier[1] = host_d;
    v.blocks[0] = cfg.hbm_blocks;
    v.blocks[1] = cfg.host_blocks;
    v.L = cfg.num_layers;
    v.Hkv = cfg.num_kv_heads;
    v.D = cfg.head_dim;
    v.T = cfg.block_tokens;
    v.layout = cfg.layout;
    v.status = d_status;
    return v;
  }
};

namespace dkv {

constexpr int kPoolScratchInts = 64;
constexpr int kApplyCounterIdx = 32;

int set_error(int code, const char* fmt, ...);
int cuda_check(cudaError_t e, const char* what);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Arguments of the split-K attention kernel.
struct AttnParams {
  PoolView pool;
  int layer;
  const int32_t* table;
  const int32_t* seq_lens;
  const uint8_t* tier_map;
  int max_blocks;
  int Hq;
  int S;
  const float* qs;   // [B][Hq][D], scaled by log2(e)/sqrt(D)
  float2* part_ml;   // [B][Hq][S] (m, l)
  float* part_acc;   // [B][Hq][S][D]
  // fused combine (when out != nullptr): the last CTA of each (b, kv head) merges
  int* cnt;          // [B][Hkv] arrival counters (zero on entry)
  const float* knew; // [B][Hkv][D]
  const float* vnew; // [B][Hkv][D]
  uint16_t* out;     // [B][Hq*D] bf16, or nullptr
  int lsu_hbm;       // bit 0: HBM-tier blocks by cp.async instead of bulk copies; bit 1:
                     // host-tier blocks by bulk copies instead of cp.async
  int pdl;           // launch with programmatic dependent launch
  int early_kv;      // the kernel ahead is this step's projection: stream KV before it ends
  int signal_next;   // let the next kernel in the stream launch early (programmatic launch)
  uint64_t wait_ns;  // limit of each bounded wait
  int withhold;      // test hook: CTA (0, 0, 0) withholds its first block (bounded-wait test)
};

int launch_attention(const AttnParams& p, int B, int Hkv, int D, int G, int variant, cudaStream_t st);
int attention_ctas_per_sm(int G, int variant);
int launch_combine(int B, int Hq, int Hkv, int D, int S, const float2* ml, const float* acc,
                   const float* qs, const float* knew, const float* vnew, uint16_t* out, cudaStream_t st);

// Arguments of one projection launch (see dkv_projection.cu).
struct ProjArgs {
  PoolView pool;
  int layer;
  const uint16_t* x;
  const uint16_t* W;
  const int32_t* table;
  const int32_t* seq_lens;
  const uint8_t* tier_map;
  int max_blocks;
  int B, H, Hq, Hkv, D;
  double theta;
  float qscale;   // log2(e) / sqrt(D)
  float* qs;      // [B][Hq][D]
  float* knew;    // [B][Hkv][D]  k_hat as fp32
  float* vnew;    // [B][Hkv][D]  v_hat as fp32
  int* attn_cnt;  // [B][Hkv] attention split counters, reset by the projection
  int cluster;    // cluster size request (0 = automatic)
  int pdl;        // launch with programmatic dependent launch
};

int launch_projection(const ProjArgs& a, cudaStream_t st);

// 2-D bf16 tensor map over a row-major [rows][cols] array, box [box_rows][64], 128B swizzle.
int encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// NUMA placement of the host tier (dkv_numa.cu).
int numa_node_of_pci(const char* sysfs_root, const char* pci_bus_id);
int gpu_numa_node(int device);
struct SavedPolicy;
int alloc_host_on_node(size_t bytes, unsigned flags, int node, void** out);

// Workspace carve-up of one decode step (all offsets 256-byte aligned).
struct DecodeWs {
  int B, Hq, Hkv, D, rows, S, G, max_blocks, hidden;
  size_t off_qs, off_knew, off_vnew, off_cnt, off_ml, off_acc, total;
};

// Fills `w` for a shape; returns DKV_OK or an error (unsupported shape).
int decode_ws_layout(const dkv_pool* pool, int B, int max_blocks, int Hq, int hidden,
                     DecodeWs* w);

}  // namespace dkv
