// The decode step: projection stage (QKV GEMM, RoPE, single cache write, new-token
// partial), attention stage, combine stage; workspace layout and the C entry points.
//
// DirectKV ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", 核心方法) fuses KV generation
// (the QKV projection) with attention so that the new K/V are consumed on chip and never
// written out and read back. Here the projection's epilogue rotates q and k, writes bf16
// k_hat / v_hat to the cache exactly once, and leaves q, k_hat, v_hat (fp32) in the
// workspace; the attention stage reads only the cached blocks, and its combine folds in
// the new token's term (score q . k_hat, value v_hat) without re-reading the cache.
#include <math.h>

#include "dkv_internal.h"

namespace dkv {

// ----------------------------------------------------------------- workspace

// Automatic split count. Tensor-core kernels: one wave of about 7/8 of the resident CTA
// slots, at most 32 splits (the last split CTA of each (sequence, kv head) merges all of
// them). CUDA-core kernels, measured on B200 (attention alone, all blocks in HBM, B in
// {1, 2, 4, 8, 16, 32} x {8 K, 32 K} tokens and B in {1, 4} x 128 K, split counts from
// 0.3 to 3.5 waves of each shape's CTA slots): a grid just under a whole number of waves
// is fast and one just over it slow (its last CTAs run alone), and fewer, longer splits
// pay less per-CTA setup and merge work. G = 4: the most splits that fit in one wave up
// to 64 (sequence, kv head) units, two waves above that (B=16 x 32 K: 334 us at 9 splits
// vs 349 at 13; B=32 x 32 K: 660 vs 711 at 7; B=1 x 128 K: 102 vs 121 at 161; B=4 x 32 K:
// 97 vs 114). The one-CTA-per-SM G = 8 shape: one wave (B=1 x 32 K: 66 vs 76 us at 54).
// The three-CTA G = 8 shape: the most splits within 2.33 waves (B=4 x 8 K: 63.0 vs 67.0 us
// at 2.9 waves; B=32 x 32 K: 1108 vs 1119; B=16 x 32 K: 566 vs 573). Group sizes not
// measured: about 2.9 waves. Host-bound configurations are insensitive (70B layer with 80%
// of its blocks in the host tier: 70.75 ms at 4 and 5 splits).
static int auto_splits(const dkv_pool* pool, int B, int Hkv, int G, int variant) {
  const int slots = pool->num_sms * attention_ctas_per_sm(G, variant);
  const int units = B * Hkv;
  if (variant == 6 || variant == 7) {
    const int s = (7 * slots + 4 * units) / (8 * units);  // round(7/8 * slots / units)
    return s > 32 ? 32 : s;
  }
  if (G == 4 || (G == 8 && variant == 1)) {
    const int waves = (G == 4 && units > 64) ? 2 : 1;
    const int s = waves * slots / units;  // the most splits that fit in `waves` waves
    return s < 1 ? 1 : s;
  }
  if (G == 8) {  // the three-CTA shape: the most splits within 2.33 waves, or, where that
                 // would be more than 64 (a single sequence), within 0.86 of a wave
    int s = 233 * slots / (100 * units);
    if (s > 64) s = 86 * slots / (100 * units);
    return s < 1 ? 1 : s;
  }
  return (29 * slots + 5 * units) / (10 * units);
}

// The automatic attention kernel (CUDA cores): variant 5 packs more CTAs per SM than
// variant 1 (G = 4: four CTAs of three one-warp slots vs three of four slots; G = 8: three
// CTAs of two two-warp slots vs one of four), which streams long contexts faster, but at
// 2.9 waves of its more numerous CTA slots it cuts short contexts into more, shorter splits.
// Measured on B200 (attention alone, all blocks in HBM, B in {1, 4, 8, 16, 32} x {2 K, 8 K,
// 32 K} tokens, automatic split counts): G = 4 takes variant 5 once its splits keep at
// least 39 blocks of the table each (B=16 x 32 K: 353 vs 375 us; B=8 x 32 K: 190 vs 202;
// B=32 x 8 K: 198 vs 205; B=4 x 32 K at 38 blocks: 118 vs 117); G = 8 takes it once its
// splits keep at least 6 blocks and there are at most 64 of them (B=8 x 32 K: 304 vs 584
// us; B=32 x 2 K: 100 vs 154; B=8 x 2 K at 6.5 blocks: 49 vs 60; a single sequence, 129-161
// splits: 55-96 vs 33-84). Other group sizes: variant 1. Re-checked at the split counts of
// auto_splits above (the same sweep): the G = 4 threshold still picks the faster shape.
static int resolve_attn_variant(const dkv_pool* pool, int B, int Hkv, int G, int max_blocks) {
  const int v = pool->tuning.attn_variant;
  if (v != 0) return v;
  if (G != 4 && G != 8) return 1;
  int s5 = pool->tuning.attn_splits > 0 ? pool->tuning.attn_splits : auto_splits(pool, B, Hkv, G, 5);
  if (s5 < 1) s5 = 1;
  const int blocks_per_split = max_blocks / s5;
  if (G == 4) return blocks_per_split >= 39 ? 5 : 1;
  // G = 8 and a single sequence (automatic splits cut to under one wave): the three-CTA
  // shape only once its splits keep >= 40 blocks (70B layer, B=1: 128 K tokens 185 vs 230
  // us, 32 K 64 vs 66, 8 K 33 vs 25)
  const int slots5 = pool->num_sms * attention_ctas_per_sm(G, 5);
  if (pool->tuning.attn_splits <= 0 && 233 * slots5 / (100 * B * Hkv) > 64) return blocks_per_split >= 40 ? 5 : 1;
  return blocks_per_split >= 6 && s5 <= 64 ? 5 : 1;
}

static int pick_attn_splits(const dkv_pool* pool, int B, int Hkv, int G, int max_blocks) {
  int s = pool->tuning.attn_splits;
  if (s <= 0) s = auto_splits(pool, B, Hkv, G, resolve_attn_variant(pool, B, Hkv, G, max_blocks));
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
  w->S = pick_attn_splits(pool, B, Hkv, G, max_blocks);
  size_t o = 0;
  w->off_qs = o;       o = align_up(o + (size_t)B * Hq * D * 4, 256);
  w->off_knew = o;     o = align_up(o + (size_t)B * Hkv * D * 4, 256);
  w->off_vnew = o;     o = align_up(o + (size_t)B * Hkv * D * 4, 256);
  w->off_cnt = o;      o = align_up(o + (size_t)B * Hkv * 4, 256);
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

int dkv_decode_attn_variant(const dkv_pool* pool, int B, int max_blocks, int num_q_heads) {
  if (!pool) return set_error(DKV_ERR_ARG, "null pool");
  DecodeWs w;
  int rc = decode_ws_layout(pool, B, max_blocks, num_q_heads, 64, &w);
  return rc ? rc : resolve_attn_variant(pool, B, w.Hkv, w.G, max_blocks);
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
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  ProjArgs a;
  a.pool = pool->view();
  a.layer = layer;
  a.x = x;
  a.W = Wqkv;
  a.table = block_table;
  a.seq_lens = seq_lens;
  a.tier_map = tier_map;
  a.max_blocks = max_blocks;
  a.B = B; a.H = hidden; a.Hq = num_q_heads; a.Hkv = w.Hkv; a.D = w.D;
  a.theta = (double)rope_theta;
  a.qscale = (float)(1.4426950408889634 / sqrt((double)w.D));
  a.qs = reinterpret_cast<float*>(ws + w.off_qs);
  a.knew = reinterpret_cast<float*>(ws + w.off_knew);
  a.vnew = reinterpret_cast<float*>(ws + w.off_vnew);
  a.attn_cnt = reinterpret_cast<int*>(ws + w.off_cnt);
  a.cluster = pool->tuning.proj_splits;
  a.pdl = pool->tuning.serial_launch == 0 || pool->tuning.serial_launch == 3;
  return launch_projection(a, (cudaStream_t)stream);
}

namespace dkv {
// early_kv: the kernel ahead in the stream is this step's projection (dkv_decode_step)
static int decode_attend(dkv_pool* pool, int layer, const int32_t* block_table, const int32_t* seq_lens,
                         const uint8_t* tier_map, int B, int max_blocks, int hidden, int num_q_heads,
                         uint16_t* out, void* workspace, size_t ws_bytes, void* stream, bool early_kv) {
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
  a.cnt = reinterpret_cast<int*>(ws + w.off_cnt);
  a.knew = reinterpret_cast<const float*>(ws + w.off_knew);
  a.vnew = reinterpret_cast<const float*>(ws + w.off_vnew);
  a.out = out;
  a.lsu_hbm = pool->tuning.attn_lsu_hbm;
  a.pdl = pool->tuning.serial_launch != 1;
  a.early_kv = early_kv && a.pdl;
  a.signal_next = pool->tuning.serial_launch == 0 || pool->tuning.serial_launch == 3;
  a.wait_ns = pool->tuning.wait_limit_us > 0 ? (uint64_t)pool->tuning.wait_limit_us * 1000ull : 4000000000ull;
  a.withhold = pool->tuning.test_withhold_block != 0;
  return launch_attention(a, B, w.Hkv, w.D, w.G, resolve_attn_variant(pool, B, w.Hkv, w.G, max_blocks),
                          (cudaStream_t)stream);
}
}  // namespace dkv

extern "C" int dkv_decode_attend(dkv_pool* pool, int layer, const int32_t* block_table, const int32_t* seq_lens,
                                 const uint8_t* tier_map, int B, int max_blocks, int hidden, int num_q_heads,
                                 uint16_t* out, void* workspace, size_t ws_bytes, void* stream) {
  return decode_attend(pool, layer, block_table, seq_lens, tier_map, B, max_blocks, hidden, num_q_heads, out,
                       workspace, ws_bytes, stream, false);
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
                        reinterpret_cast<const float*>(ws + w.off_acc), reinterpret_cast<const float*>(ws + w.off_qs),
                        reinterpret_cast<const float*>(ws + w.off_knew), reinterpret_cast<const float*>(ws + w.off_vnew),
                        out, (cudaStream_t)stream);
}

int dkv_decode_step(dkv_pool* pool, int layer, const uint16_t* x, const uint16_t* Wqkv, const int32_t* block_table,
                    const int32_t* seq_lens, const uint8_t* tier_map, int B, int max_blocks, int hidden,
                    int num_q_heads, float rope_theta, uint16_t* out, void* workspace, size_t ws_bytes,
                    void* stream) {
  if (!out) return set_error(DKV_ERR_ARG, "dkv_decode_step: null out");
  int rc = dkv_decode_project(pool, layer, x, Wqkv, block_table, seq_lens, tier_map, B, max_blocks, hidden,
                              num_q_heads, rope_theta, workspace, ws_bytes, stream);
  if (rc) return rc;
  return decode_attend(pool, layer, block_table, seq_lens, tier_map, B, max_blocks, hidden, num_q_heads, out,
                       workspace, ws_bytes, stream, true);
}

}  // extern "C"
