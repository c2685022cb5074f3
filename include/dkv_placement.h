/*
 * dkv_placement.h — adaptive placement of KV blocks over the two tiers, placement plans
 * applied on the device, and the multi-layer decode step as one CUDA graph.
 *
 * The DirectKV summary page ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", section
 * 局限与后续工作) names adaptive placement as the next step: hot KV stays in HBM, cold
 * KV is read directly from CPU memory, with no large staging buffer. The "KV Offload"
 * wiki page (section CXL 作为 KV Offload 通道, the tier table) calls the KV being decoded
 * the hot KV of HBM. The series page ("「KV Cache 内存层级」系列总纲", §2.1 DirectKV and
 * §五) blames the dynamic addresses of staged copies for keeping a decode step from being
 * replayed as a CUDA graph; with zero-copy reads every address is fixed, so a whole step
 * — the placement update and every layer — replays as one graph.
 *
 * Policy (a reading: the pages define hotness no further). With n active sequences and an
 * HBM budget of `hbm_budget` blocks, each sequence keeps its newest W = hbm_budget / n
 * logical blocks in HBM (all of them if it has fewer) and its older blocks in the host
 * tier, where the attention kernel reads them in place. A sequence with len cached tokens
 * covers len / T + 1 logical blocks (the last one holds the next token's slot). Physical
 * ids are allocated smallest-free-first per tier. Operations:
 *   add(len)    the window shrinks to budget / (n + 1): rows 0..n-1, in order, move their
 *               oldest HBM blocks to the host tier until each holds at most W; then the
 *               new row n gets blocks j = 0.., in order, the newest min(W, nb) in HBM.
 *   remove(r)   row r's blocks are freed; the last row takes row r's place (its table row
 *               is rewritten, its data does not move); the window grows and rows 0.., in
 *               order, bring their newest host blocks into HBM up to min(W, nb).
 *   step()      every row counts the token the last decode step wrote (len += 1); a row
 *               that opens a new logical block gets it in HBM when W >= 1 (else in the
 *               host tier); then each row moves its oldest HBM blocks to the host tier
 *               until it holds at most W.
 * Every operation writes one plan; dkv_apply_plan (or a decode graph that holds it)
 * carries it out on the device. Within one plan no block is both the source of a move
 * and the destination of another, so its moves run concurrently.
 */
#ifndef DKV_PLACEMENT_H_
#define DKV_PLACEMENT_H_

#include "dkv.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * A placement plan, as one buffer:
 *   dkv_plan_header | dkv_plan_move[move_cap] | dkv_plan_entry[entry_cap] | int32 seq_lens[max_rows]
 * with move_cap = entry_cap = max_rows * max_blocks. Applying a plan copies each moved
 * block (every layer, K and V, every kv head) from (src_tier, src_id) to (dst_tier, dst_id),
 * writes block_table[row][block] = id and tier_map[row][block] = tier for each entry, and
 * writes seq_lens[0..n_rows).
 */
typedef struct dkv_plan_header {
  int32_t n_moves;     /* moves used */
  int32_t n_entries;   /* table entries used (each (row, block) at most once) */
  int32_t n_rows;      /* active rows: seq_lens[0..n_rows) are written */
  int32_t max_blocks;  /* table row stride the entries assume */
  int32_t move_cap;
  int32_t entry_cap;
  int32_t max_rows;
  int32_t applied;     /* 0 while the plan is pending; dkv_apply_plan sets it to 1 once the
                          device has finished reading the buffer */
} dkv_plan_header;

typedef struct dkv_plan_move { int32_t src_tier, src_id, dst_tier, dst_id; } dkv_plan_move;
typedef struct dkv_plan_entry { int32_t row, block, tier, id; } dkv_plan_entry;

/* Bytes of one plan buffer for a table of max_rows x max_blocks (0 if out of range). */
size_t dkv_plan_bytes(int max_rows, int max_blocks);

#define DKV_PLAN_MAPPED 0  /* plans in pinned host memory mapped for the device (default) */
#define DKV_PLAN_HOST   1  /* plans in ordinary host memory (no device; host-side use only) */

typedef struct dkv_bm_config {
  int32_t max_rows;      /* table rows = most sequences at once, >= 1 */
  int32_t max_blocks;    /* table columns = most logical blocks per sequence, >= 1 */
  int32_t block_tokens;  /* T >= 1 (the pool's block_tokens) */
  int32_t plan_memory;   /* DKV_PLAN_MAPPED or DKV_PLAN_HOST */
  int64_t hbm_ids;       /* HBM-tier physical ids the manager may use: 0..hbm_ids-1 */
  int64_t host_ids;      /* host-tier physical ids the manager may use: 0..host_ids-1 */
  int64_t hbm_budget;    /* blocks kept in HBM at rest, 0 <= budget; when budget > 0,
                            hbm_ids >= budget + 1 (one id of headroom for a step) */
  int32_t wait_ms;       /* longest wait for a plan buffer to be released (0 = 10000) */
  int32_t reserved;      /* 0 */
} dkv_bm_config;

typedef struct dkv_bm dkv_bm;  /* opaque block manager (host-side state, plan buffers) */

/*
 * Create a block manager with no sequences. It holds two plan buffers: operation k writes
 * buffer k mod 2, so the host prepares plan k+1 while the device applies plan k. Every
 * plan must be applied, in order, from the buffer's device alias (dkv_apply_plan or a
 * decode graph holding it). Under DKV_PLAN_MAPPED an operation first waits until the
 * device has released the buffer it is about to rewrite (the header's `applied` word,
 * set by the apply kernel); after wait_ms it fails with DKV_ERR_TIMEOUT and changes
 * nothing. Under DKV_PLAN_HOST there is no wait: the caller moves plans itself.
 * Errors: DKV_ERR_ARG (bad config), DKV_ERR_OOM (plan buffers), DKV_ERR_CUDA.
 */
int dkv_bm_create(const dkv_bm_config* cfg, dkv_bm** out);
int dkv_bm_destroy(dkv_bm* bm);

/*
 * Placement operations (see the policy above). Each writes a plan into the next plan
 * buffer. On error (DKV_ERR_ARG; DKV_ERR_CAPACITY when a tier has too few free ids or
 * the table too few rows or columns; DKV_ERR_TIMEOUT when the buffer was not released)
 * the manager and the plan buffers are unchanged.
 *   dkv_bm_add:    *row receives the new sequence's table row (= the old row count).
 *   dkv_bm_remove: *moved_from receives the old row of the sequence now at `row`, or -1
 *                  when `row` was the last row (the caller moves its per-row inputs).
 */
int dkv_bm_add(dkv_bm* bm, int32_t seq_len, int32_t* row);
int dkv_bm_remove(dkv_bm* bm, int32_t row, int32_t* moved_from);
int dkv_bm_step(dkv_bm* bm);

/* Active rows; current window W (blocks per sequence kept in HBM). */
int dkv_bm_rows(const dkv_bm* bm);
int64_t dkv_bm_window(const dkv_bm* bm);

/*
 * The plan buffer `slot` (0 or 1), or with slot = -1 the buffer the last operation wrote.
 * Returns the slot index (>= 0) or an error. host_plan / dev_plan (either may be NULL)
 * receive its host address and its device alias (NULL under DKV_PLAN_HOST).
 */
int dkv_bm_plan(const dkv_bm* bm, int slot, const void** host_plan, const void** dev_plan);

/*
 * Host snapshot of the manager's tables: block_table int32 [max_rows][max_blocks] (-1 where
 * unused), tier_map uint8 [max_rows][max_blocks] (0 where unused), seq_lens int32
 * [max_rows] (-1 for inactive rows). Any pointer may be NULL.
 */
int dkv_bm_tables(const dkv_bm* bm, int32_t* block_table, uint8_t* tier_map, int32_t* seq_lens);

/*
 * Apply a plan on `stream`: one kernel launch of fixed shape that reads the plan where it
 * lies (`plan` is a device pointer: the device alias of a DKV_PLAN_MAPPED buffer, or a
 * device copy), copies the moved blocks between the pool's tiers, and writes the device
 * tables (block_table int32 / tier_map uint8 [max_rows][max_blocks], seq_lens int32
 * [max_rows]). The counts are read on the device, so the launch can sit in a CUDA graph
 * and be replayed with new plans written to the same buffer. When the device has finished
 * reading the plan, the kernel sets the header's `applied` word (the buffer must be
 * host-visible and writable: a mapped plan buffer's device alias). Launches on one pool
 * must not overlap (they share a completion counter). A plan whose header does not
 * match max_rows / max_blocks, or whose moves or entries name a bad tier or id, is skipped
 * or partly skipped and flagged in the pool's status word (dkv_check: DKV_ERR_BAD_TABLE).
 */
int dkv_apply_plan(dkv_pool* pool, const void* plan, int32_t* block_table, uint8_t* tier_map,
                   int32_t* seq_lens, int max_rows, int max_blocks, void* stream);

/* One layer of a multi-layer decode step: x [B][hidden] bf16, Wqkv, out [B][Hq*D] bf16. */
typedef struct dkv_layer_io {
  int32_t layer;
  int32_t reserved;
  const uint16_t* x;
  const uint16_t* Wqkv;
  uint16_t* out;
} dkv_layer_io;

typedef struct dkv_graph dkv_graph;  /* an instantiated CUDA graph of one decode step */

/*
 * Capture one decode step of n_layers layers into a CUDA graph: dkv_apply_plan(plan) when
 * plan != NULL, then dkv_decode_step for each entry of `layers` in order, all with the
 * same tables, batch and workspace (the layers run one after another, so they share it).
 * Every argument is bound at capture; what changes between replays is memory contents:
 * the plan buffer, x, the tables. Nothing runs at creation. Errors: those of the captured
 * calls (nothing is left captured), DKV_ERR_CUDA.
 */
int dkv_decode_graph_create(dkv_pool* pool, const void* plan, int max_rows,
                            const dkv_layer_io* layers, int n_layers, int32_t* block_table,
                            int32_t* seq_lens, uint8_t* tier_map, int B, int max_blocks,
                            int hidden, int num_q_heads, float rope_theta, void* workspace,
                            size_t ws_bytes, dkv_graph** out);

/* Launch (replay) the graph on `stream`. */
int dkv_graph_launch(dkv_graph* graph, void* stream);
int dkv_graph_destroy(dkv_graph* graph);

#ifdef __cplusplus
}
#endif

#endif /* DKV_PLACEMENT_H_ */
