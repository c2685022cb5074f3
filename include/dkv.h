/*
 * dkv.h — C ABI of libdkv: a zero-copy, two-tier paged KV cache and the fused decode step
 * (QKV projection + RoPE + GQA split-K decode attention) for NVIDIA B200 (sm_100a).
 *
 * The problem these calls follow is DirectKV's ("长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI
 * 2026）", sections 问题与动机 and 核心方法): conventional KV offload stages host-resident KV
 * blocks into an HBM buffer before attention reads them, which costs GPU capacity and
 * moves the data twice; DirectKV lets the attention kernel read CPU-resident KV in place,
 * fuses the QKV projection with attention so the new K/V are consumed on chip and written
 * once, and overlaps fetch with compute in a warp-level pipeline. The paged-block pool and
 * the block table are the usual PagedAttention structures ("KV Offload" wiki page,
 * sections Swap-out / Swap-in: blocks are the unit that is freed and moved).
 *
 * Conventions shared by every call:
 *  - bf16 tensors are passed as `uint16_t*` holding raw bf16 bit patterns.
 *  - "device pointer" means an address the current CUDA device can dereference: device
 *    memory, or the device alias of mapped pinned host memory.
 *  - `stream` is a `cudaStream_t` passed as `void*` (NULL = the legacy default stream).
 *    Every call that takes a stream only enqueues work on it and never synchronises,
 *    except dkv_check and the pool create/destroy calls.
 *  - Return value: DKV_OK (0) or a negative DKV_ERR_* code. Nothing throws across the ABI.
 *    dkv_last_error() returns a thread-local message for the last failing call.
 *  - The library owns the pool and both tiers (unless `hbm_base` is supplied); the
 *    caller owns every other buffer (inputs, tables, outputs, workspaces).
 *  - Device-detected faults (bad tier value, physical block id out of range, a context
 *    longer than the block table) never trap: the kernel skips the offending block, sets
 *    a bit in the pool's status word, and dkv_check() reports DKV_ERR_BAD_TABLE.
 */
#ifndef DKV_H_
#define DKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DKV_OK               0
#define DKV_ERR_ARG         (-1)  /* invalid argument (null pointer, bad size, bad enum) */
#define DKV_ERR_CUDA        (-2)  /* a CUDA runtime/driver call failed */
#define DKV_ERR_OOM         (-3)  /* device or pinned-host allocation failed */
#define DKV_ERR_UNSUPPORTED (-4)  /* shape/device not supported (see each call) */
#define DKV_ERR_BAD_TABLE   (-5)  /* device-side table validation failed (dkv_check) */
#define DKV_ERR_TIMEOUT     (-6)  /* a bounded device-side wait gave up (dkv_check) */
#define DKV_ERR_CAPACITY    (-7)  /* request exceeds a fixed capacity */
#define DKV_ERR_INTERNAL    (-8)  /* a range check of the debug build (libdkv_debug.so, built
                                     with DKV_DEBUG) failed inside a kernel (dkv_check) */

#define DKV_TIER_HBM  0
#define DKV_TIER_HOST 1

#define DKV_LAYOUT_LAYER_FIRST 0  /* tier = [L][P][2][Hkv][T][D] */
#define DKV_LAYOUT_PAGE_FIRST  1  /* tier = [P][L][2][Hkv][T][D] */

#define DKV_HOST_WRITE_COMBINED 1 /* host tier allocated write-combined */
#define DKV_HOST_NUMA_NEAREST   2 /* host tier placed on the NUMA node nearest the pool's GPU
                                     (see dkv_host_numa_node) */

typedef struct dkv_pool dkv_pool;  /* opaque; owned by the library */

/*
 * Pool geometry. One physical block holds T consecutive tokens of one sequence for every
 * layer, both K and V, every kv head: per (layer, block, K|V, kv head) a contiguous
 * [T][D] bf16 chunk (4 KiB at T=16, D=128). DirectKV reorders the KV layout so that reads
 * of CPU-resident KV coalesce (核心方法); contiguous per-head chunks are that layout here.
 * The two layouts are Strata's layer-first / page-first decoupling ("「KV Cache 内存层级」
 * 系列总纲", §2.4 Strata).
 */
typedef struct dkv_pool_config {
  int32_t num_layers;    /* L >= 1 */
  int32_t num_kv_heads;  /* Hkv >= 1 */
  int32_t head_dim;      /* D: 64 or 128 */
  int32_t block_tokens;  /* T: 16 */
  int64_t hbm_blocks;    /* physical blocks in the HBM tier (>= 0) */
  int64_t host_blocks;   /* physical blocks in the host tier (>= 0) */
  int32_t layout;        /* DKV_LAYOUT_* */
  int32_t host_flags;    /* DKV_HOST_* bits (0: write-back pages, no NUMA preference) */
  void*   hbm_base;      /* optional caller-owned device buffer of at least the HBM tier's
                            size (256-byte aligned); NULL = the library allocates it */
} dkv_pool_config;

/* Launch tunables; 0 means "choose automatically". */
typedef struct dkv_tuning {
  int32_t attn_splits;   /* split-K factor of the attention grid (per sequence, kv head) */
  int32_t proj_splits;   /* cluster size of the projection (its reduction split), 0..8;
                            above hidden/64 it is cut to hidden/64 */
  int32_t attn_variant;  /* attention kernel: 0 automatic (see dkv_decode_attn_variant),
                            5 CUDA-core products with q in registers (G <= 4: three
                            one-warp consumer slots, a 6-stage ring, 4 CTAs/SM; G = 8: two
                            slots of two warps, a 4-stage ring, 3 CTAs/SM), 1 CUDA cores
                            with four slots and an 8-stage ring (3 CTAs/SM; G = 8: slots of
                            two warps, 1 CTA/SM), 6 tensor-core products (4-stage ring,
                            4 CTAs/SM), 7 tensor cores with an 8-stage ring (3 CTAs/SM);
                            other values are invalid. The tensor-core consumers are opt-in:
                            the design reserves the tensor cores for the projection */
  int32_t attn_lsu_hbm;  /* load paths of the CUDA-core attention, bits: 1 = HBM-tier blocks
                            by 16-byte cp.async instead of bulk copies (TMA engine); 2 =
                            host-tier blocks by bulk copies from the mapped host memory
                            instead of 16-byte cp.async from all 32 lanes of the producer */
  int32_t serial_launch; /* 1: launch the decode kernels without programmatic dependent
                            launch (each starts when the one before has finished: for
                            timing the kernels one by one, or when Wqkv is written by the
                            kernel directly ahead); 2: overlap only inside a step (the
                            attention streams cached KV while the projection finishes; the
                            kernel after the attention starts when it has finished);
                            0: overlap both boundaries (the attention also lets the next
                            kernel, e.g. the next step's projection, start early) */
  int32_t wait_limit_us; /* limit of each bounded wait inside the attention kernel, in
                            microseconds (0 = 4 s). On giving up a wait the kernel sets
                            DKV_ERR_TIMEOUT in the pool's status word and returns */
  int32_t test_withhold_block; /* test hook of the bounded waits: 1 = the attention's first
                            CTA (split 0, kv head 0, sequence 0) never loads its first block
                            nor signals its stage, so that stage's consumer gives up after
                            wait_limit_us (output of that (sequence, kv head) is then
                            undefined, dkv_check reports DKV_ERR_TIMEOUT); 0 = off */
  int32_t reserved[1];
} dkv_tuning;

/*
 * Create a pool on the current device: the HBM tier (device memory) and the host tier
 * (pinned host memory allocated mapped, so kernels read it in place through its device
 * alias with no staging copy: DirectKV 核心方法). Requires an sm_100 device.
 * Errors: DKV_ERR_ARG (bad geometry), DKV_ERR_UNSUPPORTED (D not 64/128, T != 16, not
 * sm_100), DKV_ERR_OOM (either allocation failed; nothing is leaked).
 * Tier contents are uninitialised.
 */
int dkv_pool_create(const dkv_pool_config* cfg, dkv_pool** out);

/*
 * NUMA placement of the host tier. GPUs of one host each read their own host tier over
 * their own PCIe link but share the host's memory (DirectKV leaves several GPUs sharing
 * CPU memory as future work: "长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", 局限与后续
 * 工作). With DKV_HOST_NUMA_NEAREST the pool allocates its host tier under a "preferred"
 * memory policy for the node its GPU's PCIe device reports, restoring the calling thread's
 * policy afterwards (a full node falls back to others; no error).
 *  - dkv_numa_node_of_pci: the node sysfs gives for a PCI device: reads
 *    <sysfs_root>/bus/pci/devices/<bus id, lower case, 4-digit domain>/numa_node
 *    (sysfs_root NULL = "/sys"); -1 when absent or negative (no NUMA information).
 *  - dkv_host_numa_node: the same for a CUDA device (its cudaDeviceGetPCIBusId); -1 if none.
 *  - dkv_pool_host_numa_node: the node that actually backs the first page of the pool's
 *    host tier (-1 without a host tier or when the kernel does not say), or DKV_ERR_ARG.
 */
int dkv_numa_node_of_pci(const char* sysfs_root, const char* pci_bus_id);
int dkv_host_numa_node(int device);
int dkv_pool_host_numa_node(const dkv_pool* pool);

/* Free both tiers (not a caller-supplied hbm_base) and the pool. Synchronises the device. */
int dkv_pool_destroy(dkv_pool* pool);

/*
 * Base address and size in bytes of a tier. For DKV_TIER_HOST, `*dev_ptr` is the device
 * alias; `host_ptr` (may be NULL) receives the host-side address of the same memory.
 */
int dkv_pool_tier_ptr(const dkv_pool* pool, int tier, void** dev_ptr, void** host_ptr,
                      size_t* bytes);

/* Set launch tunables for later calls on this pool (copied). NULL restores defaults. */
int dkv_pool_set_tuning(dkv_pool* pool, const dkv_tuning* tuning);

/*
 * Append n_tokens new tokens per sequence (e.g. a prefill's K/V) into the cache.
 * k, v: device [B][n_tokens][Hkv][D] bf16. Token t of sequence b goes to position
 * seq_lens[b] + t: slot (pos mod T) of logical block floor(pos / T), which lives in tier
 * tier_map[b*max_blocks + j] at physical index block_table[b*max_blocks + j].
 * block_table (int32), seq_lens (int32), tier_map (uint8) are device arrays. seq_lens is
 * not modified. Bad table entries are skipped and flagged (see dkv_check).
 */
int dkv_append_kv(dkv_pool* pool, int layer, const uint16_t* k, const uint16_t* v, int B,
                  int n_tokens, const int32_t* block_table, int max_blocks,
                  const int32_t* seq_lens, const uint8_t* tier_map, void* stream);

/*
 * Copy whole blocks between tiers (swap-in / swap-out, "KV Offload" wiki page, sections
 * Swap-out / Swap-in): for i < n, block src_ids[i] of tier src_tier -> block dst_ids[i] of
 * tier dst_tier, every layer, K and V, every kv head (bit-exact). Methods:
 *   DKV_COPY_DMA     one cudaMemcpyAsync per block and layer (runs of consecutive ids on
 *                    both sides are merged): the copy engine, as conventional offload does;
 *                    src_ids / dst_ids are HOST arrays.
 *   DKV_COPY_KERNEL  one kernel whose threads move 16-byte pieces (GPU-assisted I/O,
 *                    Strata, "「KV Cache 内存层级」系列总纲" §2.4); src_ids / dst_ids are
 *                    DEVICE arrays; bad ids are skipped and flagged (dkv_check).
 * The two tiers may be the same (a move within a tier); ranges must not overlap.
 */
#define DKV_COPY_DMA    0
#define DKV_COPY_KERNEL 1
int dkv_copy_blocks(dkv_pool* pool, int src_tier, int dst_tier, const int32_t* src_ids,
                    const int32_t* dst_ids, int n, int method, void* stream);

/* Bytes of caller-provided workspace dkv_decode_step needs for this shape. */
size_t dkv_decode_workspace_bytes(const dkv_pool* pool, int B, int max_blocks,
                                  int num_q_heads, int hidden);

/*
 * One decode step of one layer for a batch of B sequences (DirectKV 核心方法: QKV
 * projection fused with attention over CPU-resident KV, no staging buffer):
 *   qkv_b = Wqkv . x_b (no norm, no bias); rows [Hq q heads][Hkv k heads][Hkv v heads] x D
 *   q, k rotated by RoPE (rotate-half pairs (i, i+D/2), angle pos * theta^(-2i/D)) at
 *   pos = seq_lens[b];
 *   k_hat = bf16(k_rot), v_hat = bf16(v) written once into slot pos mod T of logical
 *   block floor(pos/T) (the table must cover ceil((pos+1)/T) blocks);
 *   out_b[h] = softmax over keys 0..pos of (q_h . k_t / sqrt(D)) applied to v_t, with
 *   q head h attending kv head h / (Hq/Hkv); keys 0..pos-1 come from the cache (either
 *   tier, read in place), key pos is (k_hat, v_hat).
 * x: device [B][hidden] bf16. Wqkv: device [(Hq+2Hkv)*D][hidden] bf16, row-major.
 * block_table: device int32 [B][max_blocks]; tier_map: device uint8 [B][max_blocks]
 * (0 = HBM, 1 = host); seq_lens: device int32 [B] (cached tokens; NOT incremented).
 * out: device [B][Hq*D] bf16. workspace: device, >= dkv_decode_workspace_bytes(...),
 * 256-byte aligned; its contents need no initialisation.
 * Supported: 1 <= B <= 32, hidden % 64 == 0, Hq % Hkv == 0 with Hq/Hkv in {1,2,4,8}.
 * Two kernels (projection; attention with the split combine fused); no host
 * synchronisation, no allocation, so the call can be captured into a CUDA graph.
 * Unless serial_launch is set (dkv_tuning), they are launched with programmatic dependent
 * launch: the projection may start while the kernel ahead of it in the stream is still
 * running, if that kernel signals programmatic launch completion early (this library's
 * kernels do), and then fetches part of Wqkv before waiting for it; everything else
 * (x, tables, positions, workspace, cache) is touched only after that kernel has
 * finished. So Wqkv must not be written by the kernel directly ahead of this call when
 * that kernel signals early. The attention streams cached KV while the projection
 * finishes (it writes only a slot the attention masks) and reads the projection's
 * outputs after it has finished. Seen from the stream, the call is ordered as usual.
 */
int dkv_decode_step(dkv_pool* pool, int layer, const uint16_t* x, const uint16_t* Wqkv,
                    const int32_t* block_table, const int32_t* seq_lens,
                    const uint8_t* tier_map, int B, int max_blocks, int hidden,
                    int num_q_heads, float rope_theta, uint16_t* out, void* workspace,
                    size_t ws_bytes, void* stream);

/*
 * The stages of dkv_decode_step as separate calls, with the same arguments and the same
 * workspace (for timing each stage). dkv_decode_step == project; attend(out).
 *   project: projection, RoPE, the single cache write of k_hat / v_hat, and q, k_hat,
 *            v_hat (fp32) for the attention — into the workspace.
 *   attend:  split-K partial softmax states over the cached blocks of both tiers; with
 *            out != NULL the last split of each (sequence, kv head) also merges the
 *            partial states with the new token's term (score q . k_hat, value v_hat) into
 *            out (the combine, fused).
 *   combine: the merge as its own kernel, for attend(out = NULL).
 * Called on its own, attend waits for the kernel ahead of it before reading anything
 * (only inside dkv_decode_step does it stream cached KV while the projection finishes).
 */
int dkv_decode_project(dkv_pool* pool, int layer, const uint16_t* x, const uint16_t* Wqkv,
                       const int32_t* block_table, const int32_t* seq_lens,
                       const uint8_t* tier_map, int B, int max_blocks, int hidden,
                       int num_q_heads, float rope_theta, void* workspace, size_t ws_bytes,
                       void* stream);
int dkv_decode_attend(dkv_pool* pool, int layer, const int32_t* block_table,
                      const int32_t* seq_lens, const uint8_t* tier_map, int B,
                      int max_blocks, int hidden, int num_q_heads, uint16_t* out,
                      void* workspace, size_t ws_bytes, void* stream);
int dkv_decode_combine(dkv_pool* pool, int B, int max_blocks, int hidden, int num_q_heads,
                       uint16_t* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * dkv_decode_step without a caller workspace, for callers that cannot allocate device
 * memory: a serving loop whose device memory is all reserved up front by its own allocator
 * (a cudaMalloc there fails or fragments that reservation), a latency-critical loop that
 * cannot take cudaMalloc's implicit synchronisation, or a plain C host with no device
 * allocator. The paper has no counterpart to this call; it is a deployment convenience.
 * Same arguments and results as dkv_decode_step; the workspace is a fixed array of
 * dkv_decode_static_workspace_capacity() bytes (16 MiB) in the library's own device memory,
 * which every GPU that loads the library holds until the process exits. The call allocates
 * nothing (no cudaMalloc/cudaFree, no allocating library routine).
 *  - The first call on a device looks up that device's array address (cudaGetSymbolAddress
 *    with the device current); make that first call before any stream capture. Under CUDA's
 *    lazy module loading (the default) the array's 16 MiB of device memory are committed at
 *    that first call, so a caller that reserves the rest of the device's memory up front
 *    makes one call first. The pool's device must be current (else DKV_ERR_ARG).
 *  - Shape errors return the same codes as dkv_decode_step (e.g. DKV_ERR_UNSUPPORTED for
 *    B > 32).
 *  - Shapes whose workspace (dkv_decode_workspace_bytes) exceeds the capacity are rejected
 *    with DKV_ERR_CAPACITY and nothing is launched.
 *  - Every call shares the one array per device and it keeps the last call's contents;
 *    nothing in it needs to start at zero (each step writes every word it later reads).
 *    Calls whose execution overlaps on the GPU (different streams, no ordering) race on it.
 */
int dkv_decode_step_static(dkv_pool* pool, int layer, const uint16_t* x, const uint16_t* Wqkv,
                           const int32_t* block_table, const int32_t* seq_lens,
                           const uint8_t* tier_map, int B, int max_blocks, int hidden,
                           int num_q_heads, float rope_theta, uint16_t* out, void* stream);

/* Size in bytes of the per-device static workspace dkv_decode_step_static uses. */
size_t dkv_decode_static_workspace_capacity(void);

/* The attention split-K factor dkv_decode_step uses for this shape: the pool's
 * dkv_tuning.attn_splits, or, when that is 0, the automatic count. With units = B * Hkv
 * and slots = the GPU's SMs x the chosen kernel shape's CTAs per SM: Hq/Hkv = 4, the most
 * splits that fit in one wave of slots (two waves above 64 units); Hq/Hkv = 8, one wave
 * for variant 1 and the most within 2.33 waves for variant 5 (0.86 of a wave where that
 * would be more than 64 splits); other group sizes, about 2.9
 * waves; the tensor-core variants, about 7/8 of one wave and at most 32. Never more than
 * max_blocks. Returns the count (> 0) or a negative DKV_ERR_* code. */
int dkv_decode_attn_splits(const dkv_pool* pool, int B, int max_blocks, int num_q_heads);

/* The attention kernel variant dkv_decode_step runs for this shape: the pool's
 * dkv_tuning.attn_variant, or, when that is 0, the automatic choice (Hq/Hkv = 4: 5 when its
 * split-K ranges keep at least 39 blocks of the table each, else 1; Hq/Hkv = 8: 5 when they
 * keep at least 6 blocks and there are at most 64 of them (at least 40 blocks when the
 * automatic count was cut under one wave), else 1; other group sizes: 1).
 * Returns the variant (> 0) or a negative DKV_ERR_* code. */
int dkv_decode_attn_variant(const dkv_pool* pool, int B, int max_blocks, int num_q_heads);

/*
 * Block-layout permutation (Strata's layout decoupling with GPU-driven copy: "「KV Cache
 * 内存层级」系列总纲", §2.4 Strata): copy `src` laid out as [A][Bn][chunk] into `dst` as
 * [Bn][A][chunk], where for src_layout == DKV_LAYOUT_LAYER_FIRST A = num_layers and
 * Bn = num_blocks (result page-first), and for DKV_LAYOUT_PAGE_FIRST A = num_blocks and
 * Bn = num_layers (result layer-first). chunk_bytes = 2 * Hkv * T * D * 2 (one block of
 * one layer), a multiple of 16. src and dst are device pointers (either may be the device
 * alias of mapped host memory), 16-byte aligned, not overlapping. Bit-exact.
 */
int dkv_permute_layout(const void* src, void* dst, int src_layout, int num_layers,
                       int64_t num_blocks, int64_t chunk_bytes, void* stream);

/* Convert a whole tier of the pool into the other layout, written to `dst`
 * (dst_bytes >= the tier's size). The pool itself is not modified. */
int dkv_convert_layout(dkv_pool* pool, int tier, void* dst, size_t dst_bytes, void* stream);

/*
 * Zero-copy GEMM study (DirectKV's motivating experiment, Fig. 2(a) as quoted in
 * "「KV Cache 内存层级」系列总纲", §一 and §四; CPU-aware tiling, §2.1):
 *   C[M][N] (fp32) = A[M][K] (bf16, device memory) . B[K][N], with B stored column-major as
 *   Bt[N][K] (bf16; Bt[n][k] = B[k][n]) in mapped pinned host memory (pass its device
 *   alias) or, for DKV_GEMM_DEVICE, in device memory.
 * Variants:
 *   DKV_GEMM_CPU_AWARE        B-panel-major tile order: each B column panel is copied
 *                             from host memory into a rotating HBM panel buffer (inside the
 *                             workspace) exactly once and read from there, so each B tile
 *                             crosses the host link once; A is re-read from HBM per panel.
 *   DKV_GEMM_NAIVE_ZERO_COPY  row-major tile order: B re-read over the host link by every
 *                             128-row tile row of C.
 *   DKV_GEMM_STAGED_SWAP      cudaMemcpyAsync of all of B into the workspace ("swap" into a
 *                             GPU buffer), then the product from device memory.
 *   DKV_GEMM_DEVICE           A and Bt both in device memory.
 * Shapes: M % 128 == 0, N % 256 == 0, K % 64 == 0 (else DKV_ERR_UNSUPPORTED). Pointers
 * 256-byte aligned. workspace >= dkv_gemm_workspace_bytes(variant, M, N, K): its first 4
 * bytes are a device status word the kernel clears and sets on a device-side timeout;
 * DKV_GEMM_STAGED_SWAP also holds the staged copy of B there. fp32 accumulation on the
 * tensor cores (tcgen05, bf16 inputs).
 */
/*
 * Mapped pinned host memory for operands read zero-copy (e.g. B of the GEMM study):
 * cudaHostAlloc(mapped [| write-combined]); `dev_ptr` receives the device alias.
 * Free with dkv_host_free. Errors: DKV_ERR_ARG, DKV_ERR_OOM.
 */
int dkv_host_alloc_mapped(size_t bytes, int host_flags, void** host_ptr, void** dev_ptr);
int dkv_host_free(void* host_ptr);

#define DKV_GEMM_CPU_AWARE       0
#define DKV_GEMM_NAIVE_ZERO_COPY 1
#define DKV_GEMM_STAGED_SWAP     2
#define DKV_GEMM_DEVICE          3

size_t dkv_gemm_workspace_bytes(int variant, int M, int N, int K);
int dkv_gemm(int variant, const uint16_t* A, const uint16_t* Bt, float* C, int M, int N, int K,
             void* workspace, size_t ws_bytes, void* stream);

/*
 * Synchronise `stream`, then read and clear the pool's device status word.
 * Returns DKV_OK, DKV_ERR_BAD_TABLE (a kernel skipped a block with a bad tier or physical
 * id, or a context exceeding max_blocks*T), DKV_ERR_TIMEOUT, DKV_ERR_INTERNAL (debug build
 * only: a kernel's computed block, slot or workspace index fell outside its buffer; the
 * access was skipped), or DKV_ERR_CUDA.
 */
int dkv_check(dkv_pool* pool, void* stream);

/* Thread-local message describing the last failing call on this thread ("" if none). */
const char* dkv_last_error(void);

/* Library version string. */
const char* dkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DKV_H_ */
