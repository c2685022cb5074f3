// Block manager: recency-window placement of each sequence's KV blocks over the HBM and
// host tiers, written out as plans that the device applies (dkv_plan.cu).
//
// Hot KV stays in HBM and cold KV is read in place from the host tier (DirectKV summary
// page, "长上下文 LLM 的零拷贝 KV Cache 卸载（OSDI 2026）", section 局限与后续工作:
// adaptive placement with no large staging buffer; the "KV Offload" wiki page's tier
// table puts the KV being decoded in HBM). The policy, its operations and the plan format
// are stated in dkv_placement.h.
//
// State per row r: len[r] cached tokens, nb = len / T + 1 logical blocks, whose ids and
// tiers live in the host table [max_rows][max_blocks]. The policy keeps the invariant
// hbm[r] = min(W, nb): a row's HBM blocks are always its newest ones, so the oldest HBM
// block is logical block nb - hbm[r] and the newest host block is nb - hbm[r] - 1.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <functional>
#include <new>
#include <queue>
#include <thread>
#include <vector>

#include "../../include/dkv_placement.h"

namespace dkv {
int set_error(int code, const char* fmt, ...);  // thread-local message (dkv_pool.cu)
}

namespace {

using dkv::set_error;

// Free physical ids of one tier; the smallest is handed out first.
struct FreeIds {
  std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> q;
  void init(int64_t n) {
    std::vector<int64_t> v((size_t)n);
    for (int64_t i = 0; i < n; ++i) v[(size_t)i] = i;
    q = decltype(q)(std::greater<int64_t>(), std::move(v));
  }
  int64_t take() {
    const int64_t i = q.top();
    q.pop();
    return i;
  }
  void give(int64_t i) { q.push(i); }
  int64_t size() const { return (int64_t)q.size(); }
};

}  // namespace

struct dkv_bm {
  dkv_bm_config cfg;
  int n = 0;                       // active rows
  std::vector<int32_t> len;        // [max_rows]
  std::vector<int32_t> hbm;        // [max_rows] HBM blocks held (= min(W, nb) at rest)
  std::vector<int32_t> id;         // [max_rows * max_blocks]
  std::vector<uint8_t> tier;       // [max_rows * max_blocks]
  FreeIds free_ids[2];
  // plan under construction
  std::vector<dkv_plan_move> moves;
  std::vector<int64_t> dirty;      // flat (row, block) indices touched
  std::vector<uint8_t> dirty_mark;
  // plan buffers
  size_t plan_bytes = 0;
  uint8_t* plan_h[2] = {nullptr, nullptr};
  void* plan_d[2] = {nullptr, nullptr};
  int next_slot = 0;
  int last_slot = -1;

  int64_t T() const { return cfg.block_tokens; }
  int32_t nb_of(int64_t l) const { return (int32_t)(l / cfg.block_tokens + 1); }
  int64_t window_for(int rows) const { return rows > 0 ? cfg.hbm_budget / rows : 0; }
  size_t at(int r, int j) const { return (size_t)r * cfg.max_blocks + j; }

  void touch(int r, int j) {
    const size_t k = at(r, j);
    if (!dirty_mark[k]) {
      dirty_mark[k] = 1;
      dirty.push_back((int64_t)k);
    }
  }
  void begin() {
    moves.clear();
    dirty.clear();
  }
  // Oldest HBM block of row r -> host tier.
  void demote_oldest(int r) {
    const int j = nb_of(len[r]) - hbm[r];
    const size_t k = at(r, j);
    const int64_t old = id[k], nw = free_ids[DKV_TIER_HOST].take();
    free_ids[DKV_TIER_HBM].give(old);
    id[k] = (int32_t)nw;
    tier[k] = DKV_TIER_HOST;
    hbm[r] -= 1;
    moves.push_back({DKV_TIER_HBM, (int32_t)old, DKV_TIER_HOST, (int32_t)nw});
    touch(r, j);
  }
  // Newest host block of row r -> HBM.
  void promote_newest(int r) {
    const int j = nb_of(len[r]) - hbm[r] - 1;
    const size_t k = at(r, j);
    const int64_t old = id[k], nw = free_ids[DKV_TIER_HBM].take();
    free_ids[DKV_TIER_HOST].give(old);
    id[k] = (int32_t)nw;
    tier[k] = DKV_TIER_HBM;
    hbm[r] += 1;
    moves.push_back({DKV_TIER_HOST, (int32_t)old, DKV_TIER_HBM, (int32_t)nw});
    touch(r, j);
  }
  // Wait until the device released the buffer the next plan goes to (mapped plans only).
  int wait_released() const {
    if (cfg.plan_memory != DKV_PLAN_MAPPED) return DKV_OK;
    volatile int32_t* applied = &reinterpret_cast<dkv_plan_header*>(plan_h[next_slot])->applied;
    if (!*applied) {
      const int ms = cfg.wait_ms > 0 ? cfg.wait_ms : 10000;
      const auto t0 = std::chrono::steady_clock::now();
      while (!*applied) {
        if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(ms))
          return set_error(DKV_ERR_TIMEOUT, "dkv_bm: plan buffer %d still holds an unapplied plan after %d ms",
                           next_slot, ms);
        std::this_thread::yield();
      }
    }
    std::atomic_thread_fence(std::memory_order_acquire);
    return DKV_OK;
  }
  // Write the plan under construction into the next buffer.
  void finish() {
    uint8_t* p = plan_h[next_slot];
    const int64_t cap = (int64_t)cfg.max_rows * cfg.max_blocks;
    auto* mv = reinterpret_cast<dkv_plan_move*>(p + sizeof(dkv_plan_header));
    auto* en = reinterpret_cast<dkv_plan_entry*>(mv + cap);
    auto* sl = reinterpret_cast<int32_t*>(en + cap);
    std::copy(moves.begin(), moves.end(), mv);
    std::sort(dirty.begin(), dirty.end());
    for (size_t i = 0; i < dirty.size(); ++i) {
      const int64_t k = dirty[i];
      dirty_mark[(size_t)k] = 0;
      en[i] = {(int32_t)(k / cfg.max_blocks), (int32_t)(k % cfg.max_blocks), (int32_t)tier[(size_t)k],
               id[(size_t)k]};
    }
    for (int r = 0; r < n; ++r) sl[r] = len[r];
    dkv_plan_header h;
    h.n_moves = (int32_t)moves.size();
    h.n_entries = (int32_t)dirty.size();
    h.n_rows = n;
    h.max_blocks = cfg.max_blocks;
    h.move_cap = (int32_t)cap;
    h.entry_cap = (int32_t)cap;
    h.max_rows = cfg.max_rows;
    h.applied = 0;
    std::atomic_thread_fence(std::memory_order_release);
    *reinterpret_cast<dkv_plan_header*>(p) = h;
    last_slot = next_slot;
    next_slot ^= 1;
  }
};

extern "C" {

size_t dkv_plan_bytes(int max_rows, int max_blocks) {
  if (max_rows < 1 || max_blocks < 1) return 0;
  const int64_t cap = (int64_t)max_rows * max_blocks;
  if (cap > (int64_t)INT32_MAX / 2) return 0;
  return sizeof(dkv_plan_header) + (size_t)cap * (sizeof(dkv_plan_move) + sizeof(dkv_plan_entry)) +
         (size_t)max_rows * sizeof(int32_t);
}

int dkv_bm_create(const dkv_bm_config* c, dkv_bm** out) {
  if (!c || !out) return set_error(DKV_ERR_ARG, "dkv_bm_create: null argument");
  *out = nullptr;
  if (c->max_rows < 1 || c->max_blocks < 1 || c->block_tokens < 1 || c->hbm_ids < 0 || c->host_ids < 0 ||
      c->hbm_budget < 0 || c->hbm_ids > INT32_MAX || c->host_ids > INT32_MAX || c->wait_ms < 0 ||
      (c->plan_memory != DKV_PLAN_MAPPED && c->plan_memory != DKV_PLAN_HOST))
    return set_error(DKV_ERR_ARG, "dkv_bm_create: bad configuration");
  if (c->hbm_budget > 0 && c->hbm_ids < c->hbm_budget + 1)
    return set_error(DKV_ERR_ARG, "dkv_bm_create: hbm_ids must be >= hbm_budget + 1");
  const size_t bytes = dkv_plan_bytes(c->max_rows, c->max_blocks);
  if (!bytes) return set_error(DKV_ERR_ARG, "dkv_bm_create: table too large");
  dkv_bm* bm = new (std::nothrow) dkv_bm;
  if (!bm) return set_error(DKV_ERR_OOM, "dkv_bm_create: out of host memory");
  try {
    bm->cfg = *c;
    const size_t cells = (size_t)c->max_rows * c->max_blocks;
    bm->len.assign((size_t)c->max_rows, -1);
    bm->hbm.assign((size_t)c->max_rows, 0);
    bm->id.assign(cells, -1);
    bm->tier.assign(cells, 0);
    bm->dirty_mark.assign(cells, 0);
    bm->free_ids[DKV_TIER_HBM].init(c->hbm_ids);
    bm->free_ids[DKV_TIER_HOST].init(c->host_ids);
  } catch (const std::bad_alloc&) {
    delete bm;
    return set_error(DKV_ERR_OOM, "dkv_bm_create: out of host memory");
  }
  bm->plan_bytes = bytes;
  for (int s = 0; s < 2; ++s) {
    if (c->plan_memory == DKV_PLAN_MAPPED) {
      void* h = nullptr;
      cudaError_t e = cudaHostAlloc(&h, bytes, cudaHostAllocMapped);
      if (e != cudaSuccess) {
        dkv_bm_destroy(bm);
        return set_error(e == cudaErrorMemoryAllocation ? DKV_ERR_OOM : DKV_ERR_CUDA,
                         "dkv_bm_create: cudaHostAlloc: %s", cudaGetErrorString(e));
      }
      bm->plan_h[s] = static_cast<uint8_t*>(h);
      e = cudaHostGetDevicePointer(&bm->plan_d[s], h, 0);
      if (e != cudaSuccess) {
        dkv_bm_destroy(bm);
        return set_error(DKV_ERR_CUDA, "dkv_bm_create: cudaHostGetDevicePointer: %s", cudaGetErrorString(e));
      }
    } else {
      bm->plan_h[s] = static_cast<uint8_t*>(::operator new(bytes, std::align_val_t(64), std::nothrow));
      if (!bm->plan_h[s]) {
        dkv_bm_destroy(bm);
        return set_error(DKV_ERR_OOM, "dkv_bm_create: out of host memory");
      }
    }
    // an empty plan: applying it before any operation changes nothing
    std::fill(bm->plan_h[s], bm->plan_h[s] + sizeof(dkv_plan_header), 0);
    auto* h = reinterpret_cast<dkv_plan_header*>(bm->plan_h[s]);
    h->max_blocks = c->max_blocks;
    h->max_rows = c->max_rows;
    h->move_cap = h->entry_cap = c->max_rows * c->max_blocks;
    h->applied = 1;  // nothing pending: the first operations need not wait
  }
  *out = bm;
  return DKV_OK;
}

int dkv_bm_destroy(dkv_bm* bm) {
  if (!bm) return DKV_OK;
  for (int s = 0; s < 2; ++s) {
    if (!bm->plan_h[s]) continue;
    if (bm->cfg.plan_memory == DKV_PLAN_MAPPED)
      cudaFreeHost(bm->plan_h[s]);
    else
      ::operator delete(bm->plan_h[s], std::align_val_t(64));
  }
  delete bm;
  return DKV_OK;
}

int dkv_bm_add(dkv_bm* bm, int32_t seq_len, int32_t* row) {
  if (!bm || seq_len < 0) return set_error(DKV_ERR_ARG, "dkv_bm_add: bad argument");
  if (bm->n >= bm->cfg.max_rows) return set_error(DKV_ERR_CAPACITY, "dkv_bm_add: all %d rows in use", bm->n);
  const int32_t nb = bm->nb_of(seq_len);
  if (nb > bm->cfg.max_blocks)
    return set_error(DKV_ERR_CAPACITY, "dkv_bm_add: %d blocks exceed max_blocks %d", nb, bm->cfg.max_blocks);
  const int64_t W = bm->window_for(bm->n + 1);
  int64_t demote = 0;
  for (int r = 0; r < bm->n; ++r) demote += std::max<int64_t>(0, bm->hbm[r] - W);
  const int64_t hot = std::min<int64_t>(W, nb);
  if (bm->free_ids[DKV_TIER_HOST].size() < demote + (nb - hot) ||
      bm->free_ids[DKV_TIER_HBM].size() + demote < hot)
    return set_error(DKV_ERR_CAPACITY, "dkv_bm_add: not enough free blocks");
  if (int rc = bm->wait_released()) return rc;
  bm->begin();
  for (int r = 0; r < bm->n; ++r)
    while (bm->hbm[r] > W) bm->demote_oldest(r);
  const int r = bm->n;
  for (int j = 0; j < nb; ++j) {
    const int t = j >= nb - hot ? DKV_TIER_HBM : DKV_TIER_HOST;
    const size_t k = bm->at(r, j);
    bm->id[k] = (int32_t)bm->free_ids[t].take();
    bm->tier[k] = (uint8_t)t;
    bm->touch(r, j);
  }
  bm->len[r] = seq_len;
  bm->hbm[r] = (int32_t)hot;
  bm->n += 1;
  bm->finish();
  if (row) *row = r;
  return DKV_OK;
}

int dkv_bm_remove(dkv_bm* bm, int32_t row, int32_t* moved_from) {
  if (!bm || row < 0 || row >= bm->n) return set_error(DKV_ERR_ARG, "dkv_bm_remove: bad row");
  if (int rc = bm->wait_released()) return rc;
  bm->begin();
  const int32_t nb = bm->nb_of(bm->len[row]);
  for (int j = 0; j < nb; ++j) {
    const size_t k = bm->at(row, j);
    bm->free_ids[bm->tier[k]].give(bm->id[k]);
  }
  const int last = bm->n - 1;
  if (row != last) {
    const int32_t nbl = bm->nb_of(bm->len[last]);
    for (int j = 0; j < nbl; ++j) {
      bm->id[bm->at(row, j)] = bm->id[bm->at(last, j)];
      bm->tier[bm->at(row, j)] = bm->tier[bm->at(last, j)];
      bm->touch(row, j);
    }
    for (int j = nbl; j < bm->cfg.max_blocks; ++j) {
      bm->id[bm->at(row, j)] = -1;
      bm->tier[bm->at(row, j)] = 0;
    }
    bm->len[row] = bm->len[last];
    bm->hbm[row] = bm->hbm[last];
  }
  for (int j = 0; j < bm->cfg.max_blocks; ++j) {
    bm->id[bm->at(last, j)] = -1;
    bm->tier[bm->at(last, j)] = 0;
  }
  bm->len[last] = -1;
  bm->hbm[last] = 0;
  bm->n -= 1;
  const int64_t W = bm->window_for(bm->n);
  for (int r = 0; r < bm->n; ++r) {
    const int64_t want = std::min<int64_t>(W, bm->nb_of(bm->len[r]));
    while (bm->hbm[r] < want) bm->promote_newest(r);
  }
  bm->finish();
  if (moved_from) *moved_from = row != last ? last : -1;
  return DKV_OK;
}

int dkv_bm_step(dkv_bm* bm) {
  if (!bm) return set_error(DKV_ERR_ARG, "dkv_bm_step: null manager");
  const int64_t W = bm->window_for(bm->n);
  int64_t host_need = 0;
  for (int r = 0; r < bm->n; ++r) {
    const int64_t l = (int64_t)bm->len[r] + 1;
    if (l > INT32_MAX - 1) return set_error(DKV_ERR_CAPACITY, "dkv_bm_step: sequence too long");
    if (l % bm->T()) continue;
    if (bm->nb_of(l) > bm->cfg.max_blocks)
      return set_error(DKV_ERR_CAPACITY, "dkv_bm_step: row %d outgrows max_blocks", r);
    host_need += (W == 0 || bm->hbm[r] + 1 > W) ? 1 : 0;
  }
  if (bm->free_ids[DKV_TIER_HOST].size() < host_need)
    return set_error(DKV_ERR_CAPACITY, "dkv_bm_step: not enough free host blocks");
  if (int rc = bm->wait_released()) return rc;
  bm->begin();
  for (int r = 0; r < bm->n; ++r) {
    bm->len[r] += 1;
    if (bm->len[r] % bm->T() == 0) {
      const int j = bm->nb_of(bm->len[r]) - 1;
      const int t = W >= 1 ? DKV_TIER_HBM : DKV_TIER_HOST;
      const size_t k = bm->at(r, j);
      bm->id[k] = (int32_t)bm->free_ids[t].take();
      bm->tier[k] = (uint8_t)t;
      if (t == DKV_TIER_HBM) bm->hbm[r] += 1;
      bm->touch(r, j);
    }
    while (bm->hbm[r] > W) bm->demote_oldest(r);
  }
  bm->finish();
  return DKV_OK;
}

int dkv_bm_rows(const dkv_bm* bm) { return bm ? bm->n : set_error(DKV_ERR_ARG, "dkv_bm_rows: null manager"); }

int64_t dkv_bm_window(const dkv_bm* bm) {
  return bm ? bm->window_for(bm->n) : set_error(DKV_ERR_ARG, "dkv_bm_window: null manager");
}

int dkv_bm_plan(const dkv_bm* bm, int slot, const void** host_plan, const void** dev_plan) {
  if (!bm || slot < -1 || slot > 1) return set_error(DKV_ERR_ARG, "dkv_bm_plan: bad argument");
  const int s = slot >= 0 ? slot : (bm->last_slot >= 0 ? bm->last_slot : 0);
  if (host_plan) *host_plan = bm->plan_h[s];
  if (dev_plan) *dev_plan = bm->plan_d[s];
  return s;
}

int dkv_bm_tables(const dkv_bm* bm, int32_t* block_table, uint8_t* tier_map, int32_t* seq_lens) {
  if (!bm) return set_error(DKV_ERR_ARG, "dkv_bm_tables: null manager");
  if (block_table) std::copy(bm->id.begin(), bm->id.end(), block_table);
  if (tier_map) std::copy(bm->tier.begin(), bm->tier.end(), tier_map);
  if (seq_lens) std::copy(bm->len.begin(), bm->len.end(), seq_lens);
  return DKV_OK;
}

}  // extern "C"
