// NUMA placement of the pinned host tier.
//
// Several GPUs of one host can each read their own pool's host tier in place over their own
// PCIe link, but they share the host's memory: DirectKV names GPUs sharing the CPU's memory
// as future work and leaves the contention untested ("长上下文 LLM 的零拷贝 KV Cache 卸载
// （OSDI 2026）", 局限与后续工作 and 批判性分析). The one placement choice this path has is
// which NUMA node backs each GPU's host tier: the node the GPU's PCIe root hangs off, so
// its zero-copy reads do not cross the inter-socket link and replicas on different sockets
// draw on different memory controllers.
//
// The node of a GPU is read from sysfs (<root>/bus/pci/devices/<domain:bus:dev.fn>/numa_node,
// -1 when the platform reports none). The pool binds its host-tier allocation there with a
// "preferred" memory policy on the allocating thread for the duration of cudaHostAlloc
// (pinning faults the pages in on that thread), then restores the thread's policy; a full
// node falls back to other nodes instead of failing.
#include <ctype.h>
#include <errno.h>
#include <linux/mempolicy.h>
#include <stdio.h>
#include <string.h>
#include <sys/syscall.h>
#include <unistd.h>

#include "dkv_internal.h"

namespace dkv {

constexpr int kMaxNodes = 1024;
constexpr int kMaskWords = kMaxNodes / 64;

static long sys_get_mempolicy(int* mode, unsigned long* mask, unsigned long maxnode, void* addr, unsigned flags) {
  return syscall(SYS_get_mempolicy, mode, mask, maxnode, addr, flags);
}
static long sys_set_mempolicy(int mode, const unsigned long* mask, unsigned long maxnode) {
  return syscall(SYS_set_mempolicy, mode, mask, maxnode);
}

int numa_node_of_pci(const char* sysfs_root, const char* pci_bus_id) {
  if (!pci_bus_id || !*pci_bus_id) return -1;
  char id[64];
  size_t n = strlen(pci_bus_id);
  if (n >= sizeof(id)) return -1;
  for (size_t i = 0; i <= n; ++i) id[i] = (char)tolower((unsigned char)pci_bus_id[i]);
  // cudaDeviceGetPCIBusId gives "dddd:bb:dd.f" (some platforms an 8-digit domain); sysfs
  // names devices with a 4-digit domain
  const char* colon = strchr(id, ':');
  const char* tail = id;
  if (colon && colon - id > 4) tail = colon - 4;
  char path[512];
  snprintf(path, sizeof(path), "%s/bus/pci/devices/%s/numa_node", sysfs_root ? sysfs_root : "/sys", tail);
  FILE* f = fopen(path, "r");
  if (!f) return -1;
  int node = -1;
  if (fscanf(f, "%d", &node) != 1) node = -1;
  fclose(f);
  return node >= 0 && node < kMaxNodes ? node : -1;
}

int gpu_numa_node(int device) {
  char bus[64];
  if (cudaDeviceGetPCIBusId(bus, (int)sizeof(bus), device) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return numa_node_of_pci("/sys", bus);
}

// Thread memory policy, saved and restored around an allocation.
struct SavedPolicy {
  int mode = MPOL_DEFAULT;
  unsigned long mask[kMaskWords] = {};
  bool valid = false;
};

bool prefer_node(int node, SavedPolicy* saved) {
  if (node < 0 || node >= kMaxNodes) return false;
  saved->valid = sys_get_mempolicy(&saved->mode, saved->mask, kMaxNodes, nullptr, 0) == 0;
  if (!saved->valid) return false;
  unsigned long mask[kMaskWords] = {};
  mask[node / 64] = 1ul << (node % 64);
  return sys_set_mempolicy(MPOL_PREFERRED, mask, kMaxNodes) == 0;
}

void restore_policy(const SavedPolicy& saved) {
  if (!saved.valid) return;
  const bool empty_mask = saved.mode == MPOL_DEFAULT || saved.mode == MPOL_LOCAL;
  sys_set_mempolicy(saved.mode, empty_mask ? nullptr : saved.mask, empty_mask ? 0 : kMaxNodes);
}

// cudaHostAlloc with the pages preferably on `node` (< 0: no preference).
int alloc_host_on_node(size_t bytes, unsigned flags, int node, void** out) {
  SavedPolicy saved;
  const bool bound = prefer_node(node, &saved);
  const cudaError_t e = cudaHostAlloc(out, bytes, flags);
  if (bound) restore_policy(saved);
  return e == cudaSuccess ? DKV_OK : (int)e;
}

int node_of_address(const void* addr) {
  int node = -1;
  if (sys_get_mempolicy(&node, nullptr, 0, const_cast<void*>(addr), MPOL_F_NODE | MPOL_F_ADDR) != 0) return -1;
  return node;
}

}  // namespace dkv

using namespace dkv;

extern "C" {

int dkv_numa_node_of_pci(const char* sysfs_root, const char* pci_bus_id) {
  return numa_node_of_pci(sysfs_root, pci_bus_id);
}

int dkv_host_numa_node(int device) { return gpu_numa_node(device); }

int dkv_pool_host_numa_node(const dkv_pool* pool) {
  if (!pool) return set_error(DKV_ERR_ARG, "dkv_pool_host_numa_node: null pool");
  if (!pool->host_h) return -1;
  return node_of_address(pool->host_h);
}

}  // extern "C"
