"""ctypes binding of libdkv's C ABI (include/dkv.h), one Python function per C entry point
with the same name. Argument marshalling only: tensors are passed as raw pointers, the
current torch CUDA stream as the stream handle, and every computation happens in the
library's kernels. If the library is missing the calls raise; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DKV_LIBRARY=debug selects the build with device-side range checks (libdkv_debug.so)
LIB_PATH = os.path.join(_HERE, "libdkv_debug.so" if os.environ.get("DKV_LIBRARY") == "debug" else "libdkv.so")
INCLUDE = os.path.join(os.path.dirname(_HERE), "include")
HEADER = os.path.join(INCLUDE, "dkv.h")

DKV_OK = 0
DKV_ERR_ARG = -1
DKV_ERR_CUDA = -2
DKV_ERR_OOM = -3
DKV_ERR_UNSUPPORTED = -4
DKV_ERR_BAD_TABLE = -5
DKV_ERR_TIMEOUT = -6
DKV_ERR_CAPACITY = -7
DKV_ERR_INTERNAL = -8

DKV_TIER_HBM = 0
DKV_TIER_HOST = 1
DKV_LAYOUT_LAYER_FIRST = 0
DKV_LAYOUT_PAGE_FIRST = 1
DKV_HOST_WRITE_COMBINED = 1
DKV_HOST_NUMA_NEAREST = 2
DKV_COPY_DMA = 0
DKV_COPY_KERNEL = 1
DKV_GEMM_CPU_AWARE = 0
DKV_GEMM_NAIVE_ZERO_COPY = 1
DKV_GEMM_STAGED_SWAP = 2
DKV_GEMM_DEVICE = 3
DKV_PLAN_MAPPED = 0
DKV_PLAN_HOST = 1


class DkvError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("dkv error %d: %s" % (code, msg))
        self.code = code


class dkv_pool_config(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_tokens", ctypes.c_int32),
                ("hbm_blocks", ctypes.c_int64), ("host_blocks", ctypes.c_int64),
                ("layout", ctypes.c_int32), ("host_flags", ctypes.c_int32),
                ("hbm_base", ctypes.c_void_p)]


class dkv_tuning(ctypes.Structure):
    _fields_ = [("attn_splits", ctypes.c_int32), ("proj_splits", ctypes.c_int32),
                ("attn_variant", ctypes.c_int32), ("attn_lsu_hbm", ctypes.c_int32),
                ("serial_launch", ctypes.c_int32), ("wait_limit_us", ctypes.c_int32),
                ("test_withhold_block", ctypes.c_int32), ("reserved", ctypes.c_int32 * 1)]


class dkv_bm_config(ctypes.Structure):
    _fields_ = [("max_rows", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("block_tokens", ctypes.c_int32), ("plan_memory", ctypes.c_int32),
                ("hbm_ids", ctypes.c_int64), ("host_ids", ctypes.c_int64),
                ("hbm_budget", ctypes.c_int64), ("wait_ms", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class dkv_layer_io(ctypes.Structure):
    _fields_ = [("layer", ctypes.c_int32), ("reserved", ctypes.c_int32), ("x", ctypes.c_void_p),
                ("Wqkv", ctypes.c_void_p), ("out", ctypes.c_void_p)]


PLAN_HEADER_BYTES = 32

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float

_SIGS = {
    "dkv_pool_create": (_I, [ctypes.POINTER(dkv_pool_config), ctypes.POINTER(_P)]),
    "dkv_pool_destroy": (_I, [_P]),
    "dkv_pool_tier_ptr": (_I, [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_SZ)]),
    "dkv_pool_set_tuning": (_I, [_P, ctypes.POINTER(dkv_tuning)]),
    "dkv_append_kv": (_I, [_P, _I, _P, _P, _I, _I, _P, _I, _P, _P, _P]),
    "dkv_decode_workspace_bytes": (_SZ, [_P, _I, _I, _I, _I]),
    "dkv_decode_step": (_I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P, _SZ, _P]),
    "dkv_decode_project": (_I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _SZ, _P]),
    "dkv_decode_attend": (_I, [_P, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "dkv_decode_combine": (_I, [_P, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "dkv_decode_attn_splits": (_I, [_P, _I, _I, _I]),
    "dkv_decode_attn_variant": (_I, [_P, _I, _I, _I]),
    "dkv_decode_step_static": (_I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P]),
    "dkv_decode_static_workspace_capacity": (_SZ, []),
    "dkv_permute_layout": (_I, [_P, _P, _I, _I, _I64, _I64, _P]),
    "dkv_convert_layout": (_I, [_P, _I, _P, _SZ, _P]),
    "dkv_check": (_I, [_P, _P]),
    "dkv_copy_blocks": (_I, [_P, _I, _I, _P, _P, _I, _I, _P]),
    "dkv_gemm_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "dkv_host_alloc_mapped": (_I, [_SZ, _I, ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "dkv_host_free": (_I, [_P]),
    "dkv_gemm": (_I, [_I, _P, _P, _P, _I, _I, _I, _P, _SZ, _P]),
    "dkv_plan_bytes": (_SZ, [_I, _I]),
    "dkv_bm_create": (_I, [ctypes.POINTER(dkv_bm_config), ctypes.POINTER(_P)]),
    "dkv_bm_destroy": (_I, [_P]),
    "dkv_bm_add": (_I, [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]),
    "dkv_bm_remove": (_I, [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]),
    "dkv_bm_step": (_I, [_P]),
    "dkv_bm_rows": (_I, [_P]),
    "dkv_bm_window": (_I64, [_P]),
    "dkv_bm_plan": (_I, [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "dkv_bm_tables": (_I, [_P, _P, _P, _P]),
    "dkv_apply_plan": (_I, [_P, _P, _P, _P, _P, _I, _I, _P]),
    "dkv_decode_graph_create": (_I, [_P, _P, _I, ctypes.POINTER(dkv_layer_io), _I, _P, _P, _P, _I, _I,
                                     _I, _I, _F, _P, _SZ, ctypes.POINTER(_P)]),
    "dkv_graph_launch": (_I, [_P, _P]),
    "dkv_graph_destroy": (_I, [_P]),
    "dkv_numa_node_of_pci": (_I, [ctypes.c_char_p, ctypes.c_char_p]),
    "dkv_host_numa_node": (_I, [_I]),
    "dkv_pool_host_numa_node": (_I, [_P]),
    "dkv_last_error": (ctypes.c_char_p, []),
    "dkv_version": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libdkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libdkv.so is not built (%s); run kv_cache_offload_b200.build.build()" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_symbols(path: Optional[str] = None):
    """Names of the functions the headers under include/ declare (or one header's)."""
    import glob
    paths = [path] if path else sorted(glob.glob(os.path.join(INCLUDE, "*.h")))
    names = set()
    for p in paths:
        txt = re.sub(r"/\*.*?\*/", "", open(p).read(), flags=re.S)
        names |= set(re.findall(r"\b(dkv_[a-z_0-9]+)\s*\(", txt))
    return sorted(names)


def dkv_last_error() -> str:
    return lib().dkv_last_error().decode()


def dkv_version() -> str:
    return lib().dkv_version().decode()


def _chk(rc: int):
    if rc != DKV_OK:
        raise DkvError(rc, dkv_last_error())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t: torch.Tensor, dtype, name: str, cuda: bool = True):
    if t.dtype != dtype:
        raise TypeError("%s must be %s (got %s)" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if cuda and not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)


# ------------------------------------------------------------------------- pool


def dkv_pool_create(num_layers: int, num_kv_heads: int, head_dim: int, hbm_blocks: int,
                    host_blocks: int, block_tokens: int = 16, layout: int = 0,
                    host_flags: int = 0, hbm_base: Optional[torch.Tensor] = None) -> int:
    cfg = dkv_pool_config(num_layers, num_kv_heads, head_dim, block_tokens, hbm_blocks,
                          host_blocks, layout, host_flags, _ptr(hbm_base))
    out = _P()
    _chk(lib().dkv_pool_create(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def dkv_pool_destroy(pool: int):
    _chk(lib().dkv_pool_destroy(pool))


def dkv_pool_tier_ptr(pool: int, tier: int):
    """(device pointer, host pointer or None, bytes) of a tier."""
    d, h, n = _P(), _P(), _SZ()
    _chk(lib().dkv_pool_tier_ptr(pool, tier, ctypes.byref(d), ctypes.byref(h), ctypes.byref(n)))
    return d.value, h.value, n.value


def dkv_pool_set_tuning(pool: int, attn_splits: int = 0, proj_splits: int = 0,
                        attn_variant: int = 0, attn_lsu_hbm: int = 0, serial_launch: int = 0,
                        wait_limit_us: int = 0, test_withhold_block: int = 0):
    t = dkv_tuning(attn_splits, proj_splits, attn_variant, attn_lsu_hbm, serial_launch, wait_limit_us,
                   test_withhold_block)
    _chk(lib().dkv_pool_set_tuning(pool, ctypes.byref(t)))


def dkv_numa_node_of_pci(sysfs_root: Optional[str], pci_bus_id: str) -> int:
    """NUMA node sysfs reports for a PCI device (-1 if none)."""
    return lib().dkv_numa_node_of_pci(None if sysfs_root is None else sysfs_root.encode(), pci_bus_id.encode())


def dkv_host_numa_node(device: int) -> int:
    """NUMA node nearest CUDA device `device` (-1 if the platform reports none)."""
    return lib().dkv_host_numa_node(device)


def dkv_pool_host_numa_node(pool: int) -> int:
    """Node backing the first page of the pool's host tier (-1 if unknown or no host tier)."""
    r = lib().dkv_pool_host_numa_node(pool)
    if r < -1:
        raise DkvError(r, dkv_last_error())
    return r


def host_tier_tensor(pool: int) -> torch.Tensor:
    """The host tier as a flat CPU int16 tensor (raw bf16 bits) aliasing the pinned memory."""
    _, h, n = dkv_pool_tier_ptr(pool, DKV_TIER_HOST)
    if not n:
        return torch.empty(0, dtype=torch.int16)
    buf = (ctypes.c_int16 * (n // 2)).from_address(h)
    import numpy as np
    return torch.from_numpy(np.ctypeslib.as_array(buf))


def dkv_append_kv(pool: int, layer: int, k: torch.Tensor, v: torch.Tensor,
                  block_table: torch.Tensor, seq_lens: torch.Tensor, tier_map: torch.Tensor,
                  stream=None):
    """k, v: [B, n_tokens, Hkv, D] bf16 on the device."""
    _need(k, torch.bfloat16, "k"); _need(v, torch.bfloat16, "v")
    _need(block_table, torch.int32, "block_table"); _need(seq_lens, torch.int32, "seq_lens")
    _need(tier_map, torch.uint8, "tier_map")
    B, n = k.shape[0], k.shape[1]
    _chk(lib().dkv_append_kv(pool, layer, _ptr(k), _ptr(v), B, n, _ptr(block_table),
                             block_table.shape[1], _ptr(seq_lens), _ptr(tier_map), _stream(stream)))


# ---------------------------------------------------------------------- decode


def dkv_decode_workspace_bytes(pool: int, B: int, max_blocks: int, num_q_heads: int, hidden: int) -> int:
    n = lib().dkv_decode_workspace_bytes(pool, B, max_blocks, num_q_heads, hidden)
    if n == 0:
        raise DkvError(DKV_ERR_ARG, dkv_last_error())
    return n


def dkv_decode_attn_splits(pool: int, B: int, max_blocks: int, num_q_heads: int) -> int:
    r = lib().dkv_decode_attn_splits(pool, B, max_blocks, num_q_heads)
    if r < 0:
        raise DkvError(r, dkv_last_error())
    return r


def dkv_decode_attn_variant(pool: int, B: int, max_blocks: int, num_q_heads: int) -> int:
    r = lib().dkv_decode_attn_variant(pool, B, max_blocks, num_q_heads)
    if r < 0:
        raise DkvError(r, dkv_last_error())
    return r


def _decode_checks(x, Wqkv, block_table, seq_lens, tier_map):
    _need(x, torch.bfloat16, "x"); _need(Wqkv, torch.bfloat16, "Wqkv")
    _need(block_table, torch.int32, "block_table"); _need(seq_lens, torch.int32, "seq_lens")
    _need(tier_map, torch.uint8, "tier_map")
    if block_table.shape != tier_map.shape or block_table.shape[0] != x.shape[0]:
        raise ValueError("block_table/tier_map must be [B, max_blocks] with B = x.shape[0]")


def dkv_decode_step(pool: int, layer: int, x: torch.Tensor, Wqkv: torch.Tensor,
                    block_table: torch.Tensor, seq_lens: torch.Tensor, tier_map: torch.Tensor,
                    num_q_heads: int, rope_theta: float, out: torch.Tensor,
                    workspace: torch.Tensor, stream=None):
    _decode_checks(x, Wqkv, block_table, seq_lens, tier_map)
    _need(out, torch.bfloat16, "out")
    B, H = x.shape
    _chk(lib().dkv_decode_step(pool, layer, _ptr(x), _ptr(Wqkv), _ptr(block_table), _ptr(seq_lens),
                               _ptr(tier_map), B, block_table.shape[1], H, num_q_heads,
                               float(rope_theta), _ptr(out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)))


def dkv_decode_step_static(pool: int, layer: int, x: torch.Tensor, Wqkv: torch.Tensor,
                           block_table: torch.Tensor, seq_lens: torch.Tensor, tier_map: torch.Tensor,
                           num_q_heads: int, rope_theta: float, out: torch.Tensor, stream=None):
    """dkv_decode_step with the library's fixed per-device workspace: allocates nothing."""
    _decode_checks(x, Wqkv, block_table, seq_lens, tier_map)
    _need(out, torch.bfloat16, "out")
    B, H = x.shape
    _chk(lib().dkv_decode_step_static(pool, layer, _ptr(x), _ptr(Wqkv), _ptr(block_table), _ptr(seq_lens),
                                      _ptr(tier_map), B, block_table.shape[1], H, num_q_heads,
                                      float(rope_theta), _ptr(out), _stream(stream)))


def dkv_decode_static_workspace_capacity() -> int:
    return lib().dkv_decode_static_workspace_capacity()


def dkv_decode_project(pool, layer, x, Wqkv, block_table, seq_lens, tier_map, num_q_heads,
                       rope_theta, workspace, stream=None):
    _decode_checks(x, Wqkv, block_table, seq_lens, tier_map)
    B, H = x.shape
    _chk(lib().dkv_decode_project(pool, layer, _ptr(x), _ptr(Wqkv), _ptr(block_table), _ptr(seq_lens),
                                  _ptr(tier_map), B, block_table.shape[1], H, num_q_heads,
                                  float(rope_theta), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))


def dkv_decode_attend(pool, layer, block_table, seq_lens, tier_map, hidden, num_q_heads,
                      workspace, out=None, stream=None):
    """Split-K attention; with `out` the combine is fused (else call dkv_decode_combine)."""
    B = block_table.shape[0]
    if out is not None:
        _need(out, torch.bfloat16, "out")
    _chk(lib().dkv_decode_attend(pool, layer, _ptr(block_table), _ptr(seq_lens), _ptr(tier_map), B,
                                 block_table.shape[1], hidden, num_q_heads, _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))


def dkv_decode_combine(pool, B, max_blocks, hidden, num_q_heads, out, workspace, stream=None):
    _need(out, torch.bfloat16, "out")
    _chk(lib().dkv_decode_combine(pool, B, max_blocks, hidden, num_q_heads, _ptr(out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))


# ---------------------------------------------------------------------- layout


def dkv_permute_layout(src, dst, src_layout: int, num_layers: int, num_blocks: int,
                       chunk_bytes: int, stream=None):
    _chk(lib().dkv_permute_layout(_ptr(src), _ptr(dst), src_layout, num_layers, num_blocks,
                                  chunk_bytes, _stream(stream)))


def dkv_convert_layout(pool: int, tier: int, dst, dst_bytes: Optional[int] = None, stream=None):
    if dst_bytes is None:
        dst_bytes = dst.numel() * dst.element_size()
    _chk(lib().dkv_convert_layout(pool, tier, _ptr(dst), dst_bytes, _stream(stream)))


class MappedHostBuffer:
    """Mapped pinned host memory from dkv_host_alloc_mapped: `.tensor` is a CPU view of
    `numel` elements of `dtype`, `.dev_ptr` the device alias. Freed by close()."""

    def __init__(self, numel: int, dtype=torch.int16, host_flags: int = 0):
        import numpy as np
        esz = torch.empty(0, dtype=dtype).element_size()
        h, d = _P(), _P()
        _chk(lib().dkv_host_alloc_mapped(numel * esz, host_flags, ctypes.byref(h), ctypes.byref(d)))
        self.host_ptr, self.dev_ptr, self.numel = h.value, d.value, numel
        raw = (ctypes.c_uint8 * (numel * esz)).from_address(self.host_ptr)
        self.tensor = torch.from_numpy(np.ctypeslib.as_array(raw)).view(dtype)

    def close(self):
        if self.host_ptr:
            self.tensor = None
            _chk(lib().dkv_host_free(self.host_ptr))
            self.host_ptr = 0


def dkv_host_alloc_mapped(numel: int, dtype=torch.int16, host_flags: int = 0) -> "MappedHostBuffer":
    return MappedHostBuffer(numel, dtype, host_flags)


def dkv_host_free(buf: "MappedHostBuffer"):
    buf.close()


def dkv_gemm_workspace_bytes(variant: int, M: int, N: int, K: int) -> int:
    return lib().dkv_gemm_workspace_bytes(variant, M, N, K)


def dkv_gemm(variant: int, A: torch.Tensor, Bt, C: torch.Tensor, workspace: torch.Tensor, M: int = 0,
             N: int = 0, K: int = 0, stream=None):
    """C = A . B with Bt = B^T ([N][K]); Bt may be a device tensor or a raw device pointer
    (e.g. the device alias of mapped pinned host memory), then give M, N, K explicitly."""
    _need(A, torch.bfloat16, "A")
    _need(C, torch.float32, "C")
    M = M or A.shape[0]
    K = K or A.shape[1]
    N = N or C.shape[1]
    _chk(lib().dkv_gemm(variant, _ptr(A), _ptr(Bt), _ptr(C), M, N, K, _ptr(workspace),
                        workspace.numel() * workspace.element_size(), _stream(stream)))


def dkv_copy_blocks(pool: int, src_tier: int, dst_tier: int, src_ids: torch.Tensor,
                    dst_ids: torch.Tensor, method: int = DKV_COPY_KERNEL, stream=None):
    """Copy blocks between tiers; ids are int32 CPU tensors for DKV_COPY_DMA, CUDA tensors
    for DKV_COPY_KERNEL."""
    cuda = method == DKV_COPY_KERNEL
    _need(src_ids, torch.int32, "src_ids", cuda=cuda)
    _need(dst_ids, torch.int32, "dst_ids", cuda=cuda)
    if src_ids.is_cuda != cuda or dst_ids.is_cuda != cuda:
        raise ValueError("ids must be %s tensors for this method" % ("CUDA" if cuda else "CPU"))
    _chk(lib().dkv_copy_blocks(pool, src_tier, dst_tier, _ptr(src_ids), _ptr(dst_ids),
                               src_ids.numel(), method, _stream(stream)))


def dkv_check(pool: int, stream=None) -> int:
    """Synchronise and return the pool's status code (DKV_OK or a DKV_ERR_*)."""
    return lib().dkv_check(pool, _stream(stream))


# ------------------------------------------------------------ placement and graphs


def dkv_plan_bytes(max_rows: int, max_blocks: int) -> int:
    return lib().dkv_plan_bytes(max_rows, max_blocks)


def dkv_bm_create(max_rows: int, max_blocks: int, hbm_ids: int, host_ids: int, hbm_budget: int,
                  block_tokens: int = 16, plan_memory: int = DKV_PLAN_MAPPED, wait_ms: int = 0) -> int:
    cfg = dkv_bm_config(max_rows, max_blocks, block_tokens, plan_memory, hbm_ids, host_ids, hbm_budget, wait_ms, 0)
    out = _P()
    _chk(lib().dkv_bm_create(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def dkv_bm_destroy(bm: int):
    _chk(lib().dkv_bm_destroy(bm))


def dkv_bm_add(bm: int, seq_len: int) -> int:
    row = ctypes.c_int32()
    _chk(lib().dkv_bm_add(bm, seq_len, ctypes.byref(row)))
    return row.value


def dkv_bm_remove(bm: int, row: int) -> int:
    moved = ctypes.c_int32()
    _chk(lib().dkv_bm_remove(bm, row, ctypes.byref(moved)))
    return moved.value


def dkv_bm_step(bm: int):
    _chk(lib().dkv_bm_step(bm))


def dkv_bm_rows(bm: int) -> int:
    r = lib().dkv_bm_rows(bm)
    if r < 0:
        raise DkvError(r, dkv_last_error())
    return r


def dkv_bm_window(bm: int) -> int:
    return lib().dkv_bm_window(bm)


def dkv_bm_plan(bm: int, slot: int = -1):
    """(slot, host address, device alias or None) of a plan buffer."""
    h, d = _P(), _P()
    r = lib().dkv_bm_plan(bm, slot, ctypes.byref(h), ctypes.byref(d))
    if r < 0:
        raise DkvError(r, dkv_last_error())
    return r, h.value, d.value


def dkv_bm_tables(bm: int, max_rows: int, max_blocks: int):
    """Host snapshot (block_table int32, tier_map uint8, seq_lens int32) as numpy arrays."""
    import numpy as np
    bt = np.empty((max_rows, max_blocks), np.int32)
    tm = np.empty((max_rows, max_blocks), np.uint8)
    sl = np.empty((max_rows,), np.int32)
    _chk(lib().dkv_bm_tables(bm, bt.ctypes.data, tm.ctypes.data, sl.ctypes.data))
    return bt, tm, sl


def read_plan(host_addr: int):
    """Decode a plan buffer at a host address into {"moves", "entries", "seq_lens"} lists
    (tuples of ints), for inspection and tests."""
    import numpy as np
    hdr = np.ctypeslib.as_array((ctypes.c_int32 * 8).from_address(host_addr))
    n_moves, n_entries, n_rows, _, move_cap, entry_cap, _, _ = [int(v) for v in hdr]
    base = host_addr + PLAN_HEADER_BYTES
    mv = np.ctypeslib.as_array((ctypes.c_int32 * (4 * max(n_moves, 1))).from_address(base))
    en = np.ctypeslib.as_array((ctypes.c_int32 * (4 * max(n_entries, 1))).from_address(base + 16 * move_cap))
    sl = np.ctypeslib.as_array((ctypes.c_int32 * max(n_rows, 1)).from_address(base + 16 * (move_cap + entry_cap)))
    return {"moves": [tuple(int(v) for v in mv[4 * i:4 * i + 4]) for i in range(n_moves)],
            "entries": [tuple(int(v) for v in en[4 * i:4 * i + 4]) for i in range(n_entries)],
            "seq_lens": [int(v) for v in sl[:n_rows]]}


class BlockManager:
    """The library's block manager (dkv_bm_*): recency-window placement over the two tiers.
    Each operation writes a plan; `plan()` gives its device alias for dkv_apply_plan or a
    decode graph."""

    def __init__(self, max_rows: int, max_blocks: int, hbm_ids: int, host_ids: int, hbm_budget: int,
                 block_tokens: int = 16, plan_memory: int = DKV_PLAN_MAPPED, wait_ms: int = 0):
        self.max_rows, self.max_blocks = max_rows, max_blocks
        self.handle = dkv_bm_create(max_rows, max_blocks, hbm_ids, host_ids, hbm_budget, block_tokens,
                                    plan_memory, wait_ms)

    def add(self, seq_len: int) -> int:
        return dkv_bm_add(self.handle, seq_len)

    def remove(self, row: int) -> int:
        return dkv_bm_remove(self.handle, row)

    def step(self):
        dkv_bm_step(self.handle)

    @property
    def rows(self) -> int:
        return dkv_bm_rows(self.handle)

    @property
    def window(self) -> int:
        return dkv_bm_window(self.handle)

    def plan(self, slot: int = -1):
        return dkv_bm_plan(self.handle, slot)

    def last_plan(self):
        return read_plan(self.plan()[1])

    def tables(self):
        return dkv_bm_tables(self.handle, self.max_rows, self.max_blocks)

    def close(self):
        if self.handle:
            dkv_bm_destroy(self.handle)
            self.handle = 0


def dkv_apply_plan(pool: int, plan_dev: int, block_table: torch.Tensor, tier_map: torch.Tensor,
                   seq_lens: torch.Tensor, stream=None):
    _need(block_table, torch.int32, "block_table"); _need(tier_map, torch.uint8, "tier_map")
    _need(seq_lens, torch.int32, "seq_lens")
    R, MB = block_table.shape
    _chk(lib().dkv_apply_plan(pool, plan_dev, _ptr(block_table), _ptr(tier_map), _ptr(seq_lens), R, MB,
                              _stream(stream)))


def dkv_decode_graph_create(pool: int, plan_dev: Optional[int], layers, block_table: torch.Tensor,
                            seq_lens: torch.Tensor, tier_map: torch.Tensor, B: int, hidden: int,
                            num_q_heads: int, rope_theta: float, workspace: torch.Tensor) -> int:
    """layers: sequence of (layer, x, Wqkv, out) with x [B, hidden], out [B, Hq*D] (bf16).
    block_table / tier_map are the full [max_rows, max_blocks] device tables; the step
    decodes rows 0..B-1."""
    _need(block_table, torch.int32, "block_table"); _need(tier_map, torch.uint8, "tier_map")
    _need(seq_lens, torch.int32, "seq_lens")
    arr = (dkv_layer_io * len(layers))()
    for i, (layer, x, W, out) in enumerate(layers):
        _need(x, torch.bfloat16, "x"); _need(W, torch.bfloat16, "Wqkv"); _need(out, torch.bfloat16, "out")
        arr[i] = dkv_layer_io(layer, 0, _ptr(x), _ptr(W), _ptr(out))
    R, MB = block_table.shape
    g = _P()
    _chk(lib().dkv_decode_graph_create(pool, plan_dev, R, arr, len(layers), _ptr(block_table), _ptr(seq_lens),
                                       _ptr(tier_map), B, MB, hidden, num_q_heads, float(rope_theta),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       ctypes.byref(g)))
    return g.value


def dkv_graph_launch(graph: int, stream=None):
    _chk(lib().dkv_graph_launch(graph, _stream(stream)))


def dkv_graph_destroy(graph: int):
    _chk(lib().dkv_graph_destroy(graph))
