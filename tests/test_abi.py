"""The C ABI library loads on a CPU-only host and exports every symbol include/dkv.h declares.
No compute call is made here."""
import ctypes

import pytest

import kv_cache_offload_b200 as dkv


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_offload_b200.build import build
    build()


def test_every_declared_symbol_is_exported():
    L = dkv.lib()
    names = dkv.header_symbols()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_debug_library_exports_the_same_symbols():
    # libdkv_debug.so: the same sources with DKV_DEBUG range checks (loaded with
    # DKV_LIBRARY=debug); it must offer every call the header declares
    from kv_cache_offload_b200.build import LIB_DEBUG
    L = ctypes.CDLL(LIB_DEBUG)
    missing = [n for n in dkv.header_symbols() if not hasattr(L, n)]
    assert not missing, missing


def test_binding_declares_every_symbol():
    from kv_cache_offload_b200 import binding
    assert set(dkv.header_symbols()) <= set(binding._SIGS)


def test_error_paths_without_device():
    # argument validation happens before any device call
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_pool_create(0, 2, 64, 1, 1)
    assert e.value.code == dkv.DKV_ERR_ARG
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_pool_create(1, 2, 96, 1, 1)
    assert e.value.code == dkv.DKV_ERR_UNSUPPORTED
    assert dkv.lib().dkv_pool_destroy(None) == dkv.DKV_ERR_ARG
    assert "null" in dkv.dkv_last_error()
    assert dkv.lib().dkv_check(None, None) == dkv.DKV_ERR_ARG
    assert dkv.lib().dkv_permute_layout(None, None, 0, 1, 1, 16, None) == dkv.DKV_ERR_ARG
    assert dkv.lib().dkv_decode_workspace_bytes(None, 1, 1, 1, 64) == 0


def test_struct_layout_matches_header():
    assert ctypes.sizeof(dkv.binding.dkv_pool_config) == 48
    assert ctypes.sizeof(dkv.binding.dkv_tuning) == 32


def test_placement_structs_match_header():
    assert ctypes.sizeof(dkv.binding.dkv_bm_config) == 48
    assert ctypes.sizeof(dkv.binding.dkv_layer_io) == 32
    assert dkv.dkv_plan_bytes(3, 5) == 32 + 15 * 32 + 3 * 4
    assert dkv.dkv_plan_bytes(0, 5) == 0
