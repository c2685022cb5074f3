"""NUMA placement of the host tier, on the CPU: the node a GPU's PCI device reports is read
from a fake sysfs tree (bus ids as cudaDeviceGetPCIBusId prints them: upper-case hex, a
4- or 8-digit domain), and the library's own sysfs lookup runs against this host's."""
import os

import pytest

import kv_cache_offload_b200 as dkv


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_offload_b200.build import build
    build()


def _fake_sysfs(root, entries):
    for bus, node in entries.items():
        d = os.path.join(root, "bus", "pci", "devices", bus)
        os.makedirs(d, exist_ok=True)
        if node is not None:
            with open(os.path.join(d, "numa_node"), "w") as f:
                f.write("%s\n" % node)
    return str(root)


def test_node_of_pci_device_from_sysfs(tmp_path):
    root = _fake_sysfs(tmp_path, {"0000:1b:00.0": 0, "0000:9a:00.0": 1, "0000:c3:00.0": 3,
                                  "0000:05:00.0": -1, "0000:06:00.0": None})
    # cudaDeviceGetPCIBusId's spelling: upper case, sometimes an 8-digit domain
    assert dkv.dkv_numa_node_of_pci(root, "0000:1B:00.0") == 0
    assert dkv.dkv_numa_node_of_pci(root, "0000:9A:00.0") == 1
    assert dkv.dkv_numa_node_of_pci(root, "00000000:C3:00.0") == 3
    # no NUMA information: -1 (the pool then allocates with no preference)
    assert dkv.dkv_numa_node_of_pci(root, "0000:05:00.0") == -1
    assert dkv.dkv_numa_node_of_pci(root, "0000:06:00.0") == -1
    assert dkv.dkv_numa_node_of_pci(root, "0000:77:00.0") == -1
    assert dkv.dkv_numa_node_of_pci(root, "") == -1


def test_node_lookup_on_this_host_is_consistent():
    # a device this host has (if sysfs lists any): the library reads the same file
    base = "/sys/bus/pci/devices"
    if not os.path.isdir(base):
        pytest.skip("no sysfs PCI tree")
    for bus in sorted(os.listdir(base))[:8]:
        p = os.path.join(base, bus, "numa_node")
        if not os.path.exists(p):
            continue
        want = int(open(p).read().strip())
        assert dkv.dkv_numa_node_of_pci(None, bus.upper()) == (want if want >= 0 else -1)


def test_pool_rejects_unknown_host_flags():
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_pool_create(1, 2, 64, 1, 1, host_flags=4)
    assert e.value.code == dkv.DKV_ERR_ARG
