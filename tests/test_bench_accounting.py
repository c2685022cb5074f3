"""The benchmark's byte accounting and its reported fields, on the CPU.

The step roofline counts every byte a decode step must move once: the cached KV, the
QKV weight, x, the new K/V rows and the output. For the 8B-shaped all-HBM workload
(B=16, 32768 cached tokens, Hq/Hkv = 32/8, D=128, hidden 4096) that is
2^31 + 50,331,648 + 131,072 + 65,536 + 131,072 = 2,198,142,976 bytes.
"""
from types import SimpleNamespace

import pytest

import bench
import workloads as WL


def _wl(host_bytes=0):
    cfg = WL.CONFIGS["8b_hbm"]
    kv = cfg.B * cfg.ctx * cfg.Hkv * 2 * cfg.D * 2
    return SimpleNamespace(cfg=cfg, kv_hbm_bytes=kv - host_bytes, kv_host_bytes=host_bytes,
                           w_bytes=(cfg.Hq + 2 * cfg.Hkv) * cfg.D * cfg.H * 2,
                           new_kv_bytes=cfg.B * cfg.Hkv * cfg.D * 2 * 2)


def test_step_roofline_bytes_for_the_8b_layer():
    wl = _wl()
    assert wl.kv_hbm_bytes == 2 ** 31 and wl.w_bytes == 50331648
    r = bench.step_roofline(wl, 0.4, 6543.4, "measured")
    assert r["bound"] == "hbm" and r["bytes"] == 2198142976
    assert r["achieved"] == pytest.approx(2198142976 / 0.4e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6543.4)


def test_step_roofline_is_host_bound_when_blocks_live_on_the_host():
    wl = _wl(host_bytes=2 ** 30)
    r = bench.step_roofline(wl, 20.0, 6543.4, "measured")
    assert r["bound"] == "host_link" and r["host_bytes"] == 2 ** 30
    assert r["achieved_host_gbs"] == pytest.approx(2 ** 30 / 20e-3 / 1e9)


def test_replica_throughput_counts_all_ranks_over_the_slowest():
    assert bench.replica_throughput(16, 1, 0.4) == pytest.approx(40000.0)
    assert bench.replica_throughput(16, 8, 0.5) == pytest.approx(16 * 8 / 0.5e-3)


def test_workload_config_names_the_workload_without_model_keys():
    c = bench.workload_config(WL.CONFIGS["8b_hbm"], 2)
    assert c["global_batch"] == 32 and c["seq_len"] == 32768 and c["parallelism"] == "replicas x2"
    assert c["workload"].startswith("8b_hbm: B=16 hidden=4096 Hq=32 Hkv=8 D=128")
    assert "model" not in c


def test_percentiles_nearest_rank():
    assert bench.percentiles([5.0, 1.0, 3.0, 2.0, 4.0, 6.0, 7.0, 8.0, 9.0, 10.0]) == [1.0, 5.0, 9.0]
    assert bench.percentiles([2.0]) == [2.0, 2.0, 2.0]


def test_oracle_pool_runs_one_sequence_per_process():
    # the CPU baseline's process pool on the tiny workload: 2 single-threaded processes;
    # steps mode returns one wall time per step, budget mode a summed rate
    cfg = WL.CONFIGS["tiny"]
    times = bench.run_oracle_pool(cfg, 0, 2, steps=3)
    assert len(times) == 3 and all(t > 0 for t in times)
    rate, done, el = bench.run_oracle_pool(cfg, 0, 2, budget_s=0.2)
    assert done >= 2 and rate > 0 and el >= 0.2


def test_dram_reader_counts_its_bytes_and_stops():
    """The host-DRAM load of `--config host_contention`: a spawned reader adds one buffer's
    bytes per pass to the shared counter and exits once told to stop."""
    import multiprocessing as mp
    import time
    ctx = mp.get_context("spawn")
    stop, counter, ready = ctx.Event(), ctx.Value("d", 0.0), ctx.Queue()
    nbytes = 8 << 20
    p = ctx.Process(target=bench._dram_reader, args=(nbytes, stop, counter, ready), daemon=True)
    p.start()
    try:
        ready.get(timeout=120)
        t_end = time.time() + 60
        while counter.value < 3 * nbytes and time.time() < t_end:
            time.sleep(0.05)
        assert counter.value >= 3 * nbytes
        assert counter.value % nbytes == 0
    finally:
        stop.set()
        p.join(timeout=30)
    assert p.exitcode == 0


def test_gemm_cpu_baseline_extrapolates_its_sample():
    """The GEMM line's CPU baseline: the oracle's fp64 entries timed for a seeded sample on
    one thread, extrapolated by the ratio of all entries to the sample."""
    import torch
    A = (torch.rand((64, 32)) * 2 - 1).to(torch.bfloat16)
    B = (torch.rand((48, 32)) * 2 - 1).to(torch.bfloat16)
    r = bench.gemm_cpu_baseline(A, B, 64, 48, 32, n_samples=128)
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["unit"] == "ms"
    assert r["value"] == pytest.approx(r["sample_s"] * (64 * 48 / 128) * 1e3)
