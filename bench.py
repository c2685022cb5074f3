"""Benchmark: fused QKV + decode attention step on a two-tier (HBM / mapped host) paged KV cache.

Default workload (N=1): the Llama-3-70B-shaped layer, the largest single-GPU configuration —
batch 32, hidden 8192, 64 q / 8 kv heads, head_dim 128, RoPE theta 5e5, cached contexts drawn
uniformly from 8192..65536 tokens in 16-token blocks, each block in mapped pinned host memory
with probability 0.8 (read in place over PCIe) and in HBM otherwise. Its roofline is the host
link. In the same run the Llama-3-8B-shaped layer with the whole cache in HBM (batch 16,
32768 cached tokens each) is timed and reported as `hbm_line`, against the HBM roofline,
and (one GPU) the remaining configurations — the 8B layer with old blocks in the host tier,
the tiny layer and the 10240^3 zero-copy GEMM study — as `other_configs`. A
step is one decode step of one layer through the C ABI (dkv_decode_step: projection,
split-K attention, combine). Inputs are synthetic (seeded N(0,1) activations and KV,
W ~ N(0, 1/hidden)), generated on the device; steps cycle through several copies of W
(more than twice the L2 in all), as a model's layers would, so W is read from HBM.

Multi-GPU: every rank runs an independent replica of the workload (the step has no
cross-GPU exchange); value = tokens of all ranks / max-over-ranks time. Each rank's host
tier is placed on its GPU's nearest NUMA node.

Prints one JSON line on rank 0. `--impl reference` times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "fused QKV+decode-attn tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="dkv", choices=["dkv", "reference"])
    ap.add_argument("--config", default="70b_mixed",
                    choices=sorted(WL.CONFIGS) + ["gemm", "layout", "adaptive", "host_contention", "attn_sweep"],
                    help="decode workload (default: the largest single-GPU configuration; the all-HBM "
                         "8B-shaped layer is then reported beside it as hbm_line)")
    ap.add_argument("--no-hbm-line", action="store_true", help="skip the all-HBM line of the default run")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the 8b_mixed, tiny and GEMM lines of the default run (one GPU)")
    ap.add_argument("--compare-staged", action="store_true",
                    help="host-tier configs: also time swap-in (DMA and copy kernel) + HBM attention")
    ap.add_argument("--attn-splits", type=int, default=0)
    ap.add_argument("--proj-splits", type=int, default=0)
    ap.add_argument("--attn-variant", type=int, default=0,
                    help="attention kernel (dkv_tuning.attn_variant; 6/7 = the opt-in tensor-core consumer)")
    ap.add_argument("--host-flags", type=int, default=2,
                    help="dkv_pool_config.host_flags (default DKV_HOST_NUMA_NEAREST: the host tier on the "
                         "GPU's nearest NUMA node)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling)")
    ap.add_argument("--ctx", type=int, default=0, help="override the cached tokens per sequence (profiling)")
    ap.add_argument("--gemm-dim", type=int, default=0, help="override M=N=K of the GEMM study (profiling)")
    ap.add_argument("--profile", action="store_true",
                    help="warm-up + timed steps only (no clock pre-roll, e2e or CPU baseline): for ncu")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def src_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "kv_cache_offload_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(config_name: str, batch: int):
    """Per-launch traffic of the attention kernel at a full configuration, from the committed
    ncu summary (DRAM bytes for the all-HBM layer, PCIe read bytes for host-tier ones), if it
    was captured on the current kernel source and describes this batch (else None)."""
    p = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(config_name)
    if not e or e.get("src_hash") != src_hash("dkv_attention.cu", "dkv_common.cuh", "dkv_umma.cuh"):
        return None
    if e.get("batch") != batch:
        return None
    return {"bytes": e.get("bytes_per_launch"), "counter": e.get("counter")}


_NVML = {}


def sm_clock_now(index: int):
    """The GPU's SM clock (MHz) read through NVML at this moment, or None without NVML."""
    try:
        import pynvml
        if "h" not in _NVML:
            pynvml.nvmlInit()
            _NVML["h"] = {}
        h = _NVML["h"].setdefault(index, pynvml.nvmlDeviceGetHandleByIndex(index))
        return pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def reduce_max_over_ranks(vals, dist: bool, device=None):
    """Element-wise max over ranks of per-rank timings (ms); identity without a process
    group. Every rank calls it the same number of times (it is a collective)."""
    t = torch.tensor(list(vals), dtype=torch.float64, device=device)
    if dist:
        import torch.distributed as tdist
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return [float(v) for v in t]


def replica_throughput(tokens_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job tokens/s of `world` independent replicas: all ranks' tokens over the
    slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step_max * 1e-3)


# ------------------------------------------------------------------ GPU workload


def gpu_randn_bf16(shape, gen, std=1.0, device="cuda"):
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    step = 1 << 26
    for s in range(0, n, step):
        e = min(n, s + step)
        v = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            v.mul_(std)
        flat[s:e].copy_(v)
    return out


class Workload:
    """A decode workload resident on one GPU: pool (both tiers filled), tables, x, W."""

    def __init__(self, cfg: WL.DecodeConfig, seed: int, host_flags: int = 0):
        import kv_cache_offload_b200 as dkv
        self.dkv = dkv
        self.cfg = cfg
        dev = torch.device("cuda", torch.cuda.current_device())
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        self.lay = WL.block_layout(cfg, seed)
        lay = self.lay
        tier_elems = cfg.layers * 2 * cfg.Hkv * cfg.T * cfg.D
        self.hbm = gpu_randn_bf16((lay.hbm_blocks * tier_elems,), gen) if lay.hbm_blocks else None
        self.pool = dkv.dkv_pool_create(cfg.layers, cfg.Hkv, cfg.D, lay.hbm_blocks, lay.host_blocks,
                                        host_flags=host_flags, hbm_base=self.hbm)
        if lay.host_blocks:
            host = dkv.host_tier_tensor(self.pool)
            n = host.numel()
            step = 1 << 28
            for s in range(0, n, step):
                e = min(n, s + step)
                host[s:e].copy_(gpu_randn_bf16((e - s,), gen).view(torch.int16).cpu())
        self.x = gpu_randn_bf16((cfg.B, cfg.H), gen)
        # one W per layer, as in a model: steps cycle through enough copies (more than twice
        # the L2 in all) that no step finds its W left in L2 by an earlier one — a model uses
        # a layer's W again only a whole forward pass later
        self.w_bytes = cfg.rows * cfg.H * 2
        l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20)
        self.n_w = min(8, max(1, math.ceil(2 * l2 / self.w_bytes)))
        self.Ws = [gpu_randn_bf16((cfg.rows, cfg.H), gen, std=1.0 / math.sqrt(cfg.H)) for _ in range(self.n_w)]
        self.k_w = 0
        self.table = lay.block_table.to(dev)
        self.tmap = lay.tier_map.to(dev)
        self.lens = torch.tensor(lay.seq_lens, dtype=torch.int32, device=dev)
        self.out = torch.empty((cfg.B, cfg.Hq * cfg.D), dtype=torch.bfloat16, device=dev)
        self.nws = dkv.dkv_decode_workspace_bytes(self.pool, cfg.B, lay.max_blocks, cfg.Hq, cfg.H)
        self.ws = torch.empty(self.nws, dtype=torch.uint8, device=dev)
        # byte accounting (algorithmic: what the step must move)
        per_tok = 2 * cfg.Hkv * cfg.D * 2          # K and V of one token, all kv heads
        host_tok = hbm_tok = 0
        for b, c in enumerate(lay.seq_lens):
            for j in range((c + cfg.T - 1) // cfg.T):
                n = min(cfg.T, c - j * cfg.T)
                if int(lay.tier_map[b, j]):
                    host_tok += n
                else:
                    hbm_tok += n
        self.kv_host_bytes = host_tok * per_tok
        self.kv_hbm_bytes = hbm_tok * per_tok
        self.kv_bytes = self.kv_host_bytes + self.kv_hbm_bytes
        self.new_kv_bytes = cfg.B * cfg.Hkv * cfg.D * 2 * 2
        self.splits = dkv.dkv_decode_attn_splits(self.pool, cfg.B, lay.max_blocks, cfg.Hq)

    def set_tuning(self, attn_splits=0, proj_splits=0, **kw):
        c = self.cfg
        self.dkv.dkv_pool_set_tuning(self.pool, attn_splits=attn_splits, proj_splits=proj_splits, **kw)
        self.splits = self.dkv.dkv_decode_attn_splits(self.pool, c.B, self.lay.max_blocks, c.Hq)
        n = self.dkv.dkv_decode_workspace_bytes(self.pool, c.B, self.lay.max_blocks, c.Hq, c.H)
        if n > self.nws:
            self.nws = n
            self.ws = torch.empty(n, dtype=torch.uint8, device=self.ws.device)

    @property
    def W(self):
        """The next step's W (advanced by next_W)."""
        return self.Ws[self.k_w % self.n_w]

    def next_W(self):
        W = self.W
        self.k_w += 1
        return W

    def step(self):
        c = self.cfg
        self.dkv.dkv_decode_step(self.pool, 0, self.x, self.next_W(), self.table, self.lens, self.tmap, c.Hq,
                                 c.theta, self.out, self.ws)

    def attend(self):
        c = self.cfg
        self.dkv.dkv_decode_attend(self.pool, 0, self.table, self.lens, self.tmap, c.H, c.Hq, self.ws, out=self.out)

    def project(self):
        c = self.cfg
        self.dkv.dkv_decode_project(self.pool, 0, self.x, self.next_W(), self.table, self.lens, self.tmap, c.Hq,
                                    c.theta, self.ws)

    def step_timed_stages(self, ev):
        """The same step as step(), with events between its two launches."""
        c, d = self.cfg, self.dkv
        ev[0].record()
        d.dkv_decode_project(self.pool, 0, self.x, self.next_W(), self.table, self.lens, self.tmap, c.Hq,
                             c.theta, self.ws)
        ev[1].record()
        d.dkv_decode_attend(self.pool, 0, self.table, self.lens, self.tmap, c.H, c.Hq, self.ws,
                            out=self.out)
        ev[2].record()

    def close(self):
        if self.pool:
            self.dkv.dkv_pool_destroy(self.pool)
            self.pool = 0


def measure_h2d_peak(dev, nbytes=1 << 30, reps=5):
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        b.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del src, dst
    return best


# -------------------------------------------------------------------- CPU oracle
# The oracle is timed as it stands (one sequence per call, fp64 numpy) on the host's
# cores: one spawned process per core, each with single-threaded BLAS and torch, each on
# its own sequence of the workload, so the core count reported is the parallelism used.


def oracle_sample(cfg: WL.DecodeConfig, seed: int, seqs):
    """A bounded sample of the workload for the oracle: the sequences `seqs` of it (their
    context lengths), with tiers and tables drawn by the workload's own policy, generated
    on the host."""
    lens_all = WL.seq_lengths(cfg, seed)
    lens = [lens_all[b % cfg.B] for b in seqs]
    sub = WL.DecodeConfig(cfg.name, B=len(lens), H=cfg.H, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D,
                          theta=cfg.theta, ctx=cfg.ctx, ctx_range=cfg.ctx_range,
                          tier_policy=cfg.tier_policy, recent_hbm_tokens=cfg.recent_hbm_tokens,
                          host_prob=cfg.host_prob, permute=cfg.permute, layers=cfg.layers, T=cfg.T)
    return WL.make_decode_inputs(sub, seed=seed, seq_lens=lens)


def _oracle_args(inp):
    cfg, lay = inp.cfg, inp.layout
    return (WL.bf16_bits(inp.x), WL.bf16_bits(inp.W), [WL.bf16_bits(inp.hbm), WL.bf16_bits(inp.host)],
            lay.block_table.numpy(), lay.seq_lens, lay.tier_map.numpy(), cfg.Hq, cfg.Hkv, cfg.D, cfg.T,
            cfg.theta)


def _oracle_proc(name, seed, b, budget_s, steps, bar, q):
    """One oracle process: single-threaded, one sequence of the workload. With `steps`, each
    step runs between two barrier waits shared with the parent (which times the step);
    otherwise it runs until `budget_s` of its own time is spent and reports the count."""
    try:
        torch.set_num_threads(1)
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
        from oracle import dkv_oracle as O
        cfg = WL.CONFIGS[name]
        a = _oracle_args(oracle_sample(cfg, seed, [b]))
        if steps:
            for _ in range(steps):
                bar.wait(timeout=900)
                O.decode_step(*a)
                bar.wait(timeout=900)
            q.put((b, steps, 0.0, None))
            return
        bar.wait(timeout=900)
        done, t0 = 0, time.perf_counter()
        while True:
            O.decode_step(*a)
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        q.put((b, done, time.perf_counter() - t0, None))
    except Exception as e:  # reported to the parent, which raises
        try:
            bar.abort()
        except Exception:
            pass
        q.put((b, 0, 0.0, repr(e)))


def oracle_workers(cfg: WL.DecodeConfig) -> int:
    """Processes for the oracle: one per core this process may run on, at most 16, and no
    more than half the available host memory allows (W in fp64 and one sequence's KV each)."""
    n = len(os.sched_getaffinity(0))
    per = cfg.rows * cfg.H * 10 + 3 * (cfg.ctx or cfg.ctx_range[1]) * cfg.Hkv * cfg.D * 4 + (1 << 29)
    try:
        import psutil
        n = min(n, max(1, int(psutil.virtual_memory().available * 0.5 // per)))
    except Exception:
        pass
    return max(1, min(n, 16))


def run_oracle_pool(cfg: WL.DecodeConfig, seed: int, workers: int, budget_s: float = 0.0, steps: int = 0):
    """Run the oracle in `workers` spawned processes (sequences 0..workers-1 of the workload).
    Budget mode: returns (tokens/s summed over the processes, sequences done, seconds).
    Steps mode: returns the wall time of each step, a step being one sequence per process."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")  # never fork a process that has a CUDA context
    bar = ctx.Barrier(workers + 1)
    q = ctx.Queue()
    keep = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    os.environ.update({k: "1" for k in keep})
    try:
        procs = [ctx.Process(target=_oracle_proc, args=(cfg.name, seed, i, budget_s, steps, bar, q), daemon=True)
                 for i in range(workers)]
        for p in procs:
            p.start()
    finally:
        for k, v in keep.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    times = []
    try:
        if steps:
            for _ in range(steps):
                bar.wait(timeout=900)
                t0 = time.perf_counter()
                bar.wait(timeout=900)
                times.append(time.perf_counter() - t0)
        else:
            bar.wait(timeout=900)
        res = [q.get(timeout=900) for _ in procs]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    errs = [r[3] for r in res if r[3]]
    if errs:
        raise RuntimeError("oracle process failed: " + errs[0])
    if steps:
        return times
    rate = sum(d / el for _, d, el, _ in res if el > 0)
    return rate, sum(d for _, d, _, _ in res), max(el for _, _, el, _ in res)


def oracle_single_thread_tiny(seconds: float = 1.0) -> dict:
    """The oracle on the tiny configuration (1 sequence, 512 cached tokens) with one BLAS
    thread, in this process."""
    from threadpoolctl import threadpool_limits
    from oracle import dkv_oracle as O
    a = _oracle_args(WL.make_decode_inputs(WL.CONFIGS["tiny"], seed=0))
    with threadpool_limits(1):
        O.decode_step(*a)
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            O.decode_step(*a)
            done += 1
        el = time.perf_counter() - t0
    return {"ms_per_step": 1e3 * el / done, "tokens_per_s": done / el, "threads": 1,
            "workload": "tiny: B=1 hidden=256 Hq=4 Hkv=2 D=64, 512 cached tokens, all host tier"}


def cpu_baseline(cfg, seed, budget_s):
    workers = oracle_workers(cfg)
    rate, done, el = run_oracle_pool(cfg, seed, workers, budget_s=budget_s)
    return {"value": rate, "unit": "tokens/s", "cores": workers, "kind": "oracle",
            "sample": "%d processes x 1 thread, each decoding one sequence of the workload (full context, "
                      "sequences 0..%d) repeatedly for %.1f s of fp64 numpy oracle work; %d sequence steps "
                      "in all" % (workers, workers - 1, el, done),
            "tiny_single_thread": oracle_single_thread_tiny()}


# --------------------------------------------------------------------------- main


def step_roofline(wl, ms: float, hbm_peak: float, peak_kind: str) -> dict:
    """The decode step as a whole: algorithmic bytes per step over the step time, against
    the HBM peak (all-HBM workloads) or the host link (host-tier bytes dominate)."""
    c = wl.cfg
    small = c.B * c.H * 2 + wl.new_kv_bytes + c.B * c.Hq * c.D * 2  # x, new K/V rows, out
    hbm_bytes = wl.kv_hbm_bytes + wl.w_bytes + small
    if wl.kv_host_bytes:
        return {"bound": "host_link", "host_bytes": wl.kv_host_bytes, "hbm_bytes": hbm_bytes,
                "achieved_host_gbs": wl.kv_host_bytes / (ms * 1e-3) / 1e9}
    achieved = hbm_bytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "bytes": hbm_bytes, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "peak_source": peak_kind}


def workload_config(cfg: WL.DecodeConfig, world: int) -> dict:
    """The `config` object both arms report for a decode workload."""
    seq_len = cfg.ctx or cfg.ctx_range[1]
    return {"workload": "%s: B=%d hidden=%d Hq=%d Hkv=%d D=%d theta=%g, cached tokens %s, "
                        "%d-token blocks, tiers %s" % (cfg.name, cfg.B, cfg.H, cfg.Hq, cfg.Hkv, cfg.D,
                                                       cfg.theta, cfg.ctx or cfg.ctx_range, cfg.T,
                                                       cfg.tier_policy),
            "global_batch": cfg.B * world, "seq_len": seq_len, "parallelism": "replicas x%d" % world}


def run_reference(args, rank, world):
    """The oracle as the reference arm, on the host's cores: each step decodes one sequence
    of the workload in each of `workers` single-threaded processes at once; rank 0 only."""
    cfg = WL.CONFIGS[args.config]
    if rank != 0:
        return
    workers = oracle_workers(cfg)
    times = run_oracle_pool(cfg, 0, workers, steps=args.warmup + args.steps)[args.warmup:]
    ms = 1e3 * sum(times) / len(times)
    value = workers / (ms * 1e-3)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": dict(workload_config(cfg, 1),
                           step_sample="%d sequences of the workload per step, one per process" % workers),
            "step_ms_p10_p50_p90": percentiles([1e3 * t for t in times]),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": workers, "kind": "oracle",
                             "sample": "%d of %d sequences per step (full context), %d single-threaded "
                                       "processes" % (workers, cfg.B, workers)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def percentiles(v):
    """(p10, p50, p90) of a list, nearest-rank."""
    v = sorted(v)
    if not v:
        return None
    pick = lambda f: v[min(len(v) - 1, max(0, int(math.ceil(f * len(v))) - 1))]
    return [pick(0.1), pick(0.5), pick(0.9)]


def run_gemm(args, rank, world):
    """The zero-copy GEMM study as its own JSON line (`--config gemm`)."""
    from kv_cache_offload_b200.build import build
    build()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    print(json.dumps(gemm_line(args, rank, torch.device("cuda", local))), flush=True)


def gemm_line(args, rank, dev, steps=None, warmup=None):
    """The zero-copy GEMM study: C = A . B (10240^3), A in HBM, B in mapped host memory;
    CPU-aware tiling, naive zero-copy, staged swap and both operands in HBM."""
    import kv_cache_offload_b200 as dkv
    steps = steps or args.steps
    warmup = warmup or args.warmup
    cfg = WL.GEMM_CONFIGS["gemm"]
    M, N, K = cfg.M, cfg.N, cfg.K
    if args.gemm_dim:
        M = N = K = args.gemm_dim
    gen = torch.Generator(device=dev)
    gen.manual_seed(rank)
    A = (torch.rand((M, K), generator=gen, device=dev) * 2 - 1).to(torch.bfloat16)
    Btd = (torch.rand((N, K), generator=gen, device=dev) * 2 - 1).to(torch.bfloat16)
    hb = dkv.dkv_host_alloc_mapped(N * K, torch.bfloat16)
    hb.tensor.copy_(Btd.reshape(-1).cpu())
    C = torch.empty((M, N), dtype=torch.float32, device=dev)
    res = {}
    flops = 2.0 * M * N * K
    b_bytes = N * K * 2
    for name, n in (("DEVICE", steps), ("CPU_AWARE", steps), ("STAGED_SWAP", steps),
                    ("NAIVE_ZERO_COPY", max(1, min(steps, 3)))):
        v = getattr(dkv, "DKV_GEMM_" + name)
        ws = torch.empty(dkv.dkv_gemm_workspace_bytes(v, M, N, K), dtype=torch.uint8, device=dev)
        b = Btd if name == "DEVICE" else hb.dev_ptr
        for _ in range(1 if name == "NAIVE_ZERO_COPY" else warmup):
            dkv.dkv_gemm(v, A, b, C, ws, M, N, K)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            dkv.dkv_gemm(v, A, b, C, ws, M, N, K)
        e1.record()
        e1.synchronize()
        ms = e0.elapsed_time(e1) / n
        res[name] = {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12}
        del ws
    h2d = measure_h2d_peak(dev)
    hb.close()
    ca = res["CPU_AWARE"]["ms"]
    cpu = gemm_cpu_baseline(A, Btd, M, N, K) if rank == 0 else None
    del A, Btd, C
    line = {"metric": "zero-copy GEMM 10240^3 time (CPU-aware tiling)", "value": ca, "unit": "ms",
            "higher_is_better": False, "n_gpus": 1, "steps": steps, "warmup": warmup,
            "dtype": "bf16", "data": "synthetic", "impl": "dkv",
            "config": {"workload": "gemm: C = A.B, M=N=K=%d, A bf16 in HBM, B bf16 column-major in mapped "
                                   "pinned host memory, fp32 accumulate/output" % M},
            "variants": res,
            "host_link": {"h2d_peak_gbs": h2d, "algorithmic_host_bytes": b_bytes,
                          "cpu_aware_link_gbs": b_bytes / (ca * 1e-3) / 1e9,
                          "cpu_aware_frac_of_h2d": b_bytes / (ca * 1e-3) / 1e9 / h2d,
                          "naive_model_host_bytes_BM128": (M // 128) * b_bytes,
                          "link": "PCIe (not NVLink-C2C)"},
            "pages_context": {"swap_ms": 65, "naive_ms": 1122, "hardware": "PCIe platform, GPU unstated"}}
    if cpu:
        line["cpu_baseline"] = cpu
    return line


def gemm_cpu_baseline(A, Btd, M, N, K, n_samples=4096, seed=0):
    """The oracle's fp64 GEMM entries (one dot product of length K per entry), timed on one
    host thread for a seeded sample of entries and extrapolated, labelled as such, to all
    M x N entries of the GEMM."""
    import numpy as np
    from oracle import dkv_oracle as O
    A_bits = A.view(torch.int16).cpu().numpy().view(np.uint16)
    Bt_bits = Btd.view(torch.int16).cpu().numpy().view(np.uint16)
    rng = np.random.default_rng(seed)
    rows, cols = rng.integers(0, M, n_samples), rng.integers(0, N, n_samples)
    t0 = time.perf_counter()
    O.gemm_entries(A_bits, Bt_bits, rows, cols)
    t = time.perf_counter() - t0
    return {"value": t * (M * N / n_samples) * 1e3, "unit": "ms", "cores": 1, "kind": "oracle",
            "sample": "%d seeded entries of C in fp64 on one host thread (%.2f s); value = that time "
                      "extrapolated to all %d x %d entries" % (n_samples, t, M, N),
            "sample_s": t}


def run_layout(args):
    """Block-layout permutation (layer-first -> page-first) of a 2 GiB tier: L=32 layers,
    1024 blocks, 8 kv heads, D=128, T=16; HBM -> HBM and mapped host -> HBM."""
    import kv_cache_offload_b200 as dkv
    from kv_cache_offload_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    L, P, Hkv, T, D = 32, 1024, 8, 16, 128
    chunk = 2 * Hkv * T * D * 2
    nbytes = L * P * chunk
    src = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=dev).normal_()
    dst = torch.empty_like(src)
    hb = dkv.dkv_host_alloc_mapped(nbytes // 2, torch.bfloat16)
    hb.tensor.copy_(src.cpu())
    res = {}
    for name, s_ptr in (("hbm_to_hbm", src), ("host_to_hbm", hb.dev_ptr)):
        for _ in range(args.warmup):
            dkv.dkv_permute_layout(s_ptr, dst, 0, L, P, chunk)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps = args.steps if name == "hbm_to_hbm" else max(1, args.steps // 10)
        a.record()
        for _ in range(steps):
            dkv.dkv_permute_layout(s_ptr, dst, 0, L, P, chunk)
        b.record()
        b.synchronize()
        ms = a.elapsed_time(b) / steps
        res[name] = {"ms": ms, "gbs_read": nbytes / (ms * 1e-3) / 1e9}
    # bit-exact check of the last host -> HBM conversion on sampled chunks
    v = dst.view(P, L, chunk // 2)
    s2 = src.view(L, P, chunk // 2)
    for (l, pp) in ((0, 0), (31, 1023), (7, 512), (20, 3)):
        assert torch.equal(v[pp, l], s2[l, pp])
    hb.close()
    peak, kind = load_peaks()
    h2d = measure_h2d_peak(dev)
    hh = res["hbm_to_hbm"]
    line = {"metric": "block-layout conversion GB/s (layer-first -> page-first, 2 GiB tier)",
            "value": hh["gbs_read"], "unit": "GB/s (bytes read)", "higher_is_better": True, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "impl": "dkv", "data": "synthetic",
            "config": {"workload": "layout: L=32, P=1024, Hkv=8, T=16, D=128, bf16 (2 GiB)"},
            "variants": res,
            "roofline": {"bound": "hbm", "achieved": 2 * hh["gbs_read"], "peak": peak, "unit": "GB/s",
                         "frac": 2 * hh["gbs_read"] / peak, "peak_source": kind,
                         "note": "achieved counts read + write bytes, like the copy peak"},
            "host_link": {"h2d_peak_gbs": h2d, "host_to_hbm_gbs": res["host_to_hbm"]["gbs_read"],
                          "frac": res["host_to_hbm"]["gbs_read"] / h2d}}
    print(json.dumps(line), flush=True)


def run_staged_compare(args, cfg, wl, dev):
    """Conventional offload on the same workload: swap every host-tier block of the step
    into an HBM staging area (per-block cudaMemcpyAsync, or the GPU copy kernel), then
    attend over HBM only. Returns per-step times (ms)."""
    import kv_cache_offload_b200 as dkv
    lay = wl.lay
    nh, ns = lay.hbm_blocks, lay.host_blocks
    tier_elems = cfg.layers * 2 * cfg.Hkv * cfg.T * cfg.D
    hbm = torch.empty(((nh + ns) * tier_elems,), dtype=torch.bfloat16, device=dev)
    hbm[: nh * tier_elems].copy_(wl.hbm)
    pool = dkv.dkv_pool_create(cfg.layers, cfg.Hkv, cfg.D, nh + ns, ns, hbm_base=hbm)
    out = {}
    try:
        dkv.host_tier_tensor(pool).copy_(dkv.host_tier_tensor(wl.pool))
        table = lay.block_table.clone()
        table[lay.tier_map == 1] += nh
        table[lay.block_table < 0] = -1
        table = table.to(dev)
        tmap = torch.zeros_like(wl.tmap)
        src_h = torch.arange(ns, dtype=torch.int32)
        dst_h = torch.arange(nh, nh + ns, dtype=torch.int32)
        perm = torch.randperm(ns, generator=torch.Generator().manual_seed(0))
        ids = {"dma": (src_h[perm].contiguous(), dst_h[perm].contiguous()),
               "kernel": (src_h.to(dev), dst_h.to(dev))}
        steps = max(2, min(args.steps, 10))
        for name, method in (("dma", dkv.DKV_COPY_DMA), ("kernel", dkv.DKV_COPY_KERNEL)):
            s_ids, d_ids = ids[name]

            def step():
                dkv.dkv_copy_blocks(pool, 1, 0, s_ids, d_ids, method)
                dkv.dkv_decode_step(pool, 0, wl.x, wl.next_W(), table, wl.lens, tmap, cfg.Hq, cfg.theta, wl.out, wl.ws)

            step()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(steps):
                step()
            b.record()
            b.synchronize()
            out["staged_" + name + "_ms"] = a.elapsed_time(b) / steps
        assert dkv.dkv_check(pool) == dkv.DKV_OK
        out["staging_hbm_bytes"] = ns * tier_elems * 2
        out["note"] = ("dma: one cudaMemcpyAsync per block in table order (random physical ids); "
                       "kernel: one GPU copy kernel; both then attend over HBM only")
    finally:
        dkv.dkv_pool_destroy(pool)
    return out


class AdaptiveModel:
    """L layers of the 8B-shaped decode step over one pool, with the library's block manager
    placing each sequence's blocks (newest budget/B in HBM, the rest in the host tier) and
    one CUDA graph per plan buffer replaying plan application + every layer's step."""

    def __init__(self, dkv, dev, L, B, ctx, budget, headroom_tokens, seed=0):
        self.dkv, self.L, self.B, self.ctx = dkv, L, B, ctx
        H, Hq, Hkv, D, T = 4096, 32, 8, 128, 16
        self.H, self.Hq, self.Hkv, self.D, self.T, self.theta = H, Hq, Hkv, D, T, 5e5
        self.max_blocks = (ctx + headroom_tokens) // T + 1
        self.budget = budget
        hbm_ids = budget + B + 1
        host_ids = max(B * (ctx // T + 1) - budget, 0) + B * (headroom_tokens // T + 2)
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        blk = L * 2 * Hkv * T * D
        self.hbm = gpu_randn_bf16((hbm_ids * blk,), gen)
        self.pool = dkv.dkv_pool_create(L, Hkv, D, hbm_ids, host_ids, hbm_base=self.hbm)
        # host tier: random HBM blocks copied over the link by the library's copy kernel
        dst = torch.arange(host_ids, dtype=torch.int32, device=dev)
        dkv.dkv_copy_blocks(self.pool, 0, 1, (dst % hbm_ids).to(torch.int32).contiguous(), dst,
                            dkv.DKV_COPY_KERNEL)
        self.W = [gpu_randn_bf16(((Hq + 2 * Hkv) * D, H), gen, std=1.0 / math.sqrt(H)) for _ in range(L)]
        self.x = [gpu_randn_bf16((B, H), gen) for _ in range(L)]
        self.out = [torch.empty((B, Hq * D), dtype=torch.bfloat16, device=dev) for _ in range(L)]
        self.bt = torch.zeros((B, self.max_blocks), dtype=torch.int32, device=dev)
        self.tm = torch.zeros((B, self.max_blocks), dtype=torch.uint8, device=dev)
        self.sl = torch.zeros((B,), dtype=torch.int32, device=dev)
        self.bm = dkv.BlockManager(B, self.max_blocks, hbm_ids, host_ids, budget)
        for _ in range(B):
            self.bm.add(ctx)
            dkv.dkv_apply_plan(self.pool, self.bm.plan()[2], self.bt, self.tm, self.sl)
        torch.cuda.current_stream().synchronize()
        self.check_tables()
        nws = dkv.dkv_decode_workspace_bytes(self.pool, B, self.max_blocks, Hq, H)
        self.ws = torch.empty(nws, dtype=torch.uint8, device=dev)
        layers = [(l, self.x[l], self.W[l], self.out[l]) for l in range(L)]
        self.graphs = [dkv.dkv_decode_graph_create(self.pool, self.bm.plan(s)[2], layers, self.bt, self.sl,
                                                   self.tm, B, H, Hq, self.theta, self.ws) for s in (0, 1)]
        self.layers = layers
        if dkv.dkv_check(self.pool) != dkv.DKV_OK:  # synchronises: no plan buffer is still being read
            raise RuntimeError("adaptive setup: " + dkv.dkv_last_error())

    def check_tables(self):
        """The device tables must equal the manager's snapshot on every cached block."""
        bt, tm, sl = self.bm.tables()
        dbt, dtm, dsl = self.bt.cpu().numpy(), self.tm.cpu().numpy(), self.sl.cpu().numpy()
        for b in range(self.B):
            nb = int(sl[b]) // self.T + 1
            if int(dsl[b]) != int(sl[b]) or (dbt[b, :nb] != bt[b, :nb]).any() or (dtm[b, :nb] != tm[b, :nb]).any():
                raise RuntimeError("device tables differ from the block manager's (row %d)" % b)

    def bytes_per_step(self):
        """Algorithmic bytes of one L-layer step at the current placement: cached KV by tier
        (K and V of every cached token, every kv head, every layer) and W of every layer."""
        bt, tm, sl = self.bm.tables()
        per_tok = 2 * self.Hkv * self.D * 2 * self.L
        hbm = host = 0
        for b in range(self.B):
            c = int(sl[b])
            for j in range((c + self.T - 1) // self.T):
                n = min(self.T, c - j * self.T)
                if tm[b, j]:
                    host += n * per_tok
                else:
                    hbm += n * per_tok
        return hbm, host, self.L * (self.Hq + 2 * self.Hkv) * self.D * self.H * 2

    def run(self, steps, warmup, graph=True):
        """Time `steps` serving steps (host: count the last tokens, write a plan; device:
        apply it and decode every layer) after `warmup`; returns ms per step (CUDA events)."""
        dkv = self.dkv
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(warmup + steps):
            if i == warmup:
                a.record()
            self.bm.step()  # waits until the device released the plan buffer it rewrites
            slot, _, plan_dev = self.bm.plan()
            if graph:
                dkv.dkv_graph_launch(self.graphs[slot])
            else:
                dkv.dkv_apply_plan(self.pool, plan_dev, self.bt, self.tm, self.sl)
                for (l, x, W, out) in self.layers:
                    dkv.dkv_decode_step(self.pool, l, x, W, self.bt, self.sl, self.tm, self.Hq, self.theta, out,
                                        self.ws)
        b.record()
        b.synchronize()
        rc = dkv.dkv_check(self.pool)
        if rc != dkv.DKV_OK:
            raise RuntimeError("adaptive run: " + dkv.dkv_last_error())
        self.check_tables()
        return a.elapsed_time(b) / steps

    def close(self):
        for g in self.graphs:
            self.dkv.dkv_graph_destroy(g)
        self.bm.close()
        self.dkv.dkv_pool_destroy(self.pool)


def _dram_reader(nbytes, stop, counter, ready):
    """Another consumer of host DRAM bandwidth: streams through a private buffer until
    `stop` is set, adding the bytes read to `counter`."""
    import numpy as np
    a = np.ones(nbytes // 8, dtype=np.float64)  # touched, so resident
    ready.put(1)
    while not stop.is_set():
        a.max()
        with counter.get_lock():
            counter.value += nbytes


def run_host_contention(args):
    """NEXT-4 on one GPU: the host-tier decode step of the 70B-shaped layer (80% of its
    blocks read in place over PCIe) while k spawned CPU processes stream through their own
    host buffers, standing in for the host-DRAM traffic of other GPUs' replicas. Per k: the
    step's host-tier read rate, the readers' aggregate rate, and cudaMemcpy H2D under the
    same load."""
    import multiprocessing as mp
    import kv_cache_offload_b200 as dkv
    from kv_cache_offload_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = WL.CONFIGS["70b_mixed"]
    wl = Workload(cfg, seed=0, host_flags=args.host_flags)
    ctx = mp.get_context("spawn")  # never fork a process that has a CUDA context
    steps = max(3, min(args.steps, 8))
    sweep = []
    try:
        for _ in range(max(3, args.warmup)):
            wl.step()
        torch.cuda.synchronize()
        for k in (0, 2, 4, 8, 12):
            stop, counter, ready = ctx.Event(), ctx.Value("d", 0.0), ctx.Queue()
            procs = [ctx.Process(target=_dram_reader, args=(512 << 20, stop, counter, ready), daemon=True)
                     for _ in range(k)]
            for pr in procs:
                pr.start()
            try:
                for _ in procs:
                    ready.get(timeout=120)
                time.sleep(0.5)
                c0, t0 = counter.value, time.perf_counter()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(steps):
                    wl.step()
                b.record()
                b.synchronize()
                c1, t1 = counter.value, time.perf_counter()
                ms = a.elapsed_time(b) / steps
                h2d = measure_h2d_peak(dev, nbytes=512 << 20, reps=3)
            finally:
                stop.set()
                for pr in procs:
                    pr.join(timeout=30)
            assert dkv.dkv_check(wl.pool) == dkv.DKV_OK, dkv.dkv_last_error()
            sweep.append({"readers": k, "ms_per_step": ms, "tokens_per_s": cfg.B / (ms * 1e-3),
                          "host_tier_gbs": wl.kv_host_bytes / (ms * 1e-3) / 1e9,
                          "readers_gbs": (c1 - c0) / (t1 - t0) / 1e9, "h2d_memcpy_gbs": h2d})
    finally:
        wl.close()
    base = sweep[0]["host_tier_gbs"]
    line = {"metric": "host-tier zero-copy read rate under host-DRAM contention (70B-shaped layer)",
            "value": sweep[-1]["host_tier_gbs"], "unit": "GB/s", "n_gpus": 1, "higher_is_better": True,
            "config": {"workload": workload_config(cfg, 1)["workload"], "steps_per_point": steps,
                       "readers": "spawned CPU processes, each streaming a private 512 MiB buffer (max reduction)",
                       "host_cpus": os.cpu_count()},
            "sweep": sweep, "retained_at_max_readers": sweep[-1]["host_tier_gbs"] / base,
            "note": "the host-tier rate is over the whole step (projection + attention)"}
    print(json.dumps(line), flush=True)


def run_attn_sweep(args):
    """Attention alone (all blocks in HBM, serial launches) over split counts for both
    CUDA-core shapes, per batch x context, on the 8B-shaped (G = 4) and 70B-shaped (G = 8)
    layers: split counts at 0.3 to 3.5 waves of each shape's CTA slots (148 SMs x CTAs per
    SM: G = 4 variant 1 three, variant 5 four; G = 8 variant 1 one, variant 5 three), plus
    the automatic choice. 15 launches back to back between two events, best of 2 rounds."""
    import dataclasses
    import kv_cache_offload_b200 as dkv
    from kv_cache_offload_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    per_sm = {(4, 1): 3, (4, 5): 4, (8, 1): 1, (8, 5): 3}
    waves = (0.3, 0.43, 0.58, 0.72, 0.86, 1.0, 1.15, 1.45, 1.73, 2.0, 2.3, 2.9, 3.5)
    cases = ([("8b_hbm", B, c) for B in (1, 2, 4, 8, 16, 32) for c in (8192, 32768)]
             + [("8b_hbm", 1, 131072), ("8b_hbm", 4, 131072)]
             + [("70b_hbm", B, c) for B in (1, 4, 8, 32) for c in (8192, 32768)] + [("70b_hbm", 1, 131072)])
    rows = []
    for name, B, ctx in cases:
        cfg = dataclasses.replace(WL.CONFIGS[name], B=B, ctx=ctx, ctx_range=None, tier_policy="hbm")
        wl = Workload(cfg, seed=0)
        try:
            lay, units = wl.lay, cfg.B * cfg.Hkv
            auto = (dkv.dkv_decode_attn_variant(wl.pool, cfg.B, lay.max_blocks, cfg.Hq),
                    dkv.dkv_decode_attn_splits(wl.pool, cfg.B, lay.max_blocks, cfg.Hq))
            res = {}
            for variant in (1, 5):
                slots = sms * per_sm[(cfg.G, variant)]
                Ss = {max(1, min(lay.max_blocks, round(w * slots / units))) for w in waves}
                if auto[0] == variant:
                    Ss.add(auto[1])
                for S in sorted(Ss):
                    wl.set_tuning(attn_splits=S, attn_variant=variant, serial_launch=1)
                    wl.project()
                    c = wl.cfg
                    attend = lambda: dkv.dkv_decode_attend(wl.pool, 0, wl.table, wl.lens, wl.tmap, c.H, c.Hq, wl.ws,
                                                           out=wl.out)
                    for _ in range(3):
                        attend()
                    best = float("inf")
                    for _ in range(2):
                        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        torch.cuda._sleep(3_000_000)  # the host queues the launches meanwhile
                        a.record()
                        for _ in range(15):
                            attend()
                        b.record()
                        b.synchronize()
                        best = min(best, a.elapsed_time(b) * 1e3 / 15)
                    res[(variant, S)] = best
            assert dkv.dkv_check(wl.pool) == dkv.DKV_OK, dkv.dkv_last_error()
            bk = min(res, key=res.get)
            rows.append({"layer": name, "B": B, "ctx": ctx, "G": cfg.G, "units": units, "blocks": lay.max_blocks,
                         "kv_bytes": wl.kv_bytes, "auto": [auto[0], auto[1], res[auto]],
                         "best": [bk[0], bk[1], res[bk]],
                         "points_us": {"v%d S=%d" % k: v for k, v in sorted(res.items())}})
        finally:
            wl.close()
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "attention alone (us) over split counts and CUDA-core shapes, all blocks in HBM",
                      "sms": sms, "rows": rows}), flush=True)


def run_adaptive(args):
    """Adaptive placement (hot blocks in HBM, cold blocks read in place from the host tier)
    over a 4-layer slice of the 8B-shaped model, B=16 x 32768 cached tokens (8 GiB of KV),
    across HBM budgets; and CUDA-graph replay vs eager launches of a 32-layer step."""
    import kv_cache_offload_b200 as dkv
    from kv_cache_offload_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, kind = load_peaks()
    h2d = measure_h2d_peak(dev)
    L, B, ctx = 4, 16, 32768
    total = B * (ctx // 16 + 1)
    steps = max(2, min(args.steps, 6))
    warm = max(3, min(args.warmup, 3))
    sweep = []
    for frac in (1.0, 0.5, 0.25, 1.0 / 16, 0.0):
        budget = int(round(frac * total))
        m = AdaptiveModel(dkv, dev, L, B, ctx, budget, headroom_tokens=16 * 4)
        try:
            ms = m.run(steps, warm, graph=True)
            ms_eager = m.run(steps, 1, graph=False)
            hbm_b, host_b, w_b = m.bytes_per_step()
            t_roof = max((hbm_b + w_b) / (peak * 1e9), host_b / (h2d * 1e9)) * 1e3
            sweep.append({"hbm_frac": frac, "budget_blocks": budget, "window_blocks": m.bm.window,
                          "ms_per_step": ms, "tokens_per_s": B / (ms * 1e-3), "eager_ms_per_step": ms_eager,
                          "kv_hbm_bytes": hbm_b, "kv_host_bytes": host_b, "w_bytes": w_b,
                          "hbm_tier_bytes": m.hbm.numel() * 2, "t_roof_ms": t_roof, "frac_of_roofline": t_roof / ms})
        finally:
            m.close()
        torch.cuda.empty_cache()
    # launch overhead: a full-depth (32-layer) step on short contexts, all in HBM
    Lg, ctxg = 32, 2048
    m = AdaptiveModel(dkv, dev, Lg, B, ctxg, B * ((ctxg + 16 * 8) // 16 + 1), headroom_tokens=16 * 8)
    try:
        ms_g = m.run(50, warm, graph=True)
        ms_e = m.run(50, warm, graph=False)
        hbm_b, host_b, w_b = m.bytes_per_step()
        graph = {"layers": Lg, "batch": B, "cached_tokens": ctxg, "graph_ms_per_step": ms_g,
                 "eager_ms_per_step": ms_e, "speedup": ms_e / ms_g,
                 "t_roof_ms": (hbm_b + w_b) / (peak * 1e9) * 1e3,
                 "frac_of_roofline_graph": (hbm_b + w_b) / (peak * 1e9) * 1e3 / ms_g}
    finally:
        m.close()
    best = sweep[0]
    line = {"metric": "adaptive placement: 4-layer decode step tokens/s vs HBM budget", "value": best["tokens_per_s"],
            "unit": "tokens/s", "higher_is_better": True, "n_gpus": 1, "steps": steps, "warmup": warm,
            "impl": "dkv", "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "8B-shaped layers x4, B=16, 32768 cached tokens each, 16-token blocks; "
                                   "recency-window placement at HBM budget fractions 1, 1/2, 1/4, 1/16, 0; "
                                   "each step = host plan + one graph replay (plan apply + 4 layers)"},
            "h2d_peak_gbs": h2d, "hbm_peak_gbs": peak, "peak_source": kind,
            "sweep": sweep, "graph_vs_eager": graph}
    print(json.dumps(line), flush=True)


HEADLINE = "70b_mixed"  # the largest single-GPU decode configuration: the headline line
HBM_LINE = "8b_hbm"     # the all-HBM configuration, reported beside it in the same run
OTHER_CONFIGS = ("8b_mixed", "tiny")  # the remaining decode configurations (with the GEMM study)


def _nvtx(name):
    torch.cuda.nvtx.range_push(name)


def _nvtx_end():
    torch.cuda.nvtx.range_pop()


def decode_line(cfg: WL.DecodeConfig, args, world, rank, local, dist, dev, full: bool, steps: int) -> dict:
    """Time the decode step of one workload on this rank (every rank makes the same
    collective calls) and return its JSON fields. `full` adds the end-to-end loop."""
    import kv_cache_offload_b200 as dkv
    tdist = None
    if dist:
        import torch.distributed as tdist

    def barrier():
        if dist:
            tdist.barrier()
        torch.cuda.synchronize()

    _nvtx("setup " + cfg.name)
    wl = Workload(cfg, seed=rank, host_flags=args.host_flags)
    wl.set_tuning(args.attn_splits, args.proj_splits, attn_variant=args.attn_variant)
    _nvtx_end()
    try:
        _nvtx("warmup " + cfg.name)
        for _ in range(args.warmup):
            wl.step()
        assert dkv.dkv_check(wl.pool) == dkv.DKV_OK, dkv.dkv_last_error()
        _nvtx_end()

        # ---- value: K back-to-back steps, inputs resident in HBM / the host tier. The clock
        # sampler (200 ms period) starts first and the GPU is kept busy with untimed steps for
        # ~0.6 s so that samples are taken under the same load as the timed region.
        clocks = ClockSampler(local)
        barrier()
        clocks.start()
        t_end = time.perf_counter() + 0.6
        while time.perf_counter() < t_end:
            for _ in range(8 if wl.kv_host_bytes == 0 else 1):
                wl.step()
            torch.cuda.synchronize()
        _nvtx("timed " + cfg.name)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            wl.step()
        e1.record()
        barrier()
        pass_mhz = {"timed": sm_clock_now(local)}
        _nvtx_end()
        time.sleep(0.25)
        clk = clocks.stop()
        t_ms = e0.elapsed_time(e1)
        assert dkv.dkv_check(wl.pool) == dkv.DKV_OK, dkv.dkv_last_error()

        # ---- step-time spread: the same steps with an event after each one (a separate
        # pass: an event between steps ends the next step's early start)
        _nvtx("per-step " + cfg.name)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        barrier()
        evs[0].record()
        for i in range(steps):
            wl.step()
            evs[i + 1].record()
        barrier()
        pass_mhz["per_step"] = sm_clock_now(local)
        _nvtx_end()
        per_step = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]

        # ---- launch A/B under the same sustained load: interleaved blocks of back-to-back
        # steps with the two kernels overlapped (programmatic dependent launch, the default)
        # and launched serially, no events inside a block
        _nvtx("launch A/B " + cfg.name)
        # (and blocks of the attention alone, launched the same way: what the overlapped step
        # costs beyond its attention is the projection's exposed part)
        n_ab = steps if wl.kv_host_bytes == 0 else min(steps, 5)
        ab = {0: [], 1: [], 2: []}
        for _ in range(2):
            for mode in (0, 1, 2):
                wl.set_tuning(args.attn_splits, args.proj_splits, attn_variant=args.attn_variant,
                              serial_launch=1 if mode == 2 else mode)
                run = wl.step if mode < 2 else wl.attend
                run()
                barrier()
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record()
                for _ in range(n_ab):
                    run()
                a1.record()
                barrier()
                ab[mode].append(a0.elapsed_time(a1) / n_ab)
        wl.set_tuning(args.attn_splits, args.proj_splits, attn_variant=args.attn_variant)
        ab_ms = [sum(ab[m]) / len(ab[m]) for m in (0, 1, 2)]
        pass_mhz["launch_ab"] = sm_clock_now(local)
        _nvtx_end()

        # ---- per-stage durations: the same steps launched serially (no programmatic
        # dependent launch, so each kernel runs alone), with events between the two launches
        _nvtx("stages " + cfg.name)
        wl.set_tuning(args.attn_splits, args.proj_splits, attn_variant=args.attn_variant, serial_launch=1)
        for _ in range(3):
            wl.step()
        sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        barrier()
        for i in range(steps):
            wl.step_timed_stages(sevs[i])
        barrier()
        pass_mhz["stages"] = sm_clock_now(local)
        stage_ms = [sum(sevs[i][k].elapsed_time(sevs[i][k + 1]) for i in range(steps)) / steps
                    for k in range(2)]
        # ---- the projection alone, back to back: serial launches queued while a sleep kernel
        # holds the stream, timed between two events. Its GPU time per launch, including the
        # gap every kernel launch costs (~2 us on each side here) but not the two events per
        # stage above; W cycles through its copies, so it comes from HBM.
        n_proj = 100
        for _ in range(3):
            wl.project()
        barrier()
        torch.cuda._sleep(10_000_000)  # a few ms at the SM clock: the host queues the launches meanwhile
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        for _ in range(n_proj):
            wl.project()
        p1.record()
        barrier()
        proj_b2b_ms = p0.elapsed_time(p1) / n_proj
        wl.set_tuning(args.attn_splits, args.proj_splits, attn_variant=args.attn_variant)
        _nvtx_end()

        e2e_ms, h2d, d2h = 0.0, 0, 0
        if full:
            _nvtx("e2e " + cfg.name)
            e2e_ms, h2d, d2h = time_e2e(wl, steps, barrier)
            _nvtx_end()

        # ---- max over ranks
        p10, p50, p90 = percentiles(per_step)
        vals = reduce_max_over_ranks([t_ms, e2e_ms, p10, p50, p90, proj_b2b_ms] + ab_ms + stage_ms, dist, dev)
        t_ms, e2e_ms, p10, p50, p90, proj_b2b_ms = vals[:6]
        ab_ms = vals[6:9]
        stage_ms = vals[9:]
        ms = t_ms / steps
        value = replica_throughput(cfg.B, world, ms)

        peak, peak_kind = load_peaks()
        attn_ms = stage_ms[1]
        achieved = wl.kv_bytes / (attn_ms * 1e-3) / 1e9
        host_info = None
        if wl.kv_host_bytes:
            h2d_peak = measure_h2d_peak(dev)
            host_gbs = wl.kv_host_bytes / (attn_ms * 1e-3) / 1e9
            host_info = {"h2d_peak_gbs": h2d_peak, "host_kv_bytes": wl.kv_host_bytes,
                         "hbm_kv_bytes": wl.kv_hbm_bytes, "achieved_gbs": host_gbs,
                         "frac": host_gbs / h2d_peak, "link": "PCIe (not NVLink-C2C)",
                         "host_numa_node": {"gpu_nearest": host_numa_node(dkv, local),
                                            "host_tier_first_page": dkv.dkv_pool_host_numa_node(wl.pool),
                                            "policy": "preferred node = the GPU's nearest (DKV_HOST_NUMA_NEAREST)"
                                            if args.host_flags & 2 else "none"}}
        tr = profiled_traffic(cfg.name, cfg.B)
        line = {
            "value": value, "ms_per_step": ms,
            "step_ms_p10_p50_p90": [p10, p50, p90],
            "config": dict(workload_config(cfg, world), attn_splits=wl.splits, attn_variant=args.attn_variant,
                           attn_kernel_variant=dkv.dkv_decode_attn_variant(wl.pool, cfg.B, wl.lay.max_blocks, cfg.Hq),
                           l2="inputs larger than L2 (%.2f GB of KV + W per step; W cycles through %d copies, "
                              "%.2f GB)" % ((wl.kv_bytes + wl.w_bytes) / 1e9, wl.n_w, wl.n_w * wl.w_bytes / 1e9)),
            "kv_gbs": (wl.kv_bytes + wl.new_kv_bytes) / (ms * 1e-3) / 1e9,
            # the whole step against the same peak: every byte it must move (cached KV, W, x,
            # the new K/V rows, out) over the step time (host-tier bytes over the host link)
            "step_roofline": step_roofline(wl, ms, peak, peak_kind),
            "stage_ms": {"project": stage_ms[0], "attend_and_combine": stage_ms[1],
                         "timing": "each kernel alone (serial launches) between events; the step overlaps them",
                         "project_back_to_back": proj_b2b_ms,
                         "project_back_to_back_timing": "%d serial launches queued behind a sleep kernel, "
                                                        "between two events, W from HBM" % n_proj},
            "launch_ab": {"overlapped_ms_per_step": ab_ms[0], "serial_ms_per_step": ab_ms[1],
                          "attention_alone_ms": ab_ms[2], "step_minus_attention_ms": ab_ms[0] - ab_ms[2],
                          "steps_per_block": n_ab, "blocks_per_mode": 2,
                          "timing": "interleaved blocks of back-to-back steps, no events inside a block: "
                                    "the default launch (the two kernels overlapped by programmatic "
                                    "dependent launch) against serial launches and against the attention "
                                    "launched alone, under the same load"},
            "projection_roofline": {"bound": "hbm", "kernel": "proj_umma_kernel",
                                    "achieved": wl.w_bytes / (proj_b2b_ms * 1e-3) / 1e9, "peak": peak,
                                    "unit": "GB/s", "frac": wl.w_bytes / (proj_b2b_ms * 1e-3) / 1e9 / peak,
                                    "peak_source": peak_kind, "algorithmic_bytes_per_launch": wl.w_bytes,
                                    "timing": "stage_ms.project_back_to_back"},
            "roofline": ({"bound": "hbm", "kernel": "attn_splitk_kernel",
                          "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                          "peak_source": peak_kind, "traffic": tr and tr["bytes"],
                          "traffic_counter": tr and tr["counter"],
                          "algorithmic_bytes_per_launch": wl.kv_bytes}
                         if not wl.kv_host_bytes else
                         {"bound": "host_link", "kernel": "attn_splitk_kernel",
                          "achieved": host_info["achieved_gbs"], "peak": host_info["h2d_peak_gbs"], "unit": "GB/s",
                          "frac": host_info["frac"],
                          "peak_source": "measured cudaMemcpy H2D (pinned, 1 GiB) in this run",
                          "traffic": tr and tr["bytes"], "traffic_counter": tr and tr["counter"],
                          "algorithmic_bytes_per_launch": wl.kv_host_bytes}),
            "gpu_launches": 2 * steps,
            "clocks": clk,
            # SM clock (NVML) at the end of each pass: the power-capped clock differs from pass
            # to pass, and the step and stage times follow it
            "pass_end_sm_mhz": pass_mhz,
        }
        if full:
            line["e2e"] = {"value": replica_throughput(cfg.B, world, e2e_ms / steps), "unit": "tokens/s",
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        if host_info:
            line["host_link"] = host_info
            if args.compare_staged:
                line["staged_swap_baseline"] = run_staged_compare(args, cfg, wl, dev)
                line["staged_swap_baseline"]["zero_copy_ms"] = ms
        return line
    finally:
        wl.close()


def time_e2e(wl, steps, barrier):
    """The step through the public call with host buffers, as a serving loop runs it: step
    k+1's inputs are copied from pinned host memory on a copy stream into the second of two
    device buffer sets while step k computes, and step k's output is read back on that
    stream; every copy of every step is inside the timed region. Returns (ms for all
    steps, H2D bytes per step, D2H bytes per step)."""
    dkv, cfg = wl.dkv, wl.cfg
    xh = wl.x.cpu().pin_memory()
    th, mh, lh = wl.table.cpu().pin_memory(), wl.tmap.cpu().pin_memory(), wl.lens.cpu().pin_memory()
    oh = [torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory() for _ in range(2)]
    ins = [(torch.empty_like(wl.x), torch.empty_like(wl.table), torch.empty_like(wl.tmap),
            torch.empty_like(wl.lens)) for _ in range(2)]
    outs = [torch.empty_like(wl.out) for _ in range(2)]
    h2d = xh.numel() * 2 + th.numel() * 4 + mh.numel() + lh.numel() * 4
    d2h = oh[0].numel() * 2
    main, cs = torch.cuda.current_stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]

    def copy_inputs(i):
        xd, td, md, ld = ins[i]
        with torch.cuda.stream(cs):
            xd.copy_(xh, non_blocking=True); td.copy_(th, non_blocking=True)
            md.copy_(mh, non_blocking=True); ld.copy_(lh, non_blocking=True)
            ev_in[i].record(cs)

    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    cs.wait_event(a)
    copy_inputs(0)
    for k in range(steps):
        i = k % 2
        xd, td, md, ld = ins[i]
        main.wait_event(ev_in[i])
        dkv.dkv_decode_step(wl.pool, 0, xd, wl.next_W(), td, ld, md, cfg.Hq, cfg.theta, outs[i], wl.ws)
        ev_done[i].record(main)
        # copy stream, while step k computes: read back step k-1's output, then refill that
        # buffer set with step k+1's inputs (step k+1 waits for them, hence for the read-back)
        if k >= 1:
            cs.wait_event(ev_done[1 - i])
            with torch.cuda.stream(cs):
                oh[1 - i].copy_(outs[1 - i], non_blocking=True)
        if k + 1 < steps:
            copy_inputs(1 - i)
    last = (steps - 1) % 2
    cs.wait_event(ev_done[last])
    with torch.cuda.stream(cs):
        oh[last].copy_(outs[last], non_blocking=True)
    main.wait_stream(cs)
    b.record(main)
    barrier()
    return a.elapsed_time(b), h2d, d2h


def host_numa_node(dkv, device_index: int):
    """The NUMA node the pool's host tier is bound to on this GPU (None where unknown)."""
    try:
        n = dkv.dkv_host_numa_node(device_index)
        return None if n < 0 else n
    except Exception:
        return None


def main():
    args = parse()
    if args.config == "layout":
        return run_layout(args)
    if args.config == "adaptive":
        return run_adaptive(args)
    if args.config == "host_contention":
        return run_host_contention(args)
    if args.config == "attn_sweep":
        return run_attn_sweep(args)
    if args.config == "gemm":
        rank = int(os.environ.get("RANK", "0"))
        if rank == 0:
            run_gemm(args, rank, 1)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = world > 1
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.warmup < 3:
        args.warmup = 3
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=dev)
    from kv_cache_offload_b200.build import build
    if rank == 0 or not dist:
        build()
    if dist:
        tdist.barrier()
    import kv_cache_offload_b200 as dkv

    cfg = WL.CONFIGS[args.config]
    if args.batch or args.ctx:
        import dataclasses
        cfg = dataclasses.replace(cfg, B=args.batch or cfg.B)
        if args.ctx:
            cfg = dataclasses.replace(cfg, ctx=args.ctx, ctx_range=None)
    if args.profile:
        wl = Workload(cfg, seed=rank, host_flags=args.host_flags)
        wl.set_tuning(args.attn_splits, args.proj_splits, attn_variant=args.attn_variant)
        for _ in range(args.warmup):
            wl.step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            wl.step()
        b.record()
        b.synchronize()
        assert dkv.dkv_check(wl.pool) == dkv.DKV_OK, dkv.dkv_last_error()
        if rank == 0:
            print(json.dumps({"profile_run": cfg.name, "B": cfg.B, "attn_splits": wl.splits,
                              "attn_kernel_variant": dkv.dkv_decode_attn_variant(wl.pool, cfg.B, wl.lay.max_blocks,
                                                                                 cfg.Hq),
                              "kv_hbm_bytes": wl.kv_hbm_bytes, "kv_host_bytes": wl.kv_host_bytes,
                              "w_bytes": wl.w_bytes, "ms_per_step": a.elapsed_time(b) / args.steps}), flush=True)
        wl.close()
        return

    body = decode_line(cfg, args, world, rank, local, dist, dev, full=True, steps=args.steps)
    line = {"metric": METRIC, "value": body.pop("value"), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": body.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic"}
    line.update(body)
    if args.config == HEADLINE and not args.batch and not args.ctx and not args.no_hbm_line:
        # the all-HBM layer in the same run: the HBM-roofline bar beside the host-link one
        torch.cuda.empty_cache()
        hsteps = max(args.steps, 100)  # 0.4 ms steps: more of them for a stable mean
        hl = decode_line(WL.CONFIGS[HBM_LINE], args, world, rank, local, dist, dev, full=False, steps=hsteps)
        hl.update(unit="tokens/s", steps=hsteps)
        line["hbm_line"] = hl
    if args.config == HEADLINE and not args.batch and not args.ctx and world == 1 and not args.no_other_configs:
        # the remaining decode configurations and the GEMM study, in the same run (one GPU)
        torch.cuda.empty_cache()
        other = {}
        for name in OTHER_CONFIGS:
            # the 8B mixed layer also runs the conventional offload on the same workload: swap
            # the host blocks into HBM (per-block DMA or the GPU copy kernel), then attend
            args.compare_staged = name == "8b_mixed"
            o = decode_line(WL.CONFIGS[name], args, world, rank, local, dist, dev, full=False,
                            steps=min(args.steps, 20))
            o.update(unit="tokens/s", steps=min(args.steps, 20))
            other[name] = o
            torch.cuda.empty_cache()
        other["gemm"] = gemm_line(args, rank, dev, steps=min(args.steps, 5), warmup=3)
        line["other_configs"] = other
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, 0, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        tdist.barrier()
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()
