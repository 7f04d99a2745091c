#!/usr/bin/env python
"""Benchmark: paged decode attention on B200 — KV GB/s against the HBM
roofline, and decode tokens/s per layer.

A step is one pass of the whole decode path over one batch: slot reservation
(host allocator; staged before timing for the device-resident number), block
copies for copy-on-write (when any), KV append, and paged attention with its
partition merge.  The default workload is the Llama-3-8B-shaped layer:
64 sequences of U[512, 4096] tokens, 32 query / 8 KV heads, head_dim 128,
bf16, block size 16, pool 1.2x the blocks needed, seeded and synthetic.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle as the reference arm

Prints one JSON line (rank 0).  With N > 1 (torchrun, one process per GPU)
every rank runs its own batch (sequences are independent: no collective on
the data path); time is the max over ranks and ``value`` sums all ranks' bytes.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: KV GB/s (fraction of B200 HBM peak), tokens/s per layer"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_SUSTAINED = 1400.0  # TFLOP/s, dense bf16 under the power cap
STAGED_STEPS = 16  # distinct steps of metadata resident on the device, cycled
# Where a step holds more than the timed library call (copy-on-write copies,
# the prefill's append), the call is bracketed by its own CUDA events on every
# EVENT_EVERY-th timed step from the second on, or on every step from the
# second on when there are fewer than 4 such samples (a pair of timing events
# on every step added about 5 us to a 103 us decode step).  Where the call is
# the whole step, one event after the first step and the end event bracket
# steps 2..K: the first step starts on an idle GPU right after a synchronise
# and carries the host's launch latency.
EVENT_EVERY = 16

# A timed region follows a synchronize, so it would start on an idle GPU whose
# first step waits for the host to issue its launches (≈ 20-30 µs, 1-1.5 % of
# a 20-step region).  A spin kernel of about 100 µs queued before the start
# event lets the host issue the first timed steps while it runs, and the clock
# sampler's first reading falls within it; it is not part of the timed work
# (the start event follows it).
PREQUEUE_CYCLES = 200_000


def prequeue():
    torch.cuda._sleep(PREQUEUE_CYCLES)

# DRAM traffic of one pkv_append_and_decode call per workload, from the ncu
# captures summarised in profiles/ (dram__bytes_read.sum +
# dram__bytes_write.sum over the append + plan, decode and merge kernels, mean
# of the captured calls), with the hash of the decode sources they were taken
# on (kernel_source_sha()).  A pin whose hash no longer matches is reported as
# null.
TRAFFIC = {
    "llama3_8b": (608230758, "7daaec3872a1cfe9"),
    "llama3_8b_fp8": (308158284, "7daaec3872a1cfe9"),
}
# the same for one pkv_paged_attention_prefill call (prefill_tc_kernel), keyed
# by the hash of the prefill sources (kernel_source_sha(PREFILL_SOURCES))
TRAFFIC_PREFILL = {
    "prefill_llama3_8b": (329452800, "8e17c4b8b5daa237"),
}


SEQ_LEN_RECIPES = {
    "tiny": "{1,7,16,33} before the step's append",
    "llama3_8b": "U[512,4096]",
    "llama3_8b_fp8": "U[512,4096]; e4m3 K/V (scale 1/32), q and new rows float16",
    "prefix_shared": "1024-token shared prefix (refcount = num_seqs) + U[64,512] tails; KV bytes are logical "
                     "(the prefix counted once per sequence)",
    "long_splitk": "7 x 32768 + 1 x 131072",
    "mha_7b": "lognormal(median 1000, sigma 1) clipped to [16, 8192]",
}


DECODE_SOURCES = ("append.cuh", "decode.cuh", "decode_mma.cuh", "decode_tc8.cuh", "tcgen05.cuh", "device_common.cuh")
PREFILL_SOURCES = ("prefill.cuh", "tcgen05.cuh", "device_common.cuh")


def kernel_source_sha(names=DECODE_SOURCES) -> str:
    """Hash of the device sources a kernel is built from (csrc files)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_406_b200", "csrc")
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=8000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama3_8b")
    ap.add_argument("--partition-tokens", type=int, default=-1, help="-1: the workload's setting")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the CPU oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="a smaller batch of the workload's shape (for profiler captures); 0: the workload's own")
    return ap.parse_args()


def workload_of(args):
    """The named workload, with the batch cut to --num-seqs when given."""
    from dataclasses import replace
    from paged_kv_cache_406_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    if args.num_seqs > 0:
        w = replace(w, num_seqs=args.num_seqs)
    if getattr(args, "partition_tokens", -1) >= 0:
        w = replace(w, partition_tokens=args.partition_tokens)
    return w


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def combine_ranks(elapsed_ms: float, nbytes: float, ntokens: float, device) -> tuple:
    """Whole-job totals over the ranks of the default process group: the
    slowest rank's time (max), and the sums of bytes and tokens processed."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return elapsed_ms, nbytes, ntokens
    mx = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    sm = torch.tensor([nbytes, ntokens], dtype=torch.float64, device=device)
    dist.all_reduce(sm, op=dist.ReduceOp.SUM)
    return float(mx[0]), float(sm[0]), float(sm[1])


def rank_workload(w, rank: int):
    """Rank r runs its own batch of the same shape (weak scaling): seeds offset by 1000·r."""
    from dataclasses import replace
    return replace(w, seed=w.seed + 1000 * rank) if rank else w


def measured_peak_file() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return {}
    with open(p) as f:
        return json.load(f)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons of this process's GPU during
    the timed region, read through NVML (the library nvidia-smi reads): a
    background thread samples from the start of the region, pausing
    ``period_s`` between readings, and :meth:`sample` takes one reading on
    the calling thread, which the timed loops do right after their last
    launch, while the GPU still works through its queue.  One reading takes
    milliseconds, so the launching thread never samples mid-region: that
    starved the GPU of a 20-step region for the reading's duration.  Without
    the NVML binding, ``nvidia-smi -lms 200`` writes into a temporary file."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, enabled: bool, period_s: float = 0.005):
        self.readings = []  # (sm MHz, reason bits, power W)
        self.nv = self.h = self.thread = self.proc = None
        self.max_mhz = None
        if not enabled:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.bits = {name: int(getattr(pynvml, attr, 0)) for name, attr in self.REASONS}
        except Exception:
            self.nv = self.h = None
            self._start_smi(device_index)
            return
        self.stop_ev = threading.Event()
        self.go = threading.Event()
        self.period = period_s
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def begin(self):
        """Called right after the timed region's start event: readings start."""
        if self.thread is not None:
            self.go.set()

    def _handle(self, device_index: int):
        nv = self.nv
        props = torch.cuda.get_device_properties(device_index)
        uuid = str(getattr(props, "uuid", ""))
        for u in (uuid, "GPU-" + uuid):
            try:
                return nv.nvmlDeviceGetHandleByUUID(u)
            except Exception:
                pass
        try:
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(device_index)

    def sample(self):
        if self.h is None:
            return
        nv = self.nv
        try:
            mhz = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            watts = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
        except Exception:
            return
        self.readings.append((mhz, bits, watts))

    def _loop(self):
        while not self.go.wait(0.05):
            if self.stop_ev.is_set():
                return
        while not self.stop_ev.is_set():
            self.sample()
            self.stop_ev.wait(self.period)

    def _start_smi(self, device_index: int):
        try:
            fd, self.path = tempfile.mkstemp(prefix="pkv_clocks_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(device_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def _stop_smi(self):
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, smax, reasons = [], [], set()
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "nvidia-smi"}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi -lms 200"}

    def stop(self):
        if self.proc is not None:
            return self._stop_smi()
        if self.h is None:
            return None
        self.stop_ev.set()
        self.go.set()
        self.thread.join(timeout=5)
        r = list(self.readings)
        reasons = sorted({name for _, bits, _ in r for name, bit in self.bits.items() if bit and bits & bit})
        return {"sm_mhz": statistics.median(m for m, _, _ in r) if r else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(r),
                "power_w": round(statistics.median(w for _, _, w in r), 1) if r else None,
                "source": "NVML during the timed region (a thread reading from its start, %.0f ms between "
                          "readings, plus one read right after the last launch)" % (self.period * 1e3)}


# ---------------------------------------------------------------------------
# the CPU oracle, timed (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(units, budget_s: float):
    """Runs the oracle on (q rows, K, V raw blocks, table, L, scale, dtype)
    units until the budget is spent; returns (KV bytes, seconds, units done)."""
    from oracle import fp8 as of8
    from oracle import paged_attention as pa
    done, nbytes, t0 = 0, 0, time.perf_counter()
    for u in units:
        q, kb, vb, L, scale, dtype, kv_bytes = u
        table = np.arange(kb.shape[0], dtype=np.int32)[None]
        if isinstance(dtype, tuple):  # ("e4m3", k_scale, v_scale)
            of8.paged_decode_attention_fp8(q, kb, vb, table, np.array([L]), scale, dtype[1], dtype[2])
        else:
            pa.paged_decode_attention(q, kb, vb, table, np.array([L]), scale, dtype)
        done += 1
        nbytes += kv_bytes
        if time.perf_counter() - t0 > budget_s:
            break
    return nbytes, time.perf_counter() - t0, done


def _raw(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def make_units(w, k_pool, v_pool, tables, lens, q, order, count):
    G, e = w.group, torch.tensor([], dtype=w.torch_dtype).element_size()
    units = []
    for i in range(count):
        b, g = order[i % len(order)]
        L = int(lens[b])
        nblk = -(-L // w.block_size)
        idx = torch.as_tensor(tables[b, :nblk], device=k_pool.device, dtype=torch.long)
        kb = _raw(k_pool[idx, g:g + 1])
        vb = _raw(v_pool[idx, g:g + 1])
        qb = _raw(q[b:b + 1, g * G:(g + 1) * G])
        dt = ("e4m3", w.kv_scale, w.kv_scale) if w.dtype == "e4m3" else w.dtype
        units.append((qb, kb, vb, L, w.scale, dt, L * w.head_dim * 2 * e))
    return units


# ---------------------------------------------------------------------------
def setup(w, device, horizon):
    """Pools, allocator and admitted batch; ``horizon`` = tokens each sequence
    may still gain (staged + end-to-end steps), covered by pool and tables."""
    from paged_kv_cache_406_b200 import workloads as W
    from paged_kv_cache_406_b200.cache import PagedKVCache
    lens = W.seq_lens(w)
    nb = W.pool_blocks(w, lens + horizon) + (w.num_seqs if w.prefix_tokens else 0)
    shape = (nb, w.num_kv_heads, w.block_size, w.head_dim)
    k_pool = W.pool_values(shape, w, 0, device=device)
    v_pool = W.pool_values(shape, w, 1, device=device)
    maxb = -(-(int(lens.max()) + horizon) // w.block_size)
    cache = PagedKVCache(nb, w.num_kv_heads, w.head_dim, w.block_size, w.torch_dtype, maxb, device=device,
                         free_order=W.free_order(nb, w.seed), k_pool=k_pool, v_pool=v_pool,
                         k_scale=w.kv_scale, v_scale=w.kv_scale)
    if w.prefix_tokens:
        # one sequence holds the shared prefix, the others fork it (refcount =
        # num_seqs), then every sequence appends its own tail token by token
        from paged_kv_cache_406_b200 import pkv_copy_blocks
        cache.add(0, w.prefix_tokens)
        for b in range(1, w.num_seqs):
            cache.fork(0, b)
        tails = lens - w.prefix_tokens
        for r in range(int(tails.max())):
            ids = [b for b in range(w.num_seqs) if tails[b] > r]
            _, cow = cache.alloc.append_slots(ids)
            if cow.size:
                pkv_copy_blocks(cache.k_pool, cache.v_pool, torch.from_numpy(cow).to(device))
    else:
        for b, L in enumerate(lens):
            cache.add(b, int(L))
    return w, cache, lens


def sampled_steps(K: int) -> list:
    """Timed steps whose call gets its own event pair: every EVENT_EVERY-th
    from the second on, or every step from the second on when that would give
    fewer than 4 samples."""
    every = list(range(1, K, EVENT_EVERY))
    return every if len(every) >= 4 else list(range(1, K)) or [0]


def decode_launches(max_blocks: int, block_size: int, partition_tokens: int) -> int:
    """Kernels one pkv_paged_attention_decode (or pkv_append_and_decode) call
    launches: the plan (or append + plan) and decode kernels, plus the
    partition merge when a sequence of the table's capacity can span more than
    one partition."""
    pt = partition_tokens or 512
    return 2 + (1 if max_blocks * block_size > pt else 0)


def run_ours(args):
    import torch.distributed as dist
    import paged_kv_cache_406_b200 as P
    from paged_kv_cache_406_b200 import workloads as W

    ws, rank, local = dist_env()
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w0 = workload_of(args)
    horizon = STAGED_STEPS + 3 + max(0, args.e2e_steps) + 8
    w, cache, lens0 = setup(rank_workload(w0, rank), dev, horizon)
    B, hq, hkv, d, bs = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    esz = torch.tensor([], dtype=w.torch_dtype).element_size()   # stored K/V element
    qsz = torch.tensor([], dtype=w.io_dtype).element_size()      # q and new rows
    fp8 = w.dtype == "e4m3"
    ids = list(range(B))
    alloc = cache.alloc

    # ---- stage STAGED_STEPS steps of metadata and inputs on the device ----
    staged = []
    for s in range(STAGED_STEPS):
        slots, cow = alloc.append_slots(ids)
        tables, lens = alloc.block_tables(ids, cache.max_blocks)
        staged.append(dict(
            slots=torch.from_numpy(slots.copy()).to(dev), cow=torch.from_numpy(cow.copy()).to(dev),
            ncow=cow.shape[0], tables=torch.from_numpy(tables.copy()).to(dev),
            lens=torch.from_numpy(lens.copy()).to(dev), lens_host=lens.copy(),
            q=W.normal((B, hq, d), w.io_dtype, W.step_seed(w, s, 0), device=dev),
            kn=W.normal((B, hkv, d), w.io_dtype, W.step_seed(w, s, 1), device=dev),
            vn=W.normal((B, hkv, d), w.io_dtype, W.step_seed(w, s, 2), device=dev)))
    wsb = P.pkv_decode_workspace_size(B, hq, hkv, d, cache.max_blocks, bs, w.partition_tokens)
    workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    if not fp8:
        # each staged step's call checked and marshalled once (the loop then
        # pays only the C call: the GPU is never left waiting on the host)
        for st in staged:
            st["call"] = P.bind_append_and_decode(st["kn"], st["vn"], st["slots"], st["q"], cache.k_pool,
                                                  cache.v_pool, st["tables"], st["lens"], w.scale, out, workspace,
                                                  partition_tokens=w.partition_tokens)

    def kv_bytes(lens):
        return int(lens.astype(np.int64).sum()) * hkv * d * 2 * esz

    pt_eff = w.partition_tokens or 512

    def algo_bytes(lens):
        # K/V rows once per (sequence, KV head) + block-table entries + q + out,
        # + the split-partition partials (m, l, o per query head), written once and read once,
        # + the new rows of the append (read as given, written as stored) and their slots
        tab = int(sum(-(-int(L) // bs) for L in lens)) * 4
        parts = int(sum(-(-int(L) // pt_eff) for L in lens if L > pt_eff))
        append = 2 * B * hkv * d * (qsz + esz) + B * 4
        return kv_bytes(lens) + tab + B * hq * d * qsz + B * hq * d * 4 + 2 * parts * hq * (d + 2) * 4 + append

    launches_per = []

    def step(i, ev=None):
        st = staged[i % STAGED_STEPS]
        n = 0
        if st["ncow"]:
            P.pkv_copy_blocks(cache.k_pool, cache.v_pool, st["cow"])
            n += 1
        if ev is not None:
            ev[0].record()
        # the append and the decode of the step in one call (the new rows are
        # written by the launch that plans the decode)
        if fp8:
            P.pkv_append_and_decode_fp8(st["kn"], st["vn"], st["slots"], st["q"], cache.k_pool, cache.v_pool,
                                        st["tables"], st["lens"], w.scale, w.kv_scale, w.kv_scale, out=out,
                                        workspace=workspace, partition_tokens=w.partition_tokens)
        else:
            st["call"]()
        if ev is not None:
            ev[1].record()
        return n + decode_launches(cache.max_blocks, bs, w.partition_tokens)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert P.pkv_device_status(clear=True) == 0

    K = args.steps
    # roofline timing of the call (see EVENT_EVERY): the call is the whole
    # step unless the step also copies blocks for copy-on-write
    cow_in_steps = any(staged[(args.warmup + i) % STAGED_STEPS]["ncow"] for i in range(K))
    sampled = sampled_steps(K) if cow_in_steps else []
    evs = {i: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for i in sampled}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    after_first = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, not args.no_clocks)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.begin()
    prequeue()
    start.record()
    launches = 0
    for i in range(K):
        launches += step(args.warmup + i, evs.get(i))
        if i == 0:
            after_first.record()
    end.record()
    clocks.sample()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = start.elapsed_time(end)
    if sampled:
        dec_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in sampled]
        launch_timing = f"event pairs around the call on timed steps {sampled[:3]}... ({len(sampled)} samples)"
    elif K > 1:
        dec_ms = [after_first.elapsed_time(end) / (K - 1)]
        sampled = list(range(1, K))
        launch_timing = f"one event pair around timed steps 2..{K} (the call is the whole step)"
    else:
        dec_ms = [elapsed_ms]
        sampled = [0]
        launch_timing = "the single timed step"
    status = P.pkv_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    step_kv = [kv_bytes(staged[(args.warmup + i) % STAGED_STEPS]["lens_host"]) for i in range(K)]
    step_algo = [algo_bytes(staged[(args.warmup + i) % STAGED_STEPS]["lens_host"]) for i in sampled]
    my_bytes = float(sum(step_kv))
    elapsed_all, bytes_all, tokens_all = combine_ranks(elapsed_ms, my_bytes, float(B * K), dev)
    value = bytes_all / (elapsed_all * 1e-3) / 1e9
    tok_s = tokens_all / (elapsed_all * 1e-3)

    peak, peak_kind = measured_peaks()
    dec_avg_ms = float(np.mean(dec_ms))
    # the call cannot outlast the step it is part of (a check on the timing itself)
    assert dec_avg_ms <= elapsed_ms / K * 1.02, (dec_avg_ms, elapsed_ms / K)
    achieved = float(np.mean(step_algo)) / (dec_avg_ms * 1e-3) / 1e9
    sha = kernel_source_sha()
    pin = TRAFFIC.get(w.name)
    traffic = pin[0] if (pin is not None and sha == pin[1]) else None

    # ---- end to end through the public API, host buffers in and out ----
    e2e = None
    if args.e2e_steps > 0:
        E = args.e2e_steps
        host_in = []
        for s in range(min(E, STAGED_STEPS)):
            host_in.append(tuple(W.normal(shape, w.io_dtype, W.step_seed(w, 100 + s, k)).pin_memory()
                                 for k, shape in ((0, (B, hq, d)), (1, (B, hkv, d)), (2, (B, hkv, d)))))
        out_host = torch.empty((B, hq, d), dtype=torch.float32, pin_memory=True)
        ids_np = np.arange(B, dtype=np.int64)
        for s in range(3):  # warm-up
            qh, kh, vh = host_in[s % len(host_in)]
            cache.decode_step_host(ids_np, qh, kh, vh, w.scale, out_host=out_host,
                                   partition_tokens=w.partition_tokens)
        torch.cuda.synchronize()
        # lengths after the warm-up: each timed step adds one token per sequence
        base_tokens = sum(cache.alloc.seq_len(i) for i in range(B))
        meta_bytes = int(P.lib().pkv_step_meta_bytes(B, cache.max_blocks))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record()
        h0 = time.perf_counter()
        for s in range(E):
            qh, kh, vh = host_in[s % len(host_in)]
            cache.decode_step_host(ids_np, qh, kh, vh, w.scale, out_host=out_host,
                                   partition_tokens=w.partition_tokens)
        host_ms = (time.perf_counter() - h0) * 1e3
        cache.wait_copies()  # the last step's result copy back is inside the timed region
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e_bytes = sum((base_tokens + B * (s + 1)) * hkv * d * 2 * esz for s in range(E))
        e2e_ms_all, e2e_bytes_all, _ = combine_ranks(e2e_ms, float(e_bytes), float(B * E), dev)
        h2d = (B * hq * d + 2 * B * hkv * d) * qsz + meta_bytes
        e2e = {"value": round(e2e_bytes_all / (e2e_ms_all * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(B * hq * d * 4),
               "ms_per_step": round(e2e_ms_all / E, 4),
               "host_issue_ms_per_step": round(host_ms / E, 4),
               "tokens_per_s_per_layer": round(ws * B * E / (e2e_ms_all * 1e-3), 1),
               "includes": "one pkv_decode_step_host call per step: host slot reservation, pinned H2D of q/K/V rows and "
                           "metadata, kernels, D2H of out"}

    st_a = cache.stats()
    alloc_stats = {"used_blocks": st_a["used_blocks"], "free_blocks": st_a["free_blocks"],
                   "logical_tokens": st_a["logical_tokens"], "waste_tokens": st_a["waste_tokens"],
                   "waste_frac": round(st_a["waste_tokens"] / max(1, st_a["used_blocks"] * bs), 5)}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rng = np.random.default_rng(7)
        order = [(int(b), int(g)) for b in rng.permutation(B) for g in range(hkv)]
        st = staged[(args.warmup + K - 1) % STAGED_STEPS]
        units = make_units(w, cache.k_pool, cache.v_pool, st["tables"].cpu().numpy(), st["lens_host"], st["q"],
                           order, count=min(len(order), 64))
        cycle = (units[i % len(units)] for i in range(10 ** 9))  # repeat the sample until the budget is spent
        nbytes, secs, done = time_oracle(cycle, args.cpu_seconds)
        cpu = {"value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": oracle_threads(),
               "kind": "oracle", "host_cpus": os.cpu_count(),
               "sample": f"{done} (sequence, KV head) units drawn from the same batch (64 distinct, cycled), "
                         f"fp64 numpy oracle, {secs:.1f} s"}

    if rank == 0:
        res = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(elapsed_all / K, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "tokens_per_s_per_layer": round(tok_s, 1),
            "hbm_fraction": round(value / peak, 4),
            "config": {"workload": w.name, "num_seqs": B, "num_q_heads": hq, "num_kv_heads": hkv,
                       "head_dim": d, "block_size": bs, "seq_lens": SEQ_LEN_RECIPES.get(w.name.split("_bs")[0], ""),
                       "mean_seq_len": round(float(np.mean(staged[0]["lens_host"])), 1),
                       "partition_tokens": w.partition_tokens or 512, "pool_blocks": cache.num_blocks,
                       "kv_bytes_per_step": int(np.mean(step_kv)),
                       "l2": "inputs larger than L2: %.0f MB of K/V read per step vs 126 MB L2, no flush"
                             % (np.mean(step_kv) / 1e6),
                       "parallelism": f"replicas x{ws} (independent batches per GPU)"},
            "roofline": {"kernel": "pkv_append_and_decode (append + plan, decode and partition-merge kernels)",
                         "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                         "traffic": traffic, "algorithmic_bytes_per_launch": int(np.mean(step_algo)),
                         "avg_launch_ms": round(dec_avg_ms, 5), "launch_samples": len(sampled),
                         "launch_timing": launch_timing, "kernel_source_sha": sha},
            "gpu_launches": launches, "clocks": clk, "cpu_baseline": cpu, "e2e": e2e,
            "allocator": alloc_stats,
        }
        print(json.dumps(res), flush=True)
    if ws > 1:
        dist.destroy_process_group()


PREFILL_METRIC = "paged prefill attention: TFLOP/s (fraction of B200 dense bf16 peak), prompt tokens/s per layer"


def prefill_flops(ctx, n: int, hq: int, d: int) -> int:
    """Algorithmic FLOPs of causal attention for chunks of n rows behind ctx
    cached tokens: q·Kᵀ and P·V, 2·d each per visible (row, key) pair."""
    keys = sum(int(c) * n + n * (n + 1) // 2 for c in ctx)
    return 4 * d * hq * keys


def time_prefill_oracle(units, budget_s: float):
    """Runs the prefill oracle on (q rows, K, V, table, L, n, scale, dtype)
    units until the budget is spent; returns (FLOPs, seconds, units done)."""
    from oracle import paged_attention as pa
    done, flops, t0 = 0, 0, time.perf_counter()
    for q, kb, vb, L, n, scale, dtype, fl in units:
        table = np.arange(kb.shape[0], dtype=np.int32)[None]
        pa.paged_prefill_attention(q, kb, vb, table, np.array([L]), np.array([n]), scale, dtype)
        done += 1
        flops += fl
        if time.perf_counter() - t0 > budget_s:
            break
    return flops, time.perf_counter() - t0, done


def run_prefill(args, w0):
    """A step is one chunked-prefill pass over the batch: the chunk's K/V
    rows appended through their slots, then causal paged prefill attention
    of the chunk's query rows over the pool."""
    import torch.distributed as dist
    import paged_kv_cache_406_b200 as P
    from paged_kv_cache_406_b200 import workloads as W
    from paged_kv_cache_406_b200.cache import PagedKVCache

    ws, rank, local = dist_env()
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = rank_workload(w0, rank)
    B, hq, hkv, d, bs, n = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.chunk_tokens
    ctx = W.seq_lens(w)
    L = ctx + n
    nb = W.pool_blocks(w, L)
    shape = (nb, hkv, bs, d)
    maxb = -(-int(L.max()) // bs)
    cache = PagedKVCache(nb, hkv, d, bs, w.torch_dtype, maxb, device=dev, free_order=W.free_order(nb, w.seed),
                         k_pool=W.pool_values(shape, w, 0, device=dev), v_pool=W.pool_values(shape, w, 1, device=dev))
    ids = list(range(B))
    for b in ids:
        cache.add(b, int(ctx[b]))
    # the chunk's slots (host allocator), row r of sequence b at q row b·n + r
    slots = np.stack([cache.alloc.append_slots(ids)[0].copy() for _ in range(n)], axis=1).reshape(-1)
    tables, lens = cache.alloc.block_tables(ids, maxb)
    slot_d = torch.from_numpy(slots.astype(np.int32)).to(dev)
    tables_d, lens_d = torch.from_numpy(tables.copy()).to(dev), torch.from_numpy(lens.copy()).to(dev)
    q_start = torch.arange(0, B * n + 1, n, dtype=torch.int32, device=dev)
    T = B * n
    q = W.normal((T, hq, d), w.torch_dtype, W.step_seed(w, 0, 0), device=dev)
    kn = W.normal((T, hkv, d), w.torch_dtype, W.step_seed(w, 0, 1), device=dev)
    vn = W.normal((T, hkv, d), w.torch_dtype, W.step_seed(w, 0, 2), device=dev)
    out = torch.empty((T, hq, d), dtype=torch.float32, device=dev)
    # bf16 pools: V of the batch staged as f16 once per call (one f16 P·V pass)
    pf_ws = torch.empty(max(1, P.pkv_prefill_workspace_size(B, hkv, d, maxb, bs, w.torch_dtype)), dtype=torch.uint8,
                        device=dev)
    staged = w.torch_dtype == torch.bfloat16

    def step(ev=None):
        P.pkv_kv_append(kn, vn, slot_d, cache.k_pool, cache.v_pool)
        if ev is not None:
            ev[0].record()
        P.pkv_paged_attention_prefill(q, cache.k_pool, cache.v_pool, tables_d, lens_d, q_start, n, w.scale, out=out,
                                      workspace=pf_ws)
        if ev is not None:
            ev[1].record()
        return 4 if staged else 2  # append, V staging and the two prefill instances (one returns at once)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert P.pkv_device_status(clear=True) == 0
    K = args.steps
    evs = {i: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for i in sampled_steps(K)}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, not args.no_clocks)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.begin()
    prequeue()
    start.record()
    launches = 0
    for i in range(K):
        launches += step(evs.get(i))
    end.record()
    clocks.sample()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    status = P.pkv_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    elapsed_ms = start.elapsed_time(end)
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b in evs.values()]))
    flops = prefill_flops(ctx, n, hq, d)
    elapsed_all, flops_all, tokens_all = combine_ranks(elapsed_ms, float(flops) * K, float(T * K), dev)
    value = flops_all / (elapsed_all * 1e-3) / 1e12
    peaks = measured_peak_file()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_BF16_SUSTAINED))
    peak_kind = "measured bf16_tflops_sustained" if "bf16_tflops_sustained" in peaks else "fallback sustained"
    achieved = flops / (attn_ms * 1e-3) / 1e12
    pf_sha = kernel_source_sha(PREFILL_SOURCES)
    pin = TRAFFIC_PREFILL.get(w.name)
    traffic = pin[0] if (pin is not None and pf_sha == pin[1]) else None

    # ---- end to end: host q / K / V rows and metadata in, out back to host ----
    e2e = None
    if args.e2e_steps > 0:
        E = args.e2e_steps
        hq_in, hk_in, hv_in = (t.cpu().pin_memory() for t in (q, kn, vn))
        meta_h = torch.from_numpy(np.concatenate([slots.astype(np.int32), tables.reshape(-1), lens,
                                                  np.arange(0, T + 1, n, dtype=np.int32)])).pin_memory()
        meta_d = torch.empty_like(meta_h, device=dev)
        out_h = torch.empty((T, hq, d), dtype=torch.float32, pin_memory=True)
        qd, kd, vd = torch.empty_like(q), torch.empty_like(kn), torch.empty_like(vn)
        ns, nt = slots.size, tables.size

        def e2e_step():
            meta_d.copy_(meta_h, non_blocking=True)
            qd.copy_(hq_in, non_blocking=True)
            kd.copy_(hk_in, non_blocking=True)
            vd.copy_(hv_in, non_blocking=True)
            P.pkv_kv_append(kd, vd, meta_d[:ns], cache.k_pool, cache.v_pool)
            P.pkv_paged_attention_prefill(qd, cache.k_pool, cache.v_pool, meta_d[ns:ns + nt].view(B, maxb),
                                          meta_d[ns + nt:ns + nt + B], meta_d[ns + nt + B:], n, w.scale, out=out,
                                          workspace=pf_ws)
            out_h.copy_(out, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(E):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e2e_all, e2e_flops, _ = combine_ranks(e2e_ms, float(flops) * E, float(T * E), dev)
        e2e = {"value": round(e2e_flops / (e2e_all * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int((q.numel() + kn.numel() + vn.numel()) * q.element_size() + meta_h.numel() * 4),
               "d2h_bytes_per_step": int(out.numel() * 4), "ms_per_step": round(e2e_all / E, 4),
               "tokens_per_s_per_layer": round(ws * T * E / (e2e_all * 1e-3), 1),
               "includes": "pinned H2D of the chunk's q/K/V rows and metadata, append, prefill, D2H of out"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rng = np.random.default_rng(7)
        G = w.group
        units = []
        for b in rng.permutation(B)[:4]:
            g = int(rng.integers(hkv))
            nblk = -(-int(L[b]) // bs)
            idx = torch.as_tensor(tables[b, :nblk], device=dev, dtype=torch.long)
            kb, vb = _raw(cache.k_pool[idx, g:g + 1]), _raw(cache.v_pool[idx, g:g + 1])
            rows = 4  # the chunk's last rows: the most keys per row
            qb = _raw(q[b * n + n - rows:b * n + n, g * G:(g + 1) * G])
            fl = 4 * d * G * sum(int(L[b]) - rows + 1 + r for r in range(rows))
            units.append((qb, kb, vb, int(L[b]), rows, w.scale, w.dtype, fl))
        cycle = (units[i % len(units)] for i in range(10 ** 9))
        fl, secs, done = time_prefill_oracle(cycle, args.cpu_seconds)
        cpu = {"value": round(fl / secs / 1e12, 6), "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
               "host_cpus": os.cpu_count(),
               "sample": f"{done} units of 4 query rows x {G} heads (one KV head, full causal context) from the same "
                         f"batch, 4 distinct, cycled; fp64 numpy oracle, {secs:.1f} s"}

    if rank == 0:
        res = {
            "metric": PREFILL_METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ws, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(elapsed_all / K, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "tokens_per_s_per_layer": round(tokens_all / (elapsed_all * 1e-3), 1),
            "config": {"workload": w.name, "num_seqs": B, "num_q_heads": hq, "num_kv_heads": hkv, "head_dim": d,
                       "block_size": bs, "chunk_tokens": n,
                       "cached_context": "U[0,3584]" if int(ctx.max()) else "0 (whole prompts)",
                       "flops_per_step": flops,
                       "l2": "inputs larger than L2: %.0f MB of K/V + %.0f MB of q and out per step, no flush"
                             % (int(L.sum()) * hkv * d * 4 / 1e6, T * hq * d * 6 / 1e6),
                       "parallelism": f"replicas x{ws} (independent batches per GPU)"},
            "roofline": {"kernel": "pkv_paged_attention_prefill (stage_v_f16_kernel and prefill_tc_kernel for bf16 pools)",
                         "bound": "tensor",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                         "burst_peak": peaks.get("bf16_tflops"),
                         "traffic": traffic, "traffic_unit": "bytes (DRAM read + write per launch)",
                         "algorithmic_flops_per_launch": flops,
                         "tensor_flops_issued_per_launch": "algorithmic plus the masked part of diagonal chunks "
                                                          "(one f16 P·V pass; bf16 V staged as f16 by the call)",
                         "avg_launch_ms": round(attn_ms, 5), "launch_samples": len(evs),
                         "kernel_source_sha": pf_sha},
            "gpu_launches": launches, "clocks": clk, "cpu_baseline": cpu, "e2e": e2e,
        }
        print(json.dumps(res), flush=True)
    if ws > 1:
        dist.destroy_process_group()


def run_adaptive(args, w):
    """Adaptive block size (optimisation-overview page §3.3) against single
    pools of 16-, 32- and 8-token blocks on the same batch: a step appends one
    token per sequence and runs paged decode attention; the adaptive arm does
    that once per block-size class (32 / 16 / 8)."""
    import paged_kv_cache_406_b200 as P
    from paged_kv_cache_406_b200 import workloads as W
    from paged_kv_cache_406_b200.cache import AdaptivePagedKVCache, PagedKVCache, block_size_for

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = rank_workload(w, rank)
    B, hq, hkv, d = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim
    lens0 = W.seq_lens(w)
    horizon = STAGED_STEPS + 8
    maxtok = int(lens0.max()) + horizon
    per_class = {}
    for L in lens0:
        bs = block_size_for(int(L))
        per_class[bs] = per_class.get(bs, 0) + -(-(int(L) + horizon) // bs)
    per_class = {bs: int(np.ceil(1.2 * nb)) for bs, nb in per_class.items()}
    ad = AdaptivePagedKVCache(per_class, hkv, d, w.torch_dtype, maxtok, device=dev, seed=w.seed)
    fixed = {}
    for fbs in (16, 32, 8):  # one pool of a single block size for the whole batch
        nbf = int(np.ceil(1.2 * sum(-(-(int(L) + horizon) // fbs) for L in lens0)))
        fixed[fbs] = PagedKVCache(nbf, hkv, d, fbs, w.torch_dtype, -(-maxtok // fbs), device=dev,
                                  free_order=W.free_order(nbf, w.seed))
    for k, c in enumerate(list(ad.caches.values()) + list(fixed.values())):
        c.k_pool.copy_(W.normal(c.k_pool.shape, w.torch_dtype, W.pool_seed(w, 0) + 17 * k, device=dev))
        c.v_pool.copy_(W.normal(c.v_pool.shape, w.torch_dtype, W.pool_seed(w, 1) + 17 * k, device=dev))
    for i, L in enumerate(lens0):
        ad.add(i, int(L))
        for c in fixed.values():
            c.add(i, int(L))
    ids = ad.order()
    e = torch.tensor([], dtype=w.torch_dtype).element_size()
    q = W.normal((B, hq, d), w.torch_dtype, W.step_seed(w, 0, 0), device=dev)
    kn = W.normal((B, hkv, d), w.torch_dtype, W.step_seed(w, 0, 1), device=dev)
    vn = W.normal((B, hkv, d), w.torch_dtype, W.step_seed(w, 0, 2), device=dev)

    def stage(cache, members):
        out = []
        for _ in range(STAGED_STEPS):
            slots, _ = cache.alloc.append_slots(members)
            tables, lens = cache.alloc.block_tables(members, cache.max_blocks)
            out.append((torch.from_numpy(slots.copy()).to(dev), torch.from_numpy(tables.copy()).to(dev),
                        torch.from_numpy(lens.copy()).to(dev), lens.copy()))
        wsb = P.pkv_decode_workspace_size(len(members), hq, hkv, d, cache.max_blocks, cache.block_size, 0)
        return out, torch.empty(wsb, dtype=torch.uint8, device=dev)

    # "adaptive": every class in one pkv_append_and_decode_pools call per step;
    # "adaptive_per_class": one pkv_append_and_decode call per class (same
    # staged metadata); "fixed_bsN": one pool of N-token blocks for the batch
    arms = {"adaptive": [], "adaptive_per_class": [], "fixed_bs16": [], "fixed_bs32": [], "fixed_bs8": []}
    a = 0
    for bs in ad.CLASSES:
        members = [i for i in ids if ad.cls[i] == bs]
        if members:
            st, wsp = stage(ad.caches[bs], members)
            arms["adaptive_per_class"].append((ad.caches[bs], st, wsp, slice(a, a + len(members))))
            a += len(members)
    for fbs, c in fixed.items():
        st, wsp = stage(c, ids)
        arms[f"fixed_bs{fbs}"].append((c, st, wsp, slice(0, B)))
    per_class = arms["adaptive_per_class"]
    one_call = []
    for k in range(STAGED_STEPS):
        pools = [(c.k_pool, c.v_pool, st[k][1], sl.stop - sl.start) for c, st, _, sl in per_class]
        one_call.append((pools, torch.cat([st[k][0] for _, st, _, _ in per_class]),
                         torch.cat([st[k][2] for _, st, _, _ in per_class])))
    pools_ws = torch.empty(P.pkv_decode_pools_workspace_size(one_call[0][0], hq), dtype=torch.uint8, device=dev)
    arms["adaptive"] = [(c, st, None, sl) for c, st, _, sl in per_class]  # for the byte and block accounting
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)

    def step(arm, i):
        if arm == "adaptive":
            pools, slots, lens = one_call[i % STAGED_STEPS]
            P.pkv_append_and_decode_pools(pools, kn, vn, slots, q, lens, w.scale, out=out, workspace=pools_ws)
            return decode_launches(max(c.max_blocks * c.block_size for c, _, _, _ in per_class) // 16, 16, 0)
        for cache, st, wsp, sl in arms[arm]:
            slots, tables, lens, _ = st[i % STAGED_STEPS]
            P.pkv_append_and_decode(kn[sl], vn[sl], slots, q[sl], cache.k_pool, cache.v_pool, tables, lens, w.scale,
                                    out=out[sl], workspace=wsp)
        return sum(decode_launches(c.max_blocks, c.block_size, 0) for c, _, _, _ in arms[arm])

    res_arms = {}
    clocks = ClockSampler(local, not args.no_clocks)
    launches = 0
    for arm in arms:
        for i in range(args.warmup):
            step(arm, i)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks.begin()
        prequeue()
        s0.record()
        for i in range(args.steps):
            launches += step(arm, args.warmup + i)
        s1.record()
        clocks.sample()
        torch.cuda.synchronize()
        ms = s0.elapsed_time(s1)
        nbytes = sum(int(st[(args.warmup + i) % STAGED_STEPS][3].astype(np.int64).sum()) * hkv * d * 2 * e
                     for i in range(args.steps) for _, st, _, _ in arms[arm])
        res_arms[arm] = {"kv_gb_s": round(nbytes / (ms * 1e-3) / 1e9, 1), "ms_per_step": round(ms / args.steps, 5),
                         "tokens_per_s_per_layer": round(B * args.steps / (ms * 1e-3), 1),
                         "calls_per_step": 1 if arm == "adaptive" else len(arms[arm]),
                         "pool_blocks": {str(c.block_size): c.num_blocks for c, _, _, _ in arms[arm]},
                         "waste_tokens": sum(c.stats()["waste_tokens"] for c, _, _, _ in arms[arm])}
    clk = clocks.stop()
    assert P.pkv_device_status(clear=True) == 0
    peak, peak_kind = measured_peaks()
    r = res_arms["adaptive"]
    if rank == 0:
        res = {"metric": METRIC, "value": r["kv_gb_s"], "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
               "tokens_per_s_per_layer": r["tokens_per_s_per_layer"], "hbm_fraction": round(r["kv_gb_s"] / peak, 4),
               "config": {"workload": w.name, "num_seqs": B, "num_q_heads": hq, "num_kv_heads": hkv, "head_dim": d,
                          "block_size": "adaptive: 32 below 1024 tokens, 16 below 8192, 8 above",
                          "seq_lens": "80% U[128,1023], 19% U[1024,8191], 1 U[8192,16384]",
                          "class_sizes": {str(bs): sum(1 for i in ids if ad.cls[i] == bs) for bs in ad.CLASSES},
                          "l2": "no flush; K/V per step %.0f MB" % (sum(int(L) for L in lens0) * hkv * d * 2 * e / 1e6),
                          "parallelism": f"replicas x{ws}"},
               "arms": res_arms, "peak": peak, "peak_source": f"{peak_kind} hbm_gbs",
               "gpu_launches": launches, "clocks": clk, "cpu_baseline": None, "e2e": None}
        print(json.dumps(res), flush=True)


def run_prefix_cache(args, w):
    """Hash-based prefix caching in the host allocator (vLLM paging page §3
    phase 3; production page §5: reuse saves memory, hashing costs CPU time).
    Admits the workload's requests three ways - plain pkv_seq_add, and
    pkv_seq_add_cached with shared system prompts and with all-distinct
    prompts - and reports host time per admission, reuse and blocks held."""
    import paged_kv_cache_406_b200 as P
    from paged_kv_cache_406_b200 import workloads as W
    rng = np.random.default_rng(w.seed)
    suffix = W.seq_lens(w)
    systems = [rng.integers(0, 32000, size=w.prefix_tokens, dtype=np.int32) for _ in range(4)]
    prompts = [np.concatenate([systems[i % 4], rng.integers(0, 32000, size=int(suffix[i]), dtype=np.int32)])
               for i in range(w.num_seqs)]
    distinct = [rng.integers(0, 32000, size=len(p), dtype=np.int32) for p in prompts]
    bs = w.block_size
    nb = sum(-(-len(p) // bs) for p in prompts) + 16
    reps = max(1, min(args.steps, 50))

    def arm(kind, data):
        times, stats = [], None
        for _ in range(reps):
            a = P.Allocator(nb, bs, W.free_order(nb, w.seed))
            t0 = time.perf_counter()
            if kind == "add":
                for i, p in enumerate(data):
                    a.add(i, len(p))
            else:
                for i, p in enumerate(data):
                    a.add_cached(i, p)
            times.append(time.perf_counter() - t0)
            stats = a.stats()
        us = float(np.median(times)) / len(data) * 1e6
        return {"us_per_admission": round(us, 3), "used_blocks": stats["used_blocks"],
                "cache_hits": stats["cache_hits"], "cache_queries": stats["cache_queries"],
                "hit_rate": round(stats["cache_hits"] / max(1, stats["cache_queries"]), 4)}

    res_arms = {"plain_add": arm("add", prompts), "cached_shared_prompts": arm("cached", prompts),
                "cached_distinct_prompts": arm("cached", distinct)}
    c, plain = res_arms["cached_shared_prompts"], res_arms["plain_add"]
    res = {"metric": "prefix caching: host admission time per sequence, KV blocks held", "value": c["us_per_admission"],
           "unit": "us/sequence", "n_gpus": 0, "steps": reps, "warmup": 0, "ms_per_step": None,
           "higher_is_better": False, "scaling": None, "vs_baseline": None, "dtype": "int32 token ids",
           "data": "synthetic",
           "config": {"workload": w.name, "requests": w.num_seqs, "system_prompts": 4,
                      "system_prompt_tokens": w.prefix_tokens, "suffix_tokens": "U[16,512]", "block_size": bs,
                      "timing": "median over repetitions of admitting every request into a fresh allocator, "
                                "through the Python binding (one ctypes call per request)"},
           "blocks_saved": plain["used_blocks"] - c["used_blocks"],
           "blocks_saved_frac": round(1 - c["used_blocks"] / plain["used_blocks"], 4),
           "hashing_overhead_us": round(res_arms["cached_distinct_prompts"]["us_per_admission"] -
                                        plain["us_per_admission"], 3),
           "arms": res_arms, "gpu_launches": 0, "clocks": None, "cpu_baseline": None, "e2e": None,
           "device": "host only: the C++ allocator (no kernel on this path)"}
    print(json.dumps(res), flush=True)


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, on this arm's workload, each
    step a bounded sample of it (rank 0 only)."""
    ws, rank, local = dist_env()
    if rank != 0:
        return
    from paged_kv_cache_406_b200 import workloads as W
    w = workload_of(args)
    if w.chunk_tokens:
        return run_reference_prefill(args, w, ws)
    lens = W.seq_lens(w)
    rng = np.random.default_rng(w.seed)
    G, e = w.group, torch.tensor([], dtype=w.torch_dtype).element_size()
    # each step: one (sequence, KV head) unit, blocks drawn from the seeded pool values
    K, Wm = args.steps, args.warmup
    order = [(int(b), int(g)) for b in rng.permutation(w.num_seqs) for g in range(w.num_kv_heads)]
    cache = {}

    def unit(i):
        b, g = order[i % len(order)]
        if (b, g) not in cache:
            L = int(lens[b])
            nblk = -(-L // w.block_size)
            shp = (nblk, 1, w.block_size, w.head_dim)
            kb = _raw(W.normal(shp, w.torch_dtype, W.pool_seed(w, 0) + 7919 * b + g))
            vb = _raw(W.normal(shp, w.torch_dtype, W.pool_seed(w, 1) + 7919 * b + g))
            qb = _raw(W.normal((1, G, w.head_dim), w.torch_dtype, W.step_seed(w, 0, 0) + b))
            cache[(b, g)] = (qb, kb, vb, L, w.scale, w.dtype, L * w.head_dim * 2 * e)
        return cache[(b, g)]

    for i in range(Wm):
        time_oracle([unit(i)], 1e9)
    total_bytes, total_s = 0, 0.0
    for i in range(K):
        nb, s, _ = time_oracle([unit(Wm + i)], 1e9)
        total_bytes += nb
        total_s += s
    value = total_bytes / total_s / 1e9
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": ws,
           "steps": K, "warmup": Wm, "ms_per_step": round(total_s / K * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
                      "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size},
           "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "kind": "oracle", "cores": oracle_threads(),
                            "sample": "one (sequence, KV head) unit of the workload per step, fp64 numpy oracle"},
           "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def run_reference_prefill(args, w, ws):
    """Reference arm for a prefill workload: each step, the fp64 oracle on the
    last 4 chunk rows x G query heads of one (sequence, KV head) over its full
    causal context."""
    from paged_kv_cache_406_b200 import workloads as W
    L = W.seq_lens(w) + w.chunk_tokens
    rng = np.random.default_rng(w.seed)
    G, rows = w.group, 4
    order = [(int(b), int(rng.integers(w.num_kv_heads))) for b in rng.permutation(w.num_seqs)]
    cache = {}

    def unit(i):
        b, g = order[i % len(order)]
        if (b, g) not in cache:
            nblk = -(-int(L[b]) // w.block_size)
            shp = (nblk, 1, w.block_size, w.head_dim)
            kb = _raw(W.normal(shp, w.torch_dtype, W.pool_seed(w, 0) + 7919 * b + g))
            vb = _raw(W.normal(shp, w.torch_dtype, W.pool_seed(w, 1) + 7919 * b + g))
            qb = _raw(W.normal((rows, G, w.head_dim), w.torch_dtype, W.step_seed(w, 0, 0) + b))
            fl = 4 * w.head_dim * G * sum(int(L[b]) - rows + 1 + r for r in range(rows))
            cache[(b, g)] = (qb, kb, vb, int(L[b]), rows, w.scale, w.dtype, fl)
        return cache[(b, g)]

    K, Wm = args.steps, args.warmup
    for i in range(Wm):
        time_prefill_oracle([unit(i)], 1e9)
    total_fl, total_s = 0, 0.0
    for i in range(K):
        fl, s, _ = time_prefill_oracle([unit(Wm + i)], 1e9)
        total_fl += fl
        total_s += s
    value = total_fl / total_s / 1e12
    res = {"impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6), "unit": "TFLOP/s",
           "n_gpus": ws, "steps": K, "warmup": Wm, "ms_per_step": round(total_s / K * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
                      "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
                      "chunk_tokens": w.chunk_tokens},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "kind": "oracle", "cores": oracle_threads(),
                            "sample": f"{rows} chunk rows x {G} heads of one (sequence, KV head) per step, "
                                      "full causal context, fp64 numpy oracle"},
           "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "prefix_cache":
        from paged_kv_cache_406_b200 import workloads as W
        run_prefix_cache(args, W.WORKLOADS["prefix_cache"])
    else:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA GPU (B200); use --impl reference for the CPU oracle")
        w = workload_of(args)
        if w.chunk_tokens:
            run_prefill(args, w)
        elif w.name == "adaptive_mix":
            run_adaptive(args, w)
        else:
            run_ours(args)


if __name__ == "__main__":
    main()
