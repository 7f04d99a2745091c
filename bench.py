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
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: KV GB/s (fraction of B200 HBM peak), tokens/s per layer"
FALLBACK_HBM_GBS = 6650.0
STAGED_STEPS = 16  # distinct steps of metadata resident on the device, cycled

# DRAM traffic of one pkv_paged_attention_decode call on the default workload,
# from the ncu capture summarised in profiles/ (dram__bytes_read.sum +
# dram__bytes_write.sum over its kernels).  Valid only while the kernel
# sources hash to TRAFFIC_SOURCE_SHA; otherwise reported as null.
TRAFFIC_BYTES = 607263488  # plan + decode + merge kernels, mean of two captured calls
TRAFFIC_SOURCE_SHA = "62c7be410db53362"


SEQ_LEN_RECIPES = {
    "tiny": "{1,7,16,33} before the step's append",
    "llama3_8b": "U[512,4096]",
    "llama3_8b_fp8": "U[512,4096]; e4m3 K/V (scale 1/32), q and new rows float16",
    "prefix_shared": "1024-token shared prefix (refcount = num_seqs) + U[64,512] tails; KV bytes are logical "
                     "(the prefix counted once per sequence)",
    "long_splitk": "7 x 32768 + 1 x 131072",
    "mha_7b": "lognormal(median 1000, sigma 1) clipped to [16, 8192]",
}


def kernel_source_sha() -> str:
    """Hash of the device sources (every .cu / .cuh file of the library)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_406_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
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
    return ap.parse_args()


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
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool):
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_gpu{gpu_index}.csv")
        if not enabled:
            return
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


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
    w0 = W.WORKLOADS[args.workload]
    if args.partition_tokens >= 0:
        from dataclasses import replace
        w0 = replace(w0, partition_tokens=args.partition_tokens)
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

    def kv_bytes(lens):
        return int(lens.astype(np.int64).sum()) * hkv * d * 2 * esz

    pt_eff = w.partition_tokens or 512

    def algo_bytes(lens):
        # K/V rows once per (sequence, KV head) + block-table entries + q + out,
        # + the split-partition partials (m, l, o per query head), written once and read once
        tab = int(sum(-(-int(L) // bs) for L in lens)) * 4
        parts = int(sum(-(-int(L) // pt_eff) for L in lens if L > pt_eff))
        return kv_bytes(lens) + tab + B * hq * d * qsz + B * hq * d * 4 + 2 * parts * hq * (d + 2) * 4

    launches_per = []

    def step(i, ev=None):
        st = staged[i % STAGED_STEPS]
        n = 0
        if st["ncow"]:
            P.pkv_copy_blocks(cache.k_pool, cache.v_pool, st["cow"])
            n += 1
        if fp8:
            P.pkv_kv_append_fp8(st["kn"], st["vn"], st["slots"], cache.k_pool, cache.v_pool, w.kv_scale, w.kv_scale)
        else:
            P.pkv_kv_append(st["kn"], st["vn"], st["slots"], cache.k_pool, cache.v_pool)
        n += 1
        if ev is not None:
            ev[0].record()
        if fp8:
            P.pkv_paged_attention_decode_fp8(st["q"], cache.k_pool, cache.v_pool, st["tables"], st["lens"], w.scale,
                                             w.kv_scale, w.kv_scale, out=out, workspace=workspace,
                                             partition_tokens=w.partition_tokens)
        else:
            P.pkv_paged_attention_decode(st["q"], cache.k_pool, cache.v_pool, st["tables"], st["lens"], w.scale,
                                         out=out, workspace=workspace, partition_tokens=w.partition_tokens)
        if ev is not None:
            ev[1].record()
        n += 2  # plan + decode (partition merge runs inside the decode kernel)
        return n

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert P.pkv_device_status(clear=True) == 0

    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, not args.no_clocks)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    launches = 0
    for i in range(K):
        launches += step(args.warmup + i, evs[i])
    end.record()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = start.elapsed_time(end)
    dec_ms = [a.elapsed_time(b) for a, b in evs]
    status = P.pkv_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    step_kv = [kv_bytes(staged[(args.warmup + i) % STAGED_STEPS]["lens_host"]) for i in range(K)]
    step_algo = [algo_bytes(staged[(args.warmup + i) % STAGED_STEPS]["lens_host"]) for i in range(K)]
    my_bytes = float(sum(step_kv))
    elapsed_all, bytes_all, tokens_all = combine_ranks(elapsed_ms, my_bytes, float(B * K), dev)
    value = bytes_all / (elapsed_all * 1e-3) / 1e9
    tok_s = tokens_all / (elapsed_all * 1e-3)

    peak, peak_kind = measured_peaks()
    dec_avg_ms = float(np.mean(dec_ms))
    achieved = float(np.mean(step_algo)) / (dec_avg_ms * 1e-3) / 1e9
    sha = kernel_source_sha()
    traffic = TRAFFIC_BYTES if (TRAFFIC_BYTES is not None and sha == TRAFFIC_SOURCE_SHA) else None

    # ---- end to end through the public API, host buffers in and out ----
    e2e = None
    if args.e2e_steps > 0:
        E = args.e2e_steps
        host_in = []
        for s in range(min(E, STAGED_STEPS)):
            host_in.append(tuple(W.normal(shape, w.io_dtype, W.step_seed(w, 100 + s, k)).pin_memory()
                                 for k, shape in ((0, (B, hq, d)), (1, (B, hkv, d)), (2, (B, hkv, d)))))
        out_host = torch.empty((B, hq, d), dtype=torch.float32, pin_memory=True)
        for s in range(3):  # warm-up
            qh, kh, vh = host_in[s % len(host_in)]
            o = cache.decode_step(ids, qh, kh, vh, w.scale, partition_tokens=w.partition_tokens)
            out_host.copy_(o, non_blocking=True)
        torch.cuda.synchronize()
        e_lens = []
        meta_bytes = 0
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record()
        for s in range(E):
            qh, kh, vh = host_in[s % len(host_in)]
            o = cache.decode_step(ids, qh, kh, vh, w.scale, partition_tokens=w.partition_tokens)
            out_host.copy_(o, non_blocking=True)
            e_lens.append(kv_bytes(cache._meta_np[B:2 * B]))
            meta_bytes += B * (4 + cache.max_blocks) * 4
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e2e_ms_all, e2e_bytes_all, _ = combine_ranks(e2e_ms, float(sum(e_lens)), float(B * E), dev)
        h2d = (B * hq * d + 2 * B * hkv * d) * qsz + meta_bytes // E
        e2e = {"value": round(e2e_bytes_all / (e2e_ms_all * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(B * hq * d * 4),
               "ms_per_step": round(e2e_ms_all / E, 4),
               "tokens_per_s_per_layer": round(ws * B * E / (e2e_ms_all * 1e-3), 1),
               "includes": "host slot reservation, pinned H2D of q/K/V rows and metadata, kernels, D2H of out"}

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
            "roofline": {"kernel": "pkv_paged_attention_decode (plan + decode + partition-merge kernels)",
                         "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                         "traffic": traffic, "algorithmic_bytes_per_launch": int(np.mean(step_algo)),
                         "avg_launch_ms": round(dec_avg_ms, 5), "kernel_source_sha": sha},
            "gpu_launches": launches, "clocks": clk, "cpu_baseline": cpu, "e2e": e2e,
            "allocator": alloc_stats,
        }
        print(json.dumps(res), flush=True)
    if ws > 1:
        dist.destroy_process_group()


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, on this arm's workload, each
    step a bounded sample of it (rank 0 only)."""
    ws, rank, local = dist_env()
    if rank != 0:
        return
    from paged_kv_cache_406_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
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


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA GPU (B200); use --impl reference for the CPU oracle")
        run_ours(args)


if __name__ == "__main__":
    main()
