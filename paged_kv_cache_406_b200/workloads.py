"""Seeded synthetic workloads for the paged decode and prefill paths.

This module only draws inputs: sequence lengths, the order in which physical
blocks leave the free list, and N(0, 1) values for q / K / V.  It holds none
of the method's arithmetic, so the tests can feed the same inputs to the CUDA
library and to the CPU oracle.  Shapes follow Llama-3-8B-like (32 query / 8 KV
heads, head_dim 128) and 7B-MHA-like (32 / 32) decode layers with mixed
sequence lengths and shared prefixes.

Draws (each workload has its own seed):
  * lengths: numpy PCG64 generator seeded with ``seed``;
  * free-list order: a permutation from a PCG64 generator seeded ``seed + 1``;
  * values: N(0, 1) from a PCG64 generator (CPU, small cases) or from
    torch's CUDA generator (large cases, drawn directly on the device), cast
    to the workload dtype with round-to-nearest-even.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16, "e4m3": torch.float8_e4m3fn}


@dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str            # pool element type: "f32" | "bf16" | "f16" | "e4m3"
    seed: int
    steps: int = 1        # decode steps (one appended token per sequence each)
    partition_tokens: int = 0  # 0 = library default
    prefix_tokens: int = 0     # tokens shared by every sequence (refcount = num_seqs)
    pool_slack: float = 1.2    # pool size as a multiple of the blocks needed
    kv_scale: float = 1.0 / 32  # e4m3 pools: value = kv_scale * code value (K and V)
    chunk_tokens: int = 0      # prefill workloads: new query rows per sequence (0: a decode workload)

    @property
    def torch_dtype(self) -> torch.dtype:
        return TORCH_DTYPES[self.dtype]

    @property
    def io_dtype(self) -> torch.dtype:
        """Element type of q and of the new K/V rows (float16 for e4m3 pools)."""
        return torch.float16 if self.dtype == "e4m3" else TORCH_DTYPES[self.dtype]

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    # 4 sequences, lengths {1, 7, 16, 33} before the step's append, fp32, 16-block pool
    "tiny": Workload("tiny", 4, 4, 4, 64, 16, "f32", 406001, pool_slack=0.0),
    # Llama-3-8B-shaped layer: 64 sequences of U[512, 4096] tokens, GQA 32/8, bf16
    "llama3_8b": Workload("llama3_8b", 64, 32, 8, 128, 16, "bf16", 406002),
    # the same batch with an e4m3 KV cache (scale 1/32), q and new rows float16
    "llama3_8b_fp8": Workload("llama3_8b_fp8", 64, 32, 8, 128, 16, "e4m3", 406002),
    # 32 sequences sharing a 1024-token prefix plus U[64, 512]-token tails
    "prefix_shared_bs8": Workload("prefix_shared_bs8", 32, 32, 8, 128, 8, "bf16", 406003, prefix_tokens=1024),
    "prefix_shared_bs16": Workload("prefix_shared_bs16", 32, 32, 8, 128, 16, "bf16", 406003, prefix_tokens=1024),
    "prefix_shared_bs32": Workload("prefix_shared_bs32", 32, 32, 8, 128, 32, "bf16", 406003, prefix_tokens=1024),
    # long contexts split into 512-token partitions: 7 x 32768 + 1 x 131072 tokens
    "long_splitk": Workload("long_splitk", 8, 32, 8, 128, 16, "bf16", 406004, partition_tokens=512),
    # 7B MHA at high concurrency: 256 lognormal(median 1000, sigma 1) lengths in [16, 8192], 50 steps
    "mha_7b": Workload("mha_7b", 256, 32, 32, 128, 16, "f16", 406005, steps=50),
    # chunked prefill on the Llama-3-8B layer: 16 sequences, a 512-token chunk
    # each on top of U[0, 3584] cached tokens (so 512 .. 4096 tokens in all)
    "prefill_llama3_8b": Workload("prefill_llama3_8b", 16, 32, 8, 128, 16, "bf16", 406006, chunk_tokens=512),
    # the optimisation-overview page's traffic mix for adaptive block sizes:
    # 80 % of 64 sequences below 1024 tokens, the rest 1024..8191, one >= 8192
    "adaptive_mix": Workload("adaptive_mix", 64, 32, 8, 128, 16, "bf16", 406008),
    # prefix caching (host allocator): 256 requests, each one of 4 shared
    # 1024-token system prompts plus its own U[16, 512]-token suffix
    "prefix_cache": Workload("prefix_cache", 256, 32, 8, 128, 16, "bf16", 406009, prefix_tokens=1024),
    # whole 2048-token prompts from an empty cache, 8 sequences
    "prefill_prompt_2k": Workload("prefill_prompt_2k", 8, 32, 8, 128, 16, "bf16", 406007, chunk_tokens=2048),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields changed (smaller parity variants)."""
    return replace(w, **kw)


def seq_lens(w: Workload) -> np.ndarray:
    """Per-sequence token counts before the first decode step (int64).

    For prefix-shared workloads this is prefix + tail; for prefill workloads
    the context cached before the chunk of ``chunk_tokens`` new rows."""
    rng = np.random.Generator(np.random.PCG64(w.seed))
    n = w.num_seqs
    if w.name == "tiny":
        return np.array([1, 7, 16, 33], dtype=np.int64)[:n]
    if w.name.startswith("llama3_8b"):
        return rng.integers(512, 4096, size=n, endpoint=True).astype(np.int64)
    if w.name.startswith("prefix_shared"):
        return w.prefix_tokens + rng.integers(64, 512, size=n, endpoint=True).astype(np.int64)
    if w.name.startswith("long_splitk"):
        base = np.array([32768] * 7 + [131072], dtype=np.int64)
        return base[:n] if n <= 8 else np.resize(base, n)
    if w.name.startswith("adaptive_mix"):
        short = int(round(0.8 * n))
        long_ = max(0, n - short - 1)
        return np.concatenate([rng.integers(128, 1023, size=short, endpoint=True),
                               rng.integers(1024, 8191, size=long_, endpoint=True),
                               rng.integers(8192, 16384, size=n - short - long_, endpoint=True)]).astype(np.int64)
    if w.name == "prefix_cache":  # suffix lengths (the shared prompt comes on top)
        return rng.integers(16, 512, size=n, endpoint=True).astype(np.int64)
    if w.name.startswith("prefill_llama3_8b"):  # cached context before the chunk
        return rng.integers(0, 3584, size=n, endpoint=True).astype(np.int64)
    if w.name.startswith("prefill_prompt"):
        return np.zeros(n, dtype=np.int64)
    if w.name.startswith("mha_7b"):
        x = rng.lognormal(mean=math.log(1000.0), sigma=1.0, size=n)
        return np.clip(np.rint(x), 16, 8192).astype(np.int64)
    raise KeyError(w.name)


def pool_blocks(w: Workload, lens: np.ndarray) -> int:
    """Physical blocks in the pool: the blocks every sequence reaches by the
    last step (shared prefix counted once), times the slack factor; at least
    16 (the tiny workload's fixed 16-block pool when its slack is 0)."""
    bs = w.block_size
    if w.prefix_tokens:
        prefix_blocks = -(-w.prefix_tokens // bs)
        need = prefix_blocks + int(sum(-(-(int(L) + w.steps) // bs) - w.prefix_tokens // bs for L in lens))
    else:
        need = int(sum(-(-(int(L) + w.steps) // bs) for L in lens))
    return max(16, int(math.ceil(need * w.pool_slack)) if w.pool_slack else need)


def free_order(num_blocks: int, seed: int) -> np.ndarray:
    """A seeded permutation of the block ids: the order blocks leave the free list."""
    return np.random.Generator(np.random.PCG64(seed + 1)).permutation(num_blocks).astype(np.int32)


def normal(shape, dtype: torch.dtype, seed: int, device="cpu") -> torch.Tensor:
    """N(0, 1) values of ``shape`` in ``dtype``, seeded, on ``device``."""
    if torch.device(device).type == "cuda":
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        return torch.randn(shape, generator=g, device=device, dtype=dtype)
    x = np.random.Generator(np.random.PCG64(seed)).standard_normal(size=shape, dtype=np.float32)
    return torch.from_numpy(x).to(dtype)


def pool_values(shape, w: Workload, which: int, device="cpu") -> torch.Tensor:
    """Initial pool contents: N(0, 1) in the pool dtype; for e4m3 pools the
    codes of N(0, 1) / kv_scale (torch's float8 cast, round to nearest even)."""
    if w.dtype == "e4m3":
        x = normal(shape, torch.float32, pool_seed(w, which), device)
        return (x / w.kv_scale).to(torch.float8_e4m3fn)
    return normal(shape, w.torch_dtype, pool_seed(w, which), device)


def step_seed(w: Workload, step: int, what: int) -> int:
    """Seed for the per-step draws: what = 0 (q), 1 (new K), 2 (new V)."""
    return w.seed * 1000 + step * 10 + what + 7


def pool_seed(w: Workload, which: int) -> int:
    """Seed for the initial pool contents: which = 0 (K), 1 (V)."""
    return w.seed * 1000 + 900000 + which
