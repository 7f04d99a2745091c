"""Shared helpers for the GPU parity tests: seeded cases, raw views for the
oracle, the tolerance rule."""
from __future__ import annotations

import numpy as np
import torch

from oracle import paged_attention as pa
from oracle.block_allocator import BlockAllocatorModel

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
# max-abs tolerance relative to an output scale of 1 (fp32 output)
TOL = {"f32": 1e-5, "bf16": 2e-3, "f16": 2e-3}


def raw(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a tensor's storage in the oracle's raw form."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def dtype_name(t: torch.dtype) -> str:
    return {torch.float32: "f32", torch.bfloat16: "bf16", torch.float16: "f16"}[t]


def randn(shape, dtype: str, rng: np.random.Generator) -> torch.Tensor:
    return torch.from_numpy(rng.standard_normal(size=shape, dtype=np.float32)).to(DT[dtype])


def assert_close(gpu: torch.Tensor, ref: np.ndarray, dtype: str, what: str = "") -> float:
    g = gpu.detach().cpu().double().numpy()
    err = np.abs(g - ref)
    bound = TOL[dtype] * np.maximum(1.0, np.abs(ref))
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{what}: {len(bad)} elements out of tolerance, first {bad[:3].tolist()}, max err {err.max()}"
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    return float(err.max())


class Case:
    """A paged batch built by the oracle's allocator model: lengths, pools,
    tables and q; ``guard`` extra blocks stay unused."""

    def __init__(self, lens, hq, hkv, d, bs, dtype, seed, guard=4):
        rng = np.random.default_rng(seed)
        self.lens = np.asarray(lens, dtype=np.int64)
        self.B, self.hq, self.hkv, self.d, self.bs, self.dtype = len(lens), hq, hkv, d, bs, dtype
        need = int(sum(-(-int(L) // bs) for L in self.lens))
        self.nb = need + guard
        self.order = rng.permutation(self.nb).astype(np.int32)
        self.model = BlockAllocatorModel(self.nb, bs, self.order)
        for b, L in enumerate(self.lens):
            self.model.add(b, int(L))
        self.maxb = max(1, max(len(self.model.block_table(b)) for b in range(self.B)))
        self.tables = np.full((self.B, self.maxb), -1, dtype=np.int32)
        for b in range(self.B):
            t = self.model.block_table(b)
            self.tables[b, :len(t)] = t
        self.k_pool = randn((self.nb, hkv, bs, d), dtype, rng)
        self.v_pool = randn((self.nb, hkv, bs, d), dtype, rng)
        self.q = randn((self.B, hq, d), dtype, rng)
        self.scale = 1.0 / np.sqrt(d)

    def oracle(self, lens=None) -> np.ndarray:
        lens = self.lens if lens is None else lens
        return pa.paged_decode_attention(raw(self.q), raw(self.k_pool), raw(self.v_pool), self.tables, lens,
                                         self.scale, self.dtype)

    def device(self, dev="cuda"):
        return dict(q=self.q.to(dev), k_pool=self.k_pool.to(dev), v_pool=self.v_pool.to(dev),
                    block_tables=torch.from_numpy(self.tables).to(dev),
                    seq_lens=torch.from_numpy(self.lens.astype(np.int32)).to(dev))
