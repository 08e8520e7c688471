"""Seeded synthetic inputs for paged decode attention.

This module draws random numbers and builds block tables; it holds none of the
method's arithmetic (no attention, no slot formula, no score, no quantiser), so
that both the CUDA path and the fp64 oracle can take their inputs from it.

Workloads (shapes and value distributions of the decode scenarios the pages
describe; all values bf16 ~ N(0, 1) unless stated):
  c1  tiny:     B=2, old lens 37/100 (+1 appended), Hq=4, Hkv=2, d=64, bs=16,
                pool of exactly 64 blocks handed out by a seeded permutation.
  c2  Llama-3.2-1B shape: 16 layers, Hq=32, Hkv=8, d=64, B=32, old len 1024
                (+1), bs=16, pool = 1.1 x blocks in use, shuffled.
  c3  Llama-3-8B shape: 32 layers, Hq=32, Hkv=8, d=128, B=64, old lens uniform
                in [512, 8192] (+1), bs=16, pool = 1.1 x in use, shuffled; per
                layer 1% of the Hkv*d channels (10 of the 1024 (head, channel)
                pairs, rounded) of K and V scaled x8 as outliers.
  c4  128K context: 1 layer, Hq=32, Hkv=8, d=128, B=4, len 131072 (no append),
                bs=256, one tensor [2, L, N, 256, Hkv, d] (nano-vLLM layout), shuffled.
  c5  INT8 pool: 1 layer, Hq=64, Hkv=8, d=128, B=128, old len 4096 (+1), bs=16;
                K/V history drawn bf16 and quantised by the INT8 append.
  p1  prefill compression: 32 prompts of 8192 tokens, Hkv=8, d=128, bs=16,
                budget 1024 tokens per prompt (the PagedEviction budget); prompt
                K/V rows [T, Hkv, d] bf16 N(0, 1) with 1% of the (head, channel)
                pairs scaled x8.
  p2  chunked prefill: 4 sequences, each appending and attending the last
                512-token chunk of an 8192-token prompt (Sarathi's chunk size),
                Hq=32, Hkv=8, d=128, bs=16, shuffled pool; values N(0, 1).
Seeds are 396 + the workload's index (0..6).

The allocator is the on-demand block pool of the vLLM notes (ybb.press "LLM 推理
KV Cache 内存管理深度工程实践" §2.1): a shuffled free list, each sequence taking
blocks from it while its table covers fewer slots than it has tokens.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Config:
    key: str
    name: str
    layers: int
    batch: int
    hq: int
    hkv: int
    head_dim: int
    block_size: int
    old_lens: tuple = ()            # explicit per-sequence old lengths, or
    old_len_range: tuple = ()       # (lo, hi) inclusive uniform range
    append: bool = True             # one new token appended per sequence per layer
    score: bool = False             # step includes the PagedEviction score + argmin
    int8: bool = False
    fp8: bool = False               # e4m3 pools (history cast by the FP8 append)
    outlier_frac: float = 0.0
    spare: float = 0.10
    nano_layout: bool = False       # K/V in one [2, L, N, bs, Hkv, d] tensor
    pool_blocks: Optional[int] = None
    seed: int = 396


CONFIGS = {
    "c1": Config("c1", "tiny paged decode", 1, 2, 4, 2, 64, 16, old_lens=(37, 100),
                 score=True, pool_blocks=64, seed=396),
    "c2": Config("c2", "Llama-3.2-1B-shape decode", 16, 32, 32, 8, 64, 16,
                 old_lens=(1024,) * 32, score=True, seed=397),
    "c3": Config("c3", "Llama-3-8B-shape decode", 32, 64, 32, 8, 128, 16,
                 old_len_range=(512, 8192), outlier_frac=0.01, seed=398),
    "c4": Config("c4", "long-context split-KV 128K", 1, 4, 32, 8, 128, 256,
                 old_lens=(131072,) * 4, append=False, nano_layout=True, seed=399),
    "c5": Config("c5", "INT8 paged KV", 1, 128, 64, 8, 128, 16, old_lens=(4096,) * 128,
                 int8=True, seed=400),
}


def scaled(cfg: Config, **kw) -> Config:
    """A copy of cfg with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(cfg, **kw)


@dataclass
class Workload:
    cfg: Config
    old_lens: np.ndarray            # [B] int32, tokens cached before the step
    ctx_lens: np.ndarray            # [B] int32, tokens attended (old + appended)
    positions: np.ndarray           # [B] int32, position of the appended token
    block_tables: np.ndarray        # [B, MB] int32, -1 = unused entry
    num_blocks: int                 # N physical blocks per layer pool
    # device (or host) tensors
    q: torch.Tensor                 # [L, B, Hq, d] bf16
    k_new: Optional[torch.Tensor]   # [L, B, 1, Hkv, d] bf16
    v_new: Optional[torch.Tensor]
    k_pool: Optional[torch.Tensor]  # [L, N, bs, Hkv, d] bf16 (view into kv for nano layout)
    v_pool: Optional[torch.Tensor]
    kv: Optional[torch.Tensor] = None          # [2, L, N, bs, Hkv, d] (nano layout)
    k_hist: Optional[torch.Tensor] = None      # INT8 workloads: [L, B, old, Hkv, d] bf16
    v_hist: Optional[torch.Tensor] = None
    outliers: list = field(default_factory=list)  # per layer: list of (head, channel)

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.cfg.head_dim)


def _old_lens(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    if cfg.old_lens:
        assert len(cfg.old_lens) == cfg.batch
        return np.asarray(cfg.old_lens, np.int32)
    lo, hi = cfg.old_len_range
    return rng.integers(lo, hi + 1, size=cfg.batch).astype(np.int32)


def _allocate(lens: np.ndarray, bs: int, spare: float, pool_blocks: Optional[int],
              rng: np.random.Generator):
    """On-demand allocator over a shuffled free list; returns (tables, N)."""
    tables = []
    for n_tok in lens:
        t = 0
        cnt = 0
        while t < n_tok:      # grow the table one block at a time
            t += bs
            cnt += 1
        tables.append(cnt)
    used = int(sum(tables))
    n = pool_blocks if pool_blocks is not None else int(math.ceil(used * (1.0 + spare)))
    if n < used:
        raise ValueError("pool smaller than the blocks in use")
    free = list(rng.permutation(n).astype(np.int64))
    mb = max(max(tables), 1)
    bt = np.full((len(lens), mb), -1, np.int32)
    for b, cnt in enumerate(tables):
        for j in range(cnt):
            bt[b, j] = free.pop(0) if pool_blocks is not None else free.pop()
    return bt, n


def generate(cfg: Config, device="cpu", layers: Optional[int] = None,
             seed: Optional[int] = None) -> Workload:
    """Draw one decode step's inputs for cfg on `device` (seeded).

    layers: draw only the first `layers` layers (parity tests); default all."""
    seed = cfg.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    L = cfg.layers if layers is None else layers
    B, Hq, Hkv, d, bs = cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size
    old = _old_lens(cfg, rng)
    ctx = old + (1 if cfg.append else 0)
    bt, N = _allocate(ctx, bs, cfg.spare, cfg.pool_blocks, rng)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = torch.bfloat16

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(bf)

    q = randn(L, B, Hq, d)
    k_new = v_new = None
    if cfg.append:
        k_new = randn(L, B, 1, Hkv, d)
        v_new = randn(L, B, 1, Hkv, d)
    kv = k_pool = v_pool = k_hist = v_hist = None
    outliers = []
    n_out = int(round(cfg.outlier_frac * Hkv * d))
    for layer in range(L):
        if n_out:
            ch = rng.choice(Hkv * d, size=n_out, replace=False)
            outliers.append([(int(c) // d, int(c) % d) for c in ch])
        else:
            outliers.append([])
    if cfg.int8 or cfg.fp8:
        # history drawn in bf16, quantised later by the INT8 / FP8 append
        k_hist = randn(L, B, int(old.max()), Hkv, d)
        v_hist = randn(L, B, int(old.max()), Hkv, d)
    else:
        if cfg.nano_layout:
            kv = torch.empty(2, L, N, bs, Hkv, d, dtype=bf, device=device)
            k_pool, v_pool = kv[0], kv[1]
        else:
            k_pool = torch.empty(L, N, bs, Hkv, d, dtype=bf, device=device)
            v_pool = torch.empty(L, N, bs, Hkv, d, dtype=bf, device=device)
        for layer in range(L):
            # one layer at a time keeps the fp32 staging buffer small
            k_pool[layer].copy_(randn(N, bs, Hkv, d))
            v_pool[layer].copy_(randn(N, bs, Hkv, d))
    for layer, pairs in enumerate(outliers):
        for h, c in pairs:
            for t in (k_pool, v_pool, k_new, v_new, k_hist, v_hist):
                if t is not None:
                    t[layer, ..., h, c] *= 8
    return Workload(cfg=cfg, old_lens=old, ctx_lens=ctx.astype(np.int32),
                    positions=old.astype(np.int32), block_tables=bt, num_blocks=N,
                    q=q, k_new=k_new, v_new=v_new, k_pool=k_pool, v_pool=v_pool, kv=kv,
                    k_hist=k_hist, v_hist=v_hist, outliers=outliers)


def bits(t: torch.Tensor) -> np.ndarray:
    """Host uint16 bit patterns of a bf16 tensor (any device)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def compact(wl: Workload, layer: int, seqs) -> dict:
    """Host copy of the pre-step state of the sequences `seqs` of one layer:
    only the physical blocks those sequences use, renumbered 0..n-1, with the
    matching block table.  Pure gathering (no method arithmetic)."""
    seqs = list(seqs)
    bt = wl.block_tables[seqs]
    ids = bt[bt >= 0]
    remap = {int(p): i for i, p in enumerate(ids)}
    new_bt = np.full_like(bt, -1)
    for r in range(bt.shape[0]):
        for j in range(bt.shape[1]):
            if bt[r, j] >= 0:
                new_bt[r, j] = remap[int(bt[r, j])]
    out = {
        "block_tables": new_bt,
        "num_blocks": len(ids),
        "ctx_lens": wl.ctx_lens[seqs].copy(),
        "old_lens": wl.old_lens[seqs].copy(),
        "positions": wl.positions[seqs].copy(),
        "q": bits(wl.q[layer, seqs]),
    }
    if wl.k_new is not None:
        out["k_new"] = bits(wl.k_new[layer, seqs])
        out["v_new"] = bits(wl.v_new[layer, seqs])
    if wl.k_pool is not None:
        idx = torch.as_tensor(ids, dtype=torch.long, device=wl.k_pool.device)
        out["k_pool"] = bits(wl.k_pool[layer].index_select(0, idx))
        out["v_pool"] = bits(wl.v_pool[layer].index_select(0, idx))
    if wl.k_hist is not None:
        out["k_hist"] = bits(wl.k_hist[layer, seqs])
        out["v_hist"] = bits(wl.v_hist[layer, seqs])
    return out


# ----------------------------------------------------------------------------- prefill stage
@dataclass(frozen=True)
class PrefillConfig:
    key: str
    name: str
    batch: int
    prompt_lens: tuple
    hkv: int
    head_dim: int
    block_size: int
    budget: int
    outlier_frac: float = 0.01
    spare: float = 0.10
    seed: int = 401


PREFILL = {
    "p1": PrefillConfig("p1", "PagedEviction prefill compression", 32, (8192,) * 32, 8, 128, 16,
                        1024),
}


@dataclass
class PrefillWorkload:
    cfg: PrefillConfig
    k: torch.Tensor                 # [T, Hkv, d] bf16, prompts concatenated
    v: torch.Tensor
    cu_seqlens: np.ndarray          # [B+1] int32
    block_tables: np.ndarray        # [B, MB] int32: ceil(min(len, budget)/bs) blocks each
    num_blocks: int


def generate_prefill(cfg: PrefillConfig, device="cpu") -> PrefillWorkload:
    """Seeded prompt rows and the block tables for the compressed prompts."""
    rng = np.random.default_rng(cfg.seed)
    lens = np.asarray(cfg.prompt_lens, np.int64)
    kept = np.minimum(lens, cfg.budget)
    bt, N = _allocate(np.maximum(kept, 1), cfg.block_size, cfg.spare, None, rng)
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    T, Hkv, d = int(lens.sum()), cfg.hkv, cfg.head_dim
    k = torch.empty(T, Hkv, d, dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    step = 1 << 16                  # draw in slices: bounded fp32 staging
    for t0 in range(0, T, step):
        n = min(step, T - t0)
        k[t0:t0 + n].copy_(torch.randn(n, Hkv, d, generator=g, device=device))
        v[t0:t0 + n].copy_(torch.randn(n, Hkv, d, generator=g, device=device))
    n_out = int(round(cfg.outlier_frac * Hkv * d))
    for c in rng.choice(Hkv * d, size=n_out, replace=False):
        h, e = int(c) // d, int(c) % d
        k[:, h, e] *= 8
        v[:, h, e] *= 8
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return PrefillWorkload(cfg=cfg, k=k, v=v, cu_seqlens=cu, block_tables=bt, num_blocks=N)


# ----------------------------------------------------------------------------- chunked prefill
@dataclass(frozen=True)
class ChunkConfig:
    key: str
    name: str
    batch: int
    ctx_len: int                    # tokens cached after the chunk's append
    chunk: int                      # query tokens per sequence
    hq: int
    hkv: int
    head_dim: int
    block_size: int
    spare: float = 0.10
    seed: int = 402


CHUNKED = {
    "p2": ChunkConfig("p2", "chunked prefill attention", 4, 8192, 512, 32, 8, 128, 16),
}


@dataclass
class ChunkWorkload:
    cfg: ChunkConfig
    k_pool: torch.Tensor            # [N, bs, Hkv, d] bf16 (history; the chunk is appended)
    v_pool: torch.Tensor
    k_new: torch.Tensor             # [B, chunk, Hkv, d] bf16
    v_new: torch.Tensor
    q: torch.Tensor                 # [B*chunk, Hq, d] bf16
    cu_q: np.ndarray                # [B+1] int32
    ctx_lens: np.ndarray            # [B] int32 (after the append)
    positions: np.ndarray           # [B] int32, first position of the chunk
    block_tables: np.ndarray
    num_blocks: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.cfg.head_dim)


def generate_chunked(cfg: ChunkConfig, device="cpu") -> ChunkWorkload:
    rng = np.random.default_rng(cfg.seed)
    B, bs, Hkv, d = cfg.batch, cfg.block_size, cfg.hkv, cfg.head_dim
    ctx = np.full(B, cfg.ctx_len, np.int32)
    bt, N = _allocate(ctx, bs, cfg.spare, None, rng)
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device).to(torch.bfloat16)

    k_pool = randn(N, bs, Hkv, d)
    v_pool = randn(N, bs, Hkv, d)
    k_new = randn(B, cfg.chunk, Hkv, d)
    v_new = randn(B, cfg.chunk, Hkv, d)
    q = randn(B * cfg.chunk, cfg.hq, d)
    cu = (np.arange(B + 1) * cfg.chunk).astype(np.int32)
    return ChunkWorkload(cfg=cfg, k_pool=k_pool, v_pool=v_pool, k_new=k_new, v_new=v_new, q=q,
                         cu_q=cu, ctx_lens=ctx, positions=(ctx - cfg.chunk).astype(np.int32),
                         block_tables=bt, num_blocks=N)
