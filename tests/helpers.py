"""Shared helpers for the parity tests: run one decode step of a workload on the
GPU through the C ABI, run the same step in the fp64 oracle on host copies of
the generator's inputs, and compare with the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

# attention output: |err| <= ATOL + RTOL * |ref| against the fp64 oracle
ATOL, RTOL = 2e-3, 1e-2
# token scores: relative
SCORE_RTOL = 1e-5


def assert_attention_close(got_bf16: torch.Tensor, ref: np.ndarray, what=""):
    got = got_bf16.detach().float().cpu().numpy().astype(np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at "
                             f"{tuple(idx)} got {got[tuple(idx)]} ref {ref[tuple(idx)]}; "
                             f"max err {err.max():.3g}")


def assert_scores_close(got: np.ndarray, ref: np.ndarray, what=""):
    inf = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf), what
    g, r = got[~inf], ref[~inf]
    rel = np.abs(g - r) / np.maximum(np.abs(r), 1e-30)
    zero = r == 0
    assert (g[zero] == 0).all(), what
    assert (rel[~zero] <= SCORE_RTOL).all(), f"{what}: max rel err {rel[~zero].max():.3g}"


def assert_evict_consistent(got: np.ndarray, ref_idx, ref_means, ref_gap, what=""):
    """Exact where the oracle's decision margin exceeds what fp32 scores can move
    a block mean by; otherwise the GPU's block must also attain the minimum."""
    n_exact = 0
    for b in range(len(ref_idx)):
        if ref_idx[b] < 0:
            assert got[b] == -1, (what, b)
            continue
        mn = ref_means[b, ref_idx[b]]
        margin = 4 * SCORE_RTOL * abs(mn)
        if ref_gap[b] > margin:
            assert got[b] == ref_idx[b], (what, b, got[b], ref_idx[b])
            n_exact += 1
        else:
            assert 0 <= got[b] < ref_means.shape[1] and ref_means[b, got[b]] <= mn + margin, \
                (what, b)
    return n_exact


class Device:
    """Device copies of one workload plus outputs and scratch for the C ABI."""

    def __init__(self, wl: W.Workload, num_splits=0, pad=0):
        """pad > 0: every pool is a [:, :, :bs] view of a buffer with bs + pad slots per
        block, so its block stride is (bs + pad)·Hkv·d; the pad slots hold NaN (bf16),
        127 (INT8) or the e4m3 NaN code, and pads_untouched() checks they still do."""
        cfg = wl.cfg
        dev = torch.device("cuda")
        self.wl, self.dev, self.num_splits = wl, dev, num_splits
        self._pads = []

        def pool(shape, dtype, fill, src=None):
            L_, N_, bs_ = shape[:3]
            big = torch.full((L_, N_, bs_ + pad) + tuple(shape[3:]), fill, dtype=dtype,
                             device=dev)
            view = big[:, :, :bs_]
            if src is not None:
                view.copy_(src)
            if pad:
                self._pads.append((big[:, :, bs_:], fill))
            return view
        self.bt = torch.as_tensor(wl.block_tables, device=dev)
        self.ctx = torch.as_tensor(wl.ctx_lens, device=dev)
        self.pos = torch.as_tensor(wl.positions, device=dev)
        self.q = wl.q.to(dev)
        self.k_new = None if wl.k_new is None else wl.k_new.to(dev)
        self.v_new = None if wl.v_new is None else wl.v_new.to(dev)
        L, B = self.q.shape[0], cfg.batch
        N, bs, Hkv, d = wl.num_blocks, cfg.block_size, cfg.hkv, cfg.head_dim
        if cfg.fp8:
            self.k8 = pool((L, N, bs, Hkv, d), torch.uint8, 0x7f if pad else 0)
            self.v8 = pool((L, N, bs, Hkv, d), torch.uint8, 0x7f if pad else 0)
        elif cfg.int8:
            self.kq = pool((L, N, bs, Hkv, d), torch.int8, 127 if pad else 0)
            self.vq = pool((L, N, bs, Hkv, d), torch.int8, 127 if pad else 0)
            self.ks = torch.zeros(L, N, bs, Hkv, dtype=torch.float32, device=dev)
            self.vs = torch.zeros_like(self.ks)
        elif pad:
            k_src = wl.kv[0] if wl.kv is not None else wl.k_pool
            v_src = wl.kv[1] if wl.kv is not None else wl.v_pool
            self.k_pool = pool(tuple(k_src.shape), torch.bfloat16, float("nan"), k_src.to(dev))
            self.v_pool = pool(tuple(v_src.shape), torch.bfloat16, float("nan"), v_src.to(dev))
        else:
            if wl.kv is not None:
                self.kv = wl.kv.to(dev)
                self.k_pool, self.v_pool = self.kv[0], self.kv[1]
            else:
                self.k_pool = wl.k_pool.to(dev)
                self.v_pool = wl.v_pool.to(dev)
        self.out = torch.empty(L, B, cfg.hq, d, dtype=torch.bfloat16, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws = pk.alloc_workspace(B, cfg.hq, Hkv, d, bs, wl.max_blocks, num_splits, dev)
        self.slots = torch.full((B, 1), -7, dtype=torch.int64, device=dev)

    def pads_untouched(self) -> bool:
        for gap, fill in self._pads:
            if gap.dtype == torch.bfloat16:
                if not torch.isnan(gap).all():
                    return False
            elif not (gap == fill).all():
                return False
        return True

    def _append_hist(self, layer, k, v, bt, pos):
        if self.wl.cfg.fp8:
            pk.pa_append_kv_fp8(k, v, self.k8[layer], self.v8[layer], bt, pos, self.err)
        else:
            pk.pa_append_kv_int8(k, v, self.kq[layer], self.vq[layer], self.ks[layer],
                                 self.vs[layer], bt, pos, self.err)

    def fill_int8_history(self, layer):
        """Quantise the bf16 history into the INT8 (or FP8) pools with the append."""
        wl = self.wl
        zeros = torch.zeros(wl.cfg.batch, dtype=torch.int32, device=self.dev)
        kh, vh = wl.k_hist[layer].to(self.dev), wl.v_hist[layer].to(self.dev)
        if (wl.old_lens == wl.old_lens[0]).all():
            n = int(wl.old_lens[0])
            self._append_hist(layer, kh[:, :n].contiguous(), vh[:, :n].contiguous(), self.bt,
                              zeros)
        else:
            for b in range(wl.cfg.batch):
                n = int(wl.old_lens[b])
                if n == 0:
                    continue
                self._append_hist(layer, kh[b:b + 1, :n].contiguous(),
                                  vh[b:b + 1, :n].contiguous(), self.bt[b:b + 1], zeros[b:b + 1])

    def step(self, layer, score=False):
        """append (when the workload appends) then decode; optional score+select."""
        cfg = self.wl.cfg
        if cfg.fp8:
            if self.k_new is not None:
                pk.pa_append_kv_fp8(self.k_new[layer], self.v_new[layer], self.k8[layer],
                                    self.v8[layer], self.bt, self.pos, self.err,
                                    slot_out=self.slots)
            pk.pa_decode_fp8(self.out[layer], self.q[layer], self.k8[layer], self.v8[layer],
                             self.bt, self.ctx, self.wl.scale, self.err, self.ws, self.num_splits)
        elif cfg.int8:
            if self.k_new is not None:
                pk.pa_append_kv_int8(self.k_new[layer], self.v_new[layer], self.kq[layer],
                                     self.vq[layer], self.ks[layer], self.vs[layer], self.bt,
                                     self.pos, self.err, slot_out=self.slots)
            pk.pa_decode_int8(self.out[layer], self.q[layer], self.kq[layer], self.vq[layer],
                              self.ks[layer], self.vs[layer], self.bt, self.ctx, self.wl.scale,
                              self.err, self.ws, self.num_splits)
        else:
            if self.k_new is not None:
                pk.pa_append_kv(self.k_new[layer], self.v_new[layer], self.k_pool[layer],
                                self.v_pool[layer], self.bt, self.pos, self.err,
                                slot_out=self.slots)
            pk.pa_decode(self.out[layer], self.q[layer], self.k_pool[layer], self.v_pool[layer],
                         self.bt, self.ctx, self.wl.scale, self.err, self.ws, self.num_splits)
        res = {}
        if score:
            B, MB = self.bt.shape
            scores = torch.full((B, MB * cfg.block_size, cfg.hkv), float("nan"),
                                dtype=torch.float32, device=self.dev)
            evict = torch.full((B,), -9, dtype=torch.int32, device=self.dev)
            means = torch.empty(B, MB, dtype=torch.float32, device=self.dev)
            pk.pe_score_tokens(scores, self.k_pool[layer], self.v_pool[layer], self.bt, self.ctx,
                               self.err)
            pk.pe_select_evict_block(evict, scores, self.ctx, cfg.block_size, means)
            res = dict(scores=scores, evict=evict, means=means)
        return res


def oracle_step(wl: W.Workload, layer: int, seqs, score=False):
    """The same step in the fp64 oracle, on host copies of the generator's inputs
    for the sequences `seqs` only."""
    cfg = wl.cfg
    s = W.compact(wl, layer, seqs)
    Hkv, d, bs = cfg.hkv, cfg.head_dim, cfg.block_size
    stride = bs * Hkv * d
    n = s["num_blocks"]
    res = {"ctx_lens": s["ctx_lens"]}
    if cfg.fp8:
        k8 = np.zeros(n * stride, np.uint8)
        v8 = np.zeros_like(k8)
        zeros = np.zeros(len(s["ctx_lens"]), np.int32)
        for r in range(len(s["ctx_lens"])):
            m = int(s["old_lens"][r])
            if m:
                oracle.append_kv_fp8(s["k_hist"][r:r + 1, :m], s["v_hist"][r:r + 1, :m], k8, v8,
                                     stride, s["block_tables"][r:r + 1], zeros[r:r + 1], bs)
        if "k_new" in s:
            res["slots"] = oracle.append_kv_fp8(s["k_new"], s["v_new"], k8, v8, stride,
                                                s["block_tables"], s["positions"], bs)
        res["out"] = oracle.paged_decode_fp8(s["q"], k8, v8, stride, s["block_tables"],
                                             s["ctx_lens"], Hkv, bs, wl.scale)
        res.update(k8=k8, v8=v8)
    elif cfg.int8:
        kq = np.zeros(n * stride, np.int8)
        vq = np.zeros_like(kq)
        ks = np.zeros(n * bs * Hkv, np.float32)
        vs = np.zeros_like(ks)
        zeros = np.zeros(len(s["ctx_lens"]), np.int32)
        for r in range(len(s["ctx_lens"])):
            m = int(s["old_lens"][r])
            if m:
                oracle.append_kv_int8(s["k_hist"][r:r + 1, :m], s["v_hist"][r:r + 1, :m], kq, vq,
                                      ks, vs, stride, s["block_tables"][r:r + 1], zeros[r:r + 1],
                                      bs)
        if "k_new" in s:
            res["slots"] = oracle.append_kv_int8(s["k_new"], s["v_new"], kq, vq, ks, vs, stride,
                                                 s["block_tables"], s["positions"], bs)
        res["out"] = oracle.paged_decode_int8(s["q"], kq, vq, ks, vs, stride, s["block_tables"],
                                              s["ctx_lens"], Hkv, bs, wl.scale)
        res.update(kq=kq, vq=vq, ks=ks, vs=vs)
    else:
        kc = s["k_pool"].ravel().copy()
        vc = s["v_pool"].ravel().copy()
        if "k_new" in s:
            res["slots"] = oracle.append_kv(s["k_new"], s["v_new"], kc, vc, stride,
                                            s["block_tables"], s["positions"], bs)
        res["out"] = oracle.paged_decode(s["q"], kc, vc, stride, s["block_tables"], s["ctx_lens"],
                                         Hkv, bs, wl.scale)
        if score:
            sc = oracle.score_tokens(kc, vc, stride, s["block_tables"], s["ctx_lens"], Hkv, d, bs)
            ev, means, gap = oracle.select_evict_block(sc, s["ctx_lens"], bs)
            res.update(scores=sc, evict=ev, means=means, gap=gap)
        res.update(kc=kc, vc=vc)
    res["compact"] = s
    return res
