#!/usr/bin/env python
"""Decode-step benchmark of the paged KV decode attention library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3] [--impl ours|reference]

One step is one decode step of the chosen workload through the C ABI:
for every layer, the KV append of the new token and paged decode attention
(c2 adds the PagedEviction score pass and block selection per layer).  Default
workload: c3, the Llama-3-8B-shape decode (32 layers, 32/8 heads, d=128,
batch 64, contexts uniform in [512, 8192], block 16), whose pools (~40 GB)
exceed L2, so no flush is needed between steps.

Prints ONE JSON line (rank 0).  value = decode tokens/s of the whole job
(batch x ranks / step time, device-timed, max over ranks); the roofline object
covers the decode kernel (algorithmic bytes / event-timed duration).
N > 1 (torchrun): every rank runs its own replica of the batch on its own GPU
(sequences are independent; no collective on the data path), weak scaling.

--impl reference times the fp64 CPU oracle (the correctness reference) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_396_b200 import workloads as W  # noqa: E402

METRIC = "paged decode-attention HBM GB/s (% of B200 peak) and decode tokens/s at 1 GPU"
FALLBACK_HBM_GBS = 6650.0
DECODE_SOURCES = ["decode_simple.cu", "decode_tc.cu", "kernels.h", "common.cuh", "ptx.cuh"]
# sources of the other workloads' dominant kernels (their recorded traffic is keyed by them)
PREFILL_SOURCES = {"p1": ["prefill.cu", "prefill.h", "kernels.h", "common.cuh"],
                   "p2": ["prefill_attn_tc.cu", "prefill_attn.h", "kernels.h", "common.cuh",
                          "ptx.cuh"]}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c3", choices=["c2", "c3", "c4", "c5", "p1", "p2"],
                    help="c2..c5: decode steps; p1: PagedEviction prefill compression; "
                         "p2: chunked prefill attention")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kv", default=None, choices=["bf16", "int8", "fp8"],
                    help="KV storage type (default: the workload's own)")
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--evict", default="full", choices=["full", "incremental"],
                    help="workloads with a score pass: rescore the whole context per layer "
                         "(full) or score each token once at append into a paged score pool "
                         "and select blocks from it (incremental)")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling aid: keep only this many layers of the workload")
    ap.add_argument("--plan", default="step", choices=["step", "call"],
                    help="staged decode: make the partition plan once per step "
                         "(pa_decode_prepare + planned calls) or inside every decode call")
    ap.add_argument("--select", default="call", choices=["call", "stream"],
                    help="incremental eviction: the block selection inside the decode call "
                         "(pa_decode*_select_pooled: extra CTAs of its merge launch) or as its "
                         "own kernel on a second stream beside the decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--secondary", default=None,
                    help="comma-separated workloads also measured and reported under "
                         "'secondary' in the same JSON line (c5-fp8 = c5 on e4m3 pools); "
                         f"default for the c3 line: {'c4,c2,c5,c5-fp8,p1,p2'}, else none; "
                         "'none' for no secondary lines")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every call from Python instead of replaying a CUDA graph")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers
def reduce_max(x: float, world: int) -> float:
    """Max of x over all ranks (device times are reported as the slowest rank's)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, batch: int, ms_per_step: float) -> float:
    """Whole-job decode throughput: every rank decodes its own batch of sequences
    (weak scaling), so the job emits world * batch tokens per (slowest) step."""
    return world * batch / (ms_per_step / 1000.0)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """The source without // comments and blank lines (whitespace collapsed), so a
    comment edit does not invalidate a recorded capture; a // inside a string
    literal is kept."""
    out = []
    for line in text.splitlines():
        q, cut = False, len(line)
        for i, ch in enumerate(line):
            if ch == '"' and (i == 0 or line[i - 1] != "\\"):
                q = not q
            elif not q and line.startswith("//", i):
                cut = i
                break
        code = " ".join(line[:cut].split())
        if code:
            out.append(code)
    return "\n".join(out)


def source_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        p = os.path.join(ROOT, "paged_kv_cache_396_b200", "csrc", f)
        if os.path.exists(p):
            h.update(_code_only(open(p, encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def decode_source_hash() -> str:
    return source_hash(DECODE_SOURCES)


def recorded_traffic(workload: str, record="decode_traffic.txt", sources=None):
    """dram bytes per launch of the dominant kernel from a committed ncu summary
    (profiles/<record>), if it was taken on the current sources (else None)."""
    p = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(p):
        return None
    want = source_hash(sources if sources is not None else DECODE_SOURCES)
    for line in open(p):
        kv = dict(x.split("=", 1) for x in line.split() if "=" in x)
        if kv.get("workload") == workload and kv.get("sources") == want:
            return float(kv["bytes_per_launch"])
    return None


class Clocks:
    """nvidia-smi sampler (200 ms) running during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", ident, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- model
def clocks_under_load(clk, device, run_steps, timed_s, seconds=0.8):
    """The clock record of a run.  The sampler polls every 200 ms and starts 0.3 s
    before the timed region, so a timed region shorter than a second (c2's 20 steps
    take about 7 ms) yields mostly samples of the idle GPU around it.  The timed
    region's own samples stand when it lasted at least 1 s (timed_s) and gave at
    least 3.  Otherwise the same step runs back to back, untimed, for `seconds` right
    after the timed region, and its samples are the record; the timed region's own
    are kept under 'timed_region'."""
    if clk is not None and clk.get("samples", 0) >= 3 and timed_s >= 1.0:
        return dict(clk, window="timed region")
    soak = Clocks(device)
    t_end = time.perf_counter() + seconds
    while time.perf_counter() < t_end:
        run_steps()
        torch.cuda.synchronize(device)
    rec = soak.stop()
    if rec is None:
        return clk
    return dict(rec, window=f"the same step back to back for {seconds} s after the timed "
                            "region (shorter than 1 s: mostly idle samples)", timed_region=clk)


def decode_algorithmic_bytes(cfg, ctx_lens, partial_slots, n_units=0):
    """Bytes one decode call (one layer) must move: K/V rows of every cached
    token (plus INT8 scales), q and out, the table entries and lengths read, the
    partition partials written and read back by the merge (partial_slots slots
    of Hq rows of d + 2 floats), and the partition list of the staged kernel."""
    elt = 1 if (cfg.int8 or cfg.fp8) else 2
    tok = int(np.sum(ctx_lens))
    kv = tok * cfg.hkv * cfg.head_dim * 2 * elt
    if cfg.int8:
        kv += tok * cfg.hkv * 2 * 4
    qo = 2 * cfg.batch * cfg.hq * cfg.head_dim * 2
    nblk = int(sum(-(-int(n) // cfg.block_size) for n in ctx_lens))
    table = nblk * 4 + 2 * cfg.batch * 4
    parts = 2 * partial_slots * cfg.hq * (cfg.head_dim + 2) * 4
    plan = 2 * n_units * 16 + 2 * cfg.batch * 4
    return kv + qo + table + parts + plan


class Runner:
    """Device state and one decode step of a workload through the binding."""

    def __init__(self, cfg, device, num_splits=0, wl=None, evict="full", plan="step",
                 overlap_select=True, select="call"):
        from paged_kv_cache_396_b200 import pagedkv as pk
        self.pk, self.cfg, self.dev = pk, cfg, device
        wl = W.generate(cfg, device) if wl is None else wl
        self.wl = wl
        self.L = cfg.layers
        self.bt = torch.as_tensor(wl.block_tables, device=device)
        self.ctx = torch.as_tensor(wl.ctx_lens, device=device)
        self.pos = torch.as_tensor(wl.positions, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        B, Hq, Hkv, d, bs = cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size
        MB = wl.max_blocks
        self.out = torch.empty(self.L, B, Hq, d, dtype=torch.bfloat16, device=device)
        self.ws = pk.alloc_workspace(B, Hq, Hkv, d, bs, MB, num_splits, device)
        self.num_splits = num_splits
        self.S, self.chunk, self.dec_launches, self.staged = pk.pa_decode_plan(
            B, Hq, Hkv, d, bs, MB, num_splits)
        # the staged kernel's partition plan: once per step (pa_decode_prepare, then the
        # planned calls) or inside every decode call; the general kernel keeps no plan
        self.per_step_plan = self.staged and plan == "step" and not (
            (cfg.int8 or cfg.fp8) and d != 128)
        if cfg.fp8:
            N = wl.num_blocks
            self.k8 = torch.zeros(self.L, N, bs, Hkv, d, dtype=torch.uint8, device=device)
            self.v8 = torch.zeros_like(self.k8)
            zeros = torch.zeros(B, dtype=torch.int32, device=device)
            for l in range(self.L):
                for b in range(B):  # one prompt-style append per sequence
                    n = int(wl.old_lens[b])
                    pk.pa_append_kv_fp8(wl.k_hist[l, b:b + 1, :n].contiguous(),
                                        wl.v_hist[l, b:b + 1, :n].contiguous(), self.k8[l],
                                        self.v8[l], self.bt[b:b + 1], zeros[b:b + 1], self.err)
        if cfg.int8:
            N = wl.num_blocks
            self.kq = torch.zeros(self.L, N, bs, Hkv, d, dtype=torch.int8, device=device)
            self.vq = torch.zeros_like(self.kq)
            self.ks = torch.zeros(self.L, N, bs, Hkv, dtype=torch.float32, device=device)
            self.vs = torch.zeros_like(self.ks)
            zeros = torch.zeros(B, dtype=torch.int32, device=device)
            for l in range(self.L):
                if (wl.old_lens == wl.old_lens[0]).all():
                    n = int(wl.old_lens[0])
                    pk.pa_append_kv_int8(wl.k_hist[l, :, :n].contiguous(),
                                         wl.v_hist[l, :, :n].contiguous(), self.kq[l], self.vq[l],
                                         self.ks[l], self.vs[l], self.bt, zeros, self.err)
                    continue
                for b in range(B):  # unequal lengths: one prompt-style append per sequence
                    n = int(wl.old_lens[b])
                    pk.pa_append_kv_int8(wl.k_hist[l, b:b + 1, :n].contiguous(),
                                         wl.v_hist[l, b:b + 1, :n].contiguous(), self.kq[l],
                                         self.vq[l], self.ks[l], self.vs[l], self.bt[b:b + 1],
                                         zeros[b:b + 1], self.err)
        self.incremental = bool(cfg.score) and evict == "incremental"
        # incremental eviction on bf16 pools: the block choice inside the decode call
        self.select_in_call = (self.incremental and select == "call" and not cfg.int8
                               and not cfg.fp8)
        if cfg.score:
            self.scores = torch.zeros(B, MB * bs, Hkv, dtype=torch.float32, device=device)
            self.evict = torch.zeros(B, dtype=torch.int32, device=device)
        # incremental eviction: the block choice of a layer overlaps its decode (a second
        # stream joined at the end of the step) unless overlap is off
        self.side = (torch.cuda.Stream(device)
                     if self.incremental and overlap_select and not self.select_in_call
                     else None)
        self.ev_app = [torch.cuda.Event() for _ in range(self.L)]
        self.ev_join = torch.cuda.Event()
        if self.incremental:
            # paged score pools, filled for the cached history once (set-up): score
            # every cached token, then place each score at its token's slot
            N = wl.num_blocks
            self.score_pool = torch.zeros(self.L, N, bs, Hkv, dtype=torch.float32, device=device)
            old = torch.as_tensor(wl.old_lens, device=device)
            t = torch.arange(MB * bs, device=device)
            live = t[None, :] < old[:, None]
            bidx, tidx = live.nonzero(as_tuple=True)
            slots = self.bt[bidx, tidx // bs].long() * bs + tidx % bs
            for l in range(self.L):
                pk.pe_score_tokens(self.scores, wl.k_pool[l], wl.v_pool[l], self.bt, self.ctx,
                                   self.err)
                self.score_pool[l].view(N * bs, Hkv)[slots] = self.scores[bidx, tidx]
        torch.cuda.synchronize(device)
        self.q = wl.q
        self.k_new, self.v_new = wl.k_new, wl.v_new
        self.decode_bytes = None

    def account_bytes(self):
        """Algorithmic bytes of one decode call, with the partition counts the
        last call actually used (read back from the workspace)."""
        cfg, pk = self.cfg, self.pk
        n_sub = max(1, 8 // cfg.hkv)
        if self.staged:
            n_units, chunk, ns = pk.workspace_plan(self.ws, cfg.batch)
            slots = sum(n * n_sub for n in ns if n > 1 or n_sub > 1)
            self.chunk_used = chunk
        else:
            n_units = 0
            slots = 0
            if self.S > 1:
                slots = sum(max(1, -(-int(n) // self.chunk)) for n in self.wl.ctx_lens)
            self.chunk_used = self.chunk
        self.decode_bytes = decode_algorithmic_bytes(cfg, self.wl.ctx_lens, slots, n_units)
        self.partitions = slots

    def selection_rides_on_merge(self):
        """Whether the decode call's merge launch carries the block selection: the
        staged kernel with a warp-per-row merge (the library's rule: with the balanced
        split B + SMs <= 8 B, with an explicit one S * wph <= 8)."""
        cfg = self.cfg
        if not (self.select_in_call and self.staged and self.dec_launches >= 3):
            return False
        P = torch.cuda.get_device_properties(self.dev).multi_processor_count
        wph = max(1, 8 // cfg.hkv)
        if self.num_splits == 0 and P < 1024:
            return cfg.batch + P <= 8 * cfg.batch
        return self.S * wph <= 8

    def launches_per_step(self):
        dec = self.dec_launches - (1 if self.per_step_plan else 0)
        per_layer = (1 if self.cfg.append else 0) + dec
        if self.cfg.score:
            per_layer += (0 if self.selection_rides_on_merge() else 1) if self.incremental else 2
        return per_layer * self.L + (1 if self.per_step_plan else 0)

    def decode_calls(self):
        """The step's decode calls alone, back to back: the partition plan (once per
        step) and one decode call per layer, with no other kernel or event between
        them (an event recorded between two kernels of a graph stops the second from
        starting while the first drains)."""
        pk, cfg = self.pk, self.cfg
        if self.per_step_plan:
            pk.pa_decode_prepare(self.q[0], self.wl.k_pool[0] if self.wl.k_pool is not None
                                 else self.kq[0] if cfg.int8 else self.k8[0], self.bt, self.ctx,
                                 self.err, self.ws, self.num_splits)
        for l in range(self.L):
            if cfg.fp8:
                (pk.pa_decode_fp8_planned if self.per_step_plan else pk.pa_decode_fp8)(
                    self.out[l], self.q[l], self.k8[l], self.v8[l], self.bt, self.ctx,
                    self.wl.scale, self.err, self.ws, self.num_splits)
            elif cfg.int8:
                (pk.pa_decode_int8_planned if self.per_step_plan else pk.pa_decode_int8)(
                    self.out[l], self.q[l], self.kq[l], self.vq[l], self.ks[l], self.vs[l],
                    self.bt, self.ctx, self.wl.scale, self.err, self.ws, self.num_splits)
            else:
                (pk.pa_decode_planned if self.per_step_plan else pk.pa_decode)(
                    self.out[l], self.q[l], self.wl.k_pool[l], self.wl.v_pool[l], self.bt,
                    self.ctx, self.wl.scale, self.err, self.ws, self.num_splits)

    def step(self, ev=None):
        pk, cfg = self.pk, self.cfg
        if self.per_step_plan:
            # every layer of the step has the same context lengths: one partition plan
            pk.pa_decode_prepare(self.q[0], self.wl.k_pool[0] if self.wl.k_pool is not None
                                 else self.kq[0] if cfg.int8 else self.k8[0], self.bt, self.ctx,
                                 self.err, self.ws, self.num_splits)
        dec = pk.pa_decode_planned if self.per_step_plan else pk.pa_decode
        dec8 = pk.pa_decode_int8_planned if self.per_step_plan else pk.pa_decode_int8
        decf8 = pk.pa_decode_fp8_planned if self.per_step_plan else pk.pa_decode_fp8
        for l in range(self.L):
            if cfg.fp8:
                pk.pa_append_kv_fp8(self.k_new[l], self.v_new[l], self.k8[l], self.v8[l], self.bt,
                                    self.pos, self.err)
                if ev is not None:
                    ev[l][0].record()
                decf8(self.out[l], self.q[l], self.k8[l], self.v8[l], self.bt, self.ctx,
                      self.wl.scale, self.err, self.ws, self.num_splits)
            elif cfg.int8:
                pk.pa_append_kv_int8(self.k_new[l], self.v_new[l], self.kq[l], self.vq[l],
                                     self.ks[l], self.vs[l], self.bt, self.pos, self.err)
                if ev is not None:
                    ev[l][0].record()
                dec8(self.out[l], self.q[l], self.kq[l], self.vq[l], self.ks[l], self.vs[l],
                     self.bt, self.ctx, self.wl.scale, self.err, self.ws, self.num_splits)
            else:
                kp = self.wl.k_pool[l]
                vp = self.wl.v_pool[l]
                if cfg.append and self.incremental:
                    pk.pa_append_kv_scored(self.k_new[l], self.v_new[l], kp, vp,
                                           self.score_pool[l], self.bt, self.pos, self.err)
                    if self.side is not None:
                        # the block choice needs only this layer's score pool: it runs on
                        # a second stream beside the decode
                        self.ev_app[l].record()
                        self.side.wait_event(self.ev_app[l])
                elif cfg.append:
                    pk.pa_append_kv(self.k_new[l], self.v_new[l], kp, vp, self.bt, self.pos,
                                    self.err)
                if ev is not None:
                    ev[l][0].record()
                if self.select_in_call:   # decode and this layer's block choice, one call
                    (pk.pa_decode_planned_select_pooled if self.per_step_plan
                     else pk.pa_decode_select_pooled)(
                        self.out[l], self.q[l], kp, vp, self.bt, self.ctx, self.wl.scale,
                        self.err, self.evict, self.score_pool[l], None, self.ws,
                        self.num_splits)
                else:
                    dec(self.out[l], self.q[l], kp, vp, self.bt, self.ctx, self.wl.scale,
                        self.err, self.ws, self.num_splits)
            if ev is not None:
                ev[l][1].record()
            if self.incremental:
                if not self.select_in_call:
                    pk.pe_select_evict_block_pooled(self.evict, self.score_pool[l], self.bt,
                                                    self.ctx, self.err, stream=self.side)
            elif cfg.score:
                pk.pe_score_tokens(self.scores, self.wl.k_pool[l], self.wl.v_pool[l], self.bt,
                                   self.ctx, self.err)
                pk.pe_select_evict_block(self.evict, self.scores, self.ctx, cfg.block_size)
        if self.side is not None:   # the step ends when the block choices are made
            self.ev_join.record(self.side)
            torch.cuda.current_stream().wait_event(self.ev_join)


# ----------------------------------------------------------------------------- oracle
def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def with_single_core(cpu, fn, budget_s):
    """Add the same oracle timing on one thread (a quarter of the budget) and the
    host CPU model to a cpu_baseline dict."""
    import oracle
    n = oracle.threads()
    oracle.set_threads(1)
    try:
        v1, _, d1 = fn(budget_s / 4)
    finally:
        oracle.set_threads(n)
    cpu["single_core"] = {"value": v1, "unit": cpu["unit"], "sample": d1}
    cpu["cpu_model"] = cpu_model()
    return cpu


def oracle_throughput(wl, budget_s, max_layers=None):
    """Time the fp64 oracle (append + decode, plus score + select for c2) on
    (layer, sequence-batch) samples of the workload for about budget_s seconds;
    scale to decode tokens/s of the whole step.  Returns (tokens/s, cores, desc)."""
    import oracle
    cfg = wl.cfg
    cores = oracle.threads()
    per_call = max(8, min(cfg.batch, cores))
    Hkv, d, bs = cfg.hkv, cfg.head_dim, cfg.block_size
    stride = bs * Hkv * d
    t_total, tok_total, n_calls = 0.0, 0, 0
    layers = wl.q.shape[0] if max_layers is None else min(max_layers, wl.q.shape[0])
    order = [(l, s) for l in range(layers) for s in range(0, cfg.batch, per_call)]
    for l, s0 in order:
        seqs = list(range(s0, min(cfg.batch, s0 + per_call)))
        c = W.compact(wl, l, seqs)
        t0 = time.perf_counter()
        if cfg.fp8:
            n = c["num_blocks"]
            k8 = np.zeros(n * stride, np.uint8); v8 = np.zeros_like(k8)
            oracle.append_kv_fp8(c["k_hist"], c["v_hist"], k8, v8, stride, c["block_tables"],
                                 np.zeros(len(seqs), np.int32), bs)
            t0 = time.perf_counter()   # the history fill is set-up, not the step
            oracle.append_kv_fp8(c["k_new"], c["v_new"], k8, v8, stride, c["block_tables"],
                                 c["positions"], bs)
            oracle.paged_decode_fp8(c["q"], k8, v8, stride, c["block_tables"], c["ctx_lens"], Hkv,
                                    bs, wl.scale)
        elif cfg.int8:
            n = c["num_blocks"]
            kq = np.zeros(n * stride, np.int8); vq = np.zeros_like(kq)
            ks = np.zeros(n * bs * Hkv, np.float32); vs = np.zeros_like(ks)
            oracle.append_kv_int8(c["k_hist"], c["v_hist"], kq, vq, ks, vs, stride,
                                  c["block_tables"], np.zeros(len(seqs), np.int32), bs)
            t0 = time.perf_counter()   # the history fill is set-up, not the step
            oracle.append_kv_int8(c["k_new"], c["v_new"], kq, vq, ks, vs, stride,
                                  c["block_tables"], c["positions"], bs)
            oracle.paged_decode_int8(c["q"], kq, vq, ks, vs, stride, c["block_tables"],
                                     c["ctx_lens"], Hkv, bs, wl.scale)
        else:
            kc, vc = c["k_pool"].ravel(), c["v_pool"].ravel()
            if "k_new" in c:
                oracle.append_kv(c["k_new"], c["v_new"], kc, vc, stride, c["block_tables"],
                                 c["positions"], bs)
            oracle.paged_decode(c["q"], kc, vc, stride, c["block_tables"], c["ctx_lens"], Hkv, bs,
                                wl.scale)
            if cfg.score:
                sc = oracle.score_tokens(kc, vc, stride, c["block_tables"], c["ctx_lens"], Hkv, d,
                                         bs)
                oracle.select_evict_block(sc, c["ctx_lens"], bs)
        t_total += time.perf_counter() - t0
        tok_total += int(np.sum(c["ctx_lens"]))
        n_calls += 1
        if t_total >= budget_s:
            break
    full_tok = int(np.sum(wl.ctx_lens)) * cfg.layers
    step_s = t_total / tok_total * full_tok
    desc = (f"{n_calls} oracle calls over {tok_total} context tokens "
            f"({per_call} sequences per call, layers 0..{layers - 1}), {t_total:.1f} s, "
            f"scaled by {full_tok} context tokens per step")
    return cfg.batch / step_s, cores, desc


def reference_samples(args, sample):
    """The reference arm's timing loop: W warm-up samples (a quarter of the budget
    each) and K timed ones.  sample(budget_s) runs the oracle on a bounded part of the
    workload for about budget_s seconds and returns (throughput, cores, description).
    Returns the median throughput, the cores, the last description and the host wall
    time of one timed sample in ms (the reference arm's "step")."""
    per = max(1.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        sample(per / 4)
    vals, walls, desc, cores = [], [], "", 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        v, cores, desc = sample(per)
        walls.append(1000.0 * (time.perf_counter() - t0))
        vals.append(v)
    return statistics.median(vals), cores, desc, statistics.mean(walls)


def reference_line(args, metric, unit, value, cores, desc, wall_ms, full_step_ms, config):
    """One JSON line of the reference arm.  A step here is one bounded sample of the
    workload's step (ms_per_step is its measured host wall time, so steps x
    ms_per_step is the time actually spent); value is the oracle's throughput over
    the samples, and ms_per_full_step_extrapolated the whole step at that rate."""
    return {
        "impl": "reference", "metric": metric, "value": value, "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall_ms, "ms_per_full_step_extrapolated": full_step_ms,
        "step": "one bounded sample of the workload's step on the host cores",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config,
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.workload in W.PREFILL:
        return run_reference_prefill(args)
    if args.workload in W.CHUNKED:
        return run_reference_chunked(args)
    cfg = workload_cfg(args)
    wl = W.generate(cfg, "cpu", layers=1)
    value, cores, desc, wall = reference_samples(
        args, lambda t: oracle_throughput(wl, t, max_layers=1))
    line = reference_line(args, METRIC, "tokens/s", value, cores, desc, wall,
                          1000.0 * cfg.batch / value,
                          dict(workload_config(cfg), parallelism="replicas1"))
    print(json.dumps(line), flush=True)
    return 0


def kv_name(cfg):
    return "fp8_e4m3" if cfg.fp8 else "int8" if cfg.int8 else "bf16"


def workload_cfg(args):
    """The named workload, with its KV storage type replaced when --kv asks."""
    cfg = W.CONFIGS[args.workload]
    if args.kv is not None:
        cfg = W.scaled(cfg, int8=args.kv == "int8", fp8=args.kv == "fp8")
    return cfg


def traffic_key(args, cfg):
    return args.workload + ("" if args.kv is None else "-" + kv_name(cfg))


METRIC_P1 = "PagedEviction prefill compression: prompt tokens/s and score-kernel HBM GB/s"
METRIC_P2 = "chunked prefill attention: chunk tokens/s and tensor TFLOP/s"


def prefill_config(cfg, world):
    return {"workload": f"{cfg.key} {cfg.name}", "prompts": cfg.batch,
            "prompt_tokens": cfg.prompt_lens[0], "kv_heads": cfg.hkv, "head_dim": cfg.head_dim,
            "block_size": cfg.block_size, "budget": cfg.budget, "parallelism": f"replicas{world}",
            "l2": "prompt rows (1 GiB) larger than L2 every step (no flush needed)"}


def chunked_config(cfg, world):
    return {"workload": f"{cfg.key} {cfg.name}", "sequences": cfg.batch, "chunk": cfg.chunk,
            "context": cfg.ctx_len, "q_heads": cfg.hq, "kv_heads": cfg.hkv,
            "head_dim": cfg.head_dim, "block_size": cfg.block_size,
            "parallelism": f"replicas{world}",
            "l2": "flushed (256 MB write) before every timed step"}


def run_reference_prefill(args):
    """The oracle's prefill stage timed on bounded samples of the prefill workload."""
    import dataclasses
    cfg = W.PREFILL[args.workload]
    # one prompt's worth of rows per sample keeps the host footprint small
    small = dataclasses.replace(cfg, batch=4, prompt_lens=cfg.prompt_lens[:4])
    wl = W.generate_prefill(small, "cpu")
    value, cores, desc, wall = reference_samples(
        args, lambda t: prefill_oracle_throughput(wl, t))
    T = sum(cfg.prompt_lens)
    line = reference_line(args, METRIC_P1, "prompt tokens/s", value, cores, desc, wall,
                          1000.0 * T / value, prefill_config(cfg, 1))
    print(json.dumps(line), flush=True)
    return 0


def run_reference_chunked(args):
    """The oracle's chunked prefill attention timed on row samples of the workload."""
    cfg = W.CHUNKED[args.workload]
    wl = W.generate_chunked(cfg, "cpu")
    value, cores, desc, wall = reference_samples(
        args, lambda t: chunk_oracle_throughput(wl, t))
    line = reference_line(args, METRIC_P2, "chunk tokens/s", value, cores, desc, wall,
                          1000.0 * cfg.batch * cfg.chunk / value, chunked_config(cfg, 1))
    print(json.dumps(line), flush=True)
    return 0


def workload_config(cfg):
    lens = (f"{cfg.old_lens[0]}" if cfg.old_lens and len(set(cfg.old_lens)) == 1
            else f"uniform[{cfg.old_len_range[0]},{cfg.old_len_range[1]}]"
            if cfg.old_len_range else "mixed")
    return {
        "workload": f"{cfg.key} {cfg.name}", "layers": cfg.layers, "global_batch": cfg.batch,
        "q_heads": cfg.hq, "kv_heads": cfg.hkv, "head_dim": cfg.head_dim,
        "block_size": cfg.block_size, "cached_tokens": lens,
        "append": cfg.append, "score_pass": cfg.score, "kv_dtype": kv_name(cfg),
        "l2": "working set larger than L2 every step (no flush needed)",
    }


# ----------------------------------------------------------------------------- prefill
def prefill_oracle_throughput(wl, budget_s):
    """The oracle's score + select + pack over whole prompts of the prefill
    workload for about budget_s seconds; returns (prompt tokens/s, cores, desc)."""
    import oracle
    cfg = wl.cfg
    cu = wl.cu_seqlens
    Hkv, d, bs = cfg.hkv, cfg.head_dim, cfg.block_size
    stride = bs * Hkv * d
    cores = oracle.threads()
    t_total, tok, n = 0.0, 0, 0
    for i in range(100000):
        b = i % cfg.batch
        kb = W.bits(wl.k[int(cu[b]):int(cu[b + 1])])
        vb = W.bits(wl.v[int(cu[b]):int(cu[b + 1])])
        bt = wl.block_tables[b:b + 1]
        nb = int((bt >= 0).sum())
        bt_c = np.where(bt >= 0, np.arange(bt.shape[1], dtype=np.int32), -1).astype(np.int32)
        kc = np.zeros(nb * stride, np.uint16)
        vc = np.zeros_like(kc)
        lcu = np.array([0, kb.shape[0]], np.int32)
        t0 = time.perf_counter()
        sc = oracle.prefill_scores(kb, vb)
        keep, kept = oracle.prefill_select(sc, lcu, cfg.budget)
        oracle.prefill_pack(kb, vb, lcu, keep, kept, kc, vc, stride, bt_c, bs)
        t_total += time.perf_counter() - t0
        tok += kb.shape[0]
        n += 1
        if t_total >= budget_s:
            break
    desc = (f"{n} whole prompts ({tok} tokens) through the oracle's score, select and pack "
            f"({cores} threads), "
            f"{t_total:.1f} s")
    return tok / t_total, cores, desc


def run_prefill(args, device, world, rank, cpu_baseline=True):
    """One step = the prefill stage of one layer for every prompt of the
    workload: token scores, keep sets, packing of the kept rows into the pool."""
    import paged_kv_cache_396_b200.pagedkv as pk
    cfg = W.PREFILL[args.workload]
    wl = W.generate_prefill(cfg, device)
    B, Hkv, d, bs, budget = cfg.batch, cfg.hkv, cfg.head_dim, cfg.block_size, cfg.budget
    T = int(wl.cu_seqlens[-1])
    N = wl.num_blocks
    kc = torch.zeros(N, bs, Hkv, d, dtype=torch.bfloat16, device=device)
    vc = torch.zeros_like(kc)
    bt = torch.as_tensor(wl.block_tables, device=device)
    cu = torch.as_tensor(wl.cu_seqlens, device=device)
    scores = torch.empty(T, dtype=torch.float32, device=device)
    keep = torch.empty(B, budget, dtype=torch.int32, device=device)
    kept = torch.empty(B, dtype=torch.int32, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        pk.pe_prefill_scores(scores, wl.k, wl.v)
        if ev:
            ev[1].record(stream)
        pk.pe_prefill_select(keep, kept, scores, cu, err)
        if ev:
            ev[2].record(stream)
        pk.pe_prefill_pack(kc, vc, bt, wl.k, wl.v, cu, keep, kept, err)
        if ev:
            ev[3].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    if err.item() != 0:
        raise SystemExit(f"device error flag {err.item()} during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks = Clocks(device)
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks_under_load(clocks.stop(), device, lambda: [step() for _ in range(8)],
                            t0.elapsed_time(t1) / 1000.0)
    ms = reduce_max(t0.elapsed_time(t1), world) / args.steps
    per = [[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in evs]
    score_s = statistics.median(p[0] for p in per) / 1000.0
    select_s = statistics.median(p[1] for p in per) / 1000.0
    pack_s = statistics.median(p[2] for p in per) / 1000.0
    # algorithmic bytes: every prompt row of K and V read once plus one fp32 score
    # written per token (score kernel); kept rows read and written (pack)
    score_bytes = T * Hkv * d * 2 * 2 + T * 4
    n_kept = int(kept.sum().item())
    pack_bytes = n_kept * Hkv * d * 2 * 2 * 2 + B * budget * 4
    peak, peak_kind = peaks()
    achieved = score_bytes / score_s / 1e9

    # end to end: prompt rows from pinned host memory, keep sets back to the host
    hk = torch.empty(wl.k.shape, dtype=torch.bfloat16, pin_memory=True)
    hv = torch.empty_like(hk, pin_memory=True)
    hk.copy_(wl.k)
    hv.copy_(wl.v)
    hkeep = torch.empty(keep.shape, dtype=torch.int32, pin_memory=True)
    hkept = torch.empty(kept.shape, dtype=torch.int32, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 10))
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        wl.k.copy_(hk, non_blocking=True)
        wl.v.copy_(hv, non_blocking=True)
        pk.pe_prefill_compress(kc, vc, bt, wl.k, wl.v, cu, scores, keep, kept, err)
        hkeep.copy_(keep, non_blocking=True)
        hkept.copy_(kept, non_blocking=True)
    z.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(a.elapsed_time(z) / e2e_steps, world)
    if err.item() != 0:
        raise SystemExit(f"device error flag {err.item()} during timing")
    cpu = None
    if cpu_baseline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        host_wl = W.PrefillWorkload(cfg, wl.k.cpu(), wl.v.cpu(), wl.cu_seqlens, wl.block_tables, N)
        v_, cores, desc = prefill_oracle_throughput(host_wl, args.cpu_seconds)
        cpu = {"value": v_, "unit": "prompt tokens/s", "cores": cores, "kind": "oracle",
               "sample": desc}
        cpu = with_single_core(cpu, lambda t: prefill_oracle_throughput(host_wl, t),
                               args.cpu_seconds)
    line = {
        "metric": METRIC_P1, "value": world * T / (ms / 1000.0), "unit": "prompt tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": prefill_config(cfg, world),
        "roofline": {"bound": "hbm", "kernel": "pe_prefill_scores", "achieved": achieved,
                     "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic("p1", "prefill_traffic.txt",
                                                 PREFILL_SOURCES["p1"]),
                     "algorithmic_bytes_per_launch": score_bytes,
                     "avg_launch_us": score_s * 1e6,
                     "launch_time_statistic": f"median of {args.steps} launches"},
        "kernels_us": {"pe_prefill_scores": score_s * 1e6,
                       "pe_prefill_select": select_s * 1e6,
                       "pe_prefill_pack": pack_s * 1e6},
        "pack_gbs": pack_bytes / pack_s / 1e9,
        "cpu_baseline": cpu,
        "e2e": {"value": world * T / (e2e_ms / 1000.0), "unit": "prompt tokens/s",
                "h2d_bytes_per_step": 2 * T * Hkv * d * 2,
                "d2h_bytes_per_step": (B * budget + B) * 4, "ms_per_step": e2e_ms},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }
    return line


# ----------------------------------------------------------------------------- chunked prefill
def chunk_flops(cfg):
    """QK^T and PV flops of one chunk step: query token i of a chunk ending at
    context n sees n - chunk + i + 1 tokens; 4*d flops per (row, token, head)."""
    seen = sum(cfg.ctx_len - cfg.chunk + i + 1 for i in range(cfg.chunk))
    return 4.0 * cfg.head_dim * cfg.hq * seen * cfg.batch


def chunk_oracle_throughput(wl, budget_s):
    """The oracle's append + multi-query attention on query-row samples: one
    sequence's chunk, a slice of its query rows at a time (rows cost in
    proportion to the tokens they see, so the sample is scaled by that)."""
    import oracle
    cfg = wl.cfg
    Hkv, d, bs = cfg.hkv, cfg.head_dim, cfg.block_size
    stride = bs * Hkv * d
    kc = W.bits(wl.k_pool).ravel().copy()
    vc = W.bits(wl.v_pool).ravel().copy()
    bt = wl.block_tables[:1]
    oracle.append_kv(W.bits(wl.k_new[:1]), W.bits(wl.v_new[:1]), kc, vc, stride, bt,
                     wl.positions[:1], bs)
    t_total, seen, rows = 0.0, 0, 0
    step = 16
    for r0 in range(0, cfg.chunk, step):
        # rows r0 .. r0+step-1 of the chunk as their own causal chunk ending at their position
        n = cfg.ctx_len - cfg.chunk + r0 + step
        q = W.bits(wl.q[r0:r0 + step])
        t0 = time.perf_counter()
        oracle.paged_prefill(q, np.array([0, step], np.int32), kc, vc, stride, bt,
                             np.array([n], np.int32), Hkv, bs, wl.scale)
        t_total += time.perf_counter() - t0
        seen += sum(n - step + i + 1 for i in range(step))
        rows += step
        if t_total >= budget_s:
            break
    full_seen = cfg.batch * sum(cfg.ctx_len - cfg.chunk + i + 1 for i in range(cfg.chunk))
    step_s = t_total / seen * full_seen
    desc = (f"{rows} query rows of one chunk ({seen} row-token pairs, all heads), "
            f"{t_total:.1f} s, scaled by the {full_seen} row-token pairs of a step")
    return cfg.batch * cfg.chunk / step_s, oracle.threads(), desc


def run_chunked(args, device, world, rank, cpu_baseline=True):
    """One step = append the chunk's K/V rows and run the multi-query attention
    for every sequence of the workload."""
    import paged_kv_cache_396_b200.pagedkv as pk
    cfg = W.CHUNKED[args.workload]
    wl = W.generate_chunked(cfg, device)
    B = cfg.batch
    Tq = B * cfg.chunk
    bt = torch.as_tensor(wl.block_tables, device=device)
    ctx = torch.as_tensor(wl.ctx_lens, device=device)
    pos = torch.as_tensor(wl.positions, device=device)
    cu = torch.as_tensor(wl.cu_q, device=device)
    out = torch.empty(Tq, cfg.hq, cfg.head_dim, dtype=torch.bfloat16, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    # the balanced mode (a workspace given): 256 query tiles are 1.73 waves on 148 SMs;
    # a plan kernel, the first 148 tiles whole and one equal range of the rest per SM
    # (347 against 356 us for one CTA per tile on the same box)
    ws = pk.alloc_prefill_workspace(B, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size,
                                    cfg.chunk, device)
    attn_launches = 3 if ws is not None else 1

    def step(ev=None):
        pk.pa_append_kv(wl.k_new, wl.v_new, wl.k_pool, wl.v_pool, bt, pos, err)
        if ev:
            ev[0].record(stream)
        pk.pa_prefill_attention(out, wl.q, cu, cfg.chunk, wl.k_pool, wl.v_pool, bt, ctx,
                                wl.scale, err, workspace=ws)
        if ev:
            ev[1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    if err.item() != 0:
        raise SystemExit(f"device error flag {err.item()} during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks = Clocks(device)
    time.sleep(0.3)
    total = 0.0
    for k in range(args.steps):
        flush.zero_()                 # L2 flushed between timed steps (K/V is ~140 MB)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        step(evs[k])
        t1.record(stream)
        torch.cuda.synchronize(device)
        total += t0.elapsed_time(t1)
    clk = clocks_under_load(clocks.stop(), device, lambda: [step() for _ in range(8)],
                            total / 1000.0)
    ms = reduce_max(total / args.steps, world)
    attn_s = statistics.median(e[0].elapsed_time(e[1]) for e in evs) / 1000.0
    flops = chunk_flops(cfg)
    peak_t = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"] \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else 1590.0
    achieved = flops / attn_s / 1e12

    # end to end: queries and chunk rows from pinned host memory, output back
    h_in = []
    for t in (wl.q, wl.k_new, wl.v_new):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        h_in.append((h, t))
    h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 20))
    a.record(stream)
    for _ in range(e2e_steps):
        for h, t in h_in:
            t.copy_(h, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)
    z.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(a.elapsed_time(z) / e2e_steps, world)
    if err.item() != 0:
        raise SystemExit(f"device error flag {err.item()} during timing")
    cpu = None
    if cpu_baseline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        host_wl = W.ChunkWorkload(cfg, wl.k_pool.cpu(), wl.v_pool.cpu(), wl.k_new.cpu(),
                                  wl.v_new.cpu(), wl.q.cpu(), wl.cu_q, wl.ctx_lens, wl.positions,
                                  wl.block_tables, wl.num_blocks)
        v_, cores, desc = chunk_oracle_throughput(host_wl, args.cpu_seconds)
        cpu = {"value": v_, "unit": "chunk tokens/s", "cores": cores, "kind": "oracle",
               "sample": desc}
        cpu = with_single_core(cpu, lambda t: chunk_oracle_throughput(host_wl, t),
                               args.cpu_seconds)
    line = {
        "metric": METRIC_P2,
        "value": world * Tq / (ms / 1000.0), "unit": "chunk tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(chunked_config(cfg, world),
                       attention_mode="balanced" if ws is not None else "one CTA per tile"),
        "roofline": {"bound": "tensor", "kernel": "pa_prefill_attention",
                     "achieved": achieved, "peak": peak_t, "peak_source": "measured burst",
                     "unit": "TFLOP/s", "frac": achieved / peak_t,
                     "traffic": recorded_traffic("p2", "prefill_traffic.txt",
                                                 PREFILL_SOURCES["p2"]),
                     "algorithmic_flops_per_launch": flops, "avg_launch_us": attn_s * 1e6,
                     "launch_time_statistic": f"median of {args.steps} launches"},
        "cpu_baseline": cpu,
        "e2e": {"value": world * Tq / (e2e_ms / 1000.0), "unit": "chunk tokens/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for _, t in h_in),
                "d2h_bytes_per_step": out.numel() * out.element_size(),
                "ms_per_step": e2e_ms},
        "gpu_launches": (1 + attn_launches) * args.steps,
        "clocks": clk,
    }
    return line


# ----------------------------------------------------------------------------- decode
def call_stats(call_ms, layers, batch, world):
    """Median duration (ms) of the decode call over every sample, and the decode-only
    throughput it implies: a step decodes `batch` tokens per rank through `layers`
    decode calls, so tokens/s = world * batch / (layers * median call time)."""
    med = statistics.median(call_ms)
    return med, world * batch / (layers * med / 1000.0)


def chunk_plan(steps, per_graph):
    """Steps per graph replay of the timed region: full graphs of `per_graph` steps,
    then one shorter graph for the remainder."""
    full, rest = divmod(steps, per_graph)
    return [per_graph] * full + ([rest] if rest else [])


def run_decode(args, cfg, device, world, rank, cpu_baseline=True):
    """One decode workload: warm-up, K timed steps (CUDA graphs of the step), the
    decode calls' own time and their time inside the step, the end-to-end pass and,
    optionally, the oracle's CPU baseline.  Returns the JSON line as a dict (printed
    by rank 0)."""
    r = Runner(cfg, device, args.num_splits, evict=args.evict, plan=args.plan,
               select=args.select)
    stream = torch.cuda.current_stream(device)
    for _ in range(max(3, args.warmup)):
        r.step()
    torch.cuda.synchronize(device)
    if r.err.item() != 0:
        raise SystemExit(f"device error flag {r.err.item()} during warm-up")
    r.account_bytes()
    use_graph = not args.no_graph
    # steps per captured graph: at least 20 decode calls per replay
    R = max(1, -(-20 // r.L))

    def capture(steps, with_events=False):
        ev = ([[torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)]
               for _ in range(r.L * steps)] if with_events else None)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for k in range(steps):
                r.step(ev[k * r.L:(k + 1) * r.L] if ev else None)
        return g, ev

    plan = chunk_plan(args.steps, R)
    if use_graph:
        # the timed steps carry no events (an event between two kernels of a graph
        # keeps the second from starting while the first drains)
        full_graph = capture(R)[0] if any(n == R for n in plan) else None
        rest_graph = capture(plan[-1])[0] if plan and plan[-1] != R else None
        order = [full_graph if n == R else rest_graph for n in plan]
        for g in {id(g): g for g in order}.values():
            g.replay()
        torch.cuda.synchronize(device)

    # --- device-timed region: exactly K steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks = Clocks(device)
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    if use_graph:
        for g in order:
            g.replay()
    else:
        for k in range(args.steps):
            r.step()
    t_end.record(stream)
    torch.cuda.synchronize(device)

    def soak_steps():
        if use_graph:
            for g in order:
                g.replay()
        else:
            for _ in range(args.steps):
                r.step()

    clk = clocks_under_load(clocks.stop(), device, soak_steps,
                            t_start.elapsed_time(t_end) / 1000.0)
    total_ms = reduce_max(t_start.elapsed_time(t_end), world)
    ms_per_step = total_ms / args.steps
    value = job_tokens_per_s(world, cfg.batch, ms_per_step)

    # --- each decode call inside the step: the step with an event pair around every
    # call, >= 20 calls (after the timed region, so its events do not slow it)
    n_ev = max(1, -(-max(20, args.steps) // r.L))
    if use_graph:
        ge, evs = capture(n_ev, with_events=True)
        ge.replay()
    else:
        evs = [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
               for _ in range(r.L * n_ev)]
        for k in range(n_ev):
            r.step(evs[k * r.L:(k + 1) * r.L])
    torch.cuda.synchronize(device)
    call_ms = [a.elapsed_time(b) for a, b in evs]
    med_in_step_ms, _ = call_stats(call_ms, r.L, cfg.batch, world)

    # --- the decode calls' own time: the step's decode calls back to back (plan once,
    # then one call per layer) in a graph, >= 20 replays, an event pair per replay
    reps = max(20, args.steps)
    if use_graph:
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd):
            r.decode_calls()
        gd.replay()
    torch.cuda.synchronize(device)
    evd = [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
           for _ in range(reps)]
    for e0_, e1_ in evd:
        e0_.record(stream)
        if use_graph:
            gd.replay()
        else:
            r.decode_calls()
        e1_.record(stream)
    torch.cuda.synchronize(device)
    per_call_ms = [a.elapsed_time(b) / r.L for a, b in evd]
    med_ms = reduce_max(statistics.median(per_call_ms), world)
    _, decode_only = call_stats([med_ms], r.L, cfg.batch, world)
    achieved = r.decode_bytes / (med_ms / 1000.0) / 1e9
    peak, peak_kind = peaks()

    # --- end to end: host inputs -> C ABI -> host outputs, copies inside the timed region
    B = cfg.batch
    h_q = torch.empty(r.q.shape, dtype=torch.bfloat16, pin_memory=True)
    h_q.copy_(r.q)
    h_out = torch.empty(r.out.shape, dtype=torch.bfloat16, pin_memory=True)
    h_in = [h_q]
    d_in = [r.q]
    if cfg.append:
        for t in (r.k_new, r.v_new):
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            h.copy_(t)
            h_in.append(h)
            d_in.append(t)
    h_ctx = torch.as_tensor(r.wl.ctx_lens).pin_memory()
    h_pos = torch.as_tensor(r.wl.positions).pin_memory()
    h_in += [h_ctx, h_pos]
    d_in += [r.ctx, r.pos]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = h_out.numel() * h_out.element_size()
    e2e_steps = max(3, min(args.steps, 50))

    def e2e_step():
        for h, dv in zip(h_in, d_in):
            dv.copy_(h, non_blocking=True)
        r.step()
        h_out.copy_(r.out, non_blocking=True)

    if use_graph:
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge):
            e2e_step()
        ge.replay()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        if use_graph:
            ge.replay()
        else:
            e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, world)
    e2e = {"value": job_tokens_per_s(world, B, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
    if r.err.item() != 0:
        raise SystemExit(f"device error flag {r.err.item()} during timing")

    cpu = None
    if cpu_baseline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc = oracle_throughput(r.wl, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
        cpu = with_single_core(cpu, lambda t: oracle_throughput(r.wl, t), args.cpu_seconds)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"fp8_e4m3": "e4m3"}.get(kv_name(cfg), kv_name(cfg)), "data": "synthetic",
        "config": dict(workload_config(cfg), parallelism=f"replicas{world}"),
        "launch": {"decode_kernel": "staged-tc" if r.staged else "general",
                   "evict_scoring": ("incremental score pool" if r.incremental else
                                     "full pass per layer") if cfg.score else None,
                   "partitions": r.partitions, "chunk_tokens": r.chunk_used,
                   "partition_plan": "once per step" if r.per_step_plan else "every call",
                   "block_selection": (("inside the decode call" if r.select_in_call else
                                        "own kernel, second stream" if r.side is not None else
                                        "own kernel") if r.incremental else None),
                   "cuda_graph": use_graph, "steps_per_graph": R if use_graph else None},
        "roofline": {"bound": "hbm", "kernel": {"bf16": "pa_decode", "int8": "pa_decode_int8",
                                               "fp8_e4m3": "pa_decode_fp8"}[kv_name(cfg)],
                     "achieved": achieved, "peak": peak, "peak_source": peak_kind,
                     "unit": "GB/s", "frac": achieved / peak,
                     "frac_of_nominal_8tbs": achieved / 8000.0,
                     "traffic": recorded_traffic(traffic_key(args, cfg)),
                     "algorithmic_bytes_per_launch":
                         r.decode_bytes,
                     "avg_launch_us": med_ms * 1000.0, "launch_time_statistic":
                         f"median over {reps} replays of the step's {r.L} decode calls back "
                         f"to back (plan included), per call",
                     "avg_launch_us_in_step": med_in_step_ms * 1000.0,
                     "in_step_statistic": f"median of {len(call_ms)} decode calls inside "
                         "steps replayed after the timed region, an event pair around each "
                         "(the events keep each call from overlapping its neighbours' "
                         "launch)"},
        "decode_only_tokens_per_s": decode_only,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": r.launches_per_step() * args.steps,
        "clocks": clk,
    }
    del r
    torch.cuda.empty_cache()
    return line


SECONDARY_DEFAULT = "c4,c2,c5,c5-fp8,p1,p2"


def secondary_args(args, spec):
    """The parsed arguments for one secondary workload ("c5-fp8": c5 on e4m3 pools; c2
    runs with the incremental score pool)."""
    import copy
    a = copy.copy(args)
    name, _, kv = spec.partition("-")
    a.workload = name
    a.kv = kv or None
    a.layers = 0
    a.evict = "incremental" if name == "c2" else args.evict
    return a


def run_one(args, device, world, rank, cpu_baseline=True):
    if args.workload in W.PREFILL:
        return run_prefill(args, device, world, rank, cpu_baseline)
    if args.workload in W.CHUNKED:
        return run_chunked(args, device, world, rank, cpu_baseline)
    cfg = workload_cfg(args)
    if args.layers:
        cfg = W.scaled(cfg, layers=args.layers)
    return run_decode(args, cfg, device, world, rank, cpu_baseline)


# ----------------------------------------------------------------------------- main
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    line = run_one(args, device, world, rank)
    spec = args.secondary
    if spec is None:
        spec = SECONDARY_DEFAULT if (args.workload == "c3" and args.kv is None and
                                     not args.layers) else ""
    extra = [w for w in spec.split(",") if w and w != "none"]
    if extra:
        line["secondary"] = [run_one(secondary_args(args, w), device, world, rank,
                                     cpu_baseline=False) for w in extra]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
