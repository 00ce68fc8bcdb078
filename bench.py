#!/usr/bin/env python
"""Benchmark of the CSA / HCA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of seeded synthetic
input already resident in HBM.  The default workload is CSA decode (batch 64,
128K context each, 64 heads x 128 on one shared KV head, m = 4, indexer
8 x 64, top-k 2048, window 128): step = indexer + top-k + sparse attention.
Other workloads: csa_prefill_L4096, csa_prefill_L65536,
hca_decode_B8_N1048576, mixed_decode_B16_N256K_1M, and
csa_decode_B64_N131072_mxfp4_indexer (the default decode with the indexer keys
and queries in 4-bit storage) and csa_decode_B64_N131072_lowprec (also the main
entries in FP8 content + bf16 rotary storage).

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch (weak
scaling, no data-path collective); the step time is the max over ranks.

Rank 0 prints ONE JSON line.  ``--impl reference`` times the fp64 CPU oracle
on the host cores instead (bounded samples of the same workload).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "CSA decode tokens/s & HBM GB/s at 128K–1M ctx; prefill tokens/s & TC util"
DEFAULT_WORKLOAD = synth.CFG_DECODE_128K.name
L2_BYTES = 126 * 1024 * 1024


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------
# workloads (device side)
# ---------------------------------------------------------------------------
class CsaDecode:
    """Step = csa_indexer_topk + csa_sparse_attn_decode over B sequences."""

    def __init__(self, cfg, seed_offset=0):
        import compressed_sparse_kv_03_b200 as csa
        self.csa, self.cfg = csa, cfg
        c = cfg if not seed_offset else synth.CsaDecode(**{**cfg.__dict__, "seed": cfg.seed + seed_offset})
        self.host = synth.csa_decode_inputs(c)
        self.d = {k: v.cuda() for k, v in self.host.items()}
        self.S = cfg.N // cfg.m
        self.seq_id = torch.arange(cfg.B, dtype=torch.int32, device="cuda")
        self.kI = csa.Cache.contiguous(self.d["kI_comp"])
        self.kv = csa.Cache.contiguous(self.d["kv_comp"])
        self.idx = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device="cuda")
        self.cnt = torch.empty((cfg.B,), dtype=torch.int32, device="cuda")
        self.out = torch.empty_like(self.d["q"])
        self.ws_i = csa.Workspace()
        self.ws_a = csa.Workspace()
        self.units = cfg.B
        self.dominant = csa.KERNEL_INDEXER_SCORE
        # algorithmic bytes: every eligible indexer key once, every selected
        # entry and window row once, the queries and outputs once
        sel_rows = min(cfg.k, self.S) + min(cfg.W, cfg.N + 1)
        self.dominant_bytes = cfg.B * self.S * cfg.c_I * 2
        self.step_bytes = (self.dominant_bytes + cfg.B * sel_rows * cfg.d * 2
                           + cfg.B * (2 * cfg.H * cfg.d * 2 + cfg.H_I * cfg.c_I * 2 + cfg.H_I * 4))
        self.bound = "hbm"

    def step(self):
        csa, cfg, d = self.csa, self.cfg, self.d
        csa.indexer_topk(d["qI"], d["w"], self.kI, cfg.m, cfg.k, seq_id=self.seq_id,
                         q_pos=d["pos"], max_entries=self.S, ws=self.ws_i, out=(self.idx, self.cnt, None))
        csa.sparse_attn_decode(d["q"], self.kv, d["win"], d["win_len"], self.idx, self.cnt, cfg.lam,
                               ws=self.ws_a, out=self.out)

    # a step that streams less than twice L2 would find much of its data there
    # on the next step: such workloads flush L2 between steps (outside the
    # timed events)
    def flushes(self):
        return self.step_bytes < 2 * L2_BYTES

    def between_steps(self):
        if self.flushes():
            if getattr(self, "flush", None) is None:
                self.flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
            self.flush.zero_()

    # end to end: per-step inputs come from pinned host memory, the output goes back
    def e2e_setup(self):
        self.pin = {k: self.host[k].pin_memory() for k in ("q", "qI", "w", "win")}
        self.out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.pin.values())
        self.d2h = self.out_h.numel() * self.out_h.element_size()

    def e2e_step(self):
        for k, t in self.pin.items():
            self.d[k].copy_(t, non_blocking=True)
        self.step()
        self.out_h.copy_(self.out, non_blocking=True)

    def config(self):
        c = self.cfg
        return {"workload": c.name, "batch": c.B, "context": c.N, "heads": c.H, "head_dim": c.d,
                "m": c.m, "indexer_heads": c.H_I, "indexer_dim": c.c_I, "top_k": c.k, "window": c.W,
                "l2": (f"L2 flushed between steps ({self.step_bytes / 1e6:.0f} MB streamed per step)"
                       if self.flushes() else
                       f"inputs larger than L2: {self.step_bytes / 1e6:.0f} MB streamed per step")}


class CsaDecodeMxfp4(CsaDecode):
    """CSA decode with the 4-bit indexer: the indexer-key cache holds E2M1
    codes plus one scale byte per 32 elements (quantized once, when the cache
    is built); a step scores and selects from the codes with the new bf16
    indexer queries quantized inside the scorer (csa_indexer_topk_mxfp4),
    then attends as the bf16 step."""

    def __init__(self, cfg, seed_offset=0):
        super().__init__(cfg, seed_offset)
        csa = self.csa
        kc, ks = csa.quantize_mxfp4(self.d.pop("kI_comp"))
        self.kI = csa.Cache(kc.view(-1, kc.shape[-1]), seq_stride=self.S)
        self.kI_scales = ks.view(-1, ks.shape[-1])
        torch.cuda.synchronize()
        sel_rows = min(cfg.k, self.S) + min(cfg.W, cfg.N + 1)
        self.dominant_bytes = cfg.B * self.S * (cfg.c_I // 2 + cfg.c_I // 32)
        self.step_bytes = (self.dominant_bytes + cfg.B * sel_rows * cfg.d * 2
                           + cfg.B * (2 * cfg.H * cfg.d * 2 + cfg.H_I * cfg.c_I * 2 + cfg.H_I * 4))

    def step(self):
        csa, cfg, d = self.csa, self.cfg, self.d
        csa.indexer_topk_mxfp4(d["qI"], d["w"], self.kI, self.kI_scales, cfg.m, cfg.k,
                               seq_id=self.seq_id, q_pos=d["pos"], max_entries=self.S, ws=self.ws_i,
                               out=(self.idx, self.cnt, None))
        csa.sparse_attn_decode(d["q"], self.kv, d["win"], d["win_len"], self.idx, self.cnt, cfg.lam,
                               ws=self.ws_a, out=self.out)

    def config(self):
        c = super().config()
        c["indexer_storage"] = "E2M1 codes + one power-of-two scale byte per 32 (34 B per key)"
        return c


class CsaDecodeLowPrec(CsaDecodeMxfp4):
    """CSA decode with both low-precision caches: the 4-bit indexer keys of
    CsaDecodeMxfp4 and main entries stored as E4M3 content with a scale byte
    per 32 plus the 64 rotary coordinates in bf16 (quantized when the cache is
    built); a step is csa_indexer_topk_mxfp4 + csa_sparse_attn_decode_fp8."""

    ROPE = 64

    def __init__(self, cfg, seed_offset=0):
        super().__init__(cfg, seed_offset)
        csa = self.csa
        kv = self.d.pop("kv_comp")
        codes, scales, rope = csa.quantize_entries_fp8(kv.view(-1, kv.shape[-1]), self.ROPE)
        del kv
        self.kv = csa.Cache(codes, seq_stride=self.S)
        self.kv_scales, self.kv_rope = scales, rope
        torch.cuda.synchronize()
        sel_rows = min(cfg.k, self.S)
        win_rows = min(cfg.W, cfg.N + 1)
        entry_bytes = (cfg.d - self.ROPE) + (cfg.d - self.ROPE) // 32 + 2 * self.ROPE
        self.step_bytes = (self.dominant_bytes + cfg.B * (sel_rows * entry_bytes + win_rows * cfg.d * 2)
                           + cfg.B * (2 * cfg.H * cfg.d * 2 + cfg.H_I * cfg.c_I * 2 + cfg.H_I * 4))

    def step(self):
        csa, cfg, d = self.csa, self.cfg, self.d
        csa.indexer_topk_mxfp4(d["qI"], d["w"], self.kI, self.kI_scales, cfg.m, cfg.k,
                               seq_id=self.seq_id, q_pos=d["pos"], max_entries=self.S, ws=self.ws_i,
                               out=(self.idx, self.cnt, None))
        csa.sparse_attn_decode_fp8(d["q"], self.kv, self.kv_scales, self.kv_rope, d["win"],
                                   d["win_len"], self.idx, self.cnt, cfg.lam, ws=self.ws_a,
                                   out=self.out)

    def config(self):
        c = super().config()
        c["entry_storage"] = ("E4M3 content + one power-of-two scale byte per 32 + 64 bf16 rotary "
                              "coordinates (194 B per entry)")
        return c


class HcaDecode:
    def __init__(self, cfg, seed_offset=0):
        import compressed_sparse_kv_03_b200 as csa
        self.csa, self.cfg = csa, cfg
        self.host = synth.hca_decode_inputs(cfg)
        self.d = {k: v.cuda() for k, v in self.host.items()}
        self.S = cfg.N // cfg.m
        self.kv = csa.Cache.contiguous(self.d["kv_comp"])
        self.out = torch.empty_like(self.d["q"])
        self.ws = csa.Workspace()
        self.units = cfg.B
        self.dominant = csa.KERNEL_ATTENTION
        rows = self.S + min(cfg.W, cfg.N + 1)
        self.dominant_bytes = cfg.B * (rows * cfg.d * 2 + cfg.H * cfg.d * 2)
        self.step_bytes = self.dominant_bytes + cfg.B * cfg.H * cfg.d * 2
        self.bound = "hbm"
        self.flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")

    def step(self):
        cfg, d = self.cfg, self.d
        self.csa.hca_attn(d["q"], self.kv, d["win"], cfg.m, cfg.W, cfg.lam, win_len=d["win_len"],
                          q_pos=d["pos"], max_entries=self.S, ws=self.ws, out=self.out)

    def between_steps(self):
        self.flush.zero_()

    def e2e_setup(self):
        self.pin = {k: self.host[k].pin_memory() for k in ("q", "win")}
        self.out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.pin.values())
        self.d2h = self.out_h.numel() * self.out_h.element_size()

    def e2e_step(self):
        for k, t in self.pin.items():
            self.d[k].copy_(t, non_blocking=True)
        self.step()
        self.out_h.copy_(self.out, non_blocking=True)

    def config(self):
        c = self.cfg
        return {"workload": c.name, "batch": c.B, "context": c.N, "heads": c.H, "head_dim": c.d,
                "m": c.m, "window": c.W, "l2": "L2 flushed between steps (252 MB write)"}


class CsaPrefill:
    """Step = compress main KV + compress indexer keys + indexer/top-k + attention."""

    def __init__(self, cfg, seed_offset=0):
        import compressed_sparse_kv_03_b200 as csa
        self.csa, self.cfg = csa, cfg
        self.host = synth.csa_prefill_inputs(cfg)
        self.d = {k: v.cuda() for k, v in self.host.items()}
        L, m = cfg.L, cfg.m
        S = L // m
        self.kv_comp = torch.empty((S, cfg.d), dtype=torch.bfloat16, device="cuda")
        self.kI_comp = torch.empty((S, cfg.c_I), dtype=torch.bfloat16, device="cuda")
        self.idx = torch.empty((L, cfg.k), dtype=torch.int32, device="cuda")
        self.cnt = torch.empty((L,), dtype=torch.int32, device="cuda")
        self.out = torch.empty_like(self.d["q"])
        self.ws_i, self.ws_a = csa.Workspace(), csa.Workspace()
        self.units = L
        self.dominant = csa.KERNEL_ATTENTION
        elig = [t // m for t in range(L)]
        att_pairs = sum(min(cfg.k, e) + min(cfg.W, t + 1) for t, e in enumerate(elig))
        idx_pairs = sum(elig)
        self.dominant_flops = 4.0 * cfg.H * cfg.d * att_pairs
        self.step_flops = self.dominant_flops + 2.0 * cfg.H_I * cfg.c_I * idx_pairs
        self.bound = "tensor"
        self.flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if L <= 8192 else None

    def step(self):
        csa, cfg, d = self.csa, self.cfg, self.d
        csa.compress_kv(d["kv_raw"], d["Z"], cfg.m, out=self.kv_comp)
        csa.compress_kv(d["kI_raw"], d["ZI"], cfg.m, out=self.kI_comp)
        csa.indexer_topk(d["qI"], d["w"], csa.Cache(self.kI_comp), cfg.m, cfg.k, ws=self.ws_i,
                         out=(self.idx, self.cnt, None))
        csa.sparse_attn_prefill(d["q"], self.kv_comp, d["kv_raw"], self.idx, self.cnt, cfg.W, cfg.lam,
                                ws=self.ws_a, out=self.out)

    def between_steps(self):
        if self.flush is not None:
            self.flush.zero_()

    def e2e_setup(self):
        keys = ("q", "kv_raw", "Z", "kI_raw", "ZI", "qI", "w")
        self.pin = {k: self.host[k].pin_memory() for k in keys}
        self.out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.pin.values())
        self.d2h = self.out_h.numel() * self.out_h.element_size()

    def e2e_step(self):
        for k, t in self.pin.items():
            self.d[k].copy_(t, non_blocking=True)
        self.step()
        self.out_h.copy_(self.out, non_blocking=True)

    def config(self):
        c = self.cfg
        return {"workload": c.name, "seq_len": c.L, "heads": c.H, "head_dim": c.d, "m": c.m,
                "indexer_heads": c.H_I, "indexer_dim": c.c_I, "top_k": c.k, "window": c.W,
                "l2": "L2 flushed between steps" if self.flush is not None
                else "inputs larger than L2 (1.1 GB of queries per step)"}


class MixedDecode:
    def __init__(self, cfg, seed_offset=0):
        import compressed_sparse_kv_03_b200 as csa
        self.csa, self.cfg = csa, cfg
        self.host = synth.mixed_decode_inputs(cfg)
        self.pos = self.host["pos"].cuda()
        self.seq_id = torch.arange(cfg.B, dtype=torch.int32, device="cuda")
        self.layers = []
        step_bytes = dom = 0
        for lay in self.host["layers"]:
            L = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
            S = [int(s) for s in lay["S"]]
            L["max_S"] = max(S)
            L["kv"] = csa.Cache(L["kv_pool"], page_table=L["page_table"], page_size=cfg.page_size)
            L["out"] = torch.empty_like(L["q"])
            L["ws"] = csa.Workspace()
            if lay["kind"] == "csa":
                L["kI"] = csa.Cache(L["kI_pool"], page_table=L["page_table"], page_size=cfg.page_size)
                L["idx"] = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device="cuda")
                L["cnt"] = torch.empty((cfg.B,), dtype=torch.int32, device="cuda")
                L["ws_i"] = csa.Workspace()
                kb = sum(S) * cfg.c_I * 2
                dom += kb
                step_bytes += kb + sum(min(cfg.k, s) + cfg.W for s in S) * cfg.d * 2
            else:
                step_bytes += sum(s + cfg.W for s in S) * cfg.d * 2
            step_bytes += cfg.B * 2 * cfg.H * cfg.d * 2
            self.layers.append(L)
        self.units = cfg.B
        self.dominant = csa.KERNEL_INDEXER_SCORE
        self.dominant_bytes = dom / 2      # per launch: two CSA layers launch it
        self.step_bytes = step_bytes
        self.bound = "hbm"

    def step(self):
        csa, cfg = self.csa, self.cfg
        for L in self.layers:
            if L["kind"] == "csa":
                csa.indexer_topk(L["qI"], L["w"], L["kI"], L["m"], cfg.k, seq_id=self.seq_id,
                                 q_pos=self.pos, max_entries=L["max_S"], ws=L["ws_i"],
                                 out=(L["idx"], L["cnt"], None))
                csa.sparse_attn_decode(L["q"], L["kv"], L["win"], L["win_len"], L["idx"], L["cnt"],
                                       cfg.lam, ws=L["ws"], out=L["out"])
            else:
                csa.hca_attn(L["q"], L["kv"], L["win"], L["m"], cfg.W, cfg.lam, win_len=L["win_len"],
                             q_pos=self.pos, max_entries=L["max_S"], ws=L["ws"], out=L["out"])

    def e2e_setup(self):
        self.pin = []
        for L, lay in zip(self.layers, self.host["layers"]):
            for k in ("q", "win") + (("qI", "w") if lay["kind"] == "csa" else ()):
                self.pin.append((L[k], lay[k].pin_memory()))
        self.out_h = [torch.empty(L["out"].shape, dtype=torch.bfloat16).pin_memory() for L in self.layers]
        self.h2d = sum(t.numel() * t.element_size() for _, t in self.pin)
        self.d2h = sum(t.numel() * t.element_size() for t in self.out_h)

    def e2e_step(self):
        for dst, src in self.pin:
            dst.copy_(src, non_blocking=True)
        self.step()
        for L, oh in zip(self.layers, self.out_h):
            oh.copy_(L["out"], non_blocking=True)

    def config(self):
        c = self.cfg
        return {"workload": c.name, "batch": c.B, "context": f"U[{c.N_lo}, {c.N_hi}]",
                "layers": "/".join(c.layers), "heads": c.H, "head_dim": c.d, "top_k": c.k,
                "window": c.W, "page_size": c.page_size,
                "l2": f"inputs larger than L2: {self.step_bytes / 1e6:.0f} MB streamed per step"}


KERNEL_NAMES = {0: "indexer_score", 1: "topk_select", 2: "attention", 3: "merge", 4: "compress",
                5: "quantize", 6: "topk_sample"}

RUNNERS = {
    synth.CFG_DECODE_128K.name: (CsaDecode, synth.CFG_DECODE_128K),
    synth.CFG_HCA_1M.name: (HcaDecode, synth.CFG_HCA_1M),
    synth.CFG_PREFILL_4K.name: (CsaPrefill, synth.CFG_PREFILL_4K),
    synth.CFG_PREFILL_64K.name: (CsaPrefill, synth.CFG_PREFILL_64K),
    synth.CFG_MIXED.name: (MixedDecode, synth.CFG_MIXED),
    synth.CFG_DECODE_128K_MXFP4.name: (CsaDecodeMxfp4, synth.CFG_DECODE_128K_MXFP4),
    synth.CFG_DECODE_128K_LOWPREC.name: (CsaDecodeLowPrec, synth.CFG_DECODE_128K_LOWPREC),
}


# ---------------------------------------------------------------------------
# multi-rank aggregation (weak scaling: every rank runs its own batch)
# ---------------------------------------------------------------------------
def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity when the
    process group is not initialised)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_rank, world, ms_per_step):
    """Whole-job units per second: every rank processed units_per_rank in
    (at most) the slowest rank's step time."""
    return units_per_rank * world / (ms_per_step / 1e3)


def rank_seed_offset(rank):
    """Each rank draws its own batch."""
    return int(rank)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(name, budget_s):
    """Run the oracle on a bounded sample of the workload; returns
    (units done, seconds, description, threads)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        threads = 1
    cls, cfg = RUNNERS[name]
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    if cls is CsaDecodeMxfp4 or cls is CsaDecodeLowPrec:
        from oracle import fp8_entry as ofp8
        from oracle import mxfp4 as ofp4
        host = synth.csa_decode_inputs(cfg, B=min(cfg.B, 16))
        done, secs = 0, 0.0
        while done < host["q"].shape[0] and secs < budget_s:
            b = done
            kc, ks = ofp4.mxfp4_quantize(f(host["kI_comp"][b]))   # cache contents: not timed
            kv_b = f(host["kv_comp"][b])
            if cls is CsaDecodeLowPrec:                           # cache contents: not timed
                kv_b = ofp8.entry_dequantize(*ofp8.entry_quantize(kv_b, CsaDecodeLowPrec.ROPE))
            t0 = time.perf_counter()
            qc, qs = ofp4.mxfp4_quantize(f(host["qI"][b]))
            n = oracle.eligible_entries(int(host["pos"][b]), cfg.m)
            sel = oracle.topk_select(ofp4.indexer_scores_mxfp4(qc, qs, f(host["w"][b]), kc[:n], ks[:n]),
                                     cfg.k)
            rows = np.concatenate([kv_b[sel], f(host["win"][b])[:int(host["win_len"][b])]])
            oracle.attend_shared_kv(f(host["q"][b]), rows, cfg.lam)
            secs += time.perf_counter() - t0
            done += 1
        return (done, secs, f"{done} of {cfg.B} sequences, full decode step each "
                f"(key quantization of the cache not timed)", threads)
    if cls is CsaDecode:
        host = synth.csa_decode_inputs(synth.CsaDecode(**{**cfg.__dict__, "B": min(cfg.B, 64)}))
        done, t0 = 0, time.perf_counter()
        while done < cfg.B and (time.perf_counter() - t0) < budget_s:
            b = done
            oracle.csa_decode(f(host["q"][b:b + 1]), [f(host["kv_comp"][b])], [f(host["kI_comp"][b])],
                              f(host["qI"][b:b + 1]), f(host["w"][b:b + 1]), f(host["win"][b:b + 1]),
                              host["win_len"][b:b + 1].numpy(), host["pos"][b:b + 1].numpy(),
                              cfg.m, cfg.k, cfg.lam)
            done += 1
        return done, time.perf_counter() - t0, f"{done} of {cfg.B} sequences, full decode step each", threads
    if cls is HcaDecode:
        host = synth.hca_decode_inputs(cfg)
        done, t0 = 0, time.perf_counter()
        while done < cfg.B and (time.perf_counter() - t0) < budget_s:
            b = done
            oracle.hca_decode(f(host["q"][b:b + 1]), [f(host["kv_comp"][b])], f(host["win"][b:b + 1]),
                              host["win_len"][b:b + 1].numpy(), host["pos"][b:b + 1].numpy(), cfg.m, cfg.lam)
            done += 1
        return done, time.perf_counter() - t0, f"{done} of {cfg.B} sequences", threads
    if cls is CsaPrefill:
        host = synth.csa_prefill_inputs(cfg)
        t0 = time.perf_counter()
        kvc = oracle.bf16_round(oracle.pool_block(f(host["kv_raw"]), f(host["Z"]), cfg.m))
        kIc = oracle.bf16_round(oracle.pool_block(f(host["kI_raw"]), f(host["ZI"]), cfg.m))
        rng = np.random.default_rng(0)
        order = rng.permutation(cfg.L)
        done = 0
        kv_raw = f(host["kv_raw"])
        qv, qIv, wv = (_RowView(f, host[k]) for k in ("q", "qI", "w"))
        while done < cfg.L and (time.perf_counter() - t0) < budget_s:
            t = int(order[done])
            idx, cnt = oracle.csa_prefill_topk(qIv, wv, kIc, cfg.m, cfg.k, rows=[t])
            oracle.csa_prefill_attention(qv, kvc, kv_raw, idx, cnt, cfg.W, cfg.lam, rows=[t])
            done += 1
        return (done, time.perf_counter() - t0,
                f"compression of all {cfg.L} tokens + {done} random query rows (scaled per token)", threads)
    # mixed
    host = synth.mixed_decode_inputs(cfg)
    done, t0 = 0, time.perf_counter()
    while done < cfg.B and (time.perf_counter() - t0) < budget_s:
        b = done
        for lay in host["layers"]:
            S = int(lay["S"][b])
            kv_b = f(oracle.unpage(lay["kv_pool"], lay["page_table"][b], S, cfg.page_size))
            if lay["kind"] == "csa":
                kI_b = f(oracle.unpage(lay["kI_pool"], lay["page_table"][b], S, cfg.page_size))
                oracle.csa_decode(f(lay["q"][b:b + 1]), [kv_b], [kI_b], f(lay["qI"][b:b + 1]),
                                  f(lay["w"][b:b + 1]), f(lay["win"][b:b + 1]),
                                  lay["win_len"][b:b + 1].numpy(), host["pos"][b:b + 1].numpy(),
                                  lay["m"], cfg.k, cfg.lam)
            else:
                oracle.hca_decode(f(lay["q"][b:b + 1]), [kv_b], f(lay["win"][b:b + 1]),
                                  lay["win_len"][b:b + 1].numpy(), host["pos"][b:b + 1].numpy(),
                                  lay["m"], cfg.lam)
        done += 1
    return done, time.perf_counter() - t0, f"{done} of {cfg.B} sequences, all 4 layers", threads


class _RowView:
    """Tensor-like object whose rows are materialised in float64 on demand."""

    def __init__(self, f, t):
        self.f, self.t = f, t
        self.shape = tuple(t.shape)

    def __getitem__(self, i):
        return self.f(self.t[i])


# ---------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The base contract's reference arm: the fp64 oracle on host cores."""
    if rank != 0:
        return
    name = args.workload
    cls, cfg = RUNNERS[name]
    per_step = max(args.step_budget, 0.5)
    for _ in range(args.warmup):
        oracle_sample(name, per_step / 4)
    units = secs = 0.0
    desc, threads = "", 1
    for _ in range(args.steps):
        u, s, desc, threads = oracle_sample(name, per_step)
        units += u
        secs += s
    value = units / secs if secs else 0.0
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": name, "arm": "fp64 CPU oracle, bounded samples"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import compressed_sparse_kv_03_b200 as csa
    torch.cuda.set_device(local_rank)
    cls, cfg = RUNNERS[args.workload]
    if args.batch and hasattr(cfg, "B"):
        cfg = dataclasses.replace(cfg, B=args.batch, name=f"{cfg.name}_B{args.batch}")
    if args.seq_len and hasattr(cfg, "L"):
        cfg = dataclasses.replace(cfg, L=args.seq_len, name=f"{cfg.name}_L{args.seq_len}")
    if args.batch_invariant:
        csa.set_batch_invariant(True)
    line = measure(args, args.workload, cls, cfg, args.steps, args.warmup, rank, world, local_rank)
    # the metric's prefill half: the L=65536 prefill measured in the same run
    # (one GPU, default decode workload), as a sub-record with its own
    # roofline (tensor) and oracle baseline
    if (args.workload == DEFAULT_WORKLOAD and world == 1 and not args.no_prefill
            and not args.batch and not args.batch_invariant):
        import gc
        gc.collect()
        torch.cuda.empty_cache()
        pname = synth.CFG_PREFILL_64K.name
        pcls, pcfg = RUNNERS[pname]
        sub = measure(args, pname, pcls, pcfg, max(3, min(args.steps, 5)), 3, rank, world,
                      local_rank)
        keep = ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "higher_is_better",
                "dtype", "config", "roofline", "e2e", "clocks", "gpu_launches", "kernels_us",
                "cpu_baseline")
        line["prefill"] = {k: sub[k] for k in keep if k in sub}
        line["prefill"]["metric"] = "CSA prefill tokens/s & tensor-core utilisation"
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure(args, name, cls, cfg, K, warmup, rank, world, local_rank):
    """Time one workload (warm-up, K timed graph replays, per-kernel
    breakdown, end to end, oracle baseline on rank 0 at N=1) and return its
    JSON record."""
    import compressed_sparse_kv_03_b200 as csa
    import torch.distributed as dist
    W = cls(cfg, seed_offset=rank_seed_offset(rank))
    pk = peaks()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    def between():
        if hasattr(W, "between_steps"):
            W.between_steps()

    # warm-up (eager)
    for _ in range(warmup):
        W.step()
        between()
    torch.cuda.synchronize()

    # one CUDA graph per timed step, each with its own events around the
    # dominant kernel; L2 flushes (where a workload needs them) run between
    # the step events, outside the timed time
    kids = list(KERNEL_NAMES)
    kev = {k: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)] for k in kids}
    ev = kev[W.dominant]
    st = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for pair in st:              # torch creates CUDA events lazily, on first record
        pair[0].record(stream)
        pair[1].record(stream)
    for pair in [p for k in kids for p in kev[k]]:
        pair[1].record(stream)   # end before begin: a kernel that never runs in the step
        pair[0].record(stream)   # keeps a negative interval and is left out
    torch.cuda.synchronize()

    def attach(i):
        for k in kids:
            csa.set_timing_events(k, kev[k][i][0], kev[k][i][1])

    def detach():
        for k in kids:
            csa.set_timing_events(k)
    use_graph = not args.no_graph
    launches_before = csa.launch_count()
    graphs, bgraphs = [], []
    if use_graph:
        # timed graphs hold the step alone (an event node between two kernels
        # would also stop them overlapping); the per-kernel times, the dominant
        # kernel's included, come from separate, untimed replays of graphs with
        # events around every kernel
        for i in range(K):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                W.step()
            graphs.append(g)
        launches = csa.launch_count() - launches_before
        for i in range(K):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                attach(i)
                W.step()
                detach()
            bgraphs.append(g)
        for g in graphs[:2]:         # untimed warm replays
            g.replay()
            between()
        torch.cuda.synchronize()
    clocks = Clocks(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    launches_before = csa.launch_count()
    for i in range(K):
        st[i][0].record(stream)
        if use_graph:
            graphs[i].replay()
        else:
            csa.set_timing_events(W.dominant, ev[i][0], ev[i][1])
            W.step()
            csa.set_timing_events(W.dominant)
        st[i][1].record(stream)
        between()
    if not use_graph:
        launches = csa.launch_count() - launches_before
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = sum(b.elapsed_time(e) for b, e in st)
    # per-kernel breakdown, outside the timed region
    for i in range(K):
        if use_graph:
            bgraphs[i].replay()
        else:
            attach(i)
            W.step()
            detach()
        between()
    torch.cuda.synchronize()
    # the dominant kernel: event times of its launches in the breakdown replays
    # (graph mode) or in the timed eager steps
    dom_ms = [b.elapsed_time(e) for b, e in ev]
    kernels_us = {}
    for k in kids:
        t = statistics.median(b.elapsed_time(e) for b, e in kev[k]) * 1e3
        if t > 0.05:
            kernels_us[KERNEL_NAMES[k]] = round(t, 2)
    del graphs, bgraphs
    ms = max_over_ranks([ms], device="cuda")[0]
    ms_per_step = ms / K
    flush_note = ""
    value = job_throughput(W.units, world, ms_per_step)

    # end to end through the public API: host inputs in, result out, every step
    W.e2e_setup()
    for _ in range(2):
        W.e2e_step()
    torch.cuda.synchronize()
    barrier()
    # events around each step, so that an L2 flush between steps stays outside
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        eev[i][0].record(stream)
        W.e2e_step()
        eev[i][1].record(stream)
        between()
    torch.cuda.synchronize()
    e_ms = max_over_ranks([sum(b.elapsed_time(e) for b, e in eev)], device="cuda")[0]
    e2e_value = job_throughput(W.units, world, e_ms / K)

    dom_avg = sum(dom_ms) / len(dom_ms)
    kname = "indexer_score" if W.dominant == csa.KERNEL_INDEXER_SCORE else "attention"
    traffic = args.traffic if args.traffic is not None else recorded_traffic(kname, W.config())
    if W.bound == "hbm":
        achieved = W.dominant_bytes / (dom_avg / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic, "kernel": kname,
                "kernel_ms": dom_avg, "algorithmic_bytes": W.dominant_bytes,
                "peak_source": f"{pk['source']} hbm_gbs",
                "step_hbm_frac": W.step_bytes / (ms_per_step / 1e3) / 1e9 / pk["hbm_gbs"]}
    else:
        achieved = W.dominant_flops / (dom_avg / 1e3) / 1e12
        peak = pk["bf16_tflops_sustained"] if K * dom_avg > 1000 else pk["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "kernel": kname,
                "kernel_ms": dom_avg, "algorithmic_flops": W.dominant_flops,
                "peak_source": f"{pk['source']} bf16",
                "step_tc_frac": W.step_flops / (ms_per_step / 1e3) / 1e12 / peak}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded torch CPU generator, N(0,1) / U(0,1))",
            "config": {**W.config(), "parallelism": f"dp{world}" + flush_note,
                       **({"batch_invariant": True} if args.batch_invariant else {}),
                       "timing": "one CUDA graph per step, CUDA events per step" if use_graph
                       else "eager launches, CUDA events per step"},
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": W.h2d,
                    "d2h_bytes_per_step": W.d2h},
            "clocks": clk, "gpu_launches": int(launches),
            "kernels_us": {"median_per_step": kernels_us,
                           "note": "CUDA events around each library kernel in untimed replays "
                                   "of the step (event nodes add about a microsecond or two to "
                                   "each); for a kernel launched more than once in a step, its "
                                   "last launch"}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        u, s, desc, threads = oracle_sample(name, args.cpu_budget)
        line["cpu_baseline"] = {"value": u / s if s else 0.0, "unit": "tokens/s", "cores": threads,
                                "kind": "oracle", "sample": desc}
    del W
    return line



def recorded_traffic(kernel, config, root=None):
    """DRAM bytes per launch of `kernel` on this workload from a committed ncu
    capture (profiles/dram_traffic.json under `root`, default this directory),
    or None when there is none or the kernel's source changed since it was
    taken."""
    import hashlib
    here = root or os.path.dirname(os.path.abspath(__file__))
    try:
        with open(os.path.join(here, "profiles", "dram_traffic.json")) as f:
            entries = json.load(f)["entries"]
    except (OSError, ValueError, KeyError):
        return None
    for e in entries:
        if e.get("kernel") != kernel or any(config.get(k) != v for k, v in e["config"].items()):
            continue
        try:
            with open(os.path.join(here, e["source"]), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != e["source_sha256"]:
                    return None
        except OSError:
            return None
        return float(e["bytes_per_launch"])
    return None

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(RUNNERS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-graph", action="store_true", help="time eager launches instead of a graph")
    ap.add_argument("--batch", type=int, default=0, help="override the decode batch (profiling runs)")
    ap.add_argument("--seq-len", type=int, default=0, help="override the prefill length (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill sub-record of the default decode run")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work (cpu_baseline)")
    ap.add_argument("--step-budget", type=float, default=4.0, help="seconds per reference-arm step")
    ap.add_argument("--batch-invariant", action="store_true",
                    help="decode attention in batch-invariant mode (fixed 512-row slices)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the dominant kernel, if captured for the current kernel source")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
