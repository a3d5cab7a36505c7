"""Benchmark of the CSA / HCA attention forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
        NAME: csa_prefill (default) | hca_prefill | decode128k | decode1m | decode128k_fp4 (MXFP4 indexer)
              | hca_decode1m | append128k (compressor decode step) | out_proj (grouped output projection)
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed on this host's cores

The default line (the V4-Flash CSA prefill layer) carries a "side" object with the V4-Flash HCA
prefill layer and the two CSA decode batches (128K context, and 1M context with the FP8 cache), each
timed the same way. A step is one full pass of the layer forward over one batch of synthetic inputs
already resident in HBM: compress -> lightning indexer + top-k -> sparse + window attention for CSA prefill
(the V4-Flash layer, S=8192), compress -> dense attention for HCA prefill (S=65536), and
indexer + top-k -> attention for decode. Per-step CUDA events on the launching stream time
every kernel phase; L2 is flushed (a 256 MiB write) between steps, outside the timed events.
Multi-GPU runs are independent replicas (the path has no exchange step): every rank runs the same
workload and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import WORKLOADS, decode_inputs, prefill_inputs, proj_inputs  # noqa: E402

WORKLOAD_IDS = {"csa_prefill": 1, "hca_prefill": 2, "decode128k": 3, "decode1m": 4, "hca_decode1m": 5,
                "decode128k_fp4": 8,
                "append128k": 6, "out_proj": 7}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu record, or None when the
    kernel source changed since the counters were taken (or nothing was recorded)."""
    import hashlib
    try:
        for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
            if line.startswith("#") or not line.strip():
                continue
            wl, src, sha, nbytes = line.split()
            if wl != workload:
                continue
            path = os.path.join(ROOT, "long_context_sparse_fwd_b200", "csrc", src)
            if hashlib.sha256(open(path, "rb").read()).hexdigest()[:16] == sha:
                return int(nbytes)
    except Exception:
        return None
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---- algorithmic work (flops / bytes the method needs, not what a kernel happens to do) ----------

def csa_attention_flops(wl):
    """4*D flops per (query, head, key): QK^T and PV over the full head dim."""
    t = np.arange(wl.S, dtype=np.int64)
    n_win = np.minimum(wl.W, t + 1)
    vis = np.minimum((t + 1) // wl.m, wl.T)
    n_sel = np.minimum(wl.topk, vis) if wl.kind == "csa_prefill" else vis
    return float((n_win + n_sel).sum()) * wl.H * 4.0 * wl.D


def index_flops(wl):
    t = np.arange(wl.S, dtype=np.int64)
    vis = np.minimum((t + 1) // wl.m, wl.T)
    return float(vis.sum()) * 2.0 * wl.HI * wl.dI


def attention_bytes(wl):
    """Each tensor once: q in, o out (fp32), entries and window rows once."""
    return wl.S * wl.H * wl.D * 2 + wl.S * wl.H * wl.D * 4 + wl.T * wl.D * 2 + wl.S * wl.D * 2


def proj_flops(wl):
    """Two GEMMs per token: G groups of (H/G)*D -> R, then G*R -> hidden."""
    K = wl.H // wl.o_groups * wl.D
    return 2.0 * wl.S * (wl.o_groups * K * wl.o_rank + wl.o_groups * wl.o_rank * wl.hidden)


def append_bytes(wl, B):
    """m decode-step appends per sequence: read the token and gate, write both into the state and the
    rotated row into the window ring; the closing append reads the L-token window and writes the entry."""
    D = wl.D
    per_seq = wl.m * (4 * D + 4 * D + 2 * D) + wl.L * 4 * D + 2 * D
    return float(B * per_seq)


def decode_bytes(wl, B):
    """k^I stream + selected entries + window rows + q + o per step (HCA decode: every entry, no indexer)."""
    T, D, r = wl.T, wl.D, wl.r
    ent = (D - r) + 4 + 2 * r if wl.cache == "fp8" else 2 * D
    if wl.kind == "hca_decode":
        return float(B * (T * ent + wl.W * D * 2 + wl.H * D * 2 + wl.H * D * 4))
    if wl.index_fmt == "fp4":   # MXFP4 k^I (codes + E8M0 scales); q^I quantised each step
        ki = T * (wl.dI // 2 + wl.dI // 32)
        qi = wl.HI * (wl.dI * 2 + 2 * (wl.dI // 2 + wl.dI // 32) + 4)
    else:
        ki = T * wl.dI * 2
        qi = wl.HI * (wl.dI * 2 + 4)
    per_seq = ki + wl.topk * ent + wl.W * D * 2 + wl.H * D * 2 + wl.H * D * 4 + qi
    return float(B * per_seq)


# ---- clocks sampled during the timed region ------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, f in enumerate(fl) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


# ---- the GPU arm ---------------------------------------------------------------------------------

class Step:
    """One workload's step, split into its kernel phases with events between them."""

    def __init__(self, name, wl, csa, dev):
        self.name, self.wl, self.csa, self.dev = name, wl, csa, dev
        self.stream = torch.cuda.current_stream()
        if wl.kind == "out_proj":
            self.x = proj_inputs(wl, device=dev)
            self.z = torch.empty(wl.S, wl.o_groups * wl.o_rank, dtype=torch.bfloat16, device=dev)
            self.o = torch.empty(wl.S, wl.hidden, dtype=torch.bfloat16, device=dev)
            self.ws = torch.empty(csa.workspace_size("out_proj"), dtype=torch.uint8, device=dev)
            self.phases = ["out_proj"]
            self.units = wl.S
        elif wl.kind == "compress_append":
            # m consecutive decode-step appends (positions P0 .. P0+m-1, the last closes an entry) for B
            # sequences whose histories already fill the pooling state and the window ring
            self.B, D, L, W = wl.B, wl.D, wl.L, wl.W
            g = torch.Generator(device=dev)
            g.manual_seed(wl.seed)
            self.x = {"kv": torch.randn(wl.m, self.B, D, generator=g, device=dev).to(torch.bfloat16),   # [position, seq, D]
                      "gate": torch.randn(wl.m, self.B, D, generator=g, device=dev).to(torch.bfloat16),
                      "pos_bias": torch.randn(L, generator=g, device=dev) * 0.02}
            self.state_x = torch.randn(self.B, L, D, generator=g, device=dev).to(torch.bfloat16)
            self.state_g = torch.randn(self.B, L, D, generator=g, device=dev).to(torch.bfloat16)
            self.C = torch.empty(self.B, wl.T, D, dtype=torch.bfloat16, device=dev)
            self.win = torch.empty(self.B, W, D, dtype=torch.bfloat16, device=dev)
            self.P0 = wl.ctx - wl.m
            self.phases = ["append"]
            self.units = self.B * wl.m
        elif wl.kind in ("csa_decode", "hca_decode"):
            self.B = wl.B
            self.x = decode_inputs(wl, device=dev)
            self.P = wl.ctx - 1
            self.o = torch.empty(self.B, wl.H, wl.D, dtype=torch.float32, device=dev)
            if wl.kind == "csa_decode":
                self.idx = torch.empty(self.B, wl.topk, dtype=torch.int32, device=dev)
                if wl.index_fmt == "fp4":   # the cache holds k^I as MXFP4; q^I is quantised every step
                    self.x["kc"], self.x["ks"] = csa.quantize_mxfp4(self.x["kI"])
                    del self.x["kI"]
                    self.qc = torch.empty(self.B, wl.HI, wl.dI // 2, dtype=torch.uint8, device=dev)
                    self.qs = torch.empty(self.B, wl.HI, wl.dI // 32, dtype=torch.uint8, device=dev)
                self.ws = torch.empty(csa.workspace_size("decode", B=self.B, T=wl.T, k=wl.topk), dtype=torch.uint8,
                                      device=dev)
            else:
                self.ws = torch.empty(csa.workspace_size("hca_decode", B=self.B, T=wl.T, W=wl.W), dtype=torch.uint8,
                                      device=dev)
            self.phases = ["decode"]
            self.units = self.B
        else:
            self.x = prefill_inputs(wl, device=dev)
            S, T = wl.S, wl.T
            self.C = torch.empty(T, wl.D, dtype=torch.bfloat16, device=dev)
            self.kv_rot = torch.empty(S, wl.D, dtype=torch.bfloat16, device=dev)
            self.o = torch.empty(S, wl.H, wl.D, dtype=torch.float32, device=dev)
            if wl.kind == "csa_prefill":
                self.idx = torch.empty(S, wl.topk, dtype=torch.int32, device=dev)
                self.ws = torch.empty(csa.workspace_size("csa_forward", S=S, T=T), dtype=torch.uint8, device=dev)
                self.phases = ["compress", "index_topk", "attend"]
            else:
                self.ws = torch.empty(csa.workspace_size("hca_forward"), dtype=torch.uint8, device=dev)
                self.phases = ["compress", "attend"]
            self.units = S
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.phases) + 1)]

    def launches_per_step(self):
        # library kernels per step on the tensor-core paths these workloads take:
        # prefill: compress_entries + rotate_rows, fused index/top-k (CSA), attention;
        # decode: index scan, chunk top-k, merge, split attention, combine
        # decode: index scan, three top-k kernels, split attention, combine (plus one memset); HCA
        # decode: split attention and combine
        # CSA decode: index scan, top-k (one kernel up to 32768 entries per sequence, else three), split
        # attention, combine; the FP4 indexer adds the quantisation of q^I
        if self.wl.kind == "csa_decode":
            return (4 if self.wl.T <= 32768 else 6) + (1 if self.wl.index_fmt == "fp4" else 0)
        return {"csa_prefill": 4, "hca_prefill": 3, "hca_decode": 2,
                "compress_append": self.wl.m, "out_proj": 2}[self.wl.kind]

    def run(self, timed: bool):
        wl, x, csa = self.wl, self.x, self.csa
        ev = self.events
        if timed:
            ev[0].record(self.stream)
        if wl.kind == "out_proj":
            csa.out_proj(x["o"], x["wa"], x["wb"], z=self.z, out=self.o, workspace=self.ws)
            if timed:
                ev[1].record(self.stream)
            return
        if wl.kind == "compress_append":
            for i in range(wl.m):
                csa.compress_append(x["kv"][i], x["gate"][i], x["pos_bias"], self.state_x, self.state_g,
                                    self.P0 + i, wl.m, wl.r, wl.theta_cmp, wl.theta_tok, C=self.C, win=self.win)
            if timed:
                ev[1].record(self.stream)
            return
        if wl.kind in ("csa_decode", "hca_decode"):
            kw = dict(C=x["C"]) if wl.cache == "bf16" else dict(c8=x["c8"], c8_scale=x["scale"], c_rope=x["rope"])
            if wl.kind == "csa_decode" and wl.index_fmt == "fp4":
                csa.quantize_mxfp4(x["qI"], codes=self.qc, scales=self.qs)
                csa.decode_fp4(x["q"], self.qc, self.qs, x["w"], x["kc"], x["ks"], x["win"], x["sinks"], self.P,
                               wl.topk, wl.r, wl.theta_tok, wl.theta_cmp, o=self.o, idx=self.idx, workspace=self.ws,
                               **kw)
            elif wl.kind == "csa_decode":
                csa.decode(x["q"], x["qI"], x["w"], x["kI"], x["win"], x["sinks"], self.P, wl.topk, wl.r,
                           wl.theta_tok, wl.theta_cmp, o=self.o, idx=self.idx, workspace=self.ws, **kw)
            else:
                csa.hca_decode(x["q"], x["win"], x["sinks"], self.P, wl.r, wl.theta_tok, wl.theta_cmp, o=self.o,
                               workspace=self.ws, **kw)
            if timed:
                ev[1].record(self.stream)
            return
        csa.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok, C=self.C,
                     kv_rot=self.kv_rot)
        if timed:
            ev[1].record(self.stream)
        if wl.kind == "csa_prefill":
            csa.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, idx=self.idx, workspace=self.ws)
            if timed:
                ev[2].record(self.stream)
            csa.attend(x["q"], self.C, self.kv_rot, self.idx, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok,
                       wl.theta_cmp, o=self.o, workspace=self.ws)
            if timed:
                ev[3].record(self.stream)
        else:
            csa.hca_attend(x["q"], self.C, self.kv_rot, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp,
                           o=self.o, workspace=self.ws)
            if timed:
                ev[2].record(self.stream)

    def phase_ms(self):
        return [self.events[i].elapsed_time(self.events[i + 1]) for i in range(len(self.phases))]


def e2e_run(step, steps, warmup):
    """Same metric through the public fused call with host buffers: each step copies its inputs
    from pinned host memory, runs the forward, and reads the output back."""
    csa, wl, dev = step.csa, step.wl, step.dev
    host = {k: v.cpu().pin_memory() for k, v in step.x.items()}
    devbuf = {k: torch.empty_like(v) for k, v in step.x.items()}
    out_shape = (step.B, wl.D) if wl.kind == "compress_append" else step.o.shape
    out_dtype = torch.bfloat16 if wl.kind == "compress_append" else step.o.dtype
    o_host = torch.empty(out_shape, dtype=out_dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = o_host.numel() * o_host.element_size()
    s = torch.cuda.current_stream()

    def one():
        for k in host:
            devbuf[k].copy_(host[k], non_blocking=True)
        x = devbuf
        if wl.kind == "out_proj":
            _, o = csa.out_proj(x["o"], x["wa"], x["wb"], z=step.z, out=step.o, workspace=step.ws)
        elif wl.kind == "compress_append":
            for i in range(wl.m):
                csa.compress_append(x["kv"][i], x["gate"][i], x["pos_bias"], step.state_x, step.state_g,
                                    step.P0 + i, wl.m, wl.r, wl.theta_cmp, wl.theta_tok, C=step.C, win=step.win)
            o = step.C[:, (step.P0 + wl.m) // wl.m - 1]   # the entry the last append closed
        elif wl.kind == "csa_prefill":
            o, _, _, _ = csa.csa_forward(x["q"], x["kv"], x["gate"], x["pos_bias"], x["qI"], x["kI"], x["w"],
                                         x["sinks"], wl.m, wl.L, wl.topk, wl.W, wl.r, wl.theta_tok, wl.theta_cmp,
                                         out=(step.o, step.C, step.kv_rot, step.idx), workspace=step.ws)
        elif wl.kind == "hca_prefill":
            o, _, _ = csa.hca_forward(x["q"], x["kv"], x["gate"], x["pos_bias"], x["sinks"], wl.m, wl.L, wl.W, wl.r,
                                      wl.theta_tok, wl.theta_cmp, out=(step.o, step.C, step.kv_rot), workspace=step.ws)
        elif wl.kind == "hca_decode":
            kw = dict(C=x["C"]) if wl.cache == "bf16" else dict(c8=x["c8"], c8_scale=x["scale"], c_rope=x["rope"])
            o = csa.hca_decode(x["q"], x["win"], x["sinks"], step.P, wl.r, wl.theta_tok, wl.theta_cmp, o=step.o,
                               workspace=step.ws, **kw)
        elif wl.index_fmt == "fp4":
            kw = dict(C=x["C"]) if wl.cache == "bf16" else dict(c8=x["c8"], c8_scale=x["scale"], c_rope=x["rope"])
            csa.quantize_mxfp4(x["qI"], codes=step.qc, scales=step.qs)
            o, _ = csa.decode_fp4(x["q"], step.qc, step.qs, x["w"], x["kc"], x["ks"], x["win"], x["sinks"], step.P,
                                  wl.topk, wl.r, wl.theta_tok, wl.theta_cmp, o=step.o, idx=step.idx,
                                  workspace=step.ws, **kw)
        else:
            kw = dict(C=x["C"]) if wl.cache == "bf16" else dict(c8=x["c8"], c8_scale=x["scale"], c_rope=x["rope"])
            o, _ = csa.decode(x["q"], x["qI"], x["w"], x["kI"], x["win"], x["sinks"], step.P, wl.topk, wl.r,
                              wl.theta_tok, wl.theta_cmp, o=step.o, idx=step.idx, workspace=step.ws, **kw)
        o_host.copy_(o, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        one()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del devbuf
    return ms, h2d, d2h


# ---- the oracle (CPU baseline and reference arm) -----------------------------------------------------

def oracle_sample_rows(wl, n, seed=0):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(wl.S, size=n, replace=False)).astype(np.int64)


class OracleStep:
    """The fp64 oracle on a bounded sample of the workload: prefill rows are independent once the
    entries are pooled, so a sample of query rows (plus the pooling, amortised per token) measures
    the oracle's per-token rate; decode samples whole sequences."""

    def __init__(self, wl, target_s=4.0):
        import oracle
        self.oracle, self.wl = oracle, wl
        if wl.kind == "out_proj":
            self.x = proj_inputs(wl, device="cpu")
            self.n = 64
        elif wl.kind == "compress_append":
            g = torch.Generator().manual_seed(wl.seed)
            self.x = {"kv": torch.randn(wl.L, wl.D, generator=g).to(torch.bfloat16),
                      "gate": torch.randn(wl.L, wl.D, generator=g).to(torch.bfloat16),
                      "pos_bias": torch.randn(wl.L, generator=g) * 0.02}
        elif wl.kind in ("csa_decode", "hca_decode"):
            self.x = decode_inputs(wl, device="cpu", batch=1)
            self.P = wl.ctx - 1
            if wl.index_fmt == "fp4":   # the MXFP4 cache is built once, outside the timed steps
                self.kq = oracle.mxfp4_quantize(self.x["kI"])
        else:
            self.x = prefill_inputs(wl, device="cpu")
            t0 = time.perf_counter()
            self.C, self.kvr = oracle.compress(self.x["kv"], self.x["gate"], self.x["pos_bias"], wl.m, wl.L, wl.r,
                                               wl.theta_cmp, wl.theta_tok)
            self.compress_s = time.perf_counter() - t0
            t0 = time.perf_counter()
            self._rows(oracle_sample_rows(wl, 2, seed=99))
            per_row = (time.perf_counter() - t0) / 2
            self.n = int(max(2, min(256, target_s / max(per_row, 1e-6))))
        self.calls = 0

    def _rows(self, rows):
        wl, x, o = self.wl, self.x, self.oracle
        if wl.kind == "csa_prefill":
            ridx, _ = o.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=rows)
            idx = np.full((wl.S, wl.topk), -1, np.int32)
            idx[rows] = ridx
        else:
            idx = None
        o.attend(x["q"], self.C, self.kvr, idx, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp, rows=rows)

    def run(self):
        """Returns (units, seconds) of one sampled step."""
        wl, o, x = self.wl, self.oracle, self.x
        self.calls += 1
        t0 = time.perf_counter()
        if wl.kind == "out_proj":   # a sample of token rows (rows are independent)
            rows = oracle_sample_rows(wl, self.n, seed=self.calls)
            o.out_proj(x["o"][rows], x["wa"], x["wb"])
            return self.n, time.perf_counter() - t0
        if wl.kind == "compress_append":   # the entries of the last L tokens of one sequence (m appends' work)
            o.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
            return wl.m, time.perf_counter() - t0
        if wl.kind in ("csa_decode", "hca_decode"):
            if wl.kind == "csa_decode" and wl.index_fmt == "fp4":
                qc, qs = o.mxfp4_quantize(x["qI"])
                ridx, _ = o.decode_index_topk_fp4(qc, qs, x["w"], self.kq[0], self.kq[1], wl.topk)
            elif wl.kind == "csa_decode":
                ridx, _ = o.decode_index_topk(x["qI"], x["w"], x["kI"], wl.topk)
            else:
                ridx = np.arange(wl.T, dtype=np.int32)[None]
            kw = dict(C=x["C"]) if wl.cache == "bf16" else dict(c8=x["c8"], c8_scale=x["scale"], c_rope=x["rope"])
            o.decode_attend(x["q"], x["win"], ridx, x["sinks"], self.P, wl.r, wl.theta_tok, wl.theta_cmp, **kw)
            return 1, time.perf_counter() - t0
        rows = oracle_sample_rows(wl, self.n, seed=self.calls)
        self._rows(rows)
        dt = time.perf_counter() - t0 + self.compress_s * self.n / wl.S    # pooling amortised per token
        return self.n, dt

    def sample_desc(self):
        if self.wl.kind == "csa_decode":
            return f"1 of {self.wl.B} sequences per step (full index scan over T={self.wl.T} + attention)"
        if self.wl.kind == "out_proj":
            return f"{self.n} random token rows of S={self.wl.S} per step (both projections in fp64)"
        if self.wl.kind == "compress_append":
            return f"the pooling of the last L={self.wl.L} tokens of 1 of {self.wl.B} sequences per step"
        if self.wl.kind == "hca_decode":
            return f"1 of {self.wl.B} sequences per step (attention over all T={self.wl.T} entries + window)"
        return (f"{self.n} random query rows of S={self.wl.S} per step (index + top-k + attention per row) "
                f"plus the full pooling amortised per token")


def unit_name(wl):
    return "queries/s" if wl.kind in ("csa_decode", "hca_decode") else "tokens/s"


def metric_name(wl):
    return {"csa_prefill": "csa_prefill_tokens_per_s", "hca_prefill": "hca_prefill_tokens_per_s",
            "csa_decode": "csa_decode_queries_per_s", "hca_decode": "hca_decode_queries_per_s",
            "compress_append": "csa_append_tokens_per_s", "out_proj": "out_proj_tokens_per_s"}[wl.kind]


def config_of(wl, n_gpus):
    c = {"workload": wl.name, "S": wl.S, "H": wl.H, "D": wl.D, "m": wl.m, "window_L": wl.L, "W": wl.W,
         "rope_dim": wl.r, "theta_tok": wl.theta_tok, "theta_cmp": wl.theta_cmp, "parallelism": f"replicas{n_gpus}",
         "l2": "flushed between steps (256 MiB write outside the timed events)"}
    if wl.kind == "csa_decode":
        c.update({"B": wl.B, "ctx": wl.ctx, "T": wl.T, "topk": wl.topk, "index": f"{wl.HI}x{wl.dI}",
                  "cache": wl.cache, "index_format": "mxfp4" if wl.index_fmt == "fp4" else "bf16"})
        del c["S"]
    elif wl.kind == "hca_decode":
        c.update({"B": wl.B, "ctx": wl.ctx, "T": wl.T, "cache": wl.cache})
        del c["S"]
    elif wl.kind == "compress_append":
        c.update({"B": wl.B, "ctx": wl.ctx, "appends_per_step": wl.m})
        del c["S"]
    elif wl.kind == "out_proj":
        c = {"workload": wl.name, "S": wl.S, "H": wl.H, "D": wl.D, "o_groups": wl.o_groups, "o_lora_rank": wl.o_rank,
             "hidden": wl.hidden, "parallelism": f"replicas{n_gpus}",
             "l2": "flushed between steps (256 MiB write outside the timed events)"}
    elif wl.kind == "csa_prefill":
        c.update({"topk": wl.topk, "index": f"{wl.HI}x{wl.dI}", "T": wl.T})
    else:
        c.update({"T": wl.T})
    return c


def reference_arm(args, wl, rank, world):
    if rank != 0:
        return 0
    threads = None
    try:
        import oracle
        threads = oracle.num_threads()
        st = OracleStep(wl)
        for _ in range(args.warmup):
            st.run()
        units = secs = 0.0
        for _ in range(args.steps):
            u, s = st.run()
            units += u
            secs += s
    except Exception as e:  # the oracle is plain C; a failure here is a build problem
        print(json.dumps({"impl": "reference", "unavailable": f"oracle failed: {e}"}))
        return 0
    v = units / secs
    line = {"impl": "reference", "metric": metric_name(wl), "value": v, "unit": unit_name(wl), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, world),
            "cpu_baseline": {"value": v, "unit": unit_name(wl), "cores": threads, "kind": "oracle",
                             "sample": st.sample_desc()},
            "e2e": {"value": v, "unit": unit_name(wl), "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def cpu_baseline(wl):
    import oracle
    st = OracleStep(wl, target_s=6.0)
    units = secs = 0.0
    t_end = time.perf_counter() + 15.0
    while True:
        u, s = st.run()
        units += u
        secs += s
        if time.perf_counter() > t_end:
            break
    return {"value": units / secs, "unit": unit_name(wl), "cores": oracle.num_threads(), "kind": "oracle",
            "sample": st.sample_desc() + f"; {st.calls} steps"}


SIDE_WORKLOADS = ("hca_prefill", "decode128k", "decode1m")


def side_runs(csa, dev, steps, flush, reduce_max):
    """The other headline configurations, each timed as the main line is (device events around each
    step, L2 flushed between steps, max over ranks): the V4-Flash HCA prefill layer and the two CSA
    decode batches. Returns {workload: summary}; each workload's buffers are freed before the next."""
    peaks, peak_src = load_peaks()
    out = {}
    for name in SIDE_WORKLOADS:
        wl = WORKLOADS[WORKLOAD_IDS[name]]
        step = Step(name, wl, csa, dev)
        for _ in range(3):
            step.run(False)
        torch.cuda.synchronize()
        ph = []
        for _ in range(steps):
            flush.fill_(1)
            step.run(True)
            torch.cuda.synchronize()
            ph.append(step.phase_ms())
        ph = np.array(ph)
        total = reduce_max(float(ph.sum()))
        mean_phase = ph.mean(0)
        d = {"metric": metric_name(wl), "value": step.units * steps / (total / 1e3), "unit": unit_name(wl),
             "ms_per_step": total / steps, "steps": steps, "config": config_of(wl, 1),
             "phases_ms": {n: float(v) for n, v in zip(step.phases, mean_phase)}}
        if wl.kind == "hca_prefill":
            t_att = float(mean_phase[step.phases.index("attend")]) / 1e3
            fl, by = csa_attention_flops(wl), attention_bytes(wl)
            d["roofline"] = {"kernel": "attention", "bound": "tensor and hbm (ridge)",
                             "achieved_tflops": fl / t_att / 1e12, "peak_tflops": peaks["bf16_tflops"],
                             "frac_tensor": fl / t_att / 1e12 / peaks["bf16_tflops"],
                             "achieved_gbs": by / t_att / 1e9, "peak_gbs": peaks["hbm_gbs"],
                             "frac_hbm": by / t_att / 1e9 / peaks["hbm_gbs"], "peak_source": peak_src}
        else:
            by = decode_bytes(wl, step.B)
            t = total / steps / 1e3
            d["roofline"] = {"kernel": "whole decode step (index scan + top-k + attention + combine)",
                             "bound": "hbm", "algorithmic_bytes": by, "achieved": by / t / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": by / t / 1e9 / peaks["hbm_gbs"],
                             "peak_source": peak_src}
        d["gpu_launches"] = step.launches_per_step() * steps
        out[name] = d
        del step
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="csa_prefill", choices=sorted(WORKLOAD_IDS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true", help="skip the HCA prefill and decode objects of the default line")
    args = ap.parse_args()
    wl = WORKLOADS[WORKLOAD_IDS[args.workload]]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, wl, rank, world)

    import long_context_sparse_fwd_b200 as csa
    csa.lib()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    step = Step(args.workload, wl, csa, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        step.run(False)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    phase_ms = []
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            flush.fill_(1)
            step.run(True)
            torch.cuda.synchronize()
            phase_ms.append(step.phase_ms())
    torch.cuda.synchronize()
    barrier()
    phase_ms = np.array(phase_ms)                        # [steps, phases]
    total_ms = float(phase_ms.sum())
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    units = step.units * args.steps * world
    value = units / (total_ms / 1e3)

    peaks, peak_src = load_peaks()
    mean_phase = phase_ms.mean(0)
    dom = int(np.argmax(mean_phase))
    dom_name = step.phases[dom]
    if wl.kind == "out_proj":
        alg = proj_flops(wl)
        roof = {"bound": "tensor", "kernel": "proj_gemm_tc (o_a_proj + o_b_proj)",
                "achieved": alg / (mean_phase[dom] / 1e3) / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    elif wl.kind == "compress_append":
        alg = append_bytes(wl, step.B)
        roof = {"bound": "hbm", "kernel": "compress_append (m launches, latency-bound)",
                "achieved": alg / (mean_phase[dom] / 1e3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    elif wl.kind in ("csa_decode", "hca_decode"):
        alg = decode_bytes(wl, step.B)
        roof = {"bound": "hbm", "kernel": "csa_decode (index scan + top-k + attention)" if wl.kind == "csa_decode"
                else "hca_decode (split attention + combine)",
                "achieved": alg / (mean_phase[dom] / 1e3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    elif dom_name == "attend":
        alg = csa_attention_flops(wl)
        roof = {"bound": "tensor", "kernel": "attention", "achieved": alg / (mean_phase[dom] / 1e3) / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    elif dom_name == "index_topk":
        alg = index_flops(wl)
        roof = {"bound": "tensor", "kernel": "index_topk", "achieved": alg / (mean_phase[dom] / 1e3) / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        alg = float(wl.S * wl.D * 2 * 3 + wl.T * wl.D * 2)
        roof = {"bound": "hbm", "kernel": "compress", "achieved": alg / (mean_phase[dom] / 1e3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'profiling fallback'})"
    roof["traffic"] = recorded_traffic(args.workload)   # ncu DRAM bytes per launch (profiles/traffic.txt)
    roof["ms_per_launch"] = float(mean_phase[dom])

    def reduce_max(v):
        tv = torch.tensor([v], dtype=torch.float64, device=dev)
        if dist is not None:
            dist.all_reduce(tv, op=dist.ReduceOp.MAX)
        return float(tv.item())

    side = None
    if args.workload == "csa_prefill" and not args.no_side:
        side = side_runs(csa, dev, max(3, min(args.steps, 10)), flush, reduce_max)

    e2e = None
    if not args.no_e2e:
        ms, h2d, d2h = e2e_run(step, max(2, args.steps // 2), 1)
        te = torch.tensor([ms], dtype=torch.float64, device=dev)
        if dist is not None:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        n_e2e = max(2, args.steps // 2)
        e2e = {"value": step.units * n_e2e * world / (float(te.item()) / 1e3), "unit": unit_name(wl),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    line = {
        "metric": metric_name(wl), "value": value, "unit": unit_name(wl), "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate/out", "data": "synthetic",
        "config": config_of(wl, world),
        "phases_ms": {n: float(v) for n, v in zip(step.phases, mean_phase)},
        "roofline": roof, "e2e": e2e, "gpu_launches": step.launches_per_step() * args.steps,
        "clocks": clk.summary(),
    }
    if side is not None:
        line["side"] = side
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
