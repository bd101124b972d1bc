#!/usr/bin/env python
"""Benchmark of the HySparse hybrid block on one B200 per process.

A step is one pass of the hot path over one batch of synthetic input: the
full-attention layer with its oracle indexer, then the block's sparse layers
reusing its K^F/V^F and index set.  Default workload: the 1M-token HySparse2
prefill chunk (8192 queries at the end of a 2^20-token causal prefix, 64/4
heads, d=128, bf16, token top-k with k=1024 including the last w=128, then
11 sparse layers); --workload picks another one.

Printed value (rank 0, one JSON line): the fraction of one B200's roofline
the step reaches, summed over ranks (N x that for N replicas):
    value = (F_full / P_tensor + n_sparse * t_sparse_min) / t_step
with t_sparse_min the sparse layer's own physical bound,
    max(useful FLOPs / P_tensor, least bytes / P_hbm),
useful FLOPs = 4 d per (query head, kept key) and least bytes = every
distinct K/V row the layer's queries keep read once, plus q', outputs, lse
and index rows.  Decode steps are HBM-bound: (cache bytes + n_sparse *
selected-row bytes) / P_hbm.  P_tensor is the measured burst bf16 peak when
the SM clock stayed at its maximum with no power cap in the timed region,
else the sustained one (the line says which).  The pages' logical gather
rate ("reads k+w tokens" per query) is reported beside it as sparse_kv_gbs.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Each step replays two CUDA graphs captured from the C-ABI calls (the full
layer's launches, then the sparse layers'), so the GPU runs the kernels back
to back; --no-graph times the per-call launches instead.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the only place besides the cpu_baseline field
where this script runs the oracle).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from oracle_top_kv_b200 import accounting as A  # noqa: E402
from oracle_top_kv_b200 import dist as hdist  # noqa: E402
from oracle_top_kv_b200 import workloads as wl  # noqa: E402

METRIC = "full+index prefill TFLOP/s and sparse-reuse KV GB/s (fraction of B200 peak)"
UNIT = "fraction of one B200 roofline (step)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks while the timed region runs."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.rows, self.proc, self.err = [], None, None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception as e:  # pragma: no cover
            self.gpu_id, self.err = None, repr(e)

    def start(self):
        if self.gpu_id is None:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception as e:
            self.err = repr(e)

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 7:
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": self.err or "no nvidia-smi samples"}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


# ------------------------------------------------------------------ our arm
class HybridBlock:
    """Device buffers and C-ABI calls of one full layer + its sparse layers."""

    def __init__(self, w, device):
        from oracle_top_kv_b200 import hs
        self.hs = hs
        self.w = w
        self.dev = device
        q, k, v, _ = wl.full_layer_inputs(w, device=device)
        self.q, self.k, self.v = q, k, v
        self.p = hs.make_params(w.batch, w.hq, w.hkv, w.head_dim, w.tq, w.t, w.q_offset, w.dtype,
                                w.mode, w.block_size, w.k, w.window)
        self.o, self.lse, self.idx, self.cnt, _ = hs.full_outputs(self.p, device)
        self.ws_full = hs.workspace(self.p, hs.HS_WS_FULL, device)
        self.qs, self.kl, self.vl, self.og, self.lg, self.ol, self.ll = [], [], [], [], [], [], []
        for layer in range(w.n_sparse):
            qs = wl.sparse_layer_query(w, layer, device=device)
            self.qs.append(qs)
            self.og.append(torch.empty_like(qs))
            self.lg.append(torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32, device=device))
            if w.swa_branch:
                kl, vl = wl.sparse_layer_local_kv(w, layer, device=device)
                self.kl.append(kl)
                self.vl.append(vl)
                self.ol.append(torch.empty_like(qs))
                self.ll.append(torch.empty_like(self.lg[-1]))
            else:
                self.kl.append(None); self.vl.append(None); self.ol.append(None); self.ll.append(None)

    def full(self, stream):
        self.hs.hs_full_attn_index(self.p, self.q, self.k, self.v, self.o, self.lse, self.idx,
                                   self.cnt, None, self.ws_full, stream)

    def sparse(self, layer, stream):
        self.hs.hs_sparse_attn_reuse(self.p, self.qs[layer], self.k, self.v, self.idx, self.cnt,
                                     self.kl[layer], self.vl[layer], self.og[layer],
                                     self.lg[layer], self.ol[layer], self.ll[layer], None, stream)

    def inputs(self):
        t = [self.q, self.k, self.v] + self.qs
        if self.w.swa_branch:
            t += self.kl + self.vl
        return t

    def outputs(self):
        t = [self.o, self.lse, self.idx, self.cnt] + self.og + self.lg
        if self.w.swa_branch:
            t += self.ol + self.ll
        return t


class DecodeBlock:
    """One decode step of a HySparse2 block: the full layer's step over the
    whole cache (index selection for the new token), then the block's sparse
    layers gathering the selected rows of the same cache."""

    def __init__(self, w, device):
        from oracle_top_kv_b200 import hs
        self.hs = hs
        self.w = w
        q, kc, vc, _ = wl.full_layer_inputs(w, device=device)
        self.q, self.k, self.v = q, kc, vc
        self.seq = wl.decode_seq_lens(w, ragged=False, device=device)
        t_kv = w.t
        self.pages = None
        if w.page_size:  # the cache as a pool of pages with a shuffled block table
            self.k, self.v, self.bt = wl.paged_pool(kc, vc, w.page_size)
            del kc, vc
            self.pages = hs.make_pages(self.bt, w.page_size, self.k.shape[0])
            t_kv = self.bt.shape[1] * w.page_size
        self.p = hs.make_params(w.batch, w.hq, w.hkv, w.head_dim, 1, t_kv, 0, w.dtype, w.mode,
                                w.block_size, w.k, w.window)
        ks = self.p.ksel
        self.idx = torch.empty(w.batch, w.hkv, ks, dtype=torch.int32, device=device)
        self.cnt = torch.empty(w.batch, w.hkv, dtype=torch.int32, device=device)
        self.o = torch.empty_like(q)
        self.lse = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=device)
        self.ws_full = hs.workspace(self.p, hs.HS_WS_DECODE_FULL, device)
        self.ws_sp = hs.workspace(self.p, hs.HS_WS_DECODE_SPARSE, device)
        self.qs = [wl.sparse_layer_query(w, l, device=device) for l in range(w.n_sparse)]
        self.os = [torch.empty_like(x) for x in self.qs]
        self.ls = [torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=device)
                   for _ in self.qs]

    def full(self, stream):
        if self.pages is not None:
            self.hs.hs_decode_step_paged(self.p, self.pages, self.hs.HS_DECODE_FULL_INDEX, self.q,
                                         self.k, self.v, self.seq, self.idx, self.cnt, self.o,
                                         self.lse, None, self.ws_full, stream)
            return
        self.hs.hs_decode_step(self.p, self.hs.HS_DECODE_FULL_INDEX, self.q, self.k, self.v,
                               self.seq, self.idx, self.cnt, self.o, self.lse, None, self.ws_full,
                               stream)

    def sparse(self, layer, stream):
        if self.pages is not None:
            self.hs.hs_decode_step_paged(self.p, self.pages, self.hs.HS_DECODE_SPARSE,
                                         self.qs[layer], self.k, self.v, self.seq, self.idx,
                                         self.cnt, self.os[layer], self.ls[layer], None, None,
                                         stream)
            return
        self.hs.hs_decode_step(self.p, self.hs.HS_DECODE_SPARSE, self.qs[layer], self.k, self.v,
                               self.seq, self.idx, self.cnt, self.os[layer], self.ls[layer], None,
                               self.ws_sp, stream)

    def inputs(self):
        # per-step inputs: the new token's queries; the K/V cache is resident state
        return [self.q, self.seq] + self.qs

    def outputs(self):
        return [self.o, self.lse, self.idx, self.cnt] + self.os + self.ls


def work(w, blk):
    """Algorithmic FLOPs of the full layer and bytes of each sparse layer.
    Decode: the full layer is counted in bytes (the whole cache), returned as
    (full_bytes, sparse_bytes) with flops = None."""
    if w.decode:
        elt = 2
        full_b = A.decode_full_bytes(w.batch, w.hkv, w.head_dim, blk.seq.tolist(), elt)
        full_b += w.batch * w.hq * w.head_dim * elt * 2  # q in, o out
        rows = int(blk.cnt.sum().item())
        sp = rows * 2 * w.head_dim * elt + w.batch * w.hq * (w.head_dim * elt * 2 + 4)
        sp += w.batch * w.hkv * (w.ksel + 1) * 4
        return None, full_b, sp
    flops = A.full_layer_flops(w.batch, w.hq, w.head_dim, w.tq, w.q_offset)
    rows = A.sparse_rows_from_index(blk.idx, blk.cnt, w.mode, w.block_size, w.q_offset)
    local = A.window_rows(w.batch, w.hkv, w.tq, w.window, w.q_offset) if w.swa_branch else 0
    elt = 2 if w.dtype == "bf16" else 4
    sbytes = A.sparse_layer_bytes(rows, w.batch, w.hq, w.tq, w.head_dim, elt, w.ksel, w.hkv, local)
    return flops, None, sbytes


def sparse_useful_flops(w, blk):
    """Useful FLOPs of one sparse layer: 4*d per (query head, kept key) -- the
    selected keys clipped to the row's position plus the window branch's keys."""
    rows = A.sparse_rows_from_index(blk.idx, blk.cnt, w.mode, w.block_size, w.q_offset)
    local = A.window_rows(w.batch, w.hkv, w.tq, w.window, w.q_offset) if w.swa_branch else 0
    return (rows + local) * (w.hq // w.hkv) * 4 * w.head_dim


def sparse_on_tensor_cores(w):
    """Block mode with 64-key blocks at d = 128 in bf16 runs the row-grouped
    tcgen05 kernel (a CTA streams the union of its rows' selected blocks)."""
    return (w.mode == "block" and w.dtype == "bf16" and w.head_dim == 128 and
            w.block_size == 64 and w.ksel <= 16 and 128 % (w.hq // w.hkv) == 0)


def code_hash(paths):
    """sha256 of the sources' code: comments and whitespace removed, so that a
    comment edit does not mark a capture as stale while any code change does."""
    import re
    h = hashlib.sha256()
    for f in paths:
        text = open(os.path.join(ROOT, f), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def traffic_for(kernel, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel's
    source code is unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(f"{kernel}@{workload}")
    if not d:
        return None
    return d["bytes_per_launch"] if code_hash(d.get("sources", [])) == d.get("sha256") else None


def workload_of(args):
    w = wl.WORKLOADS[args.workload]
    kw = {}
    if args.batch:
        kw["batch"] = args.batch
    if args.seq:
        kw["t"] = args.seq
    if args.tq:  # a shorter query chunk at the end of the same prefix
        kw["t_q"] = args.tq
        kw["q_offset"] = (args.seq or w.t) - args.tq
    if kw:
        w = wl.scaled(w, name=w.name + "".join(f"_{k}{v}" for k, v in kw.items()), **kw)
    return w


def tensor_peak(peaks, clk):
    """The bf16 tensor peak that applies to the timed region: the burst figure
    while the median SM clock stayed within 3% of its maximum with no power
    cap, the sustained (power-capped) one otherwise."""
    sm, mx, reasons = clk.get("sm_mhz"), clk.get("sm_max_mhz"), clk.get("reasons") or []
    if sm and mx and sm >= 0.97 * mx and "sw_power_cap" not in reasons:
        return peaks["bf16_tflops"], "bf16_tflops"
    return peaks["bf16_tflops_sustained"], "bf16_tflops_sustained"


def sparse_bound(w, blk, p_tensor, p_hbm):
    """A sparse layer's physical roofline: max(useful FLOPs / P_tensor, least
    bytes / P_hbm).  Prefill only (decode steps are counted in bytes)."""
    if w.decode:
        return {"bound": "hbm", "t_min": 0.0}
    uf = sparse_useful_flops(w, blk)
    urows = A.sparse_unique_rows_from_index(blk.idx, blk.cnt, w.mode, w.block_size, w.q_offset)
    ulocal = (w.batch * w.hkv * min(w.t, w.q_offset + w.tq)) if w.swa_branch else 0
    elt = 2 if w.dtype == "bf16" else 4
    ub = A.sparse_layer_unique_bytes(urows, w.batch, w.hq, w.tq, w.head_dim, elt, w.ksel,
                                     w.hkv, ulocal, local=w.swa_branch)
    t_c, t_m = uf / p_tensor, ub / p_hbm
    return {"bound": "tensor" if t_c >= t_m else "hbm", "useful_flops": uf, "least_bytes": ub,
            "distinct_kv_rows": urows + ulocal, "t_min": max(t_c, t_m)}


def config_of(w, world, launch):
    return {"workload": w.name, "batch": w.batch, "seq_len": w.t, "hq": w.hq,
            "hkv": w.hkv, "head_dim": w.head_dim, "mode": w.mode,
            "block_size": w.block_size, "k": w.k, "window": w.window,
            "decode": w.decode, "t_q": w.tq, "q_offset": w.q_offset,
            "sparse_layers": w.n_sparse, "page_size": w.page_size or None,
            "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2 (K^F+V^F alone exceed 126 MB)",
            "launch": launch}


def kernel_breakdown(blk, w, sh):
    """Device time of each of the library's kernels in one untimed step (CUPTI
    kernel records through torch.profiler): which kernel dominates."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            blk.full(sh)
            for layer in range(w.n_sparse):
                blk.sparse(layer, sh)
            torch.cuda.synchronize()
        agg = {}
        for e in prof.events():
            if e.device_type.name != "CUDA":
                continue
            name = e.name.split("(")[0].replace("void ", "")
            t = getattr(e, "device_time_total", None)
            if t is None:
                t = e.cuda_time_total
            n, tot = agg.get(name, (0, 0.0))
            agg[name] = (n + 1, tot + t / 1e3)
        total = sum(v[1] for v in agg.values()) or 1.0
        return [{"kernel": k, "launches": n, "ms": ms, "share": ms / total}
                for k, (n, ms) in sorted(agg.items(), key=lambda kv: -kv[1][1])]
    except Exception as e:  # the breakdown is a diagnostic; never fail the bench for it
        return {"error": repr(e)[:200]}


def run_ours(args, rank, world, device):
    from oracle_top_kv_b200 import hs
    hs.load()
    w = workload_of(args)
    peaks, peak_kind = load_peaks()
    blk = DecodeBlock(w, device) if w.decode else HybridBlock(w, device)
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream

    def step():
        blk.full(sh)
        for layer in range(w.n_sparse):
            blk.sparse(layer, sh)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert hs.hs_device_status(sh) == 0
    flops, full_bytes, sbytes = work(w, blk)
    graphs = None if args.no_graph else capture_step(blk, w, device)
    if graphs:  # one more untimed step, through the graphs
        graphs[0].replay()
        graphs[1].replay()
        torch.cuda.synchronize(device)

    n_ev = 1 + (1 if graphs else w.n_sparse)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev + 1)]
           for _ in range(args.steps)]
    clocks = ClockSampler(device)
    clocks.start()
    time.sleep(0.5)
    hdist.barrier(device)
    torch.cuda.synchronize(device)
    launches0 = hs.hs_launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    nvtx = torch.cuda.nvtx
    for s in range(args.steps):
        nvtx.range_push(f"step {s}")
        evs[s][0].record(stream)
        if graphs:
            nvtx.range_push("full layer + index")
            graphs[0].replay()
            nvtx.range_pop()
            evs[s][1].record(stream)
            nvtx.range_push(f"{w.n_sparse} sparse layers")
            graphs[1].replay()
            nvtx.range_pop()
            evs[s][2].record(stream)
            nvtx.range_pop()
            continue
        nvtx.range_push("full layer + index")
        blk.full(sh)
        nvtx.range_pop()
        evs[s][1].record(stream)
        for layer in range(w.n_sparse):
            nvtx.range_push(f"sparse layer {layer}")
            blk.sparse(layer, sh)
            nvtx.range_pop()
            evs[s][2 + layer].record(stream)
        nvtx.range_pop()
    t1.record(stream)
    torch.cuda.synchronize(device)
    launches = hs.hs_launch_count() - launches0
    if graphs:  # replays do not pass through the library: count the captured launches
        launches = args.steps * (graphs[2] + graphs[3])
    hdist.barrier(device)
    clocks.stop()
    total_ms = hdist.max_over_ranks(t0.elapsed_time(t1), device)
    assert hs.hs_device_status(sh) == 0
    full_ms = [evs[s][0].elapsed_time(evs[s][1]) for s in range(args.steps)]
    if graphs:  # the sparse layers of a step run as one graph: per layer = step share / n
        sparse_ms = [evs[s][1].elapsed_time(evs[s][2]) / w.n_sparse for s in range(args.steps)
                     for _ in range(w.n_sparse)]
    else:
        sparse_ms = [evs[s][1 + l].elapsed_time(evs[s][2 + l]) for s in range(args.steps)
                     for l in range(w.n_sparse)]
    ms_step = total_ms / args.steps
    clk = clocks.summary()
    p_tensor_tf, tensor_kind = tensor_peak(peaks, clk)
    p_tensor = p_tensor_tf * 1e12
    p_hbm = peaks["hbm_gbs"] * 1e9
    full_s = statistics.mean(full_ms) / 1e3
    sparse_s = statistics.mean(sparse_ms) / 1e3
    sparse_gbs = sbytes / sparse_s / 1e9
    tokens = w.batch * w.tq
    sp_bound = sparse_bound(w, blk, p_tensor, p_hbm)
    if flops is not None:
        ideal = flops / p_tensor + w.n_sparse * sp_bound["t_min"]
        full_rate, full_unit, full_peak = flops / full_s / 1e12, "TFLOP/s", p_tensor_tf
        full_bound, full_peak_src = "tensor", f"{peak_kind} {tensor_kind}"
    else:
        ideal = (full_bytes + w.n_sparse * sbytes) / p_hbm
        full_rate, full_unit, full_peak = full_bytes / full_s / 1e9, "GB/s", peaks["hbm_gbs"]
        full_bound, full_peak_src = "hbm", f"{peak_kind} hbm_gbs"
    value = world * ideal / (ms_step / 1e3)
    # dominant kernel: the one with the larger share of the step
    if sum(full_ms) >= sum(sparse_ms):
        name = "decode_full_index" if w.decode else "full_attn_index"
        roof = {"kernel": name, "bound": full_bound, "achieved": full_rate, "peak": full_peak,
                "unit": full_unit, "frac": full_rate / full_peak,
                "traffic": traffic_for(name, w.name), "peak_source": full_peak_src,
                "work_per_launch": flops if flops is not None else full_bytes,
                "avg_launch_ms": full_s * 1e3}
        if flops is not None and w.mode == "token":
            roof["note"] = ("one C-ABI call = the tensor-core attention pass, then the token "
                            "selection pass (which recomputes QK^T: +50% tensor work); work = "
                            "the algorithmic FLOPs 4*d*hq per causal pair")
    elif w.decode:
        roof = {"kernel": "decode_sparse", "bound": "hbm", "achieved": sparse_gbs,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": sparse_gbs / peaks["hbm_gbs"],
                "traffic": traffic_for("decode_sparse", w.name),
                "peak_source": f"{peak_kind} hbm_gbs", "work_per_launch": sbytes,
                "avg_launch_ms": sparse_s * 1e3}
    else:
        sb = sp_bound
        if sb["bound"] == "tensor":
            ach, pk, unit, wk = sb["useful_flops"] / sparse_s / 1e12, p_tensor_tf, "TFLOP/s", \
                sb["useful_flops"]
        else:
            ach, pk, unit, wk = sb["least_bytes"] / sparse_s / 1e9, peaks["hbm_gbs"], "GB/s", \
                sb["least_bytes"]
        roof = {"kernel": "sparse_attn_reuse", "bound": sb["bound"], "achieved": ach,
                "peak": pk, "unit": unit, "frac": ach / pk,
                "traffic": traffic_for("sparse_attn_reuse", w.name),
                "peak_source": f"{peak_kind} " + (tensor_kind if sb["bound"] == "tensor"
                                                  else "hbm_gbs"),
                "work_per_launch": wk, "avg_launch_ms": sparse_s * 1e3,
                "note": "the sparse layer's physical bound: max(useful FLOPs / P_tensor, least "
                        "bytes / P_hbm), useful FLOPs = 4*d per (query head, kept key), least "
                        "bytes = distinct K/V rows kept + q' + outputs + index; the pages' "
                        "logical-bytes rate is sparse_kv_gbs"}
    full_key = "full_index_gbs" if flops is None else "full_index_tflops"

    kernels = kernel_breakdown(blk, w, sh) if not args.no_breakdown else None
    e2e = run_e2e(args, blk, w, stream, ideal, world, device) if not args.no_e2e else None
    gate_sink = None if w.decode else time_gate_sink(blk, w, stream, peaks)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": config_of(w, world, "cuda graph replays (full-layer graph, sparse-layers graph)"
                            if graphs else "per-call launches"),
        full_key: full_rate * world,
        "full_index_frac_of_peak": full_rate / full_peak,
        "sparse_kv_gbs": sparse_gbs * world,
        "sparse_kv_gbs_note": "the pages' logical accounting: every K/V row each query's "
                              "index set reads; rows shared between queries count once per "
                              "query, so this rate can exceed the HBM peak",
        "sparse_bound": {k: v for k, v in sp_bound.items() if k != "t_min"},
        "sparse_frac_of_bound": sp_bound["t_min"] / sparse_s,
        "full_ms": full_s * 1e3, "sparse_ms_per_layer": sparse_s * 1e3,
        "tokens_per_s": world * tokens / (ms_step / 1e3),
        "peaks": {"bf16_tflops": peaks["bf16_tflops"],
                  "bf16_tflops_sustained": peaks["bf16_tflops_sustained"],
                  "hbm_gbs": peaks["hbm_gbs"], "source": peak_kind,
                  "tensor_peak_used": tensor_kind,
                  "rule": "burst while the median SM clock stays within 3% of its maximum "
                          "with no power cap; sustained otherwise"},
        "roofline": roof, "gpu_launches": launches, "clocks": clk,
        "kernels": kernels,
        "e2e": e2e,
        "gate_sink": gate_sink,
    }
    return line


def time_gate_sink(blk, w, stream, peaks, reps=10):
    """The sparse-layer output epilogue (per-head sinks, sigmoid-gate fusion of
    the branches: hs_sparse_gate_sink) on layer 0's branch outputs, timed on its
    own after the step (it is not part of the step).  Algorithmic bytes: the
    branch outputs and lse read, gate pre-activations read, the fused output and
    the updated lse written."""
    hs = blk.hs
    g = torch.Generator(device="cpu").manual_seed(5)
    two = blk.ol[0] is not None
    nb = 2 if two else 1
    sink = [torch.randn(w.hq, generator=g).to(blk.dev) for _ in range(nb)]
    gate = [torch.randn(w.batch, w.hq, w.tq, generator=g).to(blk.dev) for _ in range(nb)]
    lse = [blk.lg[0].clone()] + ([blk.ll[0].clone()] if two else [])
    o = torch.empty_like(blk.og[0])

    def call():
        hs.hs_sparse_gate_sink(blk.p, blk.og[0], lse[0], o, blk.ol[0], lse[1] if two else None,
                               sink[0], sink[1] if two else None, gate[0],
                               gate[1] if two else None, stream)
    for _ in range(3):
        call()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    rows = w.batch * w.hq * w.tq
    elt = 2 if w.dtype == "bf16" else 4
    nbytes = rows * (w.head_dim * elt * (nb + 1) + 4 * 3 * nb)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "gate_sink_kernel", "ms": ms, "bytes": nbytes, "gbs": gbs,
            "frac_of_hbm": gbs / peaks["hbm_gbs"], "branches": nb,
            "note": "sparse-layer output epilogue, timed alone after the step"}


def capture_step(blk, w, device):
    """CUDA graphs of one step: (full-layer graph, sparse-layers graph, kernels
    captured in each).  The library's launches are recorded as they are
    issued on the capture stream; replaying a graph launches the same kernels
    on the same buffers without the per-call host work."""
    from oracle_top_kv_b200 import hs
    cap = torch.cuda.Stream(device)
    cap.wait_stream(torch.cuda.current_stream(device))
    g_full, g_sparse = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    c0 = hs.hs_launch_count()
    with torch.cuda.graph(g_full, stream=cap):
        blk.full(cap.cuda_stream)
    c1 = hs.hs_launch_count()
    with torch.cuda.graph(g_sparse, stream=cap):
        for layer in range(w.n_sparse):
            blk.sparse(layer, cap.cuda_stream)
    c2 = hs.hs_launch_count()
    torch.cuda.current_stream(device).wait_stream(cap)
    return g_full, g_sparse, c1 - c0, c2 - c1


def run_e2e(args, blk, w, stream, ideal, world, device):
    """Same step through the C ABI with inputs in pinned host memory: every
    step copies all its inputs host->device and all its results device->host.
    Steps are pipelined as a serving loop would run them: two device buffer
    sets and three streams, so step s+1's upload and step s-1's download
    overlap step s's kernels (per-call launches, no graphs)."""
    blks = [blk, type(blk)(w, device)]
    host_in = [t.cpu().pin_memory() for t in blk.inputs()]
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in blk.outputs()]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b, x = blks[i % 2], i % 2
        s_in.wait_event(ev_cmp[x])  # the set's previous step has read its inputs
        with torch.cuda.stream(s_in):
            for d, h in zip(b.inputs(), host_in):
                d.copy_(h, non_blocking=True)
        ev_in[x].record(s_in)
        s_cmp.wait_event(ev_in[x])
        s_cmp.wait_event(ev_out[x])  # ... and its previous results are downloaded
        b.full(s_cmp.cuda_stream)
        for layer in range(w.n_sparse):
            b.sparse(layer, s_cmp.cuda_stream)
        ev_cmp[x].record(s_cmp)
        s_out.wait_event(ev_cmp[x])
        with torch.cuda.stream(s_out):
            for h, d in zip(host_out, b.outputs()):
                h.copy_(d, non_blocking=True)
        ev_out[x].record(s_out)

    n = max(2, min(args.steps, 6))
    step(0)
    step(1)
    torch.cuda.synchronize(device)
    hdist.barrier(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(n):
        step(i)
    e1.record(s_out)
    torch.cuda.synchronize(device)
    ms = hdist.max_over_ranks(e0.elapsed_time(e1) / n, device)
    return {"value": world * ideal / (ms / 1e3), "unit": UNIT, "ms_per_step": ms,
            "steps": n, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipeline": "2 device buffer sets, copy-in / compute / copy-out streams"}


# --------------------------------------------------------------- oracle arm
def oracle_inputs(w):
    """The step's inputs on the host.  K^F/V^F are held in float64 (the oracle's
    arithmetic type) when that fits in 10 GB, so that a sample's time is the
    oracle's work on resident inputs -- as the GPU's is -- rather than a
    conversion of the whole cache; otherwise each sample converts the units it
    touches."""
    q, k, v, _ = wl.full_layer_inputs(w, device="cpu")
    if 2 * k.numel() * 8 <= 10 << 30:
        k, v = k.double().numpy(), v.double().numpy()
    layers = []
    for layer in range(w.n_sparse):
        qs = wl.sparse_layer_query(w, layer, device="cpu")
        kl, vl = wl.sparse_layer_local_kv(w, layer, device="cpu") if w.swa_branch else (None, None)
        layers.append((qs, kl, vl))
    return q, k, v, layers


def oracle_sample_time(w, inputs, budget_rows=48, seed=0):
    """Time the fp64 oracle on a bounded sample of the step and extrapolate.

    Sample: `budget_rows` query rows spread over positions (and over batch and
    kv groups), each through the full layer and every sparse layer.  The full
    layer's cost grows with the row's position, the sparse layers' does not,
    so the extrapolation weights rows by visible keys and by count respectively.
    """
    import oracle
    q, k, v, layers = inputs
    rng = np.random.default_rng(seed)
    if w.decode:
        # rows = (sequence, kv group) units at the newest position
        n_units = w.batch * w.hkv
        pick = rng.choice(n_units, size=min(n_units, max(1, budget_rows // 8)), replace=False)
        rows = np.array([(int(x) // w.hkv, int(x) % w.hkv, 0) for x in pick], np.int32)
        pos = np.full(len(rows), w.t - 1)
        n_all, full_scale = n_units, n_units / len(rows)
    else:
        # positions spread evenly over the sequence (repeated when the sample
        # holds more rows than positions), batch and kv group drawn at random
        js = np.linspace(0, w.tq - 1, budget_rows).astype(int)
        rows = np.array([(int(rng.integers(0, w.batch)), int(rng.integers(0, w.hkv)), int(j))
                         for j in js], np.int32)
        pos = w.q_offset + rows[:, 2]
        n_all = w.batch * w.hkv * w.tq
        full_scale = w.batch * w.hkv * A.causal_pairs(w.tq, w.q_offset) / float((pos + 1).sum())
    t0 = time.perf_counter()
    orc = oracle.full_attn_rows(q, k, v, rows, pos, w.mode, w.block_size, w.k, w.window)
    t_full = time.perf_counter() - t0
    t_sp = 0.0
    for (qs, kl, vl) in layers:
        t0 = time.perf_counter()
        oracle.sparse_attn_rows(qs, k, v, orc["idx"], orc["cnt"], rows, pos, w.mode,
                                w.block_size, w.k, w.window, kl, vl)
        t_sp += time.perf_counter() - t0
    est_full = t_full * full_scale
    est_sparse = t_sp * n_all / len(rows)
    sample = (f"{len(rows)} query rows (all heads of their group) through the full layer and "
              f"{w.n_sparse} sparse layers, timed {t_full + t_sp:.2f} s, extrapolated to the "
              f"whole step by visible keys (full layer) and by row count (sparse layers)")
    return est_full + est_sparse, sample, oracle.num_threads()


def cpu_ideal(w):
    """The roofline time of one step (the numerator of value) for the CPU arms,
    which have no GPU index set: the sparse layer's distinct rows are taken as
    min(rows its queries read, visible keys) per unit, and the tensor peak is
    the sustained one (the CPU arms have no GPU clock record)."""
    peaks, _ = load_peaks()
    p_hbm = peaks["hbm_gbs"] * 1e9
    p_t = peaks["bf16_tflops_sustained"] * 1e12
    if w.decode:
        full_b = A.decode_full_bytes(w.batch, w.hkv, w.head_dim, [w.t] * w.batch, 2)
        sp = w.batch * w.hkv * min(w.k, w.t) * 2 * w.head_dim * 2
        return (full_b + w.n_sparse * sp) / p_hbm
    flops = A.full_layer_flops(w.batch, w.hq, w.head_dim, w.tq, w.q_offset)
    per_unit = sum(min(w.k, w.q_offset + j + 1) for j in range(w.tq))  # keys read per unit
    visible = min(w.t, w.q_offset + w.tq)
    local = A.window_rows(w.batch, w.hkv, w.tq, w.window, w.q_offset) if w.swa_branch else 0
    uf = (w.batch * w.hkv * per_unit + local) * w.group * 4 * w.head_dim
    urows = w.batch * w.hkv * min(per_unit, visible)
    ulocal = w.batch * w.hkv * visible if w.swa_branch else 0
    ub = A.sparse_layer_unique_bytes(urows, w.batch, w.hq, w.tq, w.head_dim, 2, w.ksel, w.hkv,
                                     ulocal, local=w.swa_branch)
    return flops / p_t + w.n_sparse * max(uf / p_t, ub / p_hbm)


def cpu_value(w, t_step):
    return cpu_ideal(w) / t_step


def calibrate_rows(w, inputs, target_s, lo, hi):
    """Rows per oracle sample so that one sample takes about target_s seconds."""
    rows, took = lo, 0.0
    for _ in range(4):
        t0 = time.perf_counter()
        oracle_sample_time(w, inputs, budget_rows=rows, seed=7)
        took = time.perf_counter() - t0
        if took >= 0.5 * target_s or rows >= hi:
            break
        rows = max(rows + 1, min(hi, int(rows * target_s / max(took, 1e-3))))
    return rows


def run_reference(args, w, world):
    inputs = oracle_inputs(w)
    hi = w.batch * w.hkv * 8 if w.decode else w.batch * w.hkv * w.tq
    budget = calibrate_rows(w, inputs, 5.0, 4 if w.decode else 16, hi)
    for s in range(args.warmup):
        oracle_sample_time(w, inputs, budget_rows=budget, seed=1000 + s)
    times = []
    sample = cores = None
    for s in range(max(1, args.steps)):
        t, sample, cores = oracle_sample_time(w, inputs, budget_rows=budget, seed=s)
        times.append(t)
    t_step = statistics.mean(times)
    v = cpu_value(w, t_step)
    return {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step * 1e3,
            "ms_per_step_is": "extrapolated: each step times a bounded sample of the "
                              "workload's rows and scales it to the whole step",
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": config_of(w, world, "fp64 CPU oracle, OpenMP over the host cores"),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "per step: " + sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_1m_chunk", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0, help="override the batch (reduced replica)")
    ap.add_argument("--seq", type=int, default=0, help="override the sequence length")
    ap.add_argument("--tq", type=int, default=0,
                    help="prefill: only the last TQ query rows of the sequence (reduced replica)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time per-call launches instead of CUDA graph replays")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true",
                    help="skip the per-kernel device-time breakdown (one untimed step)")
    args = ap.parse_args()

    rank, world, local = hdist.world()
    w = workload_of(args)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w, world)), flush=True)
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        hdist.init("nccl", device)
    line = run_ours(args, rank, world, device)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a sample of about 10 s of oracle work (calibrated on smaller ones)
        inputs = oracle_inputs(w)
        max_rows = w.batch * w.hkv * 8 if w.decode else w.batch * w.hkv * w.tq
        rows = calibrate_rows(w, inputs, 10.0, 4 if w.decode else 16, max_rows)
        t, sample, cores = oracle_sample_time(w, inputs, budget_rows=rows, seed=7)
        line["cpu_baseline"] = {"value": cpu_value(w, t), "unit": UNIT, "cores": cores,
                                "kind": "oracle", "sample": sample,
                                "ms_per_step_extrapolated": t * 1e3}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
