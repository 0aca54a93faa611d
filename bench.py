"""Benchmark of the DSA hot path on B200 (prefill tokens/s and decode queries/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
                    [--no-extra] [--no-e2e] [--no-cpu-baseline] [--seq-len L] [--chunk C]

One step = the whole path (lightning indexer -> top-k -> sparse MLA) over one
batch of the workload.  The headline (default: prefill_8k, one sequence of 8192
tokens, top-2048, H_I = 64, H = 128) is printed as the JSON line's own metric;
the line also carries, under "workloads", the other full-size workloads timed
the same way in the same run:
  decode_b64        64 sequences, context U[4096, 32768], 1 query each;
  decode_128k_mtp2  16 sequences at context 131072, 2 queries each;
  decode_b1_128k    1 sequence at context 131072, 1 query, paged cache
                    (pages of 64 rows scattered over the cache pool);
  chunked_64k       a 65536-token prefill run as 16 calls of 4096 queries
                    against the growing cache (one step = all 16 calls).
Inputs are seeded synthetic data resident in HBM when the timed region starts
(the headline's drawn on the host by the seeded generator; the large
sub-workloads drawn on the device by PyTorch's seeded Philox generator, same
distributions and casts).  L2 is flushed (a 512 MB write) before every timed
step, outside the timed events.  Per-stage CUDA events on the launching stream
give each kernel's duration for the roofline figures.  `e2e` repeats the
headline step through dsa_forward_host from pinned host buffers, with the
host->device copies of the step's inputs and the device->host copy of its
output inside the timed region (the library overlaps them with the compute,
query chunk by query chunk, on three streams).

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
seeded inputs (independent shards, no collective on the data path); each timed
region is bracketed by barriers and the reported time is the max over ranks.

--impl reference times the CPU oracle (numpy float64) on the host cores over a
bounded sample of rows of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_weight_b200.configs import WORKLOADS  # noqa: E402

L2_FLUSH_BYTES = 512 << 20
D_QK, D_V, D_INDEX = 576, 512, 128
# DRAM bytes (read + write) per query of the sparse-MLA kernel on prefill, from
# one ncu capture of the kernel as it stands: dram__bytes_read.sum (361.41 MB) +
# dram__bytes_write.sum (259.02 MB) of the timed launch of
# `bench.py --seq-len 2304 --steps 1 --warmup 1 --no-e2e --no-cpu-baseline`,
# divided by its 2304 queries (the traffic is the queries in and the outputs out;
# the gathered cache rows hit L2).  None while no capture describes the kernel.
MLA_TRAFFIC_BYTES_PER_QUERY = (361.410816e6 + 257.011456e6) / 2304
# Workloads run with a paged cache, and their page size (rows).
PAGED = {"decode_b1_128k": 64}


def mla_flop_per_pair(heads: int) -> int:
    """bf16 flop of sparse MLA per (query, selected row): QK^T over 576 dims and PV over 512."""
    return heads * (D_QK + D_V) * 2


def idx_flop_per_pair(h_index: int) -> int:
    """FP8 flop of the indexer per (query, visible key): H_I dot products of 128 dims."""
    return h_index * D_INDEX * 2


def _peaks():
    """Roofline denominators: the measured copy bandwidth and bf16 GEMM rates of
    this machine's B200s; FP8 = the measured bf16 burst rate times the nominal dense
    FP8/bf16 ratio (4.5 / 2.25 PFLOP/s) unless an FP8 figure was measured."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        bf16 = float(d["bf16_tflops"])
        fp8 = float(d["fp8_tflops"]) if "fp8_tflops" in d else 2.0 * bf16
        return {"hbm": float(d["hbm_gbs"]), "bf16": bf16,
                "bf16_sustained": float(d.get("bf16_tflops_sustained", bf16)), "fp8": fp8,
                "src": "measured", "fp8_src": "measured" if "fp8_tflops" in d else "2 x measured bf16 burst"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "fp8": 3180.0, "src": "fallback",
                "fp8_src": "2 x fallback bf16"}


class ClockSampler:
    """nvidia-smi samples (every 20 ms) of the SM clock and throttle reasons.

    Started before the warm-up, so that sampling is running when the timed region
    begins; mark_start()/mark_end() bracket the timed region, and summary() keeps
    the samples taken inside it.  A region shorter than the sampling interval holds
    no sample: then the samples within 100 ms of it are used and `window` says so.
    """

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines: list[tuple[float, str]] = []
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.monotonic() + 3.0                # wait until sampling has started
            while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        t0 = self.t0 if self.t0 is not None else float("-inf")
        t1 = self.t1 if self.t1 is not None else float("inf")
        window = "timed region"
        sel = [ln for t, ln in self.lines if t0 <= t <= t1]
        if not sel:
            window = "within 100 ms of the timed region"
            sel = [ln for t, ln in self.lines if t0 - 0.1 <= t <= t1 + 0.1]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in sel:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "window": window}


def _smi_index(local: int) -> int:
    """nvidia-smi index of the CUDA device `local` (honours CUDA_VISIBLE_DEVICES)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    parts = [p.strip() for p in vis.split(",") if p.strip()]
    if parts and all(p.isdigit() for p in parts) and local < len(parts):
        return int(parts[local])
    return local


def reduce_max(value: float, device=None) -> float:
    """Max of `value` over the ranks of the default process group (identity when
    there is none); used for the timed region, which is reported as the max over
    ranks."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return units_per_rank * world / (ms / 1e3)


def rank_seed(rank: int) -> int:
    """Each rank runs its own shard: the same workload drawn from its own seed."""
    return rank


def algorithmic_pairs(q_pos: np.ndarray, k: int) -> tuple[int, int]:
    """(indexer (query, visible key) pairs, sparse-MLA (query, selected row) pairs)
    of one call: n_t = q_pos + 1 visible keys, min(n_t, k) selected rows."""
    n = np.asarray(q_pos, dtype=np.int64) + 1
    return int(n.sum()), int(np.minimum(n, k).sum())


# ----------------------------------------------------------------------------- one call of the path


class Call:
    """Device buffers and workspaces of one call (one batch) of the path."""

    def __init__(self, wl, bh, dev: dict, device, out=None, lse=None, kv_rows=None, scores=None, idx=None,
                 page_size=0, page_table=None, fused_hist=False):
        import torch

        from sparse_attention_weight_b200 import binding as B
        self.B = B
        self.wl, self.bh, self.dev = wl, bh, dev
        self.db = B.DeviceBatch.from_host(bh, device, kv_rows=kv_rows, page_size=page_size, page_table=page_table)
        T = bh.num_q
        self.T = T
        self.ld = (bh.max_kv_len + 3) // 4 * 4
        # buffers shared between calls (the chunks of a prefill) are viewed at this call's shape
        self.scores = (scores.view(-1)[:T * self.ld].view(T, self.ld) if scores is not None
                       else torch.empty((T, self.ld), dtype=torch.float32, device=device))
        self.idx = idx if idx is not None else torch.empty((T, wl.k), dtype=torch.int32, device=device)
        self.out = out if out is not None else torch.empty((T, wl.heads, D_V), dtype=torch.int16, device=device)
        self.lse = lse if lse is not None else torch.empty((T, wl.heads), dtype=torch.float32, device=device)
        self.ws_i = B.workspace(B.OP_INDEXER, self.db, H_I=wl.h_index, ld=self.ld, device=device)
        # indexer -> top-k fused through the key histogram (measured separately; the
        # default path is unfused, which is faster here)
        self.hist = (torch.empty((T, 2048), dtype=torch.int32, device=device)
                     if fused_hist and B.topk_uses_hist(self.db, wl.k) else None)
        self.ws_t = B.workspace(B.OP_TOPK, self.db, k=wl.k, device=device)
        self.ws_m = B.workspace(B.OP_SPARSE_MLA, self.db, H=wl.heads, k=wl.k, device=device)
        self.idx_pairs, self.sel_pairs = algorithmic_pairs(bh.q_pos, wl.k)

    def run(self, stream, ev=None, base=0):
        """The three stages on `stream`; with `ev`, event ev[base + i] is recorded
        before stage i and ev[base + 3] after the last."""
        B, wl, d = self.B, self.wl, self.dev
        if ev is not None:
            ev[base].record(stream)
        if self.hist is not None:
            B.dsa_indexer_scores_hist(self.db, d["q_idx"], d["k_idx"], d["w"], wl.h_index, self.scores, self.ld,
                                      self.hist, self.ws_i, stream)
        else:
            B.dsa_indexer_scores(self.db, d["q_idx"], d["k_idx"], d["w"], wl.h_index, self.scores, self.ld,
                                 self.ws_i, stream)
        if ev is not None:
            ev[base + 1].record(stream)
        if self.hist is not None:
            B.dsa_topk_hist(self.db, self.scores, self.ld, self.hist, wl.k, self.idx, self.ws_t, stream)
        else:
            B.dsa_topk(self.db, self.scores, self.ld, wl.k, self.idx, self.ws_t, stream)
        if ev is not None:
            ev[base + 2].record(stream)
        B.dsa_sparse_mla(self.db, d["q"], d["kv"], self.idx, wl.k, wl.heads, wl.sm_scale, self.out, self.lse,
                         self.ws_m, stream)
        if ev is not None:
            ev[base + 3].record(stream)

    def check_status(self):
        for ws in (self.ws_i, self.ws_t, self.ws_m):
            flags = self.B.read_device_status(ws)
            if flags:
                raise RuntimeError(f"device status flags 0x{flags:x}")


def time_calls(calls: list, args, world: int, device, clk) -> dict:
    """Warm-up, then args.steps timed steps of the calls run back to back (one step
    = every call once), L2 flushed before each step; per-stage CUDA events."""
    import torch

    from sparse_attention_weight_b200 import binding as B
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    n_ev = 4 * len(calls)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for _ in range(args.warmup):
        flush.zero_()
        for c in calls:
            c.run(stream)
    torch.cuda.synchronize()
    for c in calls:
        c.check_status()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = B.launch_count()
    clk.mark_start()
    for s in range(args.steps):
        flush.zero_()
        for i, c in enumerate(calls):
            c.run(stream, events[s], 4 * i)
    torch.cuda.synchronize()
    clk.mark_end()
    launches = B.launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    # stage[s, i, j]: step s, call i, stage j (ms)
    stage = np.array([[[events[s][4 * i + j].elapsed_time(events[s][4 * i + j + 1]) for j in range(3)]
                       for i in range(len(calls))] for s in range(args.steps)])
    step_ms = np.array([events[s][0].elapsed_time(events[s][n_ev - 1]) for s in range(args.steps)])
    total_ms = reduce_max(float(step_ms.sum()), device)
    for c in calls:
        c.check_status()
    return {"ms_per_step": total_ms / args.steps, "stage_ms": stage.sum(axis=1).mean(axis=0).tolist(),
            "launches": launches, "launches_per_step": launches / args.steps}


def rates(wl, calls, res, peaks) -> dict:
    """Per-stage rates of a timed workload against the roofline denominators."""
    idx_ms, topk_ms, mla_ms = res["stage_ms"]
    idx_pairs = sum(c.idx_pairs for c in calls)
    sel_pairs = sum(c.sel_pairs for c in calls)
    T = sum(c.T for c in calls)
    decode = wl.kind == "decode"
    idx_tflops = idx_pairs * idx_flop_per_pair(wl.h_index) / (idx_ms / 1e3) / 1e12
    mla_tflops = sel_pairs * mla_flop_per_pair(wl.heads) / (mla_ms / 1e3) / 1e12
    # sparse MLA bytes: gathered rows + queries in + outputs out + index lists
    mla_bytes = sel_pairs * D_QK * 2 + T * wl.heads * (D_QK + D_V) * 2 + T * wl.k * 4
    # indexer bytes: keys of every sequence once + queries + weights + scores written
    k_rows = sum(int(c.bh.kv_len.sum()) for c in calls) if decode else sum(int(c.bh.max_kv_len) for c in calls)
    idx_bytes = k_rows * D_INDEX + T * wl.h_index * (D_INDEX + 4) + idx_pairs * 4
    topk_bytes = idx_pairs * 4 + T * wl.k * 4
    out = {
        "indexer": {"ms": idx_ms, "fp8_tflops": idx_tflops, "fp8_frac": idx_tflops / peaks["fp8"],
                    "gbs": idx_bytes / (idx_ms / 1e3) / 1e9, "hbm_frac": idx_bytes / (idx_ms / 1e3) / 1e9 / peaks["hbm"]},
        "topk": {"ms": topk_ms, "gbs": topk_bytes / (topk_ms / 1e3) / 1e9,
                 "hbm_frac": topk_bytes / (topk_ms / 1e3) / 1e9 / peaks["hbm"]},
        "sparse_mla": {"ms": mla_ms, "bf16_tflops": mla_tflops, "bf16_frac": mla_tflops / peaks["bf16"],
                       "gbs": mla_bytes / (mla_ms / 1e3) / 1e9,
                       "hbm_frac": mla_bytes / (mla_ms / 1e3) / 1e9 / peaks["hbm"]},
    }
    if decode:
        roof = {"bound": "hbm", "kernel": "sparse_mla (gather)", "achieved": out["sparse_mla"]["gbs"],
                "peak": peaks["hbm"], "unit": "GB/s", "peak_source": peaks["src"] + " copy bandwidth",
                "algorithmic_bytes_per_launch": mla_bytes / len(calls)}
    else:
        roof = {"bound": "tensor", "kernel": "sparse_mla", "achieved": mla_tflops, "peak": peaks["bf16"],
                "unit": "TFLOP/s", "peak_source": peaks["src"] + " bf16 (burst)",
                "algorithmic_flop_per_launch": sel_pairs * mla_flop_per_pair(wl.heads) / len(calls)}
    roof["frac"] = roof["achieved"] / roof["peak"]
    return {"stages": out, "roofline": roof}


# ----------------------------------------------------------------------------- workloads


def host_call(wl, device, seed, chunk=None):
    from sparse_attention_weight_b200 import binding as B
    from sparse_attention_weight_b200 import inputs
    ins = inputs.make_inputs(wl, seed=seed, chunk_index=chunk)
    dev = {n: B.bits_to_tensor(ins[n], device) for n in ("q_idx", "k_idx", "w", "q", "kv")}
    return Call(wl, ins["batch"], dev, device), ins


def device_calls(wl, device, seed, fused_hist=False):
    """The calls of one step of a workload with device-drawn inputs (a chunked
    prefill: one call per chunk against the growing cache prefix)."""
    import torch

    from sparse_attention_weight_b200 import inputs
    if wl.kind == "chunked_prefill":
        nchunks = wl.seq_len // wl.chunk
        full = inputs.make_batch(dataclasses.replace(wl, kind="prefill"), seed)
        cache = inputs.device_cache_tensors(wl, full, device, seed)
        out = torch.empty((wl.seq_len, wl.heads, D_V), dtype=torch.int16, device=device)
        lse = torch.empty((wl.seq_len, wl.heads), dtype=torch.float32, device=device)
        scores = torch.empty(wl.chunk * wl.seq_len, dtype=torch.float32, device=device)
        idx = torch.empty((wl.chunk, wl.k), dtype=torch.int32, device=device)
        calls = []
        for c in range(nchunks):
            bh = inputs.make_batch(wl, seed, c)
            qt = inputs.device_query_tensors(wl, bh, device, seed, chunk=c)
            r = slice(c * wl.chunk, (c + 1) * wl.chunk)
            calls.append(Call(wl, bh, {**qt, **cache}, device, out=out[r], lse=lse[r], kv_rows=wl.seq_len,
                              scores=scores, idx=idx))
        return calls
    bh = inputs.make_batch(wl, seed)
    dev = {**inputs.device_query_tensors(wl, bh, device, seed), **inputs.device_cache_tensors(wl, bh, device, seed)}
    if wl.name in PAGED:
        # the same rows scattered into pages of the cache pool
        ps = PAGED[wl.name]
        table, src = inputs.paged_layout(bh, ps, seed)
        src_t = torch.as_tensor(src, device=device)
        used = src_t >= 0
        for name in ("k_idx", "kv"):
            pool = torch.zeros((src.size, dev[name].shape[1]), dtype=dev[name].dtype, device=device)
            pool[used] = dev[name][src_t[used]]
            dev[name] = pool
        return [Call(wl, bh, dev, device, kv_rows=src.size, page_size=ps, page_table=table)]
    return [Call(wl, bh, dev, device, fused_hist=fused_hist)]


def sub_record(wl, args, rank, world, device, peaks, fused_hist=False) -> dict:
    """A full-size workload timed like the headline, with device-drawn inputs."""
    import torch
    calls = device_calls(wl, device, rank_seed(rank), fused_hist)
    sub_args = argparse.Namespace(**{**vars(args), "warmup": max(3, args.warmup)})
    with ClockSampler(_smi_index(device.index or 0)) as clk:
        res = time_calls(calls, sub_args, world, device, clk)
    T = sum(c.T for c in calls)
    decode = wl.kind == "decode"
    r = rates(wl, calls, res, peaks)
    rec = {"metric": "DSA decode queries/s" if decode else "DSA prefill tokens/s",
           "value": whole_job_rate(T, world, res["ms_per_step"]), "unit": "queries/s" if decode else "tokens/s",
           "ms_per_step": res["ms_per_step"], "steps": sub_args.steps, "warmup": sub_args.warmup,
           "calls_per_step": len(calls), "queries_per_step": T, "config": config_of(wl, args),
           "roofline": r["roofline"], "stages": r["stages"], "gpu_launches": res["launches"],
           "clocks": clk.summary(), "data": "synthetic, drawn on the device (seeded Philox)",
           "indexer_topk": "fused through the emitted key histogram" if fused_hist else "unfused"}
    del calls
    torch.cuda.empty_cache()
    return rec


def project_record(args, device, peaks, seed: int) -> dict:
    """The step before the path (dsa_project_append) on the last 4096-token chunk
    of the 64K prefill: d_model 7168, H_I 64, H 128, appended to a 65536-row cache.
    One call = the stacked projection GEMM (cuBLASLt) + the RoPE/cast/append kernel."""
    import torch

    from sparse_attention_weight_b200 import binding as B
    from sparse_attention_weight_b200 import inputs
    T, d, H_I, H, rows = 4096, 7168, 64, 128, 65536
    n_all = H_I * D_INDEX + D_INDEX + H_I + D_QK + H * D_QK
    pos = np.arange(rows - T, rows, dtype=np.int32)
    bh = inputs.Batch(np.zeros(1, np.int64), np.array([rows], np.int32), np.zeros(T, np.int32), pos,
                      np.arange(T, dtype=np.int32))
    db = B.DeviceBatch.from_host(bh, device)
    g = torch.Generator(device=device)
    g.manual_seed(seed * 7919 + 7100)
    hidden = torch.randn((T, d), generator=g, device=device).to(torch.bfloat16).view(torch.int16)
    w_all = (torch.randn((n_all, d), generator=g, device=device) / np.sqrt(d)).to(torch.bfloat16).view(torch.int16)
    q_idx = torch.empty((T, H_I, D_INDEX), dtype=torch.uint8, device=device)
    w = torch.empty((T, H_I), dtype=torch.float32, device=device)
    q = torch.empty((T, H, D_QK), dtype=torch.int16, device=device)
    k_cache = torch.zeros((rows, D_INDEX), dtype=torch.uint8, device=device)
    kv_cache = torch.zeros((rows, D_QK), dtype=torch.int16, device=device)
    ws = B.workspace(B.OP_PROJECT, db, H_I=H_I, H=H, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    run = lambda: B.dsa_project_append(db, hidden, w_all, d, H_I, H, 10000.0, q_idx, w, q, k_cache, kv_cache, ws)
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        run()
    torch.cuda.synchronize()
    if B.read_device_status(ws):
        raise RuntimeError("device status flags in dsa_project_append")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    l0 = B.launch_count()
    for e0, e1 in ev:
        flush.zero_()
        e0.record()
        run()
        e1.record()
    torch.cuda.synchronize()
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    flop = 2.0 * T * d * n_all
    # the epilogue kernel's algorithmic bytes: fp32 projections in, stored outputs and cache rows out
    epi_bytes = T * n_all * 4 + T * (H_I * D_INDEX + H_I * 4 + H * D_QK * 2) + T * (D_INDEX + D_QK * 2)
    return {"metric": "projection + RoPE + cache append tokens/s", "value": T / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": args.steps, "calls_per_step": 1, "queries_per_step": T,
            "config": {"workload": "project_append_4k", "tokens": T, "d_model": d, "h_index": H_I, "heads": H,
                       "cache_rows": rows, "l2": "flushed before every timed step (512 MB write)"},
            "stages": {"gemm_plus_epilogue": {"ms": ms, "tflops": flop / (ms / 1e3) / 1e12,
                                              "bf16_frac": flop / (ms / 1e3) / 1e12 / peaks["bf16"]},
                       "epilogue_algorithmic_bytes": epi_bytes},
            "gpu_launches": B.launch_count() - l0,
            "data": "synthetic, drawn on the device (seeded Philox); GEMM by cuBLASLt (a plain library GEMM), "
                    "RoPE / casts / append by the library's own kernel"}


def backward_record(args, device, peaks, seed: int) -> dict:
    """The sparse-MLA backward (dsa_sparse_mla_backward) on a 2048-token prefill
    (k = 2048, H = 128: every query attends over all its visible rows), after a
    forward call that provides the stored output and lse."""
    import torch

    from sparse_attention_weight_b200 import binding as B
    from sparse_attention_weight_b200 import inputs
    L, k, H = 2048, 2048, 128
    wl = dataclasses.replace(WORKLOADS["prefill_8k"], name="prefill_2k_bwd", seq_len=L, k=k, heads=H)
    bh = inputs.make_batch(wl, seed)
    dev = {**inputs.device_query_tensors(wl, bh, device, seed), **inputs.device_cache_tensors(wl, bh, device, seed)}
    db = B.DeviceBatch.from_host(bh, device)
    idx = torch.full((L, k), -1, dtype=torch.int32, device=device)
    ar = torch.arange(k, device=device, dtype=torch.int32)
    for t0 in range(0, L, 256):                                 # query t selects rows 0..t
        tt = torch.arange(t0, min(L, t0 + 256), device=device, dtype=torch.int32)[:, None]
        idx[t0:t0 + tt.shape[0]] = torch.where(ar[None, :] <= tt, ar[None, :], torch.full_like(ar[None, :], -1))
    out = torch.empty((L, H, D_V), dtype=torch.int16, device=device)
    lse = torch.empty((L, H), dtype=torch.float32, device=device)
    ws = B.workspace(B.OP_SPARSE_MLA, db, H=H, k=k, device=device)
    B.dsa_sparse_mla(db, dev["q"], dev["kv"], idx, k, H, wl.sm_scale, out, lse, ws)
    g = torch.Generator(device=device)
    g.manual_seed(seed * 31 + 5)
    dout = torch.randn((L, H, D_V), generator=g, device=device).to(torch.bfloat16).view(torch.int16)
    dq = torch.empty((L, H, D_QK), dtype=torch.float32, device=device)
    dkv = torch.zeros((L, D_QK), dtype=torch.float32, device=device)
    wsb = B.workspace(B.OP_MLA_BACKWARD, db, H=H, k=k, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    run = lambda: B.dsa_sparse_mla_backward(db, dev["q"], dev["kv"], idx, k, H, wl.sm_scale, out, lse, dout, dq,
                                             dkv, wsb)
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        dkv.zero_()
        run()
    torch.cuda.synchronize()
    if B.read_device_status(wsb):
        raise RuntimeError("device status flags in dsa_sparse_mla_backward")
    steps = max(3, min(args.steps, 5))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    l0 = B.launch_count()
    for e0, e1 in ev:
        flush.zero_()
        dkv.zero_()
        e0.record()
        run()
        e1.record()
    torch.cuda.synchronize()
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    pairs = L * (L + 1) // 2
    flop = pairs * H * 2 * (2 * D_QK + D_V + D_QK + D_V)      # z, dP, dQ, dK, dV per (query, row, head)
    return {"metric": "sparse-MLA backward tokens/s", "value": L / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "steps": steps, "calls_per_step": 1, "queries_per_step": L,
            "config": {"workload": "prefill_2k_bwd", "seq_len": L, "k": k, "heads": H, "selected_pairs": pairs,
                       "l2": "flushed before every timed step (512 MB write)"},
            "stages": {"mla_backward": {"ms": ms, "tflops": flop / (ms / 1e3) / 1e12,
                                        "frac_of_bf16_tensor_peak": flop / (ms / 1e3) / 1e12 / peaks["bf16"]}},
            "gpu_launches": B.launch_count() - l0,
            "data": "synthetic, drawn on the device (seeded Philox); fp32 CUDA-core kernel with atomic d_kv"}


def config_of(wl, args) -> dict:
    decode = wl.kind == "decode"
    return {"workload": wl.name, "k": wl.k, "h_index": wl.h_index, "heads": wl.heads, "d_qk": D_QK, "d_v": D_V,
            "seq_len": wl.seq_len or None, "batch": wl.batch or None,
            "ctx": [wl.ctx_min, wl.ctx_max] if decode else None, "q_per_seq": wl.q_per_seq or None,
            "chunk": wl.chunk or None, "l2": "flushed before every timed step (512 MB write)",
            "kv_layout": f"paged, {PAGED[wl.name]}-row pages" if wl.name in PAGED else "contiguous per sequence",
            "parallelism": f"dp{args.gpus}" if args.gpus > 1 else "single"}


def e2e_headline(call, ins, args, world, device) -> dict:
    """The headline step through dsa_forward_host from pinned host buffers: the
    host->device copies of the step's inputs (cache and queries) and the
    device->host copy of its output are inside the timed region; the library
    overlaps them with the computation, query chunk by query chunk, on a copy-in,
    the compute and a copy-out stream."""
    import torch

    from sparse_attention_weight_b200 import binding as B
    wl, d = call.wl, call.dev
    stream = torch.cuda.current_stream()
    streams = (torch.cuda.Stream(device), stream, torch.cuda.Stream(device))
    ws_h = B.workspace(B.OP_FORWARD_HOST, call.db, H_I=wl.h_index, H=wl.heads, k=wl.k, device=device)
    host = {n: torch.from_numpy(ins[n].view(np.int16) if ins[n].dtype == np.uint16 else ins[n]).pin_memory()
            for n in ("q_idx", "k_idx", "w", "q", "kv")}
    out_host = torch.empty(tuple(call.out.shape), dtype=torch.int16).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        B.dsa_forward_host(call.db, host, d, wl.h_index, wl.heads, wl.k, wl.sm_scale, call.out, call.lse,
                           out_host, ws_h, streams)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    n_e2e = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / n_e2e, device)
    return {"value": whole_job_rate(call.T, world, e2e_ms), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms}


# ----------------------------------------------------------------------------- the CPU oracle


def _oracle_sample(wl, rows_max: int = 64):
    """Inputs of a seeded sample of the workload's query rows for the oracle (built
    outside any timed region): rows drawn uniformly at random (seeded), so that the
    mean time per row estimates the whole call's; per row its query tensors, per
    sequence its cache."""
    from sparse_attention_weight_b200 import inputs

    chunk = (wl.seq_len // wl.chunk - 1) if wl.kind == "chunked_prefill" else None
    bh = inputs.make_batch(wl, 0, chunk)
    order = np.random.default_rng(7).permutation(bh.num_q)[:rows_max]
    caches, rows = {}, []
    for t in order:
        b = int(bh.q_seq[t])
        if b not in caches:
            caches[b] = (inputs.cache_rows(wl, bh, "k_idx", 0, seq=b), inputs.cache_rows(wl, bh, "kv", 0, seq=b))
        rows.append((int(t), b, inputs.query_rows(wl, bh, "q_idx", 0, [t]), inputs.query_rows(wl, bh, "w", 0, [t]),
                     inputs.query_rows(wl, bh, "q", 0, [t])))
    return {"batch": bh, "caches": caches, "rows": rows}


def _time_oracle(wl, sample, budget_s: float):
    """Runs the oracle's full path on sample rows, in turn, until `budget_s` of
    oracle time is spent; returns (rows done, seconds)."""
    import oracle

    bh = sample["batch"]
    done, elapsed = 0, 0.0
    while elapsed < budget_s:
        t, b, q_idx, w, q = sample["rows"][done % len(sample["rows"])]
        k_idx, kv = sample["caches"][b]
        s = time.perf_counter()
        oracle.forward(np.zeros(1, np.int64), bh.kv_len[b:b + 1], np.zeros(1, np.int32), bh.q_pos[t:t + 1],
                       q_idx, k_idx, w, q, kv, wl.k, wl.sm_scale)
        elapsed += time.perf_counter() - s
        done += 1
    return done, elapsed


def cpu_baseline(wl, budget_s: float = 12.0, rows_max: int = 64):
    """Times the oracle on a bounded sample of the workload's rows (host cores)."""
    done, elapsed = _time_oracle(wl, _oracle_sample(wl, rows_max), budget_s)
    return {"value": done / elapsed, "cores": len(os.sched_getaffinity(0)), "rows": done, "seconds": elapsed}


# ----------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="prefill_8k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="time only the headline workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the prefill length (smaller cases for profiler captures)")
    ap.add_argument("--chunk", type=int, default=-1,
                    help="chunked workload: time only this chunk's call (default: all chunks)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the number of decode sequences (smaller cases for profiler captures)")
    args = ap.parse_args()
    wl = WORKLOADS[args.config]
    if args.seq_len:
        if wl.kind != "prefill":
            ap.error("--seq-len applies to prefill workloads")
        wl = dataclasses.replace(wl, name=f"{wl.name}@L={args.seq_len}", seq_len=args.seq_len)
    if args.batch:
        if wl.kind != "decode":
            ap.error("--batch applies to decode workloads")
        wl = dataclasses.replace(wl, name=f"{wl.name}@B={args.batch}", batch=args.batch)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    decode = wl.kind == "decode"
    metric = "DSA decode queries/s" if decode else "DSA prefill tokens/s"
    unit = "queries/s" if decode else "tokens/s"
    config = config_of(wl, args)

    if args.impl == "reference":
        if rank != 0:
            return
        # the oracle as it stands, on the host cores: W untimed and K timed steps,
        # each a bounded sample of the workload (the whole run stays within minutes)
        sample = _oracle_sample(wl)
        per_step = min(12.0, 90.0 / max(1, args.steps + args.warmup))
        for _ in range(args.warmup):
            _time_oracle(wl, sample, per_step)
        rows = secs = 0
        for _ in range(args.steps):
            r, sec = _time_oracle(wl, sample, per_step)
            rows += r
            secs += sec
        value = rows / secs
        cores = len(os.sched_getaffinity(0))
        line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / max(1, args.steps),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                                 "sample": f"each step: seeded uniformly random query rows of {wl.name} in turn "
                                           f"for {per_step:.1f} s of oracle time, full path per row (numpy "
                                           f"float64); {rows} rows in {secs:.1f} s over {args.steps} steps"},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from sparse_attention_weight_b200 import binding as B
    B.lib()
    peaks = _peaks()

    # ---- headline
    ins = None
    if wl.kind == "chunked_prefill" and args.chunk < 0:
        calls = device_calls(wl, device, rank_seed(rank))
        data = "synthetic, drawn on the device (seeded Philox)"
    else:
        call, ins = host_call(wl, device, rank_seed(rank), args.chunk if wl.kind == "chunked_prefill" else None)
        calls = [call]
        data = "synthetic (seeded host generator)"
    with ClockSampler(_smi_index(device.index or 0)) as clk:
        res = time_calls(calls, args, world, device, clk)
    T = sum(c.T for c in calls)
    r = rates(wl, calls, res, peaks)
    roof = r["roofline"]
    roof["traffic"] = (MLA_TRAFFIC_BYTES_PER_QUERY * T / len(calls)
                       if (MLA_TRAFFIC_BYTES_PER_QUERY and wl.kind == "prefill" and wl.heads == 128) else None)
    line = {
        "metric": metric, "value": whole_job_rate(T, world, res["ms_per_step"]), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16+fp8", "data": data, "config": config,
        "roofline": roof,
        "stages_ms": {"indexer": res["stage_ms"][0], "topk": res["stage_ms"][1], "sparse_mla": res["stage_ms"][2]},
        "stages": r["stages"],
        "peaks": {"hbm_gbs": peaks["hbm"], "bf16_tflops": peaks["bf16"], "fp8_tflops": peaks["fp8"],
                  "source": peaks["src"], "fp8_source": peaks["fp8_src"]},
        "gpu_launches": res["launches"],
        "clocks": clk.summary(),
    }
    if ins is not None and not args.no_e2e:
        e = e2e_headline(calls[0], ins, args, world, device)
        line["e2e"] = {"value": e["value"], "unit": unit, "h2d_bytes_per_step": e["h2d_bytes_per_step"],
                       "d2h_bytes_per_step": e["d2h_bytes_per_step"], "ms_per_step": e["ms_per_step"]}
    del calls, ins
    torch.cuda.empty_cache()

    # ---- the other full-size workloads, in the same run
    if not args.no_extra and not args.seq_len and not args.batch:
        line["workloads"] = {}
        for name in ("decode_b64", "decode_128k_mtp2", "decode_b1_128k", "chunked_64k"):
            if name != wl.name:
                line["workloads"][name] = sub_record(WORKLOADS[name], args, rank, world, device, peaks)
        # the indexer -> top-k fused through the emitted key histogram, same workload
        line["workloads"]["decode_128k_mtp2_fused_hist"] = sub_record(WORKLOADS["decode_128k_mtp2"], args, rank,
                                                                      world, device, peaks, fused_hist=True)
        line["workloads"]["project_append_4k"] = project_record(args, device, peaks, rank_seed(rank))
        line["workloads"]["prefill_2k_bwd"] = backward_record(args, device, peaks, rank_seed(rank))
        torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(wl)
        line["cpu_baseline"] = {"value": cb["value"], "unit": unit, "cores": cb["cores"], "kind": "oracle",
                                "sample": f"{cb['rows']} seeded uniformly random query rows of {wl.name} "
                                          f"(from a fixed sample of 64), full path per row (numpy float64), "
                                          f"{cb['seconds']:.1f} s"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
