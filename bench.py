"""Benchmark of the DSA hot path on B200 (prefill tokens/s or decode queries/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = the whole path (lightning indexer -> top-k -> sparse MLA) over one
call of the workload (default: prefill_8k, one sequence of 8192 tokens, top-2048,
H_I = 64, H = 128).  Inputs are seeded synthetic data resident in HBM; L2 is
flushed (a 512 MB write) before every timed step and the flush is outside the
timed events.  Per-stage CUDA events on the launching stream give each kernel's
duration for the roofline line.  `e2e` repeats the step through dsa_forward
from pinned host buffers, with the host->device copies of the step's inputs and
the device->host copy of its output inside the timed region.

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
seeded inputs (independent shards, no collective on the data path); the timed
region is bracketed by barriers and the reported time is the max over ranks.

--impl reference times the CPU oracle (numpy float64) on the host cores over a
bounded sample of rows of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
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
MLA_FLOP_PER_PAIR = 128 * (576 + 512) * 2       # per (query, selected row) at H = 128
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture
# (profiles/sparse_mla_prefill_L2304.md: 621.1 MB at 2304 queries), scaled by the
# number of queries (the traffic is the queries in and the outputs out; the cache
# gathers hit L2).  None where no capture stands for the current kernel.
MLA_TRAFFIC_BYTES_PER_QUERY = 621.1e6 / 2304
IDX_FLOP_PER_PAIR = 64 * 128 * 2                # per (query, visible key) at H_I = 64


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm": float(d["hbm_gbs"]), "bf16": float(d["bf16_tflops"]),
                "bf16_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "src": "measured"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "src": "fallback"}


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


def _algorithmic(wl, batch, idx_host=None):
    """Algorithmic work of one step: indexer (query, visible key) pairs and
    sparse-MLA (query, selected row) pairs; selected rows = min(n_t, k)."""
    n = batch.q_pos.astype(np.int64) + 1
    idx_pairs = int(n.sum())
    sel_pairs = int(np.minimum(n, wl.k).sum())
    return idx_pairs, sel_pairs


def run_ours(args, wl, rank, world, device):
    import torch

    from sparse_attention_weight_b200 import binding as B
    from sparse_attention_weight_b200 import inputs

    chunk = (wl.seq_len // wl.chunk - 1) if wl.kind == "chunked_prefill" else None
    ins = inputs.make_inputs(wl, seed=rank_seed(rank), chunk_index=chunk)
    bh = ins["batch"]
    T = bh.num_q
    B.lib()
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    db = B.DeviceBatch.from_host(bh, device)
    d = {n: B.bits_to_tensor(ins[n], device) for n in ("q_idx", "k_idx", "w", "q", "kv")}
    ld = (bh.max_kv_len + 3) // 4 * 4
    scores = torch.empty((T, ld), dtype=torch.float32, device=device)
    idx = torch.empty((T, wl.k), dtype=torch.int32, device=device)
    out = torch.empty((T, wl.heads, 512), dtype=torch.int16, device=device)
    lse = torch.empty((T, wl.heads), dtype=torch.float32, device=device)
    ws_i = B.workspace(B.OP_INDEXER, db, H_I=wl.h_index, ld=ld, device=device)
    ws_t = B.workspace(B.OP_TOPK, db, k=wl.k, device=device)
    ws_m = B.workspace(B.OP_SPARSE_MLA, db, H=wl.heads, k=wl.k, device=device)
    ws_f = B.workspace(B.OP_FORWARD, db, H_I=wl.h_index, H=wl.heads, k=wl.k, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        B.dsa_indexer_scores(db, d["q_idx"], d["k_idx"], d["w"], wl.h_index, scores, ld, ws_i, stream)
        if ev:
            ev[1].record(stream)
        B.dsa_topk(db, scores, ld, wl.k, idx, ws_t, stream)
        if ev:
            ev[2].record(stream)
        B.dsa_sparse_mla(db, d["q"], d["kv"], idx, wl.k, wl.heads, wl.sm_scale, out, lse, ws_m, stream)
        if ev:
            ev[3].record(stream)

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(_smi_index(device.index or 0)) as clk:      # sampling from before the warm-up
        for _ in range(args.warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        for ws in (ws_i, ws_t, ws_m):
            flags = B.read_device_status(ws)
            if flags:
                raise RuntimeError(f"device status flags 0x{flags:x}")
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        for k in range(args.steps):
            flush.zero_()
            step(events[k])
        torch.cuda.synchronize()
        clk.mark_end()
    if world > 1:
        torch.distributed.barrier()
    stage = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in events])   # ms
    total_ms = reduce_max(float(stage.sum()), device)
    ms_per_step = total_ms / args.steps
    idx_pairs, sel_pairs = _algorithmic(wl, bh)

    # ---- end to end through dsa_forward with host buffers
    e2e = None
    if not args.no_e2e:
        host = {n: torch.from_numpy(ins[n].view(np.int16) if ins[n].dtype == np.uint16 else ins[n]).pin_memory()
                for n in ("q_idx", "k_idx", "w", "q", "kv")}
        out_host = torch.empty((T, wl.heads, 512), dtype=torch.int16).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = out_host.numel() * out_host.element_size()

        def e2e_step():
            for n in host:
                d[n].copy_(host[n], non_blocking=True)
            B.dsa_forward(db, d["q_idx"], d["k_idx"], d["w"], wl.h_index, d["q"], d["kv"], wl.heads, wl.k,
                          wl.sm_scale, out, lse, ws_f, stream)
            out_host.copy_(out, non_blocking=True)

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
        e2e = {"value": whole_job_rate(T, world, e2e_ms), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms}
    splits = 1
    try:
        from sparse_attention_weight_b200.binding import lib  # noqa: F401
        pairs = (torch.cuda.get_device_properties(device).multi_processor_count // 2)
        splits = max(1, min(pairs // max(T, 1), (wl.k + 127) // 128, 16))
    except Exception:
        pass
    return {
        "T": T, "ms_per_step": ms_per_step, "stage_ms": stage.mean(axis=0).tolist(),
        "idx_pairs": idx_pairs, "sel_pairs": sel_pairs, "e2e": e2e, "clocks": clk.summary(),
        "launches_per_step": 4 + (1 if splits > 1 else 0),
        "k_idx_bytes": int(ins["k_idx"].nbytes), "n_vis": (bh.q_pos.astype(np.int64) + 1),
    }


def _oracle_sample(wl, rows_max: int = 64):
    """Inputs of a seeded sample of the workload's query rows for the oracle (built
    outside any timed region): per row its query tensors, per sequence its cache."""
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="prefill_8k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the prefill length (smaller cases for profiler captures)")
    args = ap.parse_args()
    wl = WORKLOADS[args.config]
    if args.seq_len:
        if wl.kind != "prefill":
            ap.error("--seq-len applies to prefill workloads")
        import dataclasses
        wl = dataclasses.replace(wl, name=f"{wl.name}@L={args.seq_len}", seq_len=args.seq_len)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    decode = wl.kind == "decode"
    metric = "DSA decode queries/s" if decode else "DSA prefill tokens/s"
    unit = "queries/s" if decode else "tokens/s"
    config = {"workload": wl.name, "k": wl.k, "h_index": wl.h_index, "heads": wl.heads,
              "d_qk": 576, "d_v": 512, "seq_len": wl.seq_len or None, "batch": wl.batch or None,
              "ctx": [wl.ctx_min, wl.ctx_max] if decode else None, "q_per_seq": wl.q_per_seq or None,
              "chunk": wl.chunk or None, "l2": "flushed before every timed step (512 MB write)",
              "parallelism": f"dp{args.gpus}" if args.gpus > 1 else "single"}

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
                                 "sample": f"each step: seeded query rows of {wl.name} in turn for "
                                           f"{per_step:.1f} s of oracle time, full path per row (numpy "
                                           f"float64); {rows} rows in {secs:.1f} s over {args.steps} steps"},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    res = run_ours(args, wl, rank, world, device)
    peaks = _peaks()
    T = res["T"]
    value = whole_job_rate(T, world, res["ms_per_step"])
    st = res["stage_ms"]
    mla_ms, idx_ms, topk_ms = st[2], st[0], st[1]
    mla_tflops = res["sel_pairs"] * MLA_FLOP_PER_PAIR * wl.heads / 128 / (mla_ms / 1e3) / 1e12
    if decode:
        # decode: the gather-bound kernel, against HBM
        gather = res["sel_pairs"] * 1152 + T * wl.heads * (576 + 512) * 2
        roof = {"bound": "hbm", "kernel": "sparse_mla", "achieved": gather / (mla_ms / 1e3) / 1e9,
                "peak": peaks["hbm"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "kernel": "sparse_mla", "achieved": mla_tflops, "peak": peaks["bf16"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peaks["src"] + (" (burst)" if roof["unit"] == "TFLOP/s" else "")
    roof["traffic"] = (MLA_TRAFFIC_BYTES_PER_QUERY * T) if wl.kind == "prefill" else None
    idx_tflops = res["idx_pairs"] * IDX_FLOP_PER_PAIR * wl.h_index / 64 / (idx_ms / 1e3) / 1e12
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16+fp8", "data": "synthetic", "config": config,
        "roofline": roof,
        "stages_ms": {"indexer": idx_ms, "topk": topk_ms, "sparse_mla": mla_ms},
        "stage_rates": {"indexer_fp8_tflops": idx_tflops, "sparse_mla_bf16_tflops": mla_tflops,
                        "topk_gbs": (res["idx_pairs"] * 4 + T * wl.k * 4) / (topk_ms / 1e3) / 1e9},
        "gpu_launches": res["launches_per_step"] * args.steps,
        "clocks": res["clocks"],
    }
    if res["e2e"]:
        e = res["e2e"]
        line["e2e"] = {"value": e["value"], "unit": unit, "h2d_bytes_per_step": e["h2d_bytes_per_step"],
                       "d2h_bytes_per_step": e["d2h_bytes_per_step"], "ms_per_step": e["ms_per_step"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(wl)
        line["cpu_baseline"] = {"value": cb["value"], "unit": unit, "cores": cb["cores"], "kind": "oracle",
                                "sample": f"{cb['rows']} seeded query rows of {wl.name}, full path per row "
                                          f"(numpy float64), {cb['seconds']:.1f} s"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
