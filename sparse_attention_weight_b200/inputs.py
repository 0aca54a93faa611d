"""Seeded synthetic inputs for the DSA path.

This module only draws random numbers and stores them in the input formats
(FP8 E4M3 bytes, bf16 bit patterns, fp32).  It holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it.

Streams.  Every tensor is drawn in row chunks of ``ROW_CHUNK`` rows; chunk c
of tensor ``tid`` in sequence ``b`` comes from
``numpy.random.default_rng([seed, cfg_id, tid, b, c])``, so any row can be
regenerated on its own (the oracle samples rows of the large workloads).
Tensor ids: 0 indexer query q_I, 1 indexer key k_I, 2 indexer head weights w,
3 MLA query Q, 4 latent KV rows, 5 decode context lengths.

Rows of per-query tensors are numbered by position for prefill (queries are
positions 0..L-1 of sequence 0) and by the query's ordinal inside its
sequence for decode.  Cache rows are numbered by position.

Quantisation: N(0,1) float32 values are clamped to +-448 and cast to E4M3 by
PyTorch's round-to-nearest-even cast; bf16 tensors use PyTorch's RNE cast.

The benchmark's largest workloads (gigabytes of queries and caches) are drawn
on the device instead (``device_query_tensors``, ``device_cache_tensors``):
the same distributions and casts from PyTorch's seeded Philox generator.  The
parity tests use the host streams above.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from .configs import D_INDEX, D_QK, Workload

ROW_CHUNK = 256
E4M3_MAX = 448.0

T_QIDX, T_KIDX, T_W, T_Q, T_KV, T_LEN = 0, 1, 2, 3, 4, 5


def _chunk_rows(seed: int, cfg_id: int, tid: int, seq: int, row0: int, nrows: int,
                row_shape: tuple[int, ...], std: float = 1.0) -> np.ndarray:
    """float32 N(0, std^2) rows [row0, row0+nrows) of one tensor of one sequence."""
    out = np.empty((nrows,) + tuple(row_shape), dtype=np.float32)
    if nrows == 0:
        return out
    c0, c1 = row0 // ROW_CHUNK, (row0 + nrows - 1) // ROW_CHUNK
    for c in range(c0, c1 + 1):
        rng = np.random.default_rng([seed, cfg_id, tid, seq, c])
        chunk = rng.standard_normal((ROW_CHUNK,) + tuple(row_shape), dtype=np.float32)
        if std != 1.0:
            chunk *= np.float32(std)
        lo = max(row0, c * ROW_CHUNK)
        hi = min(row0 + nrows, (c + 1) * ROW_CHUNK)
        out[lo - row0:hi - row0] = chunk[lo - c * ROW_CHUNK:hi - c * ROW_CHUNK]
    return out


def to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 bytes (uint8) via PyTorch's RNE cast, clamped to +-448."""
    t = torch.from_numpy(np.clip(np.ascontiguousarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16) via PyTorch's RNE cast."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@dataclass
class Batch:
    """Host copy of the batch description (mirrors ``dsa_batch`` in dsa.h)."""
    kv_offset: np.ndarray   # int64 [B]   first cache row of sequence b
    kv_len: np.ndarray      # int32 [B]   cache rows of sequence b
    q_seq: np.ndarray       # int32 [T]   sequence of query t
    q_pos: np.ndarray       # int32 [T]   position of query t; keys 0..q_pos visible
    q_row: np.ndarray       # int32 [T]   row of query t in its sequence's query streams

    @property
    def num_seqs(self) -> int:
        return int(self.kv_len.shape[0])

    @property
    def num_q(self) -> int:
        return int(self.q_pos.shape[0])

    @property
    def max_kv_len(self) -> int:
        return int(self.kv_len.max()) if self.kv_len.size else 0

    @property
    def max_q_per_seq(self) -> int:
        if self.q_seq.size == 0:
            return 0
        return int(np.bincount(self.q_seq, minlength=self.num_seqs).max())

    @property
    def total_rows(self) -> int:
        return int(self.kv_len.sum())


def decode_lengths(wl: Workload, seed: int = 0) -> np.ndarray:
    """Context lengths of a decode workload (uniform integers, inclusive bounds)."""
    rng = np.random.default_rng([seed, wl.cfg_id, T_LEN])
    return rng.integers(wl.ctx_min, wl.ctx_max, size=wl.batch, endpoint=True).astype(np.int32)


def make_batch(wl: Workload, seed: int = 0, chunk_index: int | None = None) -> Batch:
    """Batch description of one call of the workload.

    Prefill: one sequence of ``seq_len`` rows, queries at positions 0..L-1.
    Chunked prefill: call ``chunk_index`` c holds queries [c*chunk, (c+1)*chunk)
    against the cache prefix [0, (c+1)*chunk).
    Decode: ``batch`` sequences; the context length n includes the new
    token(s), so the q_per_seq queries sit at positions n-q_per_seq .. n-1.
    """
    if wl.kind == "prefill":
        L = wl.seq_len
        return Batch(np.zeros(1, np.int64), np.array([L], np.int32), np.zeros(L, np.int32),
                     np.arange(L, dtype=np.int32), np.arange(L, dtype=np.int32))
    if wl.kind == "chunked_prefill":
        c = 0 if chunk_index is None else int(chunk_index)
        lo, hi = c * wl.chunk, (c + 1) * wl.chunk
        if hi > wl.seq_len or c < 0:
            raise ValueError("chunk index out of range")
        pos = np.arange(lo, hi, dtype=np.int32)
        return Batch(np.zeros(1, np.int64), np.array([hi], np.int32), np.zeros(hi - lo, np.int32),
                     pos, pos.copy())
    if wl.kind == "decode":
        lens = decode_lengths(wl, seed)
        off = np.zeros(wl.batch, np.int64)
        off[1:] = np.cumsum(lens[:-1].astype(np.int64))
        qs = np.repeat(np.arange(wl.batch, dtype=np.int32), wl.q_per_seq)
        j = np.tile(np.arange(wl.q_per_seq, dtype=np.int32), wl.batch)
        pos = (lens[qs] - wl.q_per_seq + j).astype(np.int32)
        return Batch(off, lens, qs, pos, j)
    raise ValueError(f"unknown workload kind {wl.kind}")


def query_rows(wl: Workload, batch: Batch, which: str, seed: int = 0,
               queries: np.ndarray | None = None) -> np.ndarray:
    """Per-query tensor for the given query indices (all queries by default).

    which: "q_idx" -> uint8 [n, H_I, 128]; "w" -> float32 [n, H_I];
    "q" -> uint16 bf16 bits [n, H, 576].
    """
    if queries is None:
        queries = np.arange(batch.num_q)
    queries = np.asarray(queries, dtype=np.int64)
    if which == "q_idx":
        tid, shape, std = T_QIDX, (wl.h_index, D_INDEX), 1.0
    elif which == "w":
        tid, shape, std = T_W, (wl.h_index,), 1.0 / np.sqrt(wl.h_index)
    elif which == "q":
        tid, shape, std = T_Q, (wl.heads, D_QK), 1.0
    else:
        raise ValueError(which)
    out = np.empty((queries.size,) + shape, np.float32)
    # group consecutive queries of one sequence with consecutive rows
    i = 0
    while i < queries.size:
        t = queries[i]
        b, r = int(batch.q_seq[t]), int(batch.q_row[t])
        j = i + 1
        while (j < queries.size and batch.q_seq[queries[j]] == b
               and batch.q_row[queries[j]] == r + (j - i)):
            j += 1
        out[i:j] = _chunk_rows(seed, wl.cfg_id, tid, b, r, j - i, shape, std)
        i = j
    if which == "q_idx":
        return to_e4m3_bytes(out)
    if which == "q":
        return to_bf16_bits(out)
    return out


def cache_rows(wl: Workload, batch: Batch, which: str, seed: int = 0,
               seq: int | None = None, row0: int = 0, nrows: int | None = None) -> np.ndarray:
    """Cache tensor rows.  With ``seq`` given: rows [row0, row0+nrows) of that
    sequence.  Otherwise: the whole packed cache of the batch (sequence b at
    rows kv_offset[b] ..).

    which: "k_idx" -> uint8 [rows, 128]; "kv" -> uint16 bf16 bits [rows, 576].
    """
    if which == "k_idx":
        tid, shape, cast = T_KIDX, (D_INDEX,), to_e4m3_bytes
    elif which == "kv":
        tid, shape, cast = T_KV, (D_QK,), to_bf16_bits
    else:
        raise ValueError(which)
    if seq is not None:
        n = int(batch.kv_len[seq]) - row0 if nrows is None else nrows
        return cast(_chunk_rows(seed, wl.cfg_id, tid, seq, row0, n, shape))
    parts = [cast(_chunk_rows(seed, wl.cfg_id, tid, b, 0, int(batch.kv_len[b]), shape))
             for b in range(batch.num_seqs)]
    return np.concatenate(parts, axis=0) if parts else np.empty((0,) + shape, np.uint8)


def paged_layout(batch: Batch, page_size: int, seed: int = 0, spare_pages: int = 3):
    """A paged storage layout of the batch's caches (the block-table layout of
    paged inference caches): every sequence's rows cut into pages of
    `page_size`, the pages scattered over a physical pool in a seeded random
    order with a few unused pages.  Returns (page_table int32 [B, pages_per_seq],
    unused entries -1; src int64 [pool rows]: the contiguous row each physical
    row holds, -1 for padding).  Storage only: no values are computed."""
    lens = batch.kv_len.astype(np.int64)
    npages = (lens + page_size - 1) // page_size
    pps = int(max(1, (batch.max_kv_len + page_size - 1) // page_size))
    total = int(npages.sum()) + spare_pages
    perm = np.random.default_rng([seed, 7001, page_size]).permutation(total)
    table = np.full((batch.num_seqs, pps), -1, np.int32)
    src = np.full(total * page_size, -1, np.int64)
    k = 0
    for b in range(batch.num_seqs):
        for i in range(int(npages[b])):
            phys = int(perm[k])
            k += 1
            table[b, i] = phys
            n = int(min(page_size, lens[b] - i * page_size))
            src[phys * page_size: phys * page_size + n] = batch.kv_offset[b] + i * page_size + np.arange(n)
    return table, src


def projection_inputs(T: int, d_model: int, n_rows: int, seed: int = 0) -> dict:
    """Hidden states ~ N(0,1) and a stacked projection matrix ~ N(0, 1/d_model)
    (so every projection is ~ N(0,1), the distribution of the path's inputs), as
    bf16 bits: hidden [T, d_model], w_all [n_rows, d_model]."""
    rng_h = np.random.default_rng([seed, 7100, T, d_model])
    rng_w = np.random.default_rng([seed, 7101, n_rows, d_model])
    h = rng_h.standard_normal((T, d_model), dtype=np.float32)
    w = rng_w.standard_normal((n_rows, d_model), dtype=np.float32) * np.float32(1.0 / np.sqrt(d_model))
    return {"hidden": to_bf16_bits(h), "w_all": to_bf16_bits(w)}


def make_inputs(wl: Workload, seed: int = 0, chunk_index: int | None = None) -> dict:
    """Every input of one call of the workload, as host numpy arrays."""
    batch = make_batch(wl, seed, chunk_index)
    return {
        "batch": batch,
        "q_idx": query_rows(wl, batch, "q_idx", seed),
        "w": query_rows(wl, batch, "w", seed),
        "q": query_rows(wl, batch, "q", seed),
        "k_idx": cache_rows(wl, batch, "k_idx", seed),
        "kv": cache_rows(wl, batch, "kv", seed),
    }


# ---------------------------------------------------------------------------
# Device-drawn inputs (benchmark workloads too large to draw on the host)
# ---------------------------------------------------------------------------

def _device_normal(shape, key: tuple, device, std: float = 1.0):
    """float32 N(0, std^2) tensor drawn on `device` by PyTorch's Philox generator,
    seeded from `key` (a tuple of small ints); the same key gives the same values
    on the same device type."""
    g = torch.Generator(device=device)
    h = 0
    for v in key:
        h = (h * 1_000_003 + int(v) + 1) % (1 << 63)
    g.manual_seed(h)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def device_query_tensors(wl: Workload, batch: Batch, device, seed: int = 0, chunk: int = 0) -> dict:
    """Per-query tensors of one call drawn on the device with the distributions of
    the host generator (q_I, k_I ~ N(0,1) -> E4M3 after clamping to +-448;
    w ~ N(0, 1/H_I) fp32; Q ~ N(0,1) -> bf16), keyed by (seed, cfg, tensor, chunk)."""
    T = batch.num_q
    qi = _device_normal((T, wl.h_index, D_INDEX), (seed, wl.cfg_id, T_QIDX, chunk), device)
    w = _device_normal((T, wl.h_index), (seed, wl.cfg_id, T_W, chunk), device, 1.0 / np.sqrt(wl.h_index))
    q = _device_normal((T, wl.heads, D_QK), (seed, wl.cfg_id, T_Q, chunk), device)
    return {"q_idx": qi.clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8),
            "w": w, "q": q.to(torch.bfloat16).view(torch.int16)}


def device_cache_tensors(wl: Workload, batch: Batch, device, seed: int = 0) -> dict:
    """The packed caches of a batch (k_I -> E4M3 bytes [rows, 128], latent rows ->
    bf16 bits [rows, 576]) drawn on the device, sequence by sequence."""
    rows = int(batch.kv_len.sum())
    k_idx = torch.empty((rows, D_INDEX), dtype=torch.uint8, device=device)
    kv = torch.empty((rows, D_QK), dtype=torch.int16, device=device)
    for b in range(batch.num_seqs):
        o, n = int(batch.kv_offset[b]), int(batch.kv_len[b])
        ki = _device_normal((n, D_INDEX), (seed, wl.cfg_id, T_KIDX, b), device)
        k_idx[o:o + n] = ki.clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
        kv[o:o + n] = _device_normal((n, D_QK), (seed, wl.cfg_id, T_KV, b), device).to(torch.bfloat16).view(torch.int16)
    return {"k_idx": k_idx, "kv": kv}
