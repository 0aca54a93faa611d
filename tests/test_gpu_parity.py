"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Same seeded inputs on both sides.  Bars: top-k bit-exact given the oracle's
scores (rounded to fp32); indexer scores within 1e-4 of max(|I|, sum|w|ReLU);
attention outputs within max-abs 1e-2 / mean-abs 1e-3 of the fp64 oracle;
end to end, selection mismatches only where scores tie the k-th score to 1e-4.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import build, inputs
from sparse_attention_weight_b200.configs import WORKLOADS, Workload

from . import helpers as H

pytestmark = pytest.mark.gpu

MID_PREFILL = Workload("mid_prefill", 20, "prefill", k=2048, h_index=64, heads=128, seq_len=2600)
MID_DEC2 = Workload("mid_decode2", 21, "decode", k=2048, h_index=64, heads=128, batch=6, ctx_min=1500,
                    ctx_max=5000, q_per_seq=2)
MID_DEC1 = Workload("mid_decode1", 22, "decode", k=512, h_index=64, heads=128, batch=5, ctx_min=300,
                    ctx_max=3000, q_per_seq=1)


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    B.lib()


def _sample_rows(T, k, extra=()):
    rows = {0, 1, T - 1, T - 2, min(T - 1, k - 1), min(T - 1, k), min(T - 1, k + 1), min(T - 1, 127),
            min(T - 1, 128), T // 2}
    rows |= set(int(x) for x in extra)
    rng = np.random.default_rng(123)
    rows |= set(int(x) for x in rng.integers(0, T, size=12))
    return sorted(r for r in rows if 0 <= r < T)


def _run_indexer(dev, wl, batch_host):
    T = batch_host.num_q
    ld = (batch_host.max_kv_len + 3) // 4 * 4
    scores = torch.full((T, ld), float("nan"), device=dev["q"].device)
    ws = B.workspace(B.OP_INDEXER, dev["batch"], H_I=wl.h_index, ld=ld, device=scores.device)
    B.dsa_indexer_scores(dev["batch"], dev["q_idx"], dev["k_idx"], dev["w"], wl.h_index, scores, ld, ws)
    assert B.read_device_status(ws) == 0
    return scores.cpu().numpy()


# ----------------------------------------------------------------------------- indexer

@pytest.mark.parametrize("wl", [WORKLOADS["tiny_prefill"], MID_PREFILL, MID_DEC2, MID_DEC1,
                                Workload("hi8", 23, "prefill", k=64, h_index=8, heads=8, seq_len=700),
                                Workload("hi16", 24, "prefill", k=64, h_index=16, heads=8, seq_len=700),
                                Workload("hi32", 25, "prefill", k=64, h_index=32, heads=8, seq_len=700),
                                Workload("hi12", 31, "prefill", k=64, h_index=12, heads=8, seq_len=700),
                                Workload("hi48", 32, "prefill", k=64, h_index=48, heads=8, seq_len=700),
                                Workload("hi20_dec", 33, "decode", k=64, h_index=20, heads=8, batch=3, ctx_min=300,
                                         ctx_max=900, q_per_seq=3),
                                Workload("hi60_dec", 34, "decode", k=64, h_index=60, heads=8, batch=4, ctx_min=100,
                                         ctx_max=700, q_per_seq=1)],
                         ids=lambda w: w.name)
def test_indexer_scores_match_oracle(cuda_device, wl):
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    dev = H.to_device(ins, cuda_device)
    got = _run_indexer(dev, wl, batch)
    T = batch.num_q
    rows = list(range(T)) if T <= 1100 else _sample_rows(T, wl.k)
    ref = H.oracle_rows(ins, wl, rows)
    for i, t in enumerate(rows):
        n = int(batch.q_pos[t]) + 1
        I = ref["scores"][i]
        assert I.shape == (n,)
        H.check_indexer_row(got[t, :n], I, H.condition_scale(ins, t, n), f"{wl.name} row {t}")
        # nothing written beyond the visible keys
        assert np.isnan(got[t, n:]).all()

# ----------------------------------------------------------------------------- top-k


def _topk_case(cuda_device, rows, k):
    """rows: list of float32 arrays (row t has n_t = len(rows[t]))."""
    T = len(rows)
    nmax = max(len(r) for r in rows)
    ld = (nmax + 3) // 4 * 4
    sc = np.full((T, ld), np.nan, np.float32)
    for t, r in enumerate(rows):
        sc[t, :len(r)] = r
    bh = inputs.Batch(np.zeros(T, np.int64), np.array([len(r) for r in rows], np.int32),
                      np.arange(T, dtype=np.int32), np.array([len(r) - 1 for r in rows], np.int32),
                      np.zeros(T, np.int32))
    db = B.DeviceBatch.from_host(bh, cuda_device, kv_rows=int(nmax))
    s_dev = torch.from_numpy(sc).to(cuda_device)
    idx = torch.full((T, k), -7, dtype=torch.int32, device=cuda_device)
    ws = B.workspace(B.OP_TOPK, db, k=k, device=cuda_device)
    B.dsa_topk(db, s_dev, ld, k, idx, ws)
    assert B.read_device_status(ws) == 0
    got = idx.cpu().numpy()
    want = oracle.topk_select(sc, np.array([len(r) for r in rows]), k)
    for t in range(T):
        assert np.array_equal(got[t], want[t]), f"row {t} (n={len(rows[t])})"


def test_topk_bit_exact_on_oracle_scores(cuda_device):
    wl = WORKLOADS["tiny_prefill"]
    ins = inputs.make_inputs(wl)
    ref = H.oracle_rows(ins, wl, range(0, 1024, 7))
    _topk_case(cuda_device, [I.astype(np.float32) for I in ref["scores"]], wl.k)


def test_topk_adversarial_rows(cuda_device):
    rng = np.random.default_rng(11)
    k = 2048
    rows = [
        rng.standard_normal(5000).astype(np.float32),
        np.round(rng.standard_normal(6000), 1).astype(np.float32),          # heavy ties
        np.zeros(4000, np.float32),                                           # all equal
        np.where(rng.random(4500) < 0.5, -0.0, 0.0).astype(np.float32),      # signed zeros only
        np.concatenate([np.full(100, 3.0), np.where(rng.random(4000) < 0.5, -0.0, 0.0)]).astype(np.float32),
        rng.standard_normal(k - 1).astype(np.float32),
        rng.standard_normal(k).astype(np.float32),
        rng.standard_normal(k + 1).astype(np.float32),
        (rng.standard_normal(9000) * 1e-30).astype(np.float32),             # subnormal-range values
        np.concatenate([rng.standard_normal(3000), [np.inf, -np.inf, np.inf]]).astype(np.float32),
        rng.integers(-3, 4, size=8192).astype(np.float32),
        np.array([1.5], np.float32),
    ]
    _topk_case(cuda_device, rows, k)
    _topk_case(cuda_device, rows[:5], 64)
    _topk_case(cuda_device, [rng.standard_normal(n).astype(np.float32) for n in (300, 257, 256, 255)], 256)


def test_topk_long_rows_from_l2(cuda_device):
    """Rows longer than a cluster's eight segment caches (> 163840 keys): two reads
    and a candidate list for few rows, with the streaming fallback when the
    threshold's bin overflows the list; the streaming kernel for many rows."""
    rng = np.random.default_rng(12)
    rows = [rng.standard_normal(170000).astype(np.float32),
            np.round(rng.standard_normal(180000), 2).astype(np.float32),
            np.zeros(170000, np.float32),                                    # all tied: fallback
            rng.integers(-3, 4, size=170000).astype(np.float32),             # 7 values: fallback
            np.concatenate([np.full(3000, 2.0), rng.standard_normal(170000) - 10.0]).astype(np.float32),
            rng.standard_normal(1500).astype(np.float32)]                    # n <= k in a long launch
    _topk_case(cuda_device, rows, 2048)
    # many very long rows (more than two per SM): the streaming kernel reads them from L2
    many = [np.round(rng.standard_normal(int(n)), 3).astype(np.float32) for n in rng.integers(164000, 166000, 300)]
    _topk_case(cuda_device, many, 2048)
    # many long rows that fit eight segment caches: one cluster per row
    many = [np.round(rng.standard_normal(int(n)), 3).astype(np.float32) for n in rng.integers(33000, 70000, 320)]
    _topk_case(cuda_device, many, 2048)


def test_topk_rows_shared_by_a_cluster(cuda_device):
    """Few long rows: a cluster of CTAs per row (8, 4 or 2 of them, by the number of
    rows), each caching one segment; ties across segment boundaries go to the lower
    index, and rows with n <= k or mass ties take the same cluster path."""
    rng = np.random.default_rng(13)
    k = 2048
    base = [np.round(rng.standard_normal(20000), 1).astype(np.float32),          # ties across segments
            np.zeros(16384, np.float32),                                         # all equal
            np.concatenate([rng.standard_normal(9000), np.full(9000, 5.0)]).astype(np.float32),
            rng.standard_normal(8193).astype(np.float32),
            rng.standard_normal(2000).astype(np.float32),                        # n <= k
            np.where(rng.random(12000) < 0.5, -0.0, 0.0).astype(np.float32)]
    for T in (6, 40, 100):              # clusters of 8, 4 (6 rows -> 8; 40 -> 4...) and 2 CTAs
        rows = [base[t % len(base)] if t < len(base) else rng.standard_normal(int(rng.integers(8192, 30000)))
                .astype(np.float32) for t in range(T)]
        _topk_case(cuda_device, rows, k)
    _topk_case(cuda_device, base[:3], 100)



def test_topk_cached_rows_with_a_list(cuda_device):
    """Many rows of 10240..20480 keys (one CTA per row, the row cached in shared
    memory): rows whose keys at or above the first pass's threshold bin fit the
    list take the two later passes and the output over that list, in index order
    (ties at the threshold included); rows whose list would overflow (few distinct
    values) or exceed a quarter of the row take the passes over the cache."""
    rng = np.random.default_rng(14)
    k = 2048
    rows = []
    for t in range(320):                                      # > 2 rows per SM: no cluster
        n = int(rng.integers(10240, 20481))
        kind = t % 4
        if kind == 0:
            r = rng.standard_normal(n)
        elif kind == 1:
            r = np.round(rng.standard_normal(n), 2)           # ties at the threshold
        elif kind == 2:
            r = rng.integers(-3, 4, size=n)                   # seven values: the list overflows
        else:
            r = np.concatenate([rng.standard_normal(n - 3000), np.full(3000, 4.0)])   # top k all tied
        rows.append(r.astype(np.float32))
    _topk_case(cuda_device, rows, k)

# ----------------------------------------------------------------------------- sparse MLA


def _mla_ref_rows(ins, idx_host, rows, wl):
    """The oracle's attention for `rows` over the index rows idx_host[rows]."""
    rows = list(rows)
    ref = H.oracle_rows(ins, wl, rows, selections=idx_host[rows])
    return ref["out"], ref["lse"]


def _run_mla(dev, wl, idx_host, T):
    idx = torch.from_numpy(idx_host.astype(np.int32)).to(dev["q"].device)
    out = torch.zeros((T, wl.heads, 512), dtype=torch.int16, device=idx.device)
    lse = torch.zeros((T, wl.heads), dtype=torch.float32, device=idx.device)
    ws = B.workspace(B.OP_SPARSE_MLA, dev["batch"], H=wl.heads, k=idx_host.shape[1], device=idx.device)
    B.dsa_sparse_mla(dev["batch"], dev["q"], dev["kv"], idx, idx_host.shape[1], wl.heads, wl.sm_scale, out, lse, ws)
    assert B.read_device_status(ws) == 0
    return B.tensor_to_bits(out), lse.cpu().numpy()


def _oracle_idx(ins, wl, rows=None):
    """Index rows [T, k] of the oracle's top-k choice for `rows` (all by default); -1 elsewhere."""
    batch = ins["batch"]
    T = batch.num_q
    rows = list(range(T)) if rows is None else list(rows)
    idx = np.full((T, wl.k), -1, np.int32)
    ref = H.oracle_rows(ins, wl, rows)
    for i, t in enumerate(rows):
        idx[t] = ref["idx"][i]
    return idx


@pytest.mark.parametrize("wl", [WORKLOADS["tiny_prefill"], MID_PREFILL, MID_DEC2, MID_DEC1], ids=lambda w: w.name)
def test_sparse_mla_matches_oracle(cuda_device, wl):
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    T = batch.num_q
    rows = list(range(T)) if T <= 64 else _sample_rows(T, wl.k)
    idx = _oracle_idx(ins, wl, rows if T > 1100 else None)
    dev = H.to_device(ins, cuda_device)
    out_bits, lse = _run_mla(dev, wl, idx, T)
    ref, ref_lse = _mla_ref_rows(ins, idx, rows, wl)
    H.check_attention(out_bits[rows], ref, wl.name)
    H.check_lse(lse[rows], ref_lse, wl.name)


def test_sparse_mla_holes_unsorted_and_empty_rows(cuda_device):
    wl = Workload("holes", 26, "decode", k=640, h_index=64, heads=128, batch=4, ctx_min=700, ctx_max=2000,
                  q_per_seq=1)
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    T = batch.num_q
    rng = np.random.default_rng(3)
    idx = np.full((T, wl.k), -1, np.int32)
    for t in range(T):
        n = int(batch.q_pos[t]) + 1
        sel = rng.choice(n, size=min(n, 500), replace=False).astype(np.int32)
        slots = np.sort(rng.choice(wl.k, size=sel.size, replace=False))
        idx[t, slots] = sel                     # unsorted, with -1 holes anywhere
    idx[T - 1] = -1                             # a query with nothing selected
    dev = H.to_device(ins, cuda_device)
    out_bits, lse = _run_mla(dev, wl, idx, T)
    ref, ref_lse = _mla_ref_rows(ins, idx, range(T - 1), wl)
    H.check_attention(out_bits[:T - 1], ref, "holes")
    H.check_lse(lse[:T - 1], ref_lse, "holes")
    assert np.all(oracle.bf16_decode(out_bits[T - 1]) == 0) and np.all(np.isneginf(lse[T - 1]))


def test_sparse_mla_fewer_heads(cuda_device):
    wl = Workload("h40", 27, "prefill", k=128, h_index=8, heads=40, seq_len=300)
    ins = inputs.make_inputs(wl)
    T = ins["batch"].num_q
    idx = _oracle_idx(ins, wl)
    out_bits, lse = _run_mla(H.to_device(ins, cuda_device), wl, idx, T)
    ref, ref_lse = _mla_ref_rows(ins, idx, range(T), wl)
    H.check_attention(out_bits, ref, "h40")
    H.check_lse(lse, ref_lse, "h40")

# ----------------------------------------------------------------------------- end to end


def _forward(dev, wl, batch_host):
    T = batch_host.num_q
    d = dev["q"].device
    out = torch.zeros((T, wl.heads, 512), dtype=torch.int16, device=d)
    lse = torch.zeros((T, wl.heads), dtype=torch.float32, device=d)
    ws = B.workspace(B.OP_FORWARD, dev["batch"], H_I=wl.h_index, H=wl.heads, k=wl.k, device=d)
    B.dsa_forward(dev["batch"], dev["q_idx"], dev["k_idx"], dev["w"], wl.h_index, dev["q"], dev["kv"], wl.heads,
                  wl.k, wl.sm_scale, out, lse, ws)
    assert B.read_device_status(ws) == 0
    sp, ld, ip = B.forward_ws_views(dev["batch"], wl.h_index, wl.heads, wl.k, ws)
    base = ws.data_ptr()
    scores = ws[sp - base: sp - base + T * ld * 4].view(torch.float32).view(T, ld).cpu().numpy()
    idx = ws[ip - base: ip - base + T * wl.k * 4].view(torch.int32).view(T, wl.k).cpu().numpy()
    return B.tensor_to_bits(out), lse.cpu().numpy(), scores, idx


def check_forward_rows(ins, wl, rows, out_bits, lse, scores, idx):
    """Scores, selection and attention of the GPU's forward on `rows` against the
    oracle: attention is compared with the oracle's attention over the GPU's own
    selection (identical to the oracle's result wherever the selections agree)."""
    batch = ins["batch"]
    rows = list(rows)
    ref = H.oracle_rows(ins, wl, rows, selections=idx[rows])
    mism = 0
    for i, t in enumerate(rows):
        n = int(batch.q_pos[t]) + 1
        I = ref["scores"][i]
        H.check_indexer_row(scores[t, :n], I, H.condition_scale(ins, t, n), f"{wl.name} row {t}")
        mism += H.check_selection(idx[t], ref["idx"][i], I, n, wl.k, f"{wl.name} row {t}")
    H.check_attention(out_bits[rows], ref["out"], wl.name)
    H.check_lse(lse[rows], ref["lse"], wl.name)
    return mism


@pytest.mark.parametrize("wl", [WORKLOADS["tiny_prefill"], MID_PREFILL, MID_DEC2], ids=lambda w: w.name)
def test_forward_end_to_end(cuda_device, wl):
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    dev = H.to_device(ins, cuda_device)
    out_bits, lse, scores, idx = _forward(dev, wl, batch)
    T = batch.num_q
    rows = list(range(T)) if T <= 64 else _sample_rows(T, wl.k)
    check_forward_rows(ins, wl, rows, out_bits, lse, scores, idx)


def _full_size_rows(batch, k):
    """Rows checked at full size: every query when there are at most 64; otherwise
    the first and last rows, the rows around n = k, 36 random rows with n > k
    (real selection) and 6 with n <= k."""
    T = batch.num_q
    if T <= 64:
        return list(range(T))
    n = batch.q_pos.astype(np.int64) + 1
    rows = {0, 1, T - 3, T - 2, T - 1}
    rows |= set(int(x) for x in np.nonzero(np.abs(n - k) <= 1)[0])
    rng = np.random.default_rng(123)
    big, small = np.nonzero(n > k)[0], np.nonzero(n <= k)[0]
    rows |= set(int(x) for x in rng.choice(big, size=min(big.size, 36), replace=False))
    if small.size:
        rows |= set(int(x) for x in rng.choice(small, size=min(small.size, 6), replace=False))
    return sorted(rows)


@pytest.mark.parametrize("name,chunk", [("prefill_8k", None), ("decode_b64", None), ("decode_128k_mtp2", None),
                                        ("chunked_64k", 0), ("chunked_64k", 7), ("chunked_64k", 15)])
def test_forward_full_size_sampled(cuda_device, name, chunk):
    """The workloads at full size through dsa_forward, as the benchmark runs them
    (the chunked workload: its first, a middle and its last chunk against the
    cache prefix), checked on sampled rows that include the last ones and at
    least 32 rows that select among more than k keys."""
    wl = WORKLOADS[name]
    ins = inputs.make_inputs(wl, chunk_index=chunk)
    batch = ins["batch"]
    dev = H.to_device(ins, cuda_device)
    out_bits, lse, scores, idx = _forward(dev, wl, batch)
    rows = _full_size_rows(batch, wl.k)
    n = batch.q_pos[rows].astype(np.int64) + 1
    assert (n > wl.k).sum() >= min(32, int((batch.q_pos + 1 > wl.k).sum()))
    assert batch.num_q - 1 in rows
    check_forward_rows(ins, wl, rows, out_bits, lse, scores, idx)


def test_chunked_prefill_equals_unchunked_on_the_gpu(cuda_device):
    """A prefill of 4096 tokens run as four chunk calls against the growing cache
    gives bit-identical scores, selections and outputs to the single call."""
    full_wl = Workload("chunk_eq", 29, "prefill", k=2048, h_index=64, heads=128, seq_len=4096)
    chk_wl = Workload("chunk_eq", 29, "chunked_prefill", k=2048, h_index=64, heads=128, seq_len=4096, chunk=1024)
    ins = inputs.make_inputs(full_wl)
    full = _forward(H.to_device(ins, cuda_device), full_wl, ins["batch"])
    for c in range(4):
        ci = inputs.make_inputs(chk_wl, chunk_index=c)
        part = _forward(H.to_device(ci, cuda_device), chk_wl, ci["batch"])
        r = slice(1024 * c, 1024 * c + 1024)
        n_hi = 1024 * (c + 1)
        assert np.array_equal(part[0], full[0][r]), f"chunk {c}: outputs differ"
        assert np.array_equal(part[1], full[1][r]), f"chunk {c}: lse differs"
        assert np.array_equal(part[3], full[3][r]), f"chunk {c}: selections differ"
        for t in range(1024):
            m = 1024 * c + t + 1
            assert np.array_equal(part[2][t, :m].view(np.uint32), full[2][1024 * c + t, :m].view(np.uint32))
        assert n_hi <= part[2].shape[1]

# ----------------------------------------------------------------------------- device status


def test_device_status_flags_bad_queries_and_indices(cuda_device):
    wl = Workload("bad", 28, "decode", k=128, h_index=64, heads=128, batch=2, ctx_min=200, ctx_max=300,
                  q_per_seq=1)
    ins = inputs.make_inputs(wl)
    bh = ins["batch"]
    bad = inputs.Batch(bh.kv_offset, bh.kv_len, bh.q_seq, bh.q_pos.copy(), bh.q_row)
    bad.q_pos[1] = bh.kv_len[1] + 5                       # beyond its sequence
    dev = H.to_device({**ins, "batch": bad}, cuda_device)
    T = 2
    ld = (int(bh.kv_len.max()) + 3) // 4 * 4
    scores = torch.zeros((T, ld), device=cuda_device)
    ws = B.workspace(B.OP_INDEXER, dev["batch"], ld=ld, device=cuda_device)
    B.dsa_indexer_scores(dev["batch"], dev["q_idx"], dev["k_idx"], dev["w"], 64, scores, ld, ws)
    assert B.read_device_status(ws) & B.DEV_BAD_QUERY
    idx = torch.full((T, wl.k), -1, dtype=torch.int32, device=cuda_device)
    ws2 = B.workspace(B.OP_TOPK, dev["batch"], k=wl.k, device=cuda_device)
    B.dsa_topk(dev["batch"], scores, ld, wl.k, idx, ws2)
    assert B.read_device_status(ws2) & B.DEV_BAD_QUERY
    assert (idx[1] == -1).all()
    good = H.to_device(ins, cuda_device)
    idx_h = np.full((T, wl.k), -1, np.int32)
    idx_h[:, 0] = 0
    idx_h[0, 1] = int(bh.kv_len[0]) + 3                   # out of range
    out_bits, _ = None, None
    i_dev = torch.from_numpy(idx_h).to(cuda_device)
    out = torch.zeros((T, 128, 512), dtype=torch.int16, device=cuda_device)
    ws3 = B.workspace(B.OP_SPARSE_MLA, good["batch"], H=128, k=wl.k, device=cuda_device)
    B.dsa_sparse_mla(good["batch"], good["q"], good["kv"], i_dev, wl.k, 128, wl.sm_scale, out, None, ws3)
    assert B.read_device_status(ws3) & B.DEV_BAD_INDEX


# ----------------------------------------------------------------------------- failure detection


def test_bounded_wait_times_out_and_leaves_the_context_usable(cuda_device):
    """A barrier that nothing completes: the waiting kernel gives up after the
    limit, flags DSA_DEV_TIMEOUT, and later work on the same context runs."""
    import time
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_device)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.dsa_selftest_wait_timeout(ws, 20000)          # 20 ms
    flags = B.read_device_status(ws)
    dt = time.perf_counter() - t0
    assert flags & B.DEV_TIMEOUT
    assert 0.015 < dt < 5.0
    x = torch.arange(10, device=cuda_device).sum().item()
    assert x == 45
    _topk_case(cuda_device, [np.arange(300, dtype=np.float32)], 64)
