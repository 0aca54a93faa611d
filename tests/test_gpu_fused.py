"""Indexer -> top-k fused through the emitted key histogram (dsa_indexer_scores_hist
+ dsa_topk_hist) on the GPU: the histogram is exactly the histogram of the top 11
bits of the order-preserving keys of each row's scores, and scores and selections
are bit-identical to the unfused calls, on every top-k kernel (rows cached per
CTA, clustered rows, rows streamed from L2)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import build, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    B.lib()


def order_key_top11(scores: np.ndarray) -> np.ndarray:
    """Top 11 bits of the order-preserving key of fp32 scores (-0 == +0)."""
    b = np.ascontiguousarray(scores, dtype=np.float32).view(np.uint32).copy()
    b[(b & 0x7FFFFFFF) == 0] = 0
    key = np.where(b & 0x80000000, ~b, b | 0x80000000).astype(np.uint32)
    return key >> 21


def _case(lens, q_per_seq, H_I, seed, q_first=None):
    """Sequences of the given lengths; q_per_seq queries at the end of each (or,
    for one sequence, the queries q_first .. len-1)."""
    lens = np.asarray(lens, np.int32)
    off = np.zeros(len(lens), np.int64)
    off[1:] = np.cumsum(lens[:-1])
    if q_first is not None:
        pos = np.arange(q_first, lens[0], dtype=np.int32)
        qs = np.zeros(pos.size, np.int32)
    else:
        qs = np.repeat(np.arange(len(lens), dtype=np.int32), q_per_seq)
        pos = (lens[qs] - q_per_seq + np.tile(np.arange(q_per_seq, dtype=np.int32), len(lens))).astype(np.int32)
    batch = inputs.Batch(off, lens, qs, pos, np.zeros_like(pos))
    rng = np.random.default_rng([seed, 7200])
    T, rows = pos.size, int(lens.sum())
    return batch, {"q_idx": inputs.to_e4m3_bytes(rng.standard_normal((T, H_I, 128), dtype=np.float32)),
                   "k_idx": inputs.to_e4m3_bytes(rng.standard_normal((rows, 128), dtype=np.float32)),
                   "w": (rng.standard_normal((T, H_I), dtype=np.float32) / np.float32(np.sqrt(H_I)))}


@pytest.mark.parametrize("name,lens,qps,q_first,kernel", [
    ("cached_rows", [3000], 0, 0, 0),                         # short rows: cached per CTA (hist ignored)
    ("clustered_rows", [40000, 65536, 21000, 131072], 2, None, 8),
    ("streamed_rows", [170000], 0, 169700, -1),               # 300 rows beyond the cluster sizes
])
def test_fused_histogram_matches_unfused(cuda_device, name, lens, qps, q_first, kernel):
    H_I, k = 64, 2048
    batch, h = _case(lens, qps, H_I, seed=len(name), q_first=q_first)
    db = B.DeviceBatch.from_host(batch, cuda_device)
    T = batch.num_q
    ld = (batch.max_kv_len + 3) // 4 * 4
    dev = {n: B.bits_to_tensor(h[n], cuda_device) for n in ("q_idx", "k_idx", "w")}
    assert B.topk_uses_hist(db, k) == (kernel != 0), name
    ws_i = B.workspace(B.OP_INDEXER, db, H_I=H_I, ld=ld, device=cuda_device)
    ws_t = B.workspace(B.OP_TOPK, db, k=k, device=cuda_device)
    s0 = torch.full((T, ld), float("nan"), device=cuda_device)
    s1 = torch.full((T, ld), float("nan"), device=cuda_device)
    i0 = torch.empty((T, k), dtype=torch.int32, device=cuda_device)
    i1 = torch.empty((T, k), dtype=torch.int32, device=cuda_device)
    hist = torch.full((T, 2048), 0xDEAD, dtype=torch.int32, device=cuda_device)
    B.dsa_indexer_scores(db, dev["q_idx"], dev["k_idx"], dev["w"], H_I, s0, ld, ws_i)
    B.dsa_topk(db, s0, ld, k, i0, ws_t)
    B.dsa_indexer_scores_hist(db, dev["q_idx"], dev["k_idx"], dev["w"], H_I, s1, ld, hist, ws_i)
    B.dsa_topk_hist(db, s1, ld, hist, k, i1, ws_t)
    assert B.read_device_status(ws_i) == 0 and B.read_device_status(ws_t) == 0
    s0, s1, hist = s0.cpu().numpy(), s1.cpu().numpy(), hist.cpu().numpy().view(np.uint32)
    n = batch.q_pos.astype(np.int64) + 1
    for t in range(T):
        assert np.array_equal(s0[t, :n[t]].view(np.uint32), s1[t, :n[t]].view(np.uint32)), (name, t)
        want = np.bincount(order_key_top11(s1[t, :n[t]]), minlength=2048)
        assert np.array_equal(hist[t], want), (name, t)
    assert np.array_equal(i0.cpu().numpy(), i1.cpu().numpy()), name
