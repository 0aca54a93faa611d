"""dsa_indexer_scores_noalloc: the indexer for callers that cannot allocate.

Some callers cannot call cudaMalloc (a framework that only hands out the
operation's own tensors, a plug-in living inside someone else's memory pool),
so they cannot pass the workspace that dsa_indexer_scores plans in.  This entry
point keeps that scratch in a fixed device array inside the library.  The test
calls it through the C ABI twice in a row and checks that both results are
bit-identical to the workspace version's (the same kernels run on the same
inputs, so any difference would be a fault of the shared scratch, e.g. a
previous call's plan left behind); it also calls it at exactly its query limit
and checks that one query more is refused on the host.  This file is collected
last, so a run that stops at the first failure has already run every other test.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import build, inputs
from sparse_attention_weight_b200.configs import Workload

pytestmark = pytest.mark.gpu

# exactly DSA_NOALLOC_MAX_Q queries: 64 sequences of 256 tokens, every token a query
AT_LIMIT = Workload("noalloc_limit", 42, "decode", k=256, h_index=64, heads=128, batch=64, ctx_min=256,
                    ctx_max=256, q_per_seq=256)
PREFILL = Workload("noalloc_prefill", 40, "prefill", k=512, h_index=64, heads=128, seq_len=1500)
DECODE = Workload("noalloc_decode", 41, "decode", k=512, h_index=64, heads=128, batch=5, ctx_min=700,
                  ctx_max=4000, q_per_seq=2)


def _same_bits(a: np.ndarray, b: np.ndarray):
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), "results differ from the workspace version"


@pytest.mark.parametrize("wl", [PREFILL, DECODE, AT_LIMIT], ids=lambda w: w.name)
def test_noalloc_indexer_matches_workspace_version_twice(cuda_device, wl):
    build.build()
    bh = inputs.make_batch(wl)
    ins = {"q_idx": inputs.query_rows(wl, bh, "q_idx"), "w": inputs.query_rows(wl, bh, "w"),
           "k_idx": inputs.cache_rows(wl, bh, "k_idx")}
    db = B.DeviceBatch.from_host(bh, cuda_device)
    d = {n: B.bits_to_tensor(ins[n], cuda_device) for n in ("q_idx", "k_idx", "w")}
    T = bh.num_q
    ld = (bh.max_kv_len + 3) // 4 * 4
    ref = torch.full((T, ld), float("nan"), device=cuda_device)
    ws = B.workspace(B.OP_INDEXER, db, H_I=wl.h_index, ld=ld, device=cuda_device)
    B.dsa_indexer_scores(db, d["q_idx"], d["k_idx"], d["w"], wl.h_index, ref, ld, ws)
    assert B.read_device_status(ws) == 0
    ref_h = ref.cpu().numpy()
    assert T <= B.NOALLOC_MAX_Q and (wl is not AT_LIMIT or T == B.NOALLOC_MAX_Q)
    for _ in range(2):
        out = torch.full((T, ld), float("nan"), device=cuda_device)
        B.dsa_indexer_scores_noalloc(db, d["q_idx"], d["k_idx"], d["w"], wl.h_index, out, ld)
        torch.cuda.synchronize()
        _same_bits(out.cpu().numpy(), ref_h)


def test_noalloc_rejects_batches_above_its_limit():
    lib = B.lib()
    big = B.DsaBatch(1, B.NOALLOC_MAX_Q + 1, 4096, 0, 4096, 0x10000, 0x20000, 0x30000, 0x40000)
    p = 0x60000
    assert lib.dsa_indexer_scores_noalloc(ctypes.byref(big), p, p, p, 64, p, 4096, None) == 2
