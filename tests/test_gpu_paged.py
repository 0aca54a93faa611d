"""Paged caches (the block-table layout of paged inference caches) and the
batch-1 long-context decode workload, through the C ABI on the GPU.

A paged cache holds the same rows as a contiguous one, only elsewhere, so every
result must be bit-identical to the contiguous run (same kernels, same
arithmetic order); the batch-1 128K decode is checked against the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import build, inputs
from sparse_attention_weight_b200.configs import WORKLOADS, Workload

from . import helpers as H
from .test_gpu_parity import _forward, check_forward_rows

pytestmark = pytest.mark.gpu

DEC = Workload("paged_decode", 41, "decode", k=2048, h_index=64, heads=128, batch=6, ctx_min=1500,
               ctx_max=5000, q_per_seq=2)
PRE = Workload("paged_prefill", 42, "prefill", k=512, h_index=16, heads=64, seq_len=1400)


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    B.lib()


def paged_device(ins: dict, page_size: int, device, seed: int = 0):
    """Device copies of the inputs with the caches scattered into pages."""
    batch = ins["batch"]
    table, src = inputs.paged_layout(batch, page_size, seed)
    used = src >= 0
    k_idx = np.zeros((src.size, ins["k_idx"].shape[1]), ins["k_idx"].dtype)
    kv = np.zeros((src.size, ins["kv"].shape[1]), ins["kv"].dtype)
    k_idx[used] = ins["k_idx"][src[used]]
    kv[used] = ins["kv"][src[used]]
    dev = H.to_device(ins, device)
    dev["k_idx"] = B.bits_to_tensor(k_idx, device)
    dev["kv"] = B.bits_to_tensor(kv, device)
    dev["batch"] = B.DeviceBatch.from_host(batch, device, kv_rows=src.size, page_size=page_size,
                                           page_table=table)
    return dev, table


@pytest.mark.parametrize("wl", [DEC, PRE], ids=lambda w: w.name)
@pytest.mark.parametrize("page_size", [64, 128, 192])
def test_paged_cache_is_bit_identical_to_contiguous(cuda_device, wl, page_size):
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    ref = _forward(H.to_device(ins, cuda_device), wl, batch)
    dev, _ = paged_device(ins, page_size, cuda_device, seed=page_size)
    got = _forward(dev, wl, batch)
    n = batch.q_pos.astype(np.int64) + 1
    for t in range(batch.num_q):                        # scores: only s < n_t are defined
        assert np.array_equal(got[2][t, :n[t]].view(np.uint32), ref[2][t, :n[t]].view(np.uint32)), t
    assert np.array_equal(got[3], ref[3])                # selections
    assert np.array_equal(got[0], ref[0])                # output bits
    assert np.array_equal(got[1].view(np.uint32), ref[1].view(np.uint32))   # lse bits


def test_paged_page_outside_the_cache_is_flagged(cuda_device):
    wl = DEC
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    dev, table = paged_device(ins, 64, cuda_device)
    bad = table.copy()
    bad[2, 3] = 1 << 24                                  # far beyond the pool
    bad[4, 0] = -5
    dev["batch"] = B.DeviceBatch.from_host(batch, cuda_device, kv_rows=dev["kv"].shape[0], page_size=64,
                                           page_table=bad)
    T = batch.num_q
    d = dev["q"].device
    out = torch.zeros((T, wl.heads, 512), dtype=torch.int16, device=d)
    ws = B.workspace(B.OP_FORWARD, dev["batch"], H_I=wl.h_index, H=wl.heads, k=wl.k, device=d)
    B.dsa_forward(dev["batch"], dev["q_idx"], dev["k_idx"], dev["w"], wl.h_index, dev["q"], dev["kv"], wl.heads,
                  wl.k, wl.sm_scale, out, None, ws)
    assert B.read_device_status(ws) & 2                  # DSA_DEV_BAD_INDEX
    torch.cuda.synchronize()                             # the context stays usable
    assert torch.isfinite(out.view(torch.bfloat16).float()).all()


def test_decode_batch1_128k_paged_matches_oracle(cuda_device):
    """One sequence at context 131072, one new token, page size 64: scores of all
    131072 keys, the top-2048 selection and the attention against the oracle."""
    wl = WORKLOADS["decode_b1_128k"]
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    dev, _ = paged_device(ins, 64, cuda_device)
    out_bits, lse, scores, idx = _forward(dev, wl, batch)
    mism = check_forward_rows(ins, wl, [0], out_bits, lse, scores, idx)
    print(f"[decode_b1_128k] selection mismatches near the k-th score: {mism}")
