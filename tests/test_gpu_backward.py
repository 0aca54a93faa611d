"""Sparse-MLA backward on the GPU (dsa_sparse_mla_backward) against oracle.backward.

The oracle is given the GPU forward's stored bf16 output and fp32 lse (D and p
are formed from them, as the kernel does), so the remaining differences are the
kernel's fp32 arithmetic: sums of up to k * 576 products and an approximate exp.
Bar, per gradient tensor: max-abs error <= 2e-3 * max|ref| and mean-abs error <=
2e-4 * max|ref|.  d_q does not use atomics and must be bit-reproducible; d_kv is
accumulated with atomics (order varies) and is compared within the bar.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as BW
from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import build, inputs
from sparse_attention_weight_b200.configs import WORKLOADS, Workload

from . import helpers as H
from .test_gpu_paged import paged_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    B.lib()


def _selection(ins, wl, seed, dup=False):
    """Random usable selections with -1 holes (and repeated rows when dup)."""
    batch = ins["batch"]
    rng = np.random.default_rng(seed)
    T = batch.num_q
    idx = np.full((T, wl.k), -1, np.int32)
    for t in range(T):
        n = int(batch.q_pos[t]) + 1
        m = min(n, wl.k - wl.k // 8)
        sel = rng.choice(n, size=m, replace=dup).astype(np.int32)
        slots = np.sort(rng.choice(wl.k, size=m, replace=False))
        idx[t, slots] = sel
    return idx


def _run(dev, wl, idx, T, seed):
    d = dev["q"].device
    db = dev["batch"]
    ii = torch.as_tensor(idx, device=d)
    out = torch.empty((T, wl.heads, 512), dtype=torch.int16, device=d)
    lse = torch.empty((T, wl.heads), dtype=torch.float32, device=d)
    ws = B.workspace(B.OP_SPARSE_MLA, db, H=wl.heads, k=wl.k, device=d)
    B.dsa_sparse_mla(db, dev["q"], dev["kv"], ii, wl.k, wl.heads, wl.sm_scale, out, lse, ws)
    g = torch.Generator(device=d)
    g.manual_seed(seed)
    dout = torch.randn((T, wl.heads, 512), generator=g, device=d).to(torch.bfloat16).view(torch.int16)
    dq = torch.empty((T, wl.heads, 576), dtype=torch.float32, device=d)
    dkv = torch.zeros((dev["kv"].shape[0], 576), dtype=torch.float32, device=d)
    wsb = B.workspace(B.OP_MLA_BACKWARD, db, H=wl.heads, k=wl.k, device=d)
    B.dsa_sparse_mla_backward(db, dev["q"], dev["kv"], ii, wl.k, wl.heads, wl.sm_scale, out, lse, dout, dq, dkv, wsb)
    assert B.read_device_status(ws) == 0 and B.read_device_status(wsb) == 0
    dq2 = torch.empty_like(dq)
    dkv2 = torch.zeros_like(dkv)
    B.dsa_sparse_mla_backward(db, dev["q"], dev["kv"], ii, wl.k, wl.heads, wl.sm_scale, out, lse, dout, dq2, dkv2, wsb)
    assert torch.equal(dq, dq2)                                  # no atomics in d_q
    return (B.tensor_to_bits(out), lse.cpu().numpy(), B.tensor_to_bits(dout), dq.cpu().numpy(),
            dkv.cpu().numpy())


def _reference(ins, idx, out_bits, lse, dout_bits, wl):
    """oracle.backward per sequence (local row indices), scattered to cache rows."""
    batch = ins["batch"]
    q = oracle.bf16_decode(ins["q"])
    dq = np.zeros(q.shape)
    dkv = np.zeros((ins["kv"].shape[0], 576))
    out = oracle.bf16_decode(out_bits)
    dout = oracle.bf16_decode(dout_bits)
    for b in range(batch.num_seqs):
        ts = np.nonzero(batch.q_seq == b)[0]
        if ts.size == 0:
            continue
        off, n = int(batch.kv_offset[b]), int(batch.kv_len[b])
        rows = oracle.bf16_decode(ins["kv"][off:off + n])
        g_q, g_kv = BW.sparse_mla_backward(q[ts], rows, idx[ts], wl.sm_scale, dout[ts], out=out[ts],
                                           lse=lse[ts].astype(np.float64))
        dq[ts] = g_q
        dkv[off:off + n] += g_kv
    return dq, dkv


def _check(got, ref, what):
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    print(f"[{what}] max-abs {err.max():.3e} mean-abs {err.mean():.3e} (max |ref| {scale:.3e})")
    assert err.max() <= 2e-3 * scale and err.mean() <= 2e-4 * scale, what


@pytest.mark.parametrize("wl,dup", [
    (WORKLOADS["tiny_prefill"], False),
    (Workload("bwd_decode", 51, "decode", k=512, h_index=8, heads=32, batch=3, ctx_min=400, ctx_max=1500,
              q_per_seq=2), True),
    (Workload("bwd_h128", 52, "prefill", k=256, h_index=8, heads=128, seq_len=300), False),
], ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_backward_matches_oracle(cuda_device, wl, dup):
    ins = inputs.make_inputs(wl)
    idx = _selection(ins, wl, seed=wl.cfg_id, dup=dup)
    T = ins["batch"].num_q
    out_bits, lse, dout_bits, dq, dkv = _run(H.to_device(ins, cuda_device), wl, idx, T, seed=wl.cfg_id)
    ref_dq, ref_dkv = _reference(ins, idx, out_bits, lse, dout_bits, wl)
    _check(dq, ref_dq, f"{wl.name} d_q")
    _check(dkv, ref_dkv, f"{wl.name} d_kv")


def test_backward_paged_cache(cuda_device):
    wl = Workload("bwd_paged", 53, "decode", k=256, h_index=8, heads=16, batch=4, ctx_min=200, ctx_max=900,
                  q_per_seq=3)
    ins = inputs.make_inputs(wl)
    idx = _selection(ins, wl, seed=9, dup=True)
    T = ins["batch"].num_q
    dev, table = paged_device(ins, 64, cuda_device)
    out_bits, lse, dout_bits, dq, dkv_pool = _run(dev, wl, idx, T, seed=9)
    _, src = inputs.paged_layout(ins["batch"], 64, 0)
    dkv = np.zeros((ins["kv"].shape[0], 576))
    used = src >= 0
    dkv[src[used]] = dkv_pool[used]                              # back to the contiguous rows
    ref_dq, ref_dkv = _reference(ins, idx, out_bits, lse, dout_bits, wl)
    _check(dq, ref_dq, "paged d_q")
    _check(dkv, ref_dkv, "paged d_kv")
