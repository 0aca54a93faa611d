"""dsa_forward_host on the GPU: the forward from pinned host buffers, pipelined
over query chunks on three streams, gives bit for bit what dsa_forward gives
on the same device inputs (each chunk is an independent forward over the same
cache), and two calls queued back to back on the same buffers do not overlap."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import build, inputs
from sparse_attention_weight_b200.configs import WORKLOADS, Workload

from . import helpers as H

pytestmark = pytest.mark.gpu

NAMES = ("q_idx", "w", "q", "k_idx", "kv")


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    B.lib()


def _pinned(ins: dict) -> dict:
    return {n: torch.from_numpy(ins[n].view(np.int16) if ins[n].dtype == np.uint16
                                else np.ascontiguousarray(ins[n])).pin_memory() for n in NAMES}


def _reference(dev: dict, wl, T: int):
    """dsa_forward on device-resident copies of the same inputs."""
    d = dev["q"].device
    out = torch.empty((T, wl.heads, 512), dtype=torch.int16, device=d)
    lse = torch.empty((T, wl.heads), dtype=torch.float32, device=d)
    ws = B.workspace(B.OP_FORWARD, dev["batch"], H_I=wl.h_index, H=wl.heads, k=wl.k, device=d)
    B.dsa_forward(dev["batch"], dev["q_idx"], dev["k_idx"], dev["w"], wl.h_index, dev["q"], dev["kv"], wl.heads,
                  wl.k, wl.sm_scale, out, lse, ws)
    torch.cuda.synchronize()
    assert B.read_device_status(ws) == 0
    return out.cpu().numpy(), lse.cpu().numpy()


def _staging(dev: dict) -> dict:
    """Device buffers of the inputs' sizes, filled with garbage (the call copies in)."""
    return {n: torch.full_like(dev[n], 0x55 if dev[n].dtype == torch.uint8 else 7) for n in NAMES}


@pytest.mark.parametrize("wl", [
    Workload("fwd_host_prefill", 61, "prefill", k=256, h_index=16, heads=32, seq_len=900),
    Workload("fwd_host_decode", 62, "decode", k=512, h_index=8, heads=16, batch=6, ctx_min=700, ctx_max=2000,
             q_per_seq=2),
    WORKLOADS["tiny_prefill"],
], ids=lambda w: w.name)
@pytest.mark.parametrize("streams", ["three", "one"])
def test_forward_host_matches_forward(cuda_device, wl, streams):
    ins = inputs.make_inputs(wl)
    T = ins["batch"].num_q
    dev = H.to_device(ins, cuda_device)
    ref_out, ref_lse = _reference(dev, wl, T)
    host = _pinned(ins)
    stage = _staging(dev)
    out = torch.empty((T, wl.heads, 512), dtype=torch.int16, device=cuda_device)
    lse = torch.empty((T, wl.heads), dtype=torch.float32, device=cuda_device)
    h_out = torch.empty((T, wl.heads, 512), dtype=torch.int16).pin_memory()
    ws = B.workspace(B.OP_FORWARD_HOST, dev["batch"], H_I=wl.h_index, H=wl.heads, k=wl.k, device=cuda_device)
    cur = torch.cuda.current_stream()
    st = (torch.cuda.Stream(), cur, torch.cuda.Stream()) if streams == "three" else (cur, cur, cur)
    B.dsa_forward_host(dev["batch"], host, stage, wl.h_index, wl.heads, wl.k, wl.sm_scale, out, lse, h_out, ws, st)
    cur.synchronize()
    assert B.read_device_status(ws) == 0
    np.testing.assert_array_equal(h_out.numpy(), ref_out)
    np.testing.assert_array_equal(lse.cpu().numpy(), ref_lse)
    for n in NAMES:                                       # the staging buffers hold the copies
        assert torch.equal(stage[n].cpu(), host[n])


def test_forward_host_back_to_back_calls(cuda_device):
    """Two calls on the same device buffers with different queries, queued without
    a synchronisation between them: each host output is its own call's result."""
    wl = Workload("fwd_host_b2b", 63, "prefill", k=256, h_index=16, heads=32, seq_len=700)
    ins_a = inputs.make_inputs(wl, seed=0)
    ins_b = inputs.make_inputs(wl, seed=1)
    T = ins_a["batch"].num_q
    refs = []
    for ins in (ins_a, ins_b):
        dev = H.to_device(ins, cuda_device)
        refs.append(_reference(dev, wl, T)[0])
    dev = H.to_device(ins_a, cuda_device)
    stage = _staging(dev)
    out = torch.empty((T, wl.heads, 512), dtype=torch.int16, device=cuda_device)
    ws = B.workspace(B.OP_FORWARD_HOST, dev["batch"], H_I=wl.h_index, H=wl.heads, k=wl.k, device=cuda_device)
    cur = torch.cuda.current_stream()
    st = (torch.cuda.Stream(), cur, torch.cuda.Stream())
    h_outs = [torch.empty((T, wl.heads, 512), dtype=torch.int16).pin_memory() for _ in range(2)]
    # the pinned inputs stay referenced until the streams are done with them (the
    # caching host allocator would otherwise hand their pages to the next call)
    hosts = [_pinned(ins) for ins in (ins_a, ins_b)]
    for host, h_out in zip(hosts, h_outs):
        B.dsa_forward_host(dev["batch"], host, stage, wl.h_index, wl.heads, wl.k, wl.sm_scale, out, None, h_out,
                           ws, st)
    cur.synchronize()
    for h_out, ref in zip(h_outs, refs):
        np.testing.assert_array_equal(h_out.numpy(), ref)


def test_forward_host_refuses_pageable_memory(cuda_device):
    wl = WORKLOADS["tiny_prefill"]
    ins = inputs.make_inputs(wl)
    T = ins["batch"].num_q
    dev = H.to_device(ins, cuda_device)
    host = _pinned(ins)
    host["q"] = host["q"].clone()                         # pageable
    out = torch.empty((T, wl.heads, 512), dtype=torch.int16, device=cuda_device)
    h_out = torch.empty((T, wl.heads, 512), dtype=torch.int16).pin_memory()
    ws = B.workspace(B.OP_FORWARD_HOST, dev["batch"], H_I=wl.h_index, H=wl.heads, k=wl.k, device=cuda_device)
    with pytest.raises(B.DsaError) as e:
        B.dsa_forward_host(dev["batch"], host, _staging(dev), wl.h_index, wl.heads, wl.k, wl.sm_scale, out, None,
                           h_out, ws)
    assert e.value.status == 2
