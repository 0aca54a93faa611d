"""Pins of the sparse-MLA backward oracle (oracle.backward) to facts outside it:
PyTorch's autograd (float64) on the forward restated with PyTorch operations,
central finite differences of the oracle's own forward, and the zero gradient
of a direction the output does not depend on."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import backward as BW


def _case(T=3, H=4, S=11, k=6, seed=0, d_v=512):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, 576)) * 0.5
    kv = rng.standard_normal((S, 576)) * 0.5
    idx = np.full((T, k), -1, np.int64)
    for t in range(T):
        m = rng.integers(1, k + 1)
        sel = rng.choice(S, size=m, replace=True)          # repeats allowed: they add up
        idx[t, rng.choice(k, size=m, replace=False)] = sel
    dout = rng.standard_normal((T, H, d_v))
    return q, kv, idx, dout


def test_backward_matches_torch_autograd():
    q, kv, idx, dout = _case()
    scale = 1 / np.sqrt(576)
    dq, dkv = BW.sparse_mla_backward(q, kv, idx, scale, dout)
    tq = torch.tensor(q, requires_grad=True)
    tkv = torch.tensor(kv, requires_grad=True)
    loss = torch.zeros((), dtype=torch.float64)
    for t in range(q.shape[0]):
        sel = torch.tensor(idx[t][idx[t] >= 0])
        rows = tkv[sel]
        att = torch.softmax(scale * tq[t] @ rows.T, dim=-1)
        out = att @ rows[:, :512]
        loss = loss + (out * torch.tensor(dout[t])).sum()
    loss.backward()
    assert np.allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-13)
    assert np.allclose(dkv, tkv.grad.numpy(), rtol=1e-11, atol=1e-13)


def test_backward_matches_finite_differences():
    q, kv, idx, dout = _case(T=2, H=2, S=5, k=3, seed=1)
    scale = 0.3
    dq, dkv = BW.sparse_mla_backward(q, kv, idx, scale, dout)
    f = lambda qq, kk: float(np.sum(oracle.sparse_mla(qq, kk, idx, scale)[0] * dout))
    rng = np.random.default_rng(2)
    eps = 1e-6
    for _ in range(12):
        t, h, d = rng.integers(2), rng.integers(2), rng.integers(576)
        qp, qm = q.copy(), q.copy()
        qp[t, h, d] += eps
        qm[t, h, d] -= eps
        assert abs((f(qp, kv) - f(qm, kv)) / (2 * eps) - dq[t, h, d]) <= 1e-6 * (1 + abs(dq[t, h, d]))
        s, d2 = rng.integers(5), rng.integers(576)
        kp, km = kv.copy(), kv.copy()
        kp[s, d2] += eps
        km[s, d2] -= eps
        assert abs((f(q, kp) - f(q, km)) / (2 * eps) - dkv[s, d2]) <= 1e-6 * (1 + abs(dkv[s, d2]))


def test_unselected_rows_get_no_gradient_and_identical_rows_give_no_query_gradient():
    q, kv, idx, dout = _case(seed=3)
    dq, dkv = BW.sparse_mla_backward(q, kv, idx, 0.1, dout)
    unused = np.setdiff1d(np.arange(kv.shape[0]), idx[idx >= 0])
    assert unused.size and np.all(dkv[unused] == 0)
    # every selected entry names the same row: the softmax is uniform whatever q is,
    # so the output does not depend on q and dQ vanishes
    same = np.where(idx >= 0, 4, -1)
    dq2, _ = BW.sparse_mla_backward(q, kv, same, 0.1, dout)
    assert np.abs(dq2).max() <= 1e-12 * np.abs(dq).max()


def test_stored_forward_outputs_reproduce_the_exact_gradient():
    q, kv, idx, dout = _case(seed=4)
    scale = 0.05
    out, lse = oracle.sparse_mla(q, kv, idx, scale)
    a = BW.sparse_mla_backward(q, kv, idx, scale, dout)
    b = BW.sparse_mla_backward(q, kv, idx, scale, dout, out=out, lse=lse)
    assert np.allclose(a[0], b[0], rtol=1e-12, atol=1e-14) and np.allclose(a[1], b[1], rtol=1e-12, atol=1e-14)
