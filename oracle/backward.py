"""CPU oracle for the backward pass of the sparse MLA (training through the
sparse attention).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The product path never calls it, and
it shares no code with the CUDA library.

Plain float64 numpy.  [V3.2加速] "DeepSeek-V3.2加速技术详解", §04 (training: a
dense warm-up of the indexer, then sparse continued training in which the model
learns through the selected tokens only); [一文讀懂] "一文讀懂DeepSeek-V3.2核心技術
DSA" (the model stays trainable end to end with DSA in place).

Reading: the gradients of the sparse MLA output (see dsa_ref.sparse_mla) with
respect to the queries Q and the latent cache rows KV, for a given output
gradient dO, with the selection held fixed (top-k is a discrete choice: no
gradient flows through it).  For query t, head h, selected rows i:
  z_i = s q.kv_i,  p = softmax(z),  o = sum_i p_i v_i  (v_i = kv_i[:512])
  dP_i = dO.v_i,  D = dO.o,  dZ_i = p_i (dP_i - D)
  dQ = s sum_i dZ_i kv_i
  dKV[row_i] += s dZ_i q + p_i [dO, 0]   (the value is the latent part of the row)
Rows selected by several queries (or several times) accumulate all contributions.

Pins (tests/test_oracle_backward.py): torch.autograd in float64 on the forward
restated with PyTorch operations; central finite differences on a tiny case;
gradient of a constant-output direction.
"""
from __future__ import annotations

import numpy as np


def sparse_mla_backward(q: np.ndarray, kv: np.ndarray, idx: np.ndarray, sm_scale: float, d_out: np.ndarray,
                        d_v: int = 512, out=None, lse=None):
    """q: [T, H, 576], kv: [S, 576], idx: [T, k] (-1 unused), d_out: [T, H, d_v]
    (all float64).  Returns (dq [T, H, 576], dkv [S, 576]).

    With `out` [T, H, d_v] and `lse` [T, H] given (a forward's stored output and
    log-sum-exp), D is formed from that output and p from that lse, as a backward
    that keeps only the forward's outputs does; without them both are recomputed
    exactly."""
    T, H, D = q.shape
    dq = np.zeros_like(q, dtype=np.float64)
    dkv = np.zeros((kv.shape[0], D), dtype=np.float64)
    for t in range(T):
        pos = np.nonzero(idx[t] >= 0)[0]
        if pos.size == 0:
            continue
        sel = idx[t][pos].astype(np.int64)
        rows = kv[sel]                                  # [m, 576]
        z = sm_scale * (q[t] @ rows.T)                  # [H, m]
        if lse is None:
            e = np.exp(z - z.max(axis=1, keepdims=True))
            p = e / e.sum(axis=1, keepdims=True)
        else:
            p = np.exp(z - np.asarray(lse[t], dtype=np.float64)[:, None])
        o = p @ rows[:, :d_v] if out is None else np.asarray(out[t], dtype=np.float64)   # [H, d_v]
        dP = d_out[t] @ rows[:, :d_v].T                 # [H, m]
        Dh = np.sum(d_out[t] * o, axis=1, keepdims=True)
        dZ = p * (dP - Dh)                              # [H, m]
        dq[t] = sm_scale * (dZ @ rows)
        contrib = sm_scale * (dZ.T @ q[t])              # [m, 576]
        contrib[:, :d_v] += p.T @ d_out[t]
        np.add.at(dkv, sel, contrib)
    return dq, dkv
