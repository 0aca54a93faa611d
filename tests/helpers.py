"""Shared helpers of the GPU parity tests: device copies of seeded inputs,
oracle references per query, and the tolerance checks the tests apply."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import inputs

# Tolerances (stated per check):
#   indexer scores: |I_gpu - I_ref| <= 1e-4 * max(|I_ref|, A_ref), A_ref = sum_j |w_j| ReLU(dot_j)
#   attention output (bf16 I/O) vs the fp64 oracle: max-abs <= 1e-2 beyond the bf16 rounding of
#   the output (2^-8 |ref|), mean-abs <= 1e-3
#   lse: abs <= 2e-3 (fp32 softmax statistics; a derived bound)
IDX_RTOL = 1e-4
OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 1e-3
LSE_ABS = 2e-3


def to_device(ins: dict, device) -> dict:
    return {
        "q_idx": B.bits_to_tensor(ins["q_idx"], device),
        "k_idx": B.bits_to_tensor(ins["k_idx"], device),
        "w": B.bits_to_tensor(ins["w"], device),
        "q": B.bits_to_tensor(ins["q"], device),
        "kv": B.bits_to_tensor(ins["kv"], device),
        "batch": B.DeviceBatch.from_host(ins["batch"], device),
    }


def seq_slice(batch, t):
    b = int(batch.q_seq[t])
    off, n = int(batch.kv_offset[b]), int(batch.kv_len[b])
    return off, n


def indexer_ref_row(ins: dict, t: int):
    """(I_ref float64 [n_t], A_ref float64 [n_t]) for query t."""
    batch = ins["batch"]
    off, nb = seq_slice(batch, t)
    n = int(batch.q_pos[t]) + 1
    keys = ins["k_idx"][off:off + n]
    I = oracle.indexer_scores(ins["q_idx"][t:t + 1], keys, ins["w"][t:t + 1], np.array([n]))[0]
    qd = oracle.e4m3_decode(ins["q_idx"][t])                 # [H_I, 128]
    kd = oracle.e4m3_decode(keys)                             # [n, 128]
    dots = qd @ kd.T                                          # [H_I, n]
    A = np.abs(ins["w"][t].astype(np.float64)) @ np.maximum(dots, 0.0)
    return I, A


def check_indexer_row(got: np.ndarray, I: np.ndarray, A: np.ndarray, what: str):
    err = np.abs(got.astype(np.float64) - I)
    bound = IDX_RTOL * np.maximum(np.abs(I), A)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} scores out of tolerance; worst "
                           f"err {err.max():.3e} at s={int(err.argmax())} bound {bound[err.argmax()]:.3e}")


def check_attention(out_bits: np.ndarray, ref: np.ndarray, what: str):
    """Output of a bf16-I/O attention against the fp64 oracle.

    max-abs: |out - ref| <= 1e-2 + 2^-8 |ref|.  The second term is the rounding of
    the result into the bf16 output format (half an ulp is at most 2^-8 of the
    value; it alone reaches 0.0156 for |x| in [4, 8)), which no bf16 output can
    avoid; 1e-2 bounds the computational error on top of it.
    mean-abs: mean |out - ref| <= 1e-3.
    """
    got = oracle.bf16_decode(out_bits)
    err = np.abs(got - ref)
    excess = err - 2.0 ** -8 * np.abs(ref)
    assert excess.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (
        f"{what}: max-abs {err.max():.3e} (beyond bf16 rounding {excess.max():.3e}) mean-abs {err.mean():.3e}")
    return float(err.max()), float(err.mean())


def check_selection(gpu_idx: np.ndarray, I_ref: np.ndarray, n: int, k: int, what: str):
    """End-to-end rule: an index may differ from the oracle's only where its score
    is within 1e-4 (relative) of the oracle's k-th score."""
    ref = oracle.topk_select(I_ref[None, :n], np.array([n]), k)[0]
    g = gpu_idx[gpu_idx >= 0]
    assert len(g) == min(n, k) and np.all(np.diff(g) > 0) and g.max(initial=-1) < n, what
    if n <= k:
        assert np.array_equal(g, np.arange(n)), what
        return 0
    r = ref[ref >= 0]
    diff = np.setxor1d(g, r)
    if diff.size:
        kth = np.sort(I_ref[:n])[::-1][k - 1]
        near = np.abs(I_ref[diff] - kth) <= 1e-4 * abs(kth)
        assert near.all(), f"{what}: {int((~near).sum())} selection mismatches away from the k-th score"
    return int(diff.size)
