"""Shared helpers of the GPU parity tests: device copies of seeded inputs, the
oracle's results for chosen query rows, and the tolerance checks the tests apply.

Every reference value comes from one composition, ``oracle.forward``: it maps a
query to its sequence's cache rows and its visible keys, scores them, selects
the top k and attends over a selection (its own, or one given to it).

Tolerances (each stated where it is applied):
  indexer scores: |I_gpu - I_ref| <= 1e-4 * max(|I_ref|, A_ref) with
      A_ref = sum_j |w_j| ReLU(dot_j), the scale of the sum before cancellation;
  attention output (bf16 I/O) against the fp64 oracle: max-abs <= 1e-2 and
      mean-abs <= 1e-3; only where the result is so large (|ref| >= 4) that
      half an ulp of bf16 alone exceeds 1e-2 is that half ulp added to the bar;
  lse: abs <= 2e-3 (fp32 softmax statistics over 576-term bf16 dot products).
"""
from __future__ import annotations

import numpy as np

import oracle
from sparse_attention_weight_b200 import binding as B

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


def oracle_rows(ins: dict, wl, rows, selections=None) -> dict:
    """oracle.forward for the query rows `rows` (optionally attending over the
    given selections instead of the oracle's own top-k choice)."""
    b = ins["batch"]
    return oracle.forward(b.kv_offset, b.kv_len, b.q_seq, b.q_pos, ins["q_idx"], ins["k_idx"], ins["w"],
                          ins["q"], ins["kv"], wl.k, wl.sm_scale, queries=np.asarray(list(rows), dtype=np.int64),
                          selections=selections)


def condition_scale(ins: dict, t: int, n: int) -> np.ndarray:
    """A_ref[s] = sum_j |w[t,j]| * ReLU(q_I[t,j] . k_I[s]) for the n visible keys of
    query t: the size of the indexer sum before its signed terms cancel."""
    batch = ins["batch"]
    off = int(batch.kv_offset[int(batch.q_seq[t])])
    qd = oracle.e4m3_decode(ins["q_idx"][t])                 # [H_I, 128]
    kd = oracle.e4m3_decode(ins["k_idx"][off:off + n])       # [n, 128]
    return np.abs(ins["w"][t].astype(np.float64)) @ np.maximum(qd @ kd.T, 0.0)


def check_indexer_row(got: np.ndarray, I: np.ndarray, A: np.ndarray, what: str):
    err = np.abs(got.astype(np.float64) - I)
    bound = IDX_RTOL * np.maximum(np.abs(I), A)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} scores out of tolerance; worst "
                           f"err {err.max():.3e} at s={int(err.argmax())} bound {bound[err.argmax()]:.3e}")


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8.0), 0.0)


def check_attention(out_bits: np.ndarray, ref: np.ndarray, what: str):
    """Output of a bf16-I/O attention against the fp64 oracle: max-abs <= 1e-2 and
    mean-abs <= 1e-3, with half an ulp of bf16 added only where that half ulp
    alone exceeds 1e-2 (|ref| >= 4).  Prints the statistics."""
    got = oracle.bf16_decode(out_bits)
    err = np.abs(got - ref)
    h = bf16_half_ulp(ref)
    bound = OUT_MAX_ABS + np.where(h > OUT_MAX_ABS, h, 0.0)
    worst = int(np.argmax(err - bound))
    print(f"[{what}] attention max-abs {err.max():.3e} mean-abs {err.mean():.3e} "
          f"(largest |ref| {np.abs(ref).max():.3f})")
    assert (err <= bound).all() and err.mean() <= OUT_MEAN_ABS, (
        f"{what}: max-abs {err.max():.3e} (worst {err.flat[worst]:.3e} at |ref| {abs(ref.flat[worst]):.3f}, "
        f"bound {bound.flat[worst]:.3e}) mean-abs {err.mean():.3e}")
    return float(err.max()), float(err.mean())


def check_lse(lse: np.ndarray, ref: np.ndarray, what: str):
    err = np.abs(lse - ref)
    print(f"[{what}] lse max-abs {err.max():.3e}")
    assert err.max() <= LSE_ABS, f"{what}: lse max-abs {err.max():.3e}"


def check_selection(gpu_idx: np.ndarray, ref_idx: np.ndarray, I_ref: np.ndarray, n: int, k: int, what: str):
    """End-to-end rule: an index may differ from the oracle's only where its score
    is within 1e-4 (relative) of the oracle's k-th score."""
    g = gpu_idx[gpu_idx >= 0]
    assert len(g) == min(n, k) and np.all(np.diff(g) > 0) and g.max(initial=-1) < n, what
    if n <= k:
        assert np.array_equal(g, np.arange(n)), what
        return 0
    r = ref_idx[ref_idx >= 0]
    diff = np.setxor1d(g, r)
    if diff.size:
        kth = np.sort(I_ref[:n])[::-1][k - 1]
        near = np.abs(I_ref[diff] - kth) <= 1e-4 * abs(kth)
        assert near.all(), f"{what}: {int((~near).sum())} selection mismatches away from the k-th score"
    return int(diff.size)
