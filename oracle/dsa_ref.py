"""CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The product path never calls it, and
it shares no code with the CUDA library (it imports nothing from the package).

Plain, slow, float64 numpy.  Each function follows one step of the method as
the pages state it (titles shortened; sections as on the page):

* [V3.2加速] "DeepSeek-V3.2加速技术详解，效果惊人的秘密？", sections 03 (3.1 MHA版MLA
  VS MQA版MLA; 3.2 lightning indexer 和 fine-grained token selection mechanism).
* [推理加速] "DeepSeek-V3.2推理加速引擎深度剖析", section "DSA核心技术：重要token选择
  机制详解".
* [一文讀懂] "一文讀懂DeepSeek-V3.2核心技術DSA", sections "DSA 的兩大核心組件" and
  "DSA 的四步工作流程" (steps 2-4: indexer scoring, top-k selection, sparse MLA).
* [路线] "DeepSeek 稀疏注意力路线（V3 / V3.2 / V4）", section "DeepSeek-V3.2：DSA",
  "两阶段流程".

The pages print no formulas (they were stripped) and no worked values.  Where
they leave a step open, the reading taken is stated at the function.  The
inputs' number formats (E4M3 bytes, bf16 bit patterns) are decoded here from
the formats' definitions.

Parity pins (tests/test_oracle_pins.py): format decoders against PyTorch's
casts for every code; the indexer against exact rational arithmetic on tiny
inputs; top-k against an exhaustive subset search; sparse MLA against
PyTorch's scaled_dot_product_attention (dense when the context is <= k, masked
to the selection otherwise); softmax normalisation; permutation, chunk and
decode/prefill invariances.  No function here is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """FP8 E4M3 ("fn": no infinities) bytes -> float64, from the format definition.

    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0
    is subnormal: (m/8) * 2^-6.  Otherwise (1 + m/8) * 2^(e-7).  The single
    pattern S.1111.111 is NaN.  The indexer's keys and queries are stored in
    this format ([路线] "两阶段流程": the indexer is usually computed in FP8).
    """
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    out = sign * mag
    out = np.where((e == 0xF) & ((b & 0x7) == 0x7), np.nan, out)
    return out


def e4m3_encode_rne(x: np.ndarray) -> np.ndarray:
    """float64 -> E4M3 bytes, round to nearest even, saturating to +-448.

    Used to check the input quantisation: the representable magnitudes are
    enumerated from the format and the nearest one is chosen, ties to the code
    with an even mantissa.
    """
    x = np.asarray(x, dtype=np.float64)
    codes = np.arange(0x7F, dtype=np.uint8)                     # +0 .. 448 (0x7E); 0x7F is NaN
    vals = e4m3_decode(codes)
    ax = np.minimum(np.abs(x), 448.0)
    # nearest representable magnitude; ties go to the even code
    hi = np.searchsorted(vals, ax, side="left")
    hi = np.clip(hi, 0, vals.size - 1)
    lo = np.clip(hi - 1, 0, vals.size - 1)
    d_lo = ax - vals[lo]
    d_hi = vals[hi] - ax
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((codes[hi] & 1) == 0))
    mag = np.where(pick_hi, codes[hi], codes[lo]).astype(np.uint8)
    sign = np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
    return (mag | sign).astype(np.uint8)


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64: bf16 is the upper half of an IEEE fp32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_encode_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even on the dropped 16 bits (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    round_up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + round_up).astype(np.uint16)


# ---------------------------------------------------------------------------
# Stage 1: lightning indexer
# ---------------------------------------------------------------------------


def indexer_scores(q_idx: np.ndarray, k_idx: np.ndarray, w: np.ndarray,
                   n_vis: np.ndarray) -> np.ndarray:
    """Index scores I[t, s] = sum_j w[t, j] * ReLU(q_I[t, j, :] . k_I[s, :]).

    [一文讀懂] step 2: each query is dotted with every key of the small indexer
    key cache (128 dims per token), masked, then multiplied by the per-head
    weights projected in step 1; [路线] "两阶段流程" adds the ReLU-type
    activation and the aggregation over indexer heads.

    q_idx: [T, H_I, 128] E4M3 bytes; k_idx: [S, 128] E4M3 bytes (the keys of
    the queries' sequence); w: [T, H_I] float32; n_vis: [T] number of visible
    keys (causal, inclusive: n_t = position + 1).  Returns float64 [T, S];
    entries s >= n_t are -inf.

    Readings: no scale beyond w (a step-2 "scale" is taken as folded into w);
    the activation is ReLU.  The FP8 dot products are exact in float64 (each
    product has <= 8 significant bits within 2^-18..2^17; 128 terms add 7 bits).
    """
    q = e4m3_decode(q_idx)                         # [T, H, D]
    k = e4m3_decode(k_idx)                         # [S, D]
    wf = np.asarray(w, dtype=np.float32).astype(np.float64)
    T, H, D = q.shape
    S = k.shape[0]
    dots = (q.reshape(T * H, D) @ k.T).reshape(T, H, S)
    scores = np.einsum("th,ths->ts", wf, np.maximum(dots, 0.0))
    n_vis = np.asarray(n_vis, dtype=np.int64)
    mask = np.arange(S)[None, :] >= n_vis[:, None]
    scores[mask] = -np.inf
    return scores


# ---------------------------------------------------------------------------
# Stage 2: fine-grained top-k selection
# ---------------------------------------------------------------------------


def topk_select(scores: np.ndarray, n_vis: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k highest index scores per query.

    [一文讀懂] step 3: keep the top 2048 tokens of the whole context per query;
    if the context has <= k tokens, keep all of them (DSA is then dense
    attention).  [V3.2加速] 3.2 / [推理加速]: the rest are dropped outright
    (hard selection).

    Readings: equal scores go to the lower index; -0.0 equals +0.0; the output
    is sorted by ascending index and padded with -1 to width k.
    scores: [T, >= max n] (float32 or float64); returns int32 [T, k].
    """
    T = scores.shape[0]
    out = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = int(n_vis[t])
        if n <= k:
            out[t, :n] = np.arange(n, dtype=np.int32)
            continue
        row = np.asarray(scores[t, :n], dtype=np.float64)
        order = np.argsort(-row, kind="stable")     # stable: ties keep index order
        out[t] = np.sort(order[:k]).astype(np.int32)
    return out


# ---------------------------------------------------------------------------
# Stage 3: sparse MLA in MQA form
# ---------------------------------------------------------------------------


def sparse_mla(q: np.ndarray, kv: np.ndarray, idx: np.ndarray, sm_scale: float,
               d_v: int = 512):
    """Attention of each query over only its selected latent rows.

    [一文讀懂] step 4 / [V3.2加速] 3.1: MLA in MQA form -- all heads share one
    latent key/value row per token; attention is computed directly on the
    latent (512 dims plus the 64-dim RoPE key) and the value is the latent
    itself ("restored at the end", i.e. the up-projection is not part of this
    step).  [V3.2加速] 3.2: unselected tokens contribute nothing.

    q: [T, H, 576] float64; kv: [S, 576] float64 (rows of the queries'
    sequence); idx: [T, k] local row indices, -1 = unused.
    Returns (out [T, H, d_v] float64, lse [T, H] float64) with
    z = sm_scale * q . kv_row, p = softmax over the selected rows,
    out = sum p * kv_row[:d_v], lse = ln sum exp(z).  A query with no
    selected row gets out = 0 and lse = -inf.
    """
    T, H, _ = q.shape
    out = np.zeros((T, H, d_v), dtype=np.float64)
    lse = np.full((T, H), -np.inf, dtype=np.float64)
    for t in range(T):
        sel = idx[t][idx[t] >= 0]
        if sel.size == 0:
            continue
        rows = kv[sel]                              # [m, 576]
        z = sm_scale * (q[t] @ rows.T)              # [H, m]
        zmax = z.max(axis=1, keepdims=True)
        e = np.exp(z - zmax)
        den = e.sum(axis=1, keepdims=True)
        out[t] = (e / den) @ rows[:, :d_v]
        lse[t] = zmax[:, 0] + np.log(den[:, 0])
    return out, lse


def attention_probs(q: np.ndarray, kv: np.ndarray, sel: np.ndarray, sm_scale: float) -> np.ndarray:
    """Softmax weights [H, m] of one query over the rows ``sel`` (used by the pins)."""
    z = sm_scale * (q @ kv[sel].T)
    e = np.exp(z - z.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def dense_mla(q: np.ndarray, kv: np.ndarray, n_vis: np.ndarray, sm_scale: float, d_v: int = 512):
    """Dense causal MQA attention over keys 0..n_t-1 (the L <= k special case)."""
    T = q.shape[0]
    k = int(np.max(n_vis)) if T else 0
    idx = np.full((T, max(k, 1)), -1, dtype=np.int64)
    for t in range(T):
        idx[t, :n_vis[t]] = np.arange(n_vis[t])
    return sparse_mla(q, kv, idx, sm_scale, d_v)


# ---------------------------------------------------------------------------
# Composition over a batch of sequences
# ---------------------------------------------------------------------------


def forward(kv_offset, kv_len, q_seq, q_pos, q_idx, k_idx, w, q_bits, kv_bits,
            k: int, sm_scale: float, queries=None, d_v: int = 512, selections=None):
    """The whole path for the given queries: scores -> top-k -> sparse MLA.

    [一文讀懂] "四步工作流程", steps 2-4, applied per query against its own
    sequence's cache rows.  Arrays are the raw inputs of the call (E4M3 bytes,
    fp32 weights, bf16 bit patterns) in the packed-cache layout: sequence b
    owns cache rows kv_offset[b] .. kv_offset[b] + kv_len[b] - 1.

    ``queries`` selects a subset of query rows (default: all).  ``selections``
    (optional, one index row per entry of ``queries``) replaces step 3's own
    choice in step 4, so that the attention step can be evaluated on another
    selection (the tests compare a GPU's attention on the GPU's own choice).
    Returns a dict with per-query lists: "scores" (float64 [n_t]), "idx"
    (int32 [k], the top-k choice), and arrays "out" [n, H, d_v], "lse" [n, H].
    """
    if queries is None:
        queries = np.arange(len(q_pos))
    queries = np.asarray(queries)
    H = q_bits.shape[1]
    out = np.zeros((queries.size, H, d_v))
    lse = np.zeros((queries.size, H))
    scores_l, idx_l = [], []
    for i, t in enumerate(queries):
        b = int(q_seq[t])
        off, n_b = int(kv_offset[b]), int(kv_len[b])
        n = int(q_pos[t]) + 1
        keys = k_idx[off:off + n_b]
        s = indexer_scores(q_idx[t:t + 1], keys, w[t:t + 1], np.array([n]))[0]
        chosen = topk_select(s[None, :n].astype(np.float64), np.array([n]), k)[0]
        sel = chosen if selections is None else np.asarray(selections[i])
        # only the selected rows of the sequence are decoded: step 4 reads no other
        valid = sel[sel >= 0].astype(np.int64)
        rows = bf16_decode(kv_bits[off + valid])
        local = np.full(sel.shape, -1, dtype=np.int64)
        local[sel >= 0] = np.arange(valid.size)
        o, l = sparse_mla(bf16_decode(q_bits[t:t + 1]), rows, local[None, :], sm_scale, d_v)
        out[i], lse[i] = o[0], l[0]
        scores_l.append(s[:n])
        idx_l.append(chosen)
    return {"scores": scores_l, "idx": idx_l, "out": out, "lse": lse}
