"""CPU oracle for the step before the DSA path: projections, rotary position
embedding, FP8 quantisation and cache append.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The product path never calls it, and
it shares no code with the CUDA library.

Plain float64 numpy, following:
* [一文讀懂] "一文讀懂DeepSeek-V3.2核心技術DSA", section "DSA 的四步工作流程", step 1
  (queries and keys projected from the hidden states, rotary embeddings folded in,
  and a set of per-head weights also projected from the hidden state);
* [路线] "DeepSeek 稀疏注意力路线（V3 / V3.2 / V4）", section on V3's MLA (each
  token's hidden state is down-projected to the latent that is cached; position
  enters through a separate, decoupled RoPE channel);
* [V3.2加速] "DeepSeek-V3.2加速技术详解", 3.1 (MQA form: every query head attends to
  the shared latent row, so the query is expressed in the latent space).

Readings (the pages print no formulas; each is the plainest one the rest of the
pages support):
* One projection per output, with synthetic random weights, stacked in one
  matrix W [N_all, d_model] in this row order: indexer query (H_I x 128),
  indexer key (128), per-head weights (H_I), latent (512), RoPE key (64), latent
  query (H x 512, the MQA-form query), RoPE query (H x 64).  Y = h W^T.
* RoPE: the pairs (x[2i], x[2i+1]) of a D-dim vector are rotated by the angle
  pos * base^(-2i/D), base 10000 (the original rotary form).  It is applied to the
  whole 128-dim indexer query heads and key, and to the 64-dim RoPE parts of the
  MLA key and query; the latent parts carry no position.
* The indexer query and key are stored as E4M3 (round to nearest even,
  saturating at +-448, no scale), the latent row and the MLA query as bf16
  (round to nearest even); the weights stay fp32.
* Cache append: the new token at position pos of sequence b writes its indexer
  key and its latent row [latent, RoPE key] to the cache row of key pos.

Pins (tests/test_oracle_projection.py): RoPE against closed-form rotations of unit
vectors, its norm preservation and the relative-position identity; the
projection against explicit sums; the row order against a weight matrix that
copies chosen inputs; the append against the row mapping.
"""
from __future__ import annotations

import numpy as np

from .dsa_ref import bf16_decode, bf16_encode_rne, e4m3_encode_rne

D_INDEX, D_LATENT, D_ROPE = 128, 512, 64
ROPE_BASE = 10000.0


def rope(x: np.ndarray, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Rotates the pairs (x[..., 2i], x[..., 2i+1]) by pos * base^(-2i/D).

    x: [..., D] (D even); pos broadcasts against x's leading dims.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    i = np.arange(D // 2, dtype=np.float64)
    freq = base ** (-2.0 * i / D)                                  # [D/2]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq        # [..., D/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def layout(H_I: int, H: int) -> dict:
    """Row ranges of the stacked projection matrix (see the module readings)."""
    sizes = [("q_idx", H_I * D_INDEX), ("k_idx", D_INDEX), ("w", H_I), ("latent", D_LATENT),
             ("k_rope", D_ROPE), ("q_latent", H * D_LATENT), ("q_rope", H * D_ROPE)]
    out, o = {}, 0
    for name, n in sizes:
        out[name] = (o, o + n)
        o += n
    out["total"] = o
    return out


def project(h_bits: np.ndarray, w_bits: np.ndarray, pos: np.ndarray, H_I: int, H: int,
            base: float = ROPE_BASE) -> dict:
    """The projections of T hidden states, before storage casts (float64).

    h_bits: bf16 bits [T, d_model]; w_bits: bf16 bits [N_all, d_model];
    pos: [T] positions.  Returns q_idx [T, H_I, 128], k_idx [T, 128], w [T, H_I],
    latent [T, 512], k_rope [T, 64], q [T, H, 576] (latent part then RoPE part).
    """
    L = layout(H_I, H)
    h = bf16_decode(h_bits)
    W = bf16_decode(w_bits)
    assert W.shape == (L["total"], h.shape[1])
    Y = h @ W.T                                                      # [T, N_all]
    pos = np.asarray(pos, dtype=np.int64)
    T = h.shape[0]
    sl = lambda n: Y[:, L[n][0]:L[n][1]]
    q_idx = rope(sl("q_idx").reshape(T, H_I, D_INDEX), pos[:, None], base)
    k_idx = rope(sl("k_idx"), pos, base)
    k_rope = rope(sl("k_rope"), pos, base)
    q_rope = rope(sl("q_rope").reshape(T, H, D_ROPE), pos[:, None], base)
    q = np.concatenate([sl("q_latent").reshape(T, H, D_LATENT), q_rope], axis=-1)
    return {"q_idx": q_idx, "k_idx": k_idx, "w": sl("w").copy(), "latent": sl("latent").copy(),
            "k_rope": k_rope, "q": q}


def stored(p: dict) -> dict:
    """The storage casts of project()'s results: E4M3 codes for the indexer query
    and key, bf16 bits for the latent row [latent, k_rope] and the MLA query,
    fp32 for the weights."""
    return {"q_idx": e4m3_encode_rne(p["q_idx"]), "k_idx": e4m3_encode_rne(p["k_idx"]),
            "w": p["w"].astype(np.float32),
            "kv": bf16_encode_rne(np.concatenate([p["latent"], p["k_rope"]], axis=-1).astype(np.float32)),
            "q": bf16_encode_rne(p["q"].astype(np.float32))}


def cache_rows(kv_offset, q_seq, q_pos, page_size: int = 0, page_table=None) -> np.ndarray:
    """The cache row each new token appends to: kv_offset[b] + pos, or with a paged
    cache page_table[b, pos // page_size] * page_size + pos % page_size."""
    q_seq = np.asarray(q_seq, dtype=np.int64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    if page_size:
        pt = np.asarray(page_table, dtype=np.int64)
        return pt[q_seq, q_pos // page_size] * page_size + q_pos % page_size
    return np.asarray(kv_offset, dtype=np.int64)[q_seq] + q_pos
