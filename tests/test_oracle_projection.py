"""Pins of the projection / RoPE / quantise / append oracle (oracle.projection)
to facts outside itself: closed-form rotations, the rotation identities, explicit
sums and a weight matrix whose every row copies one known input."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import projection as P
from oracle import bf16_decode


def test_rope_closed_forms():
    # D = 2: the single pair turns by pos * 1 radian
    assert np.allclose(P.rope(np.array([1.0, 0.0]), 1), [math.cos(1.0), math.sin(1.0)], atol=1e-15)
    assert np.allclose(P.rope(np.array([0.0, 1.0]), 1), [-math.sin(1.0), math.cos(1.0)], atol=1e-15)
    # D = 4: the second pair turns at base^(-2/4) = 0.01 rad per position
    e2, e3 = np.eye(4)[2], np.eye(4)[3]
    assert np.allclose(P.rope(e2, 3), [0, 0, math.cos(0.03), math.sin(0.03)], atol=1e-15)
    assert np.allclose(P.rope(e3, 3), [0, 0, -math.sin(0.03), math.cos(0.03)], atol=1e-15)
    # the first pair of a D = 4 vector turns at 1 rad per position, independently
    assert np.allclose(P.rope(np.eye(4)[0], 2), [math.cos(2.0), math.sin(2.0), 0, 0], atol=1e-15)


def test_rope_identities():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    assert np.array_equal(P.rope(q, 0), q)
    r = P.rope(q, 777)
    assert np.allclose(r[0::2] ** 2 + r[1::2] ** 2, q[0::2] ** 2 + q[1::2] ** 2, rtol=1e-13)
    # scores depend on the relative position only
    for m, n in ((5, 2), (1000, 37), (131071, 4096)):
        a = P.rope(q, m) @ P.rope(k, n)
        b = P.rope(q, m - n) @ k
        assert abs(a - b) <= 1e-9 * (np.abs(q) @ np.abs(k))


def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_projection_against_explicit_sums():
    H_I, H, d, T = 4, 8, 5, 2
    L = P.layout(H_I, H)
    rng = np.random.default_rng(6)
    h = _bits(rng.standard_normal((T, d)))
    W = _bits(rng.standard_normal((L["total"], d)) / math.sqrt(d))
    pos = np.array([0, 3])
    got = P.project(h, W, pos, H_I, H)
    hd, Wd = bf16_decode(h), bf16_decode(W)
    Y = np.zeros((T, L["total"]))
    for t in range(T):
        for n in range(L["total"]):
            s = 0.0
            for c in range(d):
                s += hd[t, c] * Wd[n, c]
            Y[t, n] = s
    a, b = L["w"]
    assert np.allclose(got["w"], Y[:, a:b], rtol=1e-12, atol=1e-14)
    a, b = L["latent"]
    assert np.allclose(got["latent"], Y[:, a:b], rtol=1e-12, atol=1e-14)
    a, b = L["k_idx"]
    for t in range(T):
        assert np.allclose(got["k_idx"][t], P.rope(Y[t, a:b], pos[t]), rtol=1e-12, atol=1e-14)


def test_projection_row_order():
    """W[n] copies input n mod d, so at position 0 (no rotation) every output slot
    must hold the input its row number names."""
    H_I, H, d, T = 8, 16, 7, 3
    L = P.layout(H_I, H)
    W = np.zeros((L["total"], d), np.float32)
    W[np.arange(L["total"]), np.arange(L["total"]) % d] = 1.0
    h = _bits(np.arange(T * d, dtype=np.float32).reshape(T, d) + 1.0)
    got = P.project(h, _bits(W), np.zeros(T, np.int64), H_I, H)
    hd = bf16_decode(h)
    src = lambda name: hd[:, np.arange(*L[name]) % d]
    assert np.array_equal(got["q_idx"].reshape(T, -1), src("q_idx"))
    assert np.array_equal(got["k_idx"], src("k_idx"))
    assert np.array_equal(got["w"], src("w"))
    assert np.array_equal(got["latent"], src("latent"))
    assert np.array_equal(got["k_rope"], src("k_rope"))
    q = got["q"]
    assert np.array_equal(q[:, :, :512].reshape(T, -1), src("q_latent"))
    assert np.array_equal(q[:, :, 512:].reshape(T, -1), src("q_rope"))


def test_storage_casts_match_torch():
    rng = np.random.default_rng(7)
    p = {"q_idx": rng.standard_normal((3, 4, 128)) * 3, "k_idx": rng.standard_normal((3, 128)) * 600,
         "w": rng.standard_normal((3, 4)), "latent": rng.standard_normal((3, 512)),
         "k_rope": rng.standard_normal((3, 64)), "q": rng.standard_normal((3, 8, 576))}
    s = P.stored(p)
    f8 = lambda x: torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s["q_idx"], f8(p["q_idx"]))
    assert np.array_equal(s["k_idx"], f8(p["k_idx"]))      # saturating at +-448
    kv = np.concatenate([p["latent"], p["k_rope"]], -1)
    assert np.array_equal(s["kv"], _bits(kv))
    assert np.array_equal(s["q"], _bits(p["q"]))


def test_cache_rows_contiguous_and_paged():
    off = np.array([0, 100, 250])
    assert list(P.cache_rows(off, [0, 2, 1], [5, 0, 99])) == [5, 250, 199]
    pt = np.array([[3, 1, -1], [0, 2, 5]])
    assert list(P.cache_rows(None, [0, 0, 1, 1], [0, 65, 63, 130], 64, pt)) == [192, 65, 63, 322]
