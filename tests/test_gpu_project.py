"""The step before the path on the GPU (dsa_project_append): projections, RoPE,
storage casts and cache append against oracle.projection.

Bar: every stored value is the correctly rounded (E4M3 / bf16 / fp32) image of the
oracle's float64 value, up to the rounding of a value within
delta = 2^-16 * A + 2^-22 * |ref| of a rounding boundary, where A = sum_k |h_k W_nk|
bounds the fp32 GEMM's accumulated error (bf16 products are exact in fp32); so
|stored - ref| <= half an ulp of the format at ref + delta.  Cache rows other than
the appended ones stay untouched.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import projection as P
from sparse_attention_weight_b200 import binding as B
from sparse_attention_weight_b200 import build, inputs
from sparse_attention_weight_b200.configs import Workload

pytestmark = pytest.mark.gpu
SENTINEL = 0x5A


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    B.lib()


def half_ulp_bf16(x):
    ax = np.abs(x)
    return np.where(ax > 0, np.exp2(np.floor(np.log2(np.where(ax > 0, ax, 1.0))) - 8.0), 2.0 ** -134)


def half_ulp_e4m3(x):
    ax = np.minimum(np.abs(x), 448.0)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax >= 2.0 ** -6, np.exp2(e - 4.0), 2.0 ** -10)


def _run(case, device, page_size=0):
    T, d, H_I, H, base = case["T"], case["d"], case["H_I"], case["H"], case["base"]
    batch = case["batch"]
    L = P.layout(H_I, H)
    ins = inputs.projection_inputs(T, d, L["total"], seed=case["seed"])
    rows_total = int(batch.kv_len.sum())
    if page_size:
        table, src = inputs.paged_layout(batch, page_size, case["seed"])
        kv_rows = src.size
        db = B.DeviceBatch.from_host(batch, device, kv_rows=kv_rows, page_size=page_size, page_table=table)
    else:
        table, kv_rows = None, rows_total
        db = B.DeviceBatch.from_host(batch, device, kv_rows=kv_rows)
    k_cache = torch.full((kv_rows, 128), SENTINEL, dtype=torch.uint8, device=device)
    kv_cache = torch.full((kv_rows, 576), SENTINEL * 257, dtype=torch.int16, device=device)
    q_idx = torch.empty((T, H_I, 128), dtype=torch.uint8, device=device)
    w = torch.empty((T, H_I), dtype=torch.float32, device=device)
    q = torch.empty((T, H, 576), dtype=torch.int16, device=device)
    ws = B.workspace(B.OP_PROJECT, db, H_I=H_I, H=H, device=device)
    B.dsa_project_append(db, B.bits_to_tensor(ins["hidden"], device), B.bits_to_tensor(ins["w_all"], device), d,
                         H_I, H, base, q_idx, w, q, k_cache, kv_cache, ws)
    flags = B.read_device_status(ws)
    rows = P.cache_rows(batch.kv_offset, batch.q_seq, batch.q_pos, page_size, table)
    return ins, flags, rows, {"q_idx": q_idx.cpu().numpy(), "w": w.cpu().numpy(),
                              "q": B.tensor_to_bits(q), "k_cache": k_cache.cpu().numpy(),
                              "kv_cache": B.tensor_to_bits(kv_cache)}


def _check(case, ins, rows, got):
    T, H_I, H = case["T"], case["H_I"], case["H"]
    batch = case["batch"]
    L = P.layout(H_I, H)
    ref = P.project(ins["hidden"], ins["w_all"], batch.q_pos, H_I, H, case["base"])
    # sum_k |h_k W_nk| [T, N] (float32 is ample for a bound)
    A = (np.abs(oracle.bf16_decode(ins["hidden"])).astype(np.float32)
         @ np.abs(oracle.bf16_decode(ins["w_all"]).astype(np.float32)).T).astype(np.float64)
    # a rotated value mixes two projections: bound it by the larger A of its pair
    Apair = lambda a: np.repeat(np.maximum(a[..., 0::2], a[..., 1::2]), 2, axis=-1)
    sl = lambda n: A[:, L[n][0]:L[n][1]]

    def cmp(got_vals, refv, Ab, half, what):
        err = np.abs(got_vals - refv)
        bound = half(refv) + 2.0 ** -16 * Ab + 2.0 ** -22 * np.abs(refv)
        bad = err > bound
        print(f"[{what}] max err {err.max():.3e}, values off by a rounding step: "
              f"{int((err > half(refv)).sum())} of {err.size}")
        assert not bad.any(), f"{what}: {int(bad.sum())} values beyond the bound; worst {err.max():.3e}"

    cmp(oracle.e4m3_decode(got["q_idx"]), np.clip(ref["q_idx"], -448, 448),
        Apair(sl("q_idx").reshape(T, H_I, 128)), half_ulp_e4m3, "q_idx")
    cmp(got["w"].astype(np.float64), ref["w"], sl("w"), lambda x: np.abs(x) * 2.0 ** -24, "w")
    qref = ref["q"]
    Aq = np.concatenate([sl("q_latent").reshape(T, H, 512), Apair(sl("q_rope").reshape(T, H, 64))], -1)
    cmp(oracle.bf16_decode(got["q"]), qref, Aq, half_ulp_bf16, "q")
    kc, kvc = got["k_cache"], got["kv_cache"]
    cmp(oracle.e4m3_decode(kc[rows]), np.clip(ref["k_idx"], -448, 448), Apair(sl("k_idx")), half_ulp_e4m3, "k_idx")
    kvref = np.concatenate([ref["latent"], ref["k_rope"]], -1)
    Akv = np.concatenate([sl("latent"), Apair(sl("k_rope"))], -1)
    cmp(oracle.bf16_decode(kvc[rows]), kvref, Akv, half_ulp_bf16, "kv")
    untouched = np.ones(kc.shape[0], bool)
    untouched[rows] = False
    assert np.all(kc[untouched] == SENTINEL)
    assert np.all(kvc[untouched] == SENTINEL * 257)


def _case(T_per_seq, lens, d, H_I, H, seed, base=10000.0):
    lens = np.asarray(lens, np.int32)
    off = np.zeros(len(lens), np.int64)
    off[1:] = np.cumsum(lens[:-1])
    qs = np.repeat(np.arange(len(lens), dtype=np.int32), T_per_seq)
    j = np.tile(np.arange(T_per_seq, dtype=np.int32), len(lens))
    pos = (lens[qs] - T_per_seq + j).astype(np.int32)
    batch = inputs.Batch(off, lens, qs, pos, j)
    return {"T": int(pos.size), "d": d, "H_I": H_I, "H": H, "seed": seed, "base": base, "batch": batch}


@pytest.mark.parametrize("page_size", [0, 64])
def test_project_append_small(cuda_device, page_size):
    case = _case(5, [700, 4100, 131072 // 8, 96], d=512, H_I=8, H=16, seed=1)
    ins, flags, rows, got = _run(case, cuda_device, page_size)
    assert flags == 0
    _check(case, ins, rows, got)


def test_project_append_full_width(cuda_device):
    """DeepSeek-V3-sized hidden state (7168) and the workloads' head counts, one
    new token for each of 8 sequences, positions up to 131071."""
    case = _case(1, [5000, 131072, 32768, 4096, 77777, 2049, 100000, 65536], d=7168, H_I=64, H=128, seed=2)
    ins, flags, rows, got = _run(case, cuda_device)
    assert flags == 0
    _check(case, ins, rows, got)


def test_project_append_flags_a_bad_query(cuda_device):
    case = _case(2, [300, 500], d=64, H_I=4, H=8, seed=3)
    case["batch"].q_pos[1] = 300                      # beyond kv_len of sequence 0
    ins, flags, rows, got = _run(case, cuda_device)
    assert flags & 1                                  # DSA_DEV_BAD_QUERY
    kc = got["k_cache"]
    assert np.all(kc[300] == SENTINEL)                # the bad token's row (sequence 1's first) is not written
    for t in (0, 2, 3):                               # the valid tokens are appended
        assert not np.all(kc[rows[t]] == SENTINEL)
