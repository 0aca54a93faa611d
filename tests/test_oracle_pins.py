"""Pins of the CPU oracle to things other than itself.

Each test checks the oracle against an independent fact: a library cast or
routine, exact rational arithmetic, an exhaustive search, or an invariant the
method must satisfy.  A plausible slip in the oracle (dropped ReLU, wrong
mask boundary, transposed operand, wrong tie rule, missing softmax scale,
value taken from the wrong columns) fails at least one of them.
"""
from __future__ import annotations

import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_weight_b200 import inputs
from sparse_attention_weight_b200.configs import Workload

# --------------------------------------------------------------------------- formats


def test_e4m3_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref, equal_nan=True)
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9


def test_e4m3_encode_matches_torch_cast_including_ties():
    rng = np.random.default_rng(1)
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[1:] + vals[:-1]) / 2            # exact ties
    x = np.concatenate([rng.standard_normal(200_000) * 3, rng.standard_normal(2000) * 1e-3,
                        mids, -mids, vals, -vals, [0.0, -0.0, 448.0, -448.0]])
    x = x.astype(np.float32).astype(np.float64)   # torch casts from fp32
    ours = oracle.e4m3_encode_rne(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_bf16_decode_and_encode_match_torch():
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 1 << 16, size=100_000, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7F80) != 0x7F80
    bits = bits[finite]
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_decode(bits), ref)
    x = np.concatenate([rng.standard_normal(100_000).astype(np.float32),
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)], np.float32)])
    ref_bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_encode_rne(x), ref_bits)


def test_generator_quantisation_is_the_stated_rne_cast():
    wl = Workload("pin_gen", 90, "prefill", k=16, h_index=4, heads=8, seq_len=40)
    b = inputs.make_batch(wl)
    q_idx = inputs.query_rows(wl, b, "q_idx")
    raw = inputs._chunk_rows(0, wl.cfg_id, inputs.T_QIDX, 0, 0, 40, (4, 128))
    assert np.array_equal(q_idx, oracle.e4m3_encode_rne(raw.astype(np.float64)))
    q = inputs.query_rows(wl, b, "q")
    rawq = inputs._chunk_rows(0, wl.cfg_id, inputs.T_Q, 0, 0, 40, (8, 576))
    assert np.array_equal(q, oracle.bf16_encode_rne(rawq))

# --------------------------------------------------------------------------- indexer


def _exact_scores(q_idx, k_idx, w, n_vis):
    """Index scores in exact rational arithmetic, written as plain loops."""
    qv = oracle.e4m3_decode(q_idx)
    kv = oracle.e4m3_decode(k_idx)
    T, H, D = qv.shape
    S = kv.shape[0]
    out = [[None] * S for _ in range(T)]
    dots = [[[None] * S for _ in range(H)] for _ in range(T)]
    for t in range(T):
        for s in range(S):
            if s >= n_vis[t]:
                continue
            acc = Fraction(0)
            for j in range(H):
                d = Fraction(0)
                for c in range(D):
                    d += Fraction(float(qv[t, j, c])) * Fraction(float(kv[s, c]))
                dots[t][j][s] = d
                if d > 0:
                    acc += Fraction(float(np.float32(w[t, j]))) * d
            out[t][s] = acc
    return out, dots


def test_indexer_matches_exact_rational_arithmetic():
    rng = np.random.default_rng(3)
    T, H, D, S = 3, 3, 128, 7
    q_idx = oracle.e4m3_encode_rne(rng.standard_normal((T, H, D)))
    k_idx = oracle.e4m3_encode_rne(rng.standard_normal((S, D)))
    w = (rng.standard_normal((T, H)) / np.sqrt(H)).astype(np.float32)
    n_vis = np.array([1, 4, 7])
    got = oracle.indexer_scores(q_idx, k_idx, w, n_vis)
    exact, dots = _exact_scores(q_idx, k_idx, w, n_vis)
    qv, kv = oracle.e4m3_decode(q_idx), oracle.e4m3_decode(k_idx)
    for t in range(T):
        for s in range(S):
            if s >= n_vis[t]:
                assert got[t, s] == -np.inf
                continue
            scale = sum(abs(float(w[t, j])) * max(float(dots[t][j][s]), 0.0) for j in range(H))
            assert abs(got[t, s] - float(exact[t][s])) <= 1e-15 * max(scale, 1e-300)
            # the FP8 dot products themselves are exact in float64
            for j in range(H):
                assert Fraction(float(qv[t, j] @ kv[s])) == dots[t][j][s]


def test_indexer_special_cases():
    rng = np.random.default_rng(4)
    T, H, D, S = 2, 4, 128, 6
    q_idx = oracle.e4m3_encode_rne(rng.standard_normal((T, H, D)))
    k_idx = oracle.e4m3_encode_rne(rng.standard_normal((S, D)))
    n_vis = np.array([S, 3])
    qv, kv = oracle.e4m3_decode(q_idx), oracle.e4m3_decode(k_idx)
    # one-hot weights pick out ReLU of a single head's dot product
    for j in range(H):
        w = np.zeros((T, H), np.float32)
        w[:, j] = 1.0
        got = oracle.indexer_scores(q_idx, k_idx, w, n_vis)
        for t in range(T):
            for s in range(n_vis[t]):
                assert got[t, s] == max(float(qv[t, j] @ kv[s]), 0.0)
    # keys opposite to every query head give zero (ReLU cuts every term)
    k_neg = oracle.e4m3_encode_rne(-np.sign(qv[0, 0])[None, :] * np.ones((1, D)))
    q_same = np.repeat(q_idx[:1, :1], H, axis=1)
    w = rng.standard_normal((1, H)).astype(np.float32)
    assert oracle.indexer_scores(q_same, k_neg, w, np.array([1]))[0, 0] == 0.0
    # linear in w
    w1 = rng.standard_normal((T, H)).astype(np.float32)
    a = oracle.indexer_scores(q_idx, k_idx, w1, n_vis)
    b = oracle.indexer_scores(q_idx, k_idx, (2 * w1).astype(np.float32), n_vis)
    fin = np.isfinite(a)
    assert np.array_equal(2 * a[fin], b[fin])
    # causal mask is inclusive of the query's own position
    assert np.isfinite(a[1, 2]) and a[1, 3] == -np.inf

# --------------------------------------------------------------------------- top-k


def _exhaustive_topk(row, k):
    """Among all k-subsets with the largest exact score sum, the lexicographically
    smallest sorted index tuple (this is 'ties go to the lower index')."""
    best_sum, best = None, None
    fr = [Fraction(float(v)) for v in row]
    for comb in itertools.combinations(range(len(row)), k):
        s = sum(fr[i] for i in comb)
        if best_sum is None or s > best_sum or (s == best_sum and comb < best):
            best_sum, best = s, comb
    return list(best)


def test_topk_matches_exhaustive_search_with_ties_and_signed_zeros():
    rng = np.random.default_rng(5)
    pool = np.array([-1.5, -0.0, 0.0, 0.25, 0.25, 1.0, 2.0, -np.inf], dtype=np.float32)
    for trial in range(300):
        n = int(rng.integers(1, 10))
        row = rng.choice(pool[:-1] if trial % 3 else pool, size=n)
        if not np.isfinite(row).any():
            continue
        for k in range(1, 10):
            got = oracle.topk_select(row[None, :], np.array([n]), k)[0]
            if n <= k:
                assert list(got[:n]) == list(range(n)) and all(got[n:] == -1)
            else:
                fin = np.isfinite(row).all()
                if not fin:
                    continue  # -inf never appears among visible keys
                assert list(got) == _exhaustive_topk(row, k)


def test_topk_invariants_on_larger_rows():
    rng = np.random.default_rng(6)
    n, k = 5000, 700
    row = np.round(rng.standard_normal(n), 2).astype(np.float32)   # many ties
    got = oracle.topk_select(row[None, :], np.array([n]), k)[0]
    assert np.all(np.diff(got) > 0)
    sel = np.zeros(n, bool)
    sel[got] = True
    thr = row[sel].min()
    assert thr >= row[~sel].max()
    # among entries equal to the threshold, exactly the lowest indices are taken
    eq = np.flatnonzero(row == thr)
    taken = eq[sel[eq]]
    assert np.array_equal(taken, eq[:taken.size])

# --------------------------------------------------------------------------- sparse MLA


def _rand_mla(rng, T, H, S):
    q = oracle.bf16_decode(oracle.bf16_encode_rne(rng.standard_normal((T, H, 576)).astype(np.float32)))
    kv = oracle.bf16_decode(oracle.bf16_encode_rne(rng.standard_normal((S, 576)).astype(np.float32)))
    return q, kv


def _sdpa(q, kv, mask, scale):
    T, H, _ = q.shape
    S = kv.shape[0]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                     # [1, H, T, 576]
    kt = torch.from_numpy(kv)[None, None].expand(1, H, S, 576)
    vt = torch.from_numpy(kv[:, :512].copy())[None, None].expand(1, H, S, 512)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def test_dense_case_equals_library_attention():
    """Context <= k: DSA selects everything and equals dense causal attention."""
    rng = np.random.default_rng(7)
    T = S = 24
    H, k, scale = 8, 32, 1 / np.sqrt(576)
    q, kv = _rand_mla(rng, T, H, S)
    n_vis = np.arange(1, T + 1)
    idx = oracle.topk_select(np.zeros((T, S)), n_vis, k)
    out, lse = oracle.sparse_mla(q, kv, idx, scale)
    mask = np.tril(np.ones((T, S), bool))
    ref = _sdpa(q, kv, mask, scale)
    assert np.max(np.abs(out - ref)) < 1e-12
    z = scale * torch.einsum("thd,sd->ths", torch.from_numpy(q), torch.from_numpy(kv))
    z = z.masked_fill(~torch.from_numpy(mask)[:, None, :], -float("inf"))
    assert np.max(np.abs(lse - torch.logsumexp(z, dim=-1).numpy())) < 1e-12
    d_out, d_lse = oracle.dense_mla(q, kv, n_vis, scale)
    assert np.max(np.abs(d_out - ref)) < 1e-12


def test_hard_selection_equals_masked_library_attention():
    rng = np.random.default_rng(8)
    T, H, S, k, scale = 6, 8, 50, 9, 0.05
    q, kv = _rand_mla(rng, T, H, S)
    idx = np.full((T, k), -1, np.int64)
    mask = np.zeros((T, S), bool)
    for t in range(T):
        m = int(rng.integers(1, k + 1))
        sel = np.sort(rng.choice(S, size=m, replace=False))
        idx[t, :m] = sel
        mask[t, sel] = True
    out, _ = oracle.sparse_mla(q, kv, idx, scale)
    assert np.max(np.abs(out - _sdpa(q, kv, mask, scale))) < 1e-12


def test_softmax_rows_sum_to_one_and_order_does_not_matter():
    rng = np.random.default_rng(9)
    T, H, S, k, scale = 4, 8, 40, 12, 1 / np.sqrt(576)
    q, kv = _rand_mla(rng, T, H, S)
    idx = np.stack([np.sort(rng.choice(S, size=k, replace=False)) for _ in range(T)])
    for t in range(T):
        p = oracle.attention_probs(q[t], kv, idx[t], scale)
        assert np.max(np.abs(p.sum(axis=1) - 1)) < 1e-14 and p.min() >= 0
    out, lse = oracle.sparse_mla(q, kv, idx, scale)
    perm = np.stack([rng.permutation(r) for r in idx])
    out2, lse2 = oracle.sparse_mla(q, kv, perm, scale)
    assert np.max(np.abs(out - out2)) < 1e-13 and np.max(np.abs(lse - lse2)) < 1e-13
    # padding entries (-1) are skipped wherever they sit
    pad = np.concatenate([np.full((T, 3), -1), perm], axis=1)
    out3, _ = oracle.sparse_mla(q, kv, pad, scale)
    assert np.max(np.abs(out - out3)) < 1e-13

# --------------------------------------------------------------------------- composition


def _fwd(wl, batch, ins, queries=None):
    return oracle.forward(batch.kv_offset, batch.kv_len, batch.q_seq, batch.q_pos, ins["q_idx"],
                          ins["k_idx"], ins["w"], ins["q"], ins["kv"], wl.k, wl.sm_scale,
                          queries=queries)


def test_chunked_prefill_equals_unchunked():
    pre = Workload("pin_pre", 91, "prefill", k=20, h_index=4, heads=8, seq_len=96)
    chk = Workload("pin_pre", 91, "chunked_prefill", k=20, h_index=4, heads=8, seq_len=96, chunk=32)
    ins = inputs.make_inputs(pre)
    full = _fwd(pre, ins["batch"], ins)
    for c in range(3):
        ci = inputs.make_inputs(chk, chunk_index=c)
        part = _fwd(chk, ci["batch"], ci)
        rows = slice(32 * c, 32 * c + 32)
        assert np.array_equal(part["out"], full["out"][rows])
        assert all(np.array_equal(a, b) for a, b in zip(part["idx"], full["idx"][rows]))


def test_two_token_decode_equals_last_prefill_rows():
    pre = Workload("pin_dec", 92, "prefill", k=16, h_index=4, heads=8, seq_len=50)
    ins = inputs.make_inputs(pre)
    full = _fwd(pre, ins["batch"], ins)
    L = 50
    b = inputs.Batch(np.zeros(1, np.int64), np.array([L], np.int32), np.zeros(2, np.int32),
                     np.array([L - 2, L - 1], np.int32), np.array([L - 2, L - 1], np.int32))
    dec = {"q_idx": inputs.query_rows(pre, b, "q_idx"), "w": inputs.query_rows(pre, b, "w"),
           "q": inputs.query_rows(pre, b, "q"), "k_idx": ins["k_idx"], "kv": ins["kv"]}
    res = _fwd(pre, b, dec)
    assert np.array_equal(res["out"], full["out"][L - 2:])
    assert np.array_equal(res["lse"], full["lse"][L - 2:])


def test_batched_sequences_are_independent():
    dec = Workload("pin_b", 93, "decode", k=8, h_index=4, heads=8, batch=3, ctx_min=5, ctx_max=30,
                   q_per_seq=2)
    ins = inputs.make_inputs(dec)
    batch = ins["batch"]
    res = _fwd(dec, batch, ins)
    for t in range(batch.num_q):
        b = int(batch.q_seq[t])
        one = inputs.Batch(np.zeros(1, np.int64), batch.kv_len[b:b + 1], np.zeros(1, np.int32),
                           batch.q_pos[t:t + 1], batch.q_row[t:t + 1])
        off, n = int(batch.kv_offset[b]), int(batch.kv_len[b])
        r = oracle.forward(one.kv_offset, one.kv_len, one.q_seq, one.q_pos, ins["q_idx"][t:t + 1],
                           ins["k_idx"][off:off + n], ins["w"][t:t + 1], ins["q"][t:t + 1],
                           ins["kv"][off:off + n], dec.k, dec.sm_scale)
        assert np.array_equal(r["out"][0], res["out"][t])


@pytest.mark.parametrize("k", [4, 16])
def test_selection_is_a_pure_function_of_the_scores(k):
    rng = np.random.default_rng(10)
    s = rng.standard_normal((3, 30))
    a = oracle.topk_select(s, np.array([30, 10, 3]), k)
    b = oracle.topk_select(s.copy(), np.array([30, 10, 3]), k)
    assert np.array_equal(a, b)


def _composition_from_library_routines(batch, ins, k, scale):
    """The whole path for every query, written directly with PyTorch float64
    routines and none of the oracle's functions: PyTorch's casts decode the
    inputs, sequence b is sliced as rows kv_offset[b] .. + kv_len[b], query t
    sees keys 0 .. q_pos[t] (inclusive), a stable descending sort picks the k
    largest scores (ties to the lower index), and scaled_dot_product_attention
    attends over the chosen rows through a boolean mask."""
    qi = torch.from_numpy(ins["q_idx"]).view(torch.float8_e4m3fn).to(torch.float64)
    ki = torch.from_numpy(ins["k_idx"]).view(torch.float8_e4m3fn).to(torch.float64)
    w = torch.from_numpy(ins["w"]).to(torch.float64)
    q = torch.from_numpy(ins["q"].view(np.int16)).view(torch.bfloat16).to(torch.float64)
    kv = torch.from_numpy(ins["kv"].view(np.int16)).view(torch.bfloat16).to(torch.float64)
    outs, lses, chosen = [], [], []
    for t in range(batch.num_q):
        b = int(batch.q_seq[t])
        lo, hi = int(batch.kv_offset[b]), int(batch.kv_offset[b]) + int(batch.kv_len[b])
        vis = int(batch.q_pos[t]) + 1
        keys, rows = ki[lo:hi][:vis], kv[lo:hi][:vis]
        score = (torch.relu(qi[t] @ keys.T) * w[t][:, None]).sum(dim=0)          # [vis]
        order = torch.sort(score, descending=True, stable=True).indices
        pick = torch.sort(order[:k]).values
        mask = torch.zeros(vis, dtype=torch.bool)
        mask[pick] = True
        Hh = q.shape[1]
        o = torch.nn.functional.scaled_dot_product_attention(
            q[t][None, :, None, :], rows[None, None].expand(1, Hh, vis, 576),
            rows[None, None, :, :512].expand(1, Hh, vis, 512), attn_mask=mask[None, None, None, :], scale=scale)
        z = scale * (q[t] @ rows.T)
        lses.append(torch.logsumexp(z.masked_fill(~mask[None, :], -float("inf")), dim=1).numpy())
        outs.append(o[0, :, 0, :].numpy())
        chosen.append(pick.numpy())
    return np.stack(outs), np.stack(lses), chosen


@pytest.mark.parametrize("wl", [
    Workload("pin_fwd_dec", 94, "decode", k=12, h_index=4, heads=8, batch=4, ctx_min=6, ctx_max=40, q_per_seq=2),
    Workload("pin_fwd_pre", 95, "prefill", k=10, h_index=8, heads=8, seq_len=33),
    Workload("pin_fwd_chk", 96, "chunked_prefill", k=16, h_index=4, heads=8, seq_len=64, chunk=16),
], ids=lambda w: w.name)
def test_forward_equals_composition_of_library_routines(wl):
    """Pins the oracle's composition (which cache rows a query sees, how many keys
    are visible, per-sequence slicing of a packed cache) to an independent
    restatement that calls none of the oracle's functions."""
    ins = inputs.make_inputs(wl, chunk_index=2 if wl.kind == "chunked_prefill" else None)
    batch = ins["batch"]
    res = oracle.forward(batch.kv_offset, batch.kv_len, batch.q_seq, batch.q_pos, ins["q_idx"], ins["k_idx"],
                         ins["w"], ins["q"], ins["kv"], wl.k, wl.sm_scale)
    out, lse, chosen = _composition_from_library_routines(batch, ins, wl.k, wl.sm_scale)
    assert np.max(np.abs(res["out"] - out)) < 1e-12
    assert np.max(np.abs(res["lse"] - lse)) < 1e-12
    for t in range(batch.num_q):
        got = res["idx"][t]
        assert np.array_equal(got[got >= 0], chosen[t])
        assert len(res["scores"][t]) == int(batch.q_pos[t]) + 1
    # the decode and prefill batches mix contexts below and above k, so both branches of step 3 run
    n = batch.q_pos + 1
    if wl.kind != "chunked_prefill":
        assert (n <= wl.k).any() and (n > wl.k).any()


def test_forward_evaluates_attention_on_a_given_selection():
    wl = Workload("pin_fwd_sel", 97, "decode", k=8, h_index=4, heads=8, batch=2, ctx_min=20, ctx_max=30,
                  q_per_seq=1)
    ins = inputs.make_inputs(wl)
    batch = ins["batch"]
    rng = np.random.default_rng(12)
    sel = np.full((2, 8), -1, np.int32)
    for t in range(2):
        n = int(batch.q_pos[t]) + 1
        sel[t, [1, 4, 6]] = rng.choice(n, size=3, replace=False)
    res = oracle.forward(batch.kv_offset, batch.kv_len, batch.q_seq, batch.q_pos, ins["q_idx"], ins["k_idx"],
                         ins["w"], ins["q"], ins["kv"], wl.k, wl.sm_scale, selections=sel)
    for t in range(2):
        b = int(batch.q_seq[t])
        off = int(batch.kv_offset[b])
        q = oracle.bf16_decode(ins["q"][t])
        rows = oracle.bf16_decode(ins["kv"][off + sel[t][sel[t] >= 0]])
        mask = np.ones((1, rows.shape[0]), bool)
        ref = _sdpa(q[None], rows, mask, wl.sm_scale)[0]
        assert np.max(np.abs(res["out"][t] - ref)) < 1e-12
