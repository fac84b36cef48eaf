"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against a closed form, an invariant, brute force
on tiny inputs, or a library routine, so that a dropped term, a wrong sign or
index, or a transposed operand in ``oracle/oracle.c`` fails at least one.

Pages: "DeepSeek V3.2 and the lightning indexer", section "How the lightning
indexer works" (indexer = weighted sum of ReLU'd dot products per indexer
head, FP8; fixed top-k per query; MQA mode of MLA); "DeepSeek-V3.2" atlas
entry, "Design overview" (score against every preceding token, k = 2048).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from sparse_attention_08_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(t):
    return t.detach().cpu().numpy()


def _e4m3_to_f64(b):
    return torch.from_numpy(np.ascontiguousarray(b)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def _bf16_to_f64(t):
    return t.to(torch.float64).numpy()


def _bits(t_bf16):
    return _np(t_bf16.contiguous().view(torch.int16)).view(np.uint16)


# --------------------------------------------------------------------------
# Number formats: against torch's own conversions (library routines).
# --------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = _e4m3_to_f64(codes)
    for b in range(256):
        v = oracle.e4m3_decode(b)
        if math.isnan(ref[b]):
            assert math.isnan(v), hex(b)
        else:
            assert v == ref[b], (hex(b), v, ref[b])
    # spot values fixed by the format: 1.0, max normal 448, min subnormal 2^-9
    assert oracle.e4m3_decode(0x38) == 1.0
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0xB8) == -1.0


@pytest.mark.parametrize("where", ["q", "k"])
@pytest.mark.parametrize("code", [0x7F, 0xFF])
def test_indexer_refuses_e4m3_nan_codes(where, code):
    # 0x7F / 0xFF are the format's NaN encodings, not values: every oracle
    # entry that decodes e4m3 reports them as an input error
    wl = W.make_small(H_I=4, d_I=64, H=16, L=40, k=8, integer=True, seed=3)
    q8, k8 = _np(wl.q8).copy(), _np(wl.k8).copy()
    if where == "q":
        q8[7, 2, 5] = code
    else:
        k8[3, 11] = code
    qs, w, ks = _np(wl.q_scale), _np(wl.w), _np(wl.k_scale)
    pos = np.array([39], dtype=np.int64)
    with pytest.raises(ValueError, match="NaN code"):
        oracle.indexer(q8, qs, w, k8, ks)
    with pytest.raises(ValueError, match="NaN code"):
        oracle.indexer_at(q8[-1:] if where == "k" else q8[7:8], qs[:1], w[:1], k8, ks, pos)
    qb, kvb = _bits(wl.q), _bits(wl.kv)
    with pytest.raises(ValueError, match="NaN code"):
        oracle.forward(q8, qs, w, k8, ks, qb, kvb, wl.k, wl.scale)
    with pytest.raises(ValueError, match="NaN code"):
        oracle.forward_at(q8[7:8], qs[:1], w[:1], k8, ks, qb[:1], kvb, np.array([39]), wl.k,
                          wl.scale)


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(4096, generator=g) * 100).to(torch.bfloat16)
    bits = _bits(x)
    ref = x.to(torch.float64).numpy()
    got = np.array([oracle.bf16_decode(int(b)) for b in bits])
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------------
# Indexer.
# --------------------------------------------------------------------------

def test_indexer_integer_inputs_exact_vs_int_brute_force():
    # Integer-valued e4m3 codes with unit scales make every score an exact
    # integer; exact Python-int arithmetic must be matched to the last bit.
    wl = W.make_small(H_I=3, d_I=16, H=2, L=40, k=8, integer=True, seed=11)
    q8, k8 = _np(wl.q8), _np(wl.k8)
    q_int = np.vectorize(brute.int_of_e4m3_code, otypes=[object])(q8)
    k_int = np.vectorize(brute.int_of_e4m3_code, otypes=[object])(k8)
    w_int = _np(wl.w).astype(np.int64).astype(object)
    exact = brute.indexer_int(q_int, w_int, k_int)
    got = oracle.indexer(q8, _np(wl.q_scale), _np(wl.w), k8, _np(wl.k_scale))
    n = wl.T_q
    for i in range(n):
        for s in range(n):
            if s <= i:
                assert got[i, s] == float(exact[i, s]), (i, s)
            else:
                assert math.isnan(got[i, s])


def test_indexer_fold_identity_real_valued():
    # Dequantise-then-dot (oracle) equals the folded form
    # k_scale[s] * sum_j (w*q_scale)[t,j] * ReLU(q8[t,j] . k8[s]) built here from
    # torch's e4m3 decode: positive scales pass through the ReLU.
    wl = W.make_small(H_I=8, d_I=32, H=2, L=50, k=8, seed=12)
    q8, k8 = _np(wl.q8), _np(wl.k8)
    qd = _e4m3_to_f64(q8)
    kd = _e4m3_to_f64(k8)
    raw = np.einsum("tjd,sd->tjs", qd, kd)
    wq = _np(wl.w).astype(np.float64) * _np(wl.q_scale).astype(np.float64)
    folded = np.einsum("tj,tjs->ts", wq, np.maximum(raw, 0.0)) * _np(wl.k_scale).astype(
        np.float64)[None, :]
    got = oracle.indexer(q8, _np(wl.q_scale), _np(wl.w), k8, _np(wl.k_scale))
    mask = np.tril(np.ones((wl.T_q, wl.T_k), dtype=bool))
    denom = np.einsum("tj,tjs->ts", np.abs(wq), np.maximum(raw, 0.0)) * _np(wl.k_scale)[None, :]
    err = np.abs(got[mask] - folded[mask])
    assert np.all(err <= 1e-12 * denom[mask] + 1e-300)


def test_indexer_invariants():
    wl = W.make_small(H_I=4, d_I=16, H=2, L=30, k=8, seed=13)
    q8, k8 = _np(wl.q8), _np(wl.k8).copy()
    qs, w, ks = _np(wl.q_scale), _np(wl.w), _np(wl.k_scale).copy()
    base = oracle.indexer(q8, qs, w, k8, ks)
    mask = np.tril(np.ones(base.shape, dtype=bool))
    # doubling a key's scale doubles its scores exactly (power-of-two scaling)
    ks2 = ks.copy()
    ks2[7] *= 2
    dbl = oracle.indexer(q8, qs, w, k8, ks2)
    assert np.array_equal(dbl[7:, 7], 2 * base[7:, 7])
    assert np.array_equal(np.delete(dbl, 7, axis=1)[np.delete(mask, 7, axis=1)],
                          np.delete(base, 7, axis=1)[np.delete(mask, 7, axis=1)])
    # a zero key scores zero against every query
    k8z = k8.copy()
    k8z[5] = 0
    z = oracle.indexer(q8, qs, w, k8z, ks)
    assert np.all(z[5:, 5] == 0.0)
    # one-hot head weights isolate one ReLU term, which is never negative,
    # and the terms add up to the score
    acc = np.zeros_like(base)
    for j in range(4):
        wj = np.zeros_like(w)
        wj[:, j] = w[:, j]
        one = np.zeros_like(w)
        one[:, j] = 1.0
        term = oracle.indexer(q8, qs, one, k8, ks)
        assert np.all(term[mask] >= 0.0)
        acc += oracle.indexer(q8, qs, wj, k8, ks)
    assert np.allclose(acc[mask], base[mask], rtol=1e-13, atol=1e-300)
    # non-negative weights give non-negative scores
    pos = oracle.indexer(q8, qs, np.abs(w), k8, ks)
    assert np.all(pos[mask] >= 0.0)
    # a negative weight flips the sign of that head's (non-negative) term
    neg = oracle.indexer(q8, qs, -np.abs(w), k8, ks)
    assert np.all(neg[mask] <= 0.0)
    assert np.array_equal(neg[mask], -pos[mask])


# --------------------------------------------------------------------------
# Top-k.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_matches_full_sort_brute_force(seed):
    rng = np.random.default_rng(seed)
    n_q, n_k, k = 37, 60, 9
    # integer scores -> many exact ties; include signed zeros
    scores = rng.integers(-3, 4, size=(n_q, n_k)).astype(np.float64)
    scores[rng.random(scores.shape) < 0.1] = -0.0
    got = oracle.topk(scores, n_q, k)
    for i in range(n_q):
        p = n_k - n_q + i
        assert list(got[i]) == brute.topk_sorted(scores[i], p, k), i


def test_topk_counts_ties_and_zero_signs():
    n_q = n_k = 20
    k = 6
    ties = np.zeros((n_q, n_k))
    got = oracle.topk(ties, n_q, k)
    for i in range(n_q):
        m = min(k, i + 1)                       # O(Lk): min(k, p+1) entries per row
        assert list(got[i][:m]) == list(range(m))
        assert np.all(got[i][m:] == -1)
    # -0.0 and +0.0 are the same value: the lower index wins
    row = np.full((1, 4), -1.0)
    row[0, 1] = -0.0
    row[0, 3] = 0.0
    assert list(oracle.topk(row, 1, 1, rows=None)[0]) == [1]
    row[0, 1], row[0, 3] = 0.0, -0.0
    assert list(oracle.topk(row, 1, 1)[0]) == [1]


def test_topk_selects_largest_real_scores():
    rng = np.random.default_rng(5)
    scores = rng.standard_normal((1, 500))
    got = oracle.topk(scores, 1, 50)[0]
    ref = np.sort(np.argsort(-scores[0], kind="stable")[:50])
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------------
# Attention.
# --------------------------------------------------------------------------

def _sdpa_dense(q_bf16, kv_bf16, n_k, scale, d_v):
    """Dense causal MQA attention in fp64 by torch's SDPA (library routine)."""
    q = q_bf16.to(torch.float64).permute(1, 0, 2)[None]          # [1, H, n_q, d]
    k = kv_bf16.to(torch.float64)[None, None]                    # [1, 1, n_k, d]
    v = kv_bf16[:, :d_v].to(torch.float64)[None, None]
    n_q = q.shape[2]
    H = q.shape[1]
    pos = torch.arange(n_q)[:, None] + (n_k - n_q)
    mask = torch.arange(n_k)[None, :] <= pos
    out = torch.nn.functional.scaled_dot_product_attention(
        q, k.expand(1, H, n_k, -1), v.expand(1, H, n_k, -1), attn_mask=mask, scale=scale)
    return out[0].permute(1, 0, 2).numpy()                       # [n_q, H, d_v]


def test_attention_dense_limit_matches_sdpa():
    # With p+1 <= k every causal key is selected: sparse == dense causal MQA.
    wl = W.make_small(H_I=4, d_I=16, H=4, L=48, k=64, seed=21)
    scores = oracle.indexer(_np(wl.q8), _np(wl.q_scale), _np(wl.w), _np(wl.k8), _np(wl.k_scale))
    idx = oracle.topk(np.nan_to_num(scores, nan=0.0), wl.T_q, wl.k)
    out, lse = oracle.sparse_mla(_bits(wl.q), _bits(wl.kv), idx, wl.T_k, wl.scale, d_v=512)
    ref = _sdpa_dense(wl.q, wl.kv, wl.T_k, wl.scale, 512)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_attention_k_equals_L_is_dense_exactly():
    # k = L: the selection is every causal key, in ascending order, so the
    # result is bitwise that of attention over the explicit causal index list.
    wl = W.make_small(H_I=4, d_I=16, H=3, L=40, k=40, seed=22)
    idx, out, lse = oracle.forward(_np(wl.q8), _np(wl.q_scale), _np(wl.w), _np(wl.k8),
                                   _np(wl.k_scale), _bits(wl.q), _bits(wl.kv), wl.k, wl.scale)
    dense_idx = np.full((wl.T_q, wl.k), -1, dtype=np.int32)
    for i in range(wl.T_q):
        dense_idx[i, : i + 1] = np.arange(i + 1)
    assert np.array_equal(idx, dense_idx)
    out2, lse2 = oracle.sparse_mla(_bits(wl.q), _bits(wl.kv), dense_idx, wl.T_k, wl.scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    ref = _sdpa_dense(wl.q, wl.kv, wl.T_k, wl.scale, 512)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_attention_single_key_and_zero_query():
    wl = W.make_small(H_I=4, d_I=16, H=2, L=30, k=4, seed=23)
    idx = np.full((wl.T_q, 4), -1, dtype=np.int32)
    for i in range(wl.T_q):
        idx[i, 0] = i // 2
    out, _ = oracle.sparse_mla(_bits(wl.q), _bits(wl.kv), idx, wl.T_k, wl.scale)
    kvd = _bf16_to_f64(wl.kv)
    for i in range(wl.T_q):
        assert np.array_equal(out[i, 0], kvd[i // 2, :512])
        assert np.array_equal(out[i, 1], kvd[i // 2, :512])
    # q = 0: uniform softmax, output = mean of the selected values
    qz = torch.zeros_like(wl.q)
    idx2 = np.full((wl.T_q, 4), -1, dtype=np.int32)
    for i in range(wl.T_q):
        sel = sorted({0, i // 2, i})
        idx2[i, : len(sel)] = sel
    out0, lse0 = oracle.sparse_mla(_bits(qz), _bits(wl.kv), idx2, wl.T_k, wl.scale)
    for i in range(wl.T_q):
        sel = [s for s in idx2[i] if s >= 0]
        assert np.allclose(out0[i, 0], kvd[sel, :512].mean(axis=0), rtol=0, atol=1e-15)
        assert abs(lse0[i, 0] - math.log(len(sel))) < 1e-15


def test_attention_matches_explicit_loops_and_skips_invalid():
    wl = W.make_small(H_I=4, d_I=16, H=2, L=25, k=7, seed=24, q_div=2.0)
    rng = np.random.default_rng(3)
    idx = np.full((wl.T_q, 7), -1, dtype=np.int32)
    for i in range(wl.T_q):
        m = min(7, i + 1)
        idx[i, :m] = np.sort(rng.choice(i + 1, size=m, replace=False))
    idx[3, 1] = 24          # beyond p = 3: skipped
    out, lse = oracle.sparse_mla(_bits(wl.q), _bits(wl.kv), idx, wl.T_k, wl.scale)
    qd, kvd = _bf16_to_f64(wl.q), _bf16_to_f64(wl.kv)
    for i in range(wl.T_q):
        sel = [int(s) for s in idx[i] if 0 <= s <= i]
        ro, rl = brute.attention_loops(qd[i], kvd, sel, wl.scale, 512)
        assert np.max(np.abs(out[i] - ro)) < 1e-13
        assert np.max(np.abs(lse[i] - rl)) < 1e-13


def test_forward_is_the_composition():
    wl = W.make_small(H_I=4, d_I=16, H=2, lens=[30, 45], lens_q=[30, 20], k=8, seed=25)
    # second sequence is a chunk: 20 queries at positions 25..44
    b = 1
    q0, q1 = int(wl.cu_q[b]), int(wl.cu_q[b + 1])
    k0, k1 = int(wl.cu_k[b]), int(wl.cu_k[b + 1])
    args = [_np(wl.q8[q0:q1]), _np(wl.q_scale[q0:q1]), _np(wl.w[q0:q1]), _np(wl.k8[k0:k1]),
            _np(wl.k_scale[k0:k1])]
    rows = np.array([0, 3, 19], dtype=np.int64)
    idx, out, lse = oracle.forward(*args, _bits(wl.q[q0:q1]), _bits(wl.kv[k0:k1]), wl.k,
                                   wl.scale, rows=rows)
    sc = oracle.indexer(*args, rows=rows)
    assert np.all(np.isnan(sc[0, 26:])) and not np.any(np.isnan(sc[0, :26]))
    idx2 = oracle.topk(np.nan_to_num(sc, nan=0.0), q1 - q0, wl.k, rows=rows)
    out2, lse2 = oracle.sparse_mla(_bits(wl.q[q0:q1]), _bits(wl.kv[k0:k1]), idx2, k1 - k0,
                                   wl.scale, rows=rows)
    assert np.array_equal(idx, idx2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


# --------------------------------------------------------------------------
# Golden fixtures from the pages.
# --------------------------------------------------------------------------

def test_golden_sparse_budget():
    with open(os.path.join(GOLDEN, "sparse_budget.json")) as f:
        g = json.load(f)
    # "488x" at a 1M-token context with k = 2048: full L*L versus L*k work.
    L, k = g["reduction"]["L"], g["reduction"]["k"]
    assert round((L * L) / (L * k)) == g["reduction"]["ratio_rounded"]
    # every row keeps min(k, p+1) entries: count them with the oracle on a
    # small case and compare with the closed form stored beside it
    c = g["row_counts"]
    wl = W.make_small(H_I=2, d_I=16, H=1, L=c["L"], k=c["k"], seed=31)
    sc = oracle.indexer(_np(wl.q8), _np(wl.q_scale), _np(wl.w), _np(wl.k8), _np(wl.k_scale))
    idx = oracle.topk(np.nan_to_num(sc, nan=0.0), wl.T_q, wl.k)
    assert int((idx >= 0).sum()) == c["attended_pairs"]
    # closed forms for the headline shapes
    for row in g["configs"]:
        L, k = row["L"], row["k"]
        assert k * (k + 1) // 2 + (L - k) * k == row["attended_pairs"]
        assert L * (L + 1) // 2 == row["causal_pairs"]


def test_position_explicit_entries_match_row_entries():
    # the *_at entry points evaluate rows at given positions; on rows of a
    # whole sequence they must reproduce the row-indexed entry points bitwise
    wl = W.make_small(H_I=4, d_I=16, H=2, L=60, k=8, seed=32)
    rows = np.array([0, 7, 31, 59], dtype=np.int64)
    q8, qs, w = _np(wl.q8), _np(wl.q_scale), _np(wl.w)
    k8, ks = _np(wl.k8), _np(wl.k_scale)
    qb, kvb = _bits(wl.q), _bits(wl.kv)
    sc = oracle.indexer(q8, qs, w, k8, ks, rows=rows)
    sc_at = oracle.indexer_at(q8[rows], qs[rows], w[rows], k8, ks, rows)
    assert np.array_equal(np.isnan(sc), np.isnan(sc_at))
    assert np.array_equal(np.nan_to_num(sc), np.nan_to_num(sc_at))
    idx, out, lse = oracle.forward(q8, qs, w, k8, ks, qb, kvb, 8, wl.scale, rows=rows)
    i2, o2, l2 = oracle.forward_at(q8[rows], qs[rows], w[rows], k8, ks, qb[rows], kvb, rows, 8,
                                   wl.scale)
    assert np.array_equal(idx, i2) and np.array_equal(out, o2) and np.array_equal(lse, l2)
    o3, l3 = oracle.sparse_mla_at(qb[rows], kvb, idx, rows, wl.scale)
    assert np.array_equal(out, o3) and np.array_equal(lse, l3)


# --------------------------------------------------------------------------
# Indexer training signal: KL(head-averaged attention || softmax of the
# indexer scores) over the selection ("DeepSeek V3.2 and the lightning
# indexer", "Teaching a dense model to be sparse"; "DeepSeek-V3.2" atlas
# entry, "Design overview").
# --------------------------------------------------------------------------

def _kl_case(R=4, H=4, n_k=60, k=24, seed=11, q_div=24.0, holes=True):
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = (torch.randn(R, H, 576, generator=g) / q_div).to(torch.bfloat16)
    kv = torch.randn(n_k, 576, generator=g).to(torch.bfloat16)
    pos = np.arange(n_k - R, n_k, dtype=np.int64)
    idx = np.full((R, k), -1, dtype=np.int32)
    for r in range(R):
        sel = np.sort(rng.choice(int(pos[r]) + 1, size=min(k, int(pos[r]) + 1), replace=False))
        idx[r, :len(sel)] = sel
    if holes:
        idx[0, 3] = -1                       # a hole inside the prefix
        idx[1, 5] = int(pos[1]) + 7          # beyond p: not a valid entry
    logits = rng.standard_normal((R, n_k)).astype(np.float32) * 2.0
    return q, kv, idx, pos, logits


def _valid(idx, pos):
    return (idx >= 0) & (idx <= pos[:, None])


def test_kl_distributions_normalised_and_gradient_sums_to_zero():
    q, kv, idx, pos, logits = _kl_case()
    kl, grad, target = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, logits, 1 / 24)
    v = _valid(idx, pos)
    assert np.allclose(target.sum(1), 1.0, atol=1e-12)      # p sums to 1 over S
    assert np.allclose(grad.sum(1), 0.0, atol=1e-12)        # sum(q) - sum(p) = 0
    assert np.all(target[~v] == 0) and np.all(grad[~v] == 0)
    assert np.all(kl >= -1e-15)                             # Gibbs' inequality


def test_kl_vanishes_when_the_indexer_matches_the_target():
    q, kv, idx, pos, logits = _kl_case()
    _, _, target = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, logits, 1 / 24)
    # indexer scores = log of the target plus a per-row constant
    lg = np.full_like(logits, -50.0)
    for r in range(len(pos)):
        for j in range(idx.shape[1]):
            if target[r, j] > 0:
                lg[r, idx[r, j]] = np.log(target[r, j]) + 3.0 * r
    kl, grad, _ = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, lg.astype(np.float32),
                                       1 / 24)
    # float32 rounding of the scores only
    assert np.all(np.abs(kl) < 1e-12) and np.abs(grad).max() < 1e-6


def test_kl_two_keys_closed_form():
    # a zero query: every head's attention is uniform over the two keys, so
    # p = (1/2, 1/2); scores (a, 0) give q = (sigma(a), 1 - sigma(a))
    n_k, a = 5, 1.7
    q = torch.zeros(1, 3, 576).to(torch.bfloat16)
    kv = torch.randn(n_k, 576, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    idx = np.array([[1, 3, -1, -1]], dtype=np.int32)
    pos = np.array([4], dtype=np.int64)
    logits = np.zeros((1, n_k), dtype=np.float32)
    logits[0, 1] = a
    kl, grad, target = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, logits, 1 / 24)
    s = 1.0 / (1.0 + math.exp(-float(np.float32(a))))
    want = 0.5 * math.log(0.5 / s) + 0.5 * math.log(0.5 / (1.0 - s))
    assert abs(kl[0] - want) < 1e-14
    assert np.allclose(target[0], [0.5, 0.5, 0, 0], atol=1e-15)
    assert np.allclose(grad[0], [s - 0.5, 0.5 - s, 0, 0], atol=1e-15)


def test_kl_gradient_matches_finite_differences():
    q, kv, idx, pos, logits = _kl_case(R=2, seed=12)
    kl, grad, _ = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, logits, 1 / 24)
    eps = 1e-3                       # representable steps of the float32 scores
    for r, j in [(0, 0), (0, 7), (1, 2), (1, 11)]:
        s = idx[r, j]
        if s < 0 or s > pos[r]:
            continue
        up, dn = logits.copy(), logits.copy()
        up[r, s] += eps
        dn[r, s] -= eps
        d = (up[r, s] - dn[r, s]).astype(np.float64)
        kl_up, _, _ = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, up, 1 / 24)
        kl_dn, _, _ = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, dn, 1 / 24)
        fd = (kl_up[r] - kl_dn[r]) / d
        assert abs(fd - grad[r, j]) < 1e-6, (r, j, fd, grad[r, j])


def test_kl_target_is_the_mean_of_the_single_head_targets_and_matches_attention():
    q, kv, idx, pos, logits = _kl_case(R=3, H=5, seed=13, q_div=2.0)
    _, _, target = oracle.indexer_kl_at(_bits(q), _bits(kv), idx, pos, logits, 1 / 24)
    heads = [oracle.indexer_kl_at(_bits(q[:, h:h + 1]), _bits(kv), idx, pos, logits, 1 / 24)[2]
             for h in range(q.shape[1])]
    assert np.allclose(target, np.mean(heads, axis=0), atol=1e-14)
    # a single head's target weights the values like that head's attention
    out, _ = oracle.sparse_mla_at(_bits(q[:, :1]), _bits(kv), idx, pos, 1 / 24)
    vals = kv.to(torch.float64).numpy()[:, :512]
    for r in range(len(pos)):
        mix = sum(heads[0][r, j] * vals[idx[r, j]] for j in range(idx.shape[1])
                  if heads[0][r, j] > 0)
        assert np.allclose(mix, out[r, 0], atol=1e-12)


# ---------------------------------------------------------------------------
# Masked MHA mode ("DeepSeek-V3.2" atlas entry, "Design overview" and
# "Inference efficiency": short prompts are prefilled with a masked MHA
# standing in for DSA).  Reading: dense per-head
# attention restricted to the selected set.

def _mha_case(n=40, H=3, d_qk=24, d_v=8, seed=5):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(n, H, d_qk, generator=g) / 3).to(torch.bfloat16)
    k = torch.randn(n, H, d_qk, generator=g).to(torch.bfloat16)
    v = torch.randn(n, H, d_v, generator=g).to(torch.bfloat16)
    return q, k, v


def test_masked_mha_all_causal_keys_selected_is_causal_sdpa():
    """Every earlier key selected (p + 1 <= topk): the masked mode is plain
    causal multi-head attention, which torch computes in fp64."""
    n, H, scale = 40, 3, 0.3
    q, k, v = _mha_case(n, H)
    topk = 48
    rng = np.random.default_rng(1)
    idx = np.full((n, topk), -1, dtype=np.int32)
    for t in range(n):
        sel = rng.permutation(t + 1)
        idx[t, :t + 1] = sel
    out, lse = oracle.masked_mha_at(_bits(q), _bits(k), _bits(v), idx, np.arange(n), scale)
    qd, kd, vd = (x.to(torch.float64).transpose(0, 1) for x in (q, k, v))   # [H, n, d]
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=scale)
    np.testing.assert_allclose(out, ref.transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)
    sc = scale * qd @ kd.transpose(1, 2)
    sc = sc.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(sc, dim=-1).transpose(0, 1).numpy(), rtol=1e-12,
                               atol=1e-12)


def test_masked_mha_matches_explicit_loops_with_repeats_and_invalid_entries():
    n, H = 30, 2
    q, k, v = _mha_case(n, H, d_qk=16, d_v=8, seed=9)
    rng = np.random.default_rng(3)
    topk = 12
    idx = rng.integers(-3, n + 3, size=(n, topk)).astype(np.int32)
    idx[:, 5] = idx[:, 4]                                   # a repeated entry counts once
    idx[7, :] = -1                                          # an empty selection
    pos = np.arange(n)
    out, lse = oracle.masked_mha_at(_bits(q), _bits(k), _bits(v), idx, pos, 0.25)
    qf, kf, vf = (x.to(torch.float64).numpy() for x in (q, k, v))
    for t in range(n):
        o_ref, l_ref = brute.masked_mha_loops(qf[t], kf, vf, idx[t], t, 0.25)
        np.testing.assert_allclose(out[t], o_ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[t], l_ref, rtol=1e-12)
    assert np.all(out[7] == 0) and np.all(np.isneginf(lse[7]))


def test_masked_mha_ignores_keys_outside_the_selection():
    """A key that is not selected may carry any score: the result does not move."""
    n, H = 24, 2
    q, k, v = _mha_case(n, H, d_qk=16, d_v=8, seed=4)
    idx = np.array([[s for s in range(0, t + 1, 2)] + [-1] * (12 - len(range(0, t + 1, 2)))
                    for t in range(n)], dtype=np.int32)
    a = oracle.masked_mha_at(_bits(q), _bits(k), _bits(v), idx, np.arange(n), 0.5)
    k2 = k.clone()
    k2[1::2] = (q[1::2] * 40).to(torch.bfloat16)           # odd keys: huge, unselected
    b = oracle.masked_mha_at(_bits(q), _bits(k2), _bits(v), idx, np.arange(n), 0.5)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_masked_mha_is_the_mqa_mode_after_absorption():
    """The MHA and MQA forms of MLA give the same attention: with per-head keys
    k_h = [W_UK_h^T c_nope ; c_rope], values v_h = W_UV_h^T c_nope and the
    absorbed query q_abs = [W_UK_h q_nope ; q_rope], the MHA output of head h
    is W_UV_h^T applied to the MQA output over the latents.  The projections
    are signed selections of latent dims, so every product is exact in bf16
    and the identity holds to fp64 rounding."""
    rng = np.random.default_rng(7)
    n_k, H, dn, dr, dl = 50, 3, 16, 8, 64           # nope, rope, latent dims (latent > heads' dims)
    R, topk, scale = 6, 20, 0.2
    g = torch.Generator().manual_seed(2)
    c = torch.randn(n_k, dl + dr, generator=g).to(torch.bfloat16)            # [c_nope ; c_rope]
    q_nope = (torch.randn(R, H, dn, generator=g) / 2).to(torch.bfloat16)
    q_rope = (torch.randn(R, H, dr, generator=g) / 2).to(torch.bfloat16)
    k_h = torch.zeros(n_k, H, dn + dr, dtype=torch.bfloat16)
    v_h = torch.zeros(n_k, H, dn, dtype=torch.bfloat16)
    q_abs = torch.zeros(R, H, dl + dr, dtype=torch.bfloat16)
    w_uv = np.zeros((H, dn, dl))                     # W_UV_h^T as a matrix: v_h = w_uv[h] @ c_nope
    for h in range(H):
        uk = rng.permutation(dl)[:dn]
        sk = rng.choice([-1.0, 1.0], size=dn)
        uv = rng.permutation(dl)[:dn]
        sv = rng.choice([-1.0, 1.0], size=dn)
        for j in range(dn):
            k_h[:, h, j] = c[:, uk[j]] * sk[j]
            q_abs[:, h, uk[j]] = q_nope[:, h, j] * sk[j]
            v_h[:, h, j] = c[:, uv[j]] * sv[j]
            w_uv[h, j, uv[j]] = sv[j]
        k_h[:, h, dn:] = c[:, dl:]
        q_abs[:, h, dl:] = q_rope[:, h]
    q_mha = torch.cat([q_nope, q_rope], dim=2)
    pos = np.array([49, 30, 12, 40, 5, 25])
    idx = np.full((R, topk), -1, dtype=np.int32)
    for r, p in enumerate(pos):
        sel = np.sort(rng.permutation(p + 1)[:min(topk, p + 1)])
        idx[r, :len(sel)] = sel
    out_mha, lse_mha = oracle.masked_mha_at(_bits(q_mha), _bits(k_h), _bits(v_h), idx, pos, scale)
    out_mqa, lse_mqa = oracle.sparse_mla_at(_bits(q_abs), _bits(c), idx, pos, scale, d_v=dl)
    np.testing.assert_allclose(lse_mha, lse_mqa, rtol=1e-12, atol=1e-12)
    for h in range(H):
        np.testing.assert_allclose(out_mha[:, h], out_mqa[:, h] @ w_uv[h].T, rtol=1e-11, atol=1e-12)


def test_masked_mha_inputs_follow_the_recipe():
    """The masked-MHA workload's selection: per query at p, min(topk, p+1)
    distinct keys of [0, p], ascending, then -1; every key when p+1 <= topk."""
    m = W.make_mha([300, 200], [300, 40], H=2, topk=64, seed=11)
    idx = m.idx.numpy()
    row = 0
    for lq, lk in zip(m.lens_q, m.lens_k):
        for i in range(lq):
            p = lk - lq + i
            sel = idx[row + i]
            n = min(m.topk, p + 1)
            assert np.all(sel[n:] == -1)
            s = sel[:n]
            assert np.all(s >= 0) and np.all(s <= p) and np.all(np.diff(s) > 0)
            if p + 1 <= m.topk:
                assert np.array_equal(s, np.arange(p + 1))
        row += lq
    assert m.q.shape == (340, 2, 192) and m.k.shape == (500, 2, 192) and m.v.shape == (500, 2, 128)
    assert abs(m.scale - 192 ** -0.5) < 1e-12


# ---------------------------------------------------------------------------
# The indexer's backward ("DeepSeek V3.2 and the lightning indexer",
# "Teaching a dense model to be sparse": the warm-up trains the indexer alone
# on the KL signal).

def _backward_case(n_q=6, n_k=11, H=4, d=8, seed=21):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(n_q, H, d))
    w = rng.normal(size=(n_q, H))
    k = rng.normal(size=(n_k, d))
    pos = np.sort(rng.choice(np.arange(n_k), size=n_q, replace=False))
    g = rng.normal(size=(n_q, n_k))
    return q, w, k, g, pos


def test_indexer_backward_matches_torch_autograd():
    """torch's autograd differentiates the score sum_t,s g[t,s] * I[t,s]; its
    gradients are the backward for upstream g (ReLU'(0) = 0 in both)."""
    q, w, k, g, pos = _backward_case()
    dq, dw, dk = oracle.indexer_backward(q, w, k, g, pos)
    qt = torch.tensor(q, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    dots = torch.einsum("thd,sd->ths", qt, kt)
    scores = torch.einsum("th,ths->ts", wt, torch.relu(dots))
    causal = torch.arange(k.shape[0])[None, :] <= torch.tensor(pos)[:, None]
    (scores * torch.tensor(g) * causal).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_indexer_backward_of_the_kl_loss_matches_finite_differences():
    """Chained with the pinned KL oracle: the KL gradient with respect to the
    scores, pushed through the backward, is the derivative of the KL loss with
    respect to the indexer weights w (central differences; the loss recomputes
    the scores from the perturbed weights)."""
    q_t, kv_t, idx, pos_kl, _ = _kl_case(R=3, H=2, n_k=40, k=16, seed=5)
    q_kl, kv_kl = _bits(q_t), _bits(kv_t)
    R, n_k = idx.shape[0], 40
    rng = np.random.default_rng(9)
    H_I, d_I = 3, 6
    qi = rng.normal(size=(R, H_I, d_I))
    ki = rng.normal(size=(n_k, d_I))
    wi = rng.normal(size=(R, H_I))

    def scores(wv):
        return np.einsum("tj,tjs->ts", wv, np.maximum(np.einsum("tjd,sd->tjs", qi, ki), 0.0))

    def loss(wv):
        kl, _, _ = oracle.indexer_kl_at(q_kl, kv_kl, idx, pos_kl,
                                        scores(wv).astype(np.float32).astype(np.float64), 0.2)
        return kl.sum()

    # scores passed through float32 for the KL oracle's interface: use exactly
    # representable weights so the rounding does not move them
    wi = np.round(wi * 64) / 64
    qi = np.round(qi * 16) / 16
    ki = np.round(ki * 16) / 16
    lg = scores(wi).astype(np.float32)
    kl, grad, _ = oracle.indexer_kl_at(q_kl, kv_kl, idx, pos_kl, lg, 0.2)
    g = np.zeros((R, n_k))
    for r in range(R):
        for j, s in enumerate(idx[r]):
            if 0 <= s <= pos_kl[r]:
                g[r, s] += grad[r, j]
    _, dw, _ = oracle.indexer_backward(qi, wi, ki, g, pos_kl)
    h = 2.0 ** -10
    for t in range(R):
        for j in range(H_I):
            wp, wm = wi.copy(), wi.copy()
            wp[t, j] += h
            wm[t, j] -= h
            fd = (loss(wp) - loss(wm)) / (2 * h)
            assert abs(fd - dw[t, j]) <= 2e-3 * max(1.0, abs(dw[t, j])), (t, j, fd, dw[t, j])


def test_indexer_backward_relu_gates_and_causality():
    q, w, k, g, pos = _backward_case(seed=3)
    # a key that every head scores negatively carries no gradient, and
    # removing it changes nothing else
    q[..., 0] = np.abs(q[..., 0]) + 0.1
    k[0] = 0.0
    k[0, 0] = -1.0
    dq, dw, dk = oracle.indexer_backward(q, w, k, g, pos)
    assert np.all(dk[0] == 0)
    g0 = g.copy()
    g0[:, 0] = 0.0
    a = oracle.indexer_backward(q, w, k, g0, pos)
    for x, y in zip((dq, dw, dk), a):
        np.testing.assert_array_equal(x, y)
    # entries of g past a row's position are ignored
    g2 = g.copy()
    for t, p in enumerate(pos):
        g2[t, p + 1:] = 123.0
    b = oracle.indexer_backward(q, w, k, g2, pos)
    for x, y in zip((dq, dw, dk), b):
        np.testing.assert_array_equal(x, y)
