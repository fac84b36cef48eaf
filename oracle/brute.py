"""Brute-force versions of the DSA stages for TINY inputs -- TEST INFRASTRUCTURE.

These exist to pin ``oracle.c`` to something other than itself.  Each one
reaches the same result by a different route:

* ``indexer_int``: exact integer arithmetic (Python ints) for inputs whose FP8
  codes hold integers and whose scales are 1 -- the score is then an exact
  integer, so the fp64 oracle must hit it exactly.
* ``topk_sorted``: Python's ``sorted`` over (-score, index) pairs.
* ``attention_loops``: explicit softmax with ``math.exp`` over Python floats.

Pages: "DeepSeek V3.2 and the lightning indexer", section "How the lightning
indexer works" (ReLU-weighted indexer score, per-query top-k, MQA mode);
"DeepSeek-V3.2" atlas entry, "Design overview".
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

def int_of_e4m3_code(b: int) -> int:
    """Integer held by an e4m3 byte (sign, 4-bit exponent with bias 7, 3-bit
    mantissa), computed with exact fractions; fails if it is not an integer."""
    b = int(b)
    sign = -1 if b & 0x80 else 1
    e = (b >> 3) & 15
    m = b & 7
    if e == 0:
        val = Fraction(m, 8) * Fraction(2) ** (1 - 7)
    else:
        val = Fraction(8 + m, 8) * Fraction(2) ** (e - 7)
    assert val.denominator == 1, f"code {b:#x} is not an integer"
    return sign * int(val)


def indexer_int(q_int, w_int, k_int):
    """Exact integer indexer: q_int [n_q, H_I, d_I], w_int [n_q, H_I],
    k_int [n_k, d_I] (Python-int valued).  Returns an object array
    [n_q, n_k] of Python ints, None where s > p (p = n_k - n_q + i)."""
    n_q, H_I, d_I = q_int.shape
    n_k = k_int.shape[0]
    out = np.empty((n_q, n_k), dtype=object)
    for i in range(n_q):
        p = n_k - n_q + i
        for s in range(n_k):
            if s > p:
                out[i, s] = None
                continue
            total = 0
            for j in range(H_I):
                dot = sum(int(q_int[i, j, d]) * int(k_int[s, d]) for d in range(d_I))
                total += int(w_int[i, j]) * max(dot, 0)
            out[i, s] = total
    return out


def topk_sorted(scores_row, p: int, k: int):
    """Full sort of candidates 0..p by (score desc, index asc); the best
    min(k, p+1) in ascending index order, padded with -1."""
    cand = [(-(float(scores_row[s]) + 0.0), s) for s in range(p + 1)]  # +0.0 folds -0 into +0
    best = sorted(cand)[: min(k, p + 1)]
    sel = sorted(s for _, s in best)
    return sel + [-1] * (k - len(sel))


def attention_loops(q_row, kv, sel, scale, d_v):
    """q_row: float64 [H, d_qk]; kv: float64 [n_k, d_qk]; sel: list of key
    indices.  Returns (out [H, d_v], lse [H]) with explicit loops."""
    H = q_row.shape[0]
    out = np.zeros((H, d_v))
    lse = np.zeros(H)
    for h in range(H):
        xs = [scale * float(np.dot(q_row[h], kv[s])) for s in sel]
        m = max(xs)
        es = [math.exp(x - m) for x in xs]
        z = math.fsum(es)
        for e, s in zip(es, sel):
            out[h] += (e / z) * kv[s, :d_v]
        lse[h] = m + math.log(z)
    return out, lse


def masked_mha_loops(q_row, k, v, entries, p, scale):
    """Masked MHA mode by explicit loops: q_row float64 [H, d_qk], k float64
    [n_k, H, d_qk], v float64 [n_k, H, d_v]; entries is the raw index row.
    The selected set is built with a Python set (valid entries 0 <= s <= p,
    repeats once); each head takes a softmax over it with math.exp.  Returns
    (out [H, d_v], lse [H]); an empty set gives zeros and -inf."""
    sel = sorted({int(s) for s in entries if 0 <= int(s) <= p})
    H, d_v = q_row.shape[0], v.shape[2]
    out = np.zeros((H, d_v))
    lse = np.full(H, -math.inf)
    if not sel:
        return out, lse
    for h in range(H):
        xs = [scale * math.fsum(float(a) * float(b) for a, b in zip(q_row[h], k[s, h])) for s in sel]
        m = max(xs)
        es = [math.exp(x - m) for x in xs]
        z = math.fsum(es)
        for e, s in zip(es, sel):
            out[h] += (e / z) * v[s, h]
        lse[h] = m + math.log(z)
    return out, lse
