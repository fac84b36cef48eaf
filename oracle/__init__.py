"""fp64 CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.

``oracle.c`` holds the definitions (compiled to ``liboracle.so`` with gcc);
this module marshals numpy arrays into it.  ``brute.py`` holds independent
tiny-input brute-force versions used to pin ``oracle.c``.

Every function follows the plain definition of its stage, as the pages state
it ("DeepSeek V3.2 and the lightning indexer", section "How the lightning
indexer works"; "DeepSeek-V3.2" atlas entry, "Design overview"):

* indexer  I[t,s] = sum_j w[t,j] * ReLU(qhat[t,j] . khat[s])  for s <= p
* top-k    the min(k, p+1) best scores, ties to the lower index, ascending
* attention softmax over the selected latents, shared by all query heads
* indexer backward  the gradients in q_I, w and k_I of a gradient on the
  scores (the warm-up trains the indexer alone)
* masked MHA  dense per-head attention restricted to the selected set (the
  short-prefill mode the "DeepSeek-V3.2" atlas entry names in "Design overview")
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_bf16_decode.restype = ctypes.c_double
        lib.oracle_bf16_decode.argtypes = [ctypes.c_uint16]
        lib.oracle_indexer.restype = i32
        lib.oracle_indexer.argtypes = [P, P, P, P, P, i64, i64, i32, i32, P, i64, P, i64]
        lib.oracle_topk.restype = i32
        lib.oracle_topk.argtypes = [P, i64, i64, i64, P, i64, i32, P]
        lib.oracle_sparse_mla.restype = i32
        lib.oracle_sparse_mla.argtypes = [P, P, P, i64, i64, i32, i32, i32, i32, ctypes.c_double,
                                          P, i64, P, P]
        lib.oracle_forward.restype = i32
        lib.oracle_forward.argtypes = [P, P, P, P, P, P, P, i64, i64, i32, i32, i32, i32, i32, i32,
                                       ctypes.c_double, P, i64, P, P, P]
        lib.oracle_forward_at.restype = i32
        lib.oracle_forward_at.argtypes = [P, P, P, P, P, P, P, P, i64, i64, i32, i32, i32, i32, i32,
                                          i32, ctypes.c_double, P, P, P]
        lib.oracle_indexer_at.restype = i32
        lib.oracle_indexer_at.argtypes = [P, P, P, P, P, P, i64, i64, i32, i32, P, i64]
        lib.oracle_sparse_mla_at.restype = i32
        lib.oracle_sparse_mla_at.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, i32,
                                             ctypes.c_double, P, P]
        lib.oracle_num_threads.restype = i32
        lib.oracle_indexer_kl_at.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, i32,
                                             ctypes.c_double, P, P, P]
        lib.oracle_indexer_kl_at.restype = i32
        lib.oracle_indexer_backward.restype = i32
        lib.oracle_indexer_backward.argtypes = [P, P, P, P, P, i64, i64, i32, i32, P, P, P]
        lib.oracle_masked_mha_at.restype = i32
        lib.oracle_masked_mha_at.argtypes = [P, P, P, P, P, i64, i64, i32, i32, i32, i32,
                                             ctypes.c_double, P, P]
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _rows(rows, n_q):
    if rows is None:
        return np.arange(n_q, dtype=np.int64)
    return _c(rows, np.int64)


def _check(rc: int, name: str) -> None:
    if rc == -2:
        raise ValueError(f"{name}: an e4m3 input holds a NaN code (0x7F or 0xFF)")
    if rc != 0:
        raise ValueError(f"{name}: bad arguments")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def e4m3_decode(b: int) -> float:
    return float(_load().oracle_e4m3_decode(int(b) & 0xFF))


def bf16_decode(h: int) -> float:
    return float(_load().oracle_bf16_decode(int(h) & 0xFFFF))


def indexer(q8, q_scale, w, k8, k_scale, rows=None) -> np.ndarray:
    """Indexer scores for one sequence.

    q8: uint8 [n_q, H_I, d_I] (e4m3 bytes); q_scale, w: float32 [n_q, H_I];
    k8: uint8 [n_k, d_I]; k_scale: float32 [n_k].  Returns float64
    [len(rows), n_k], NaN where s > p (p = n_k - n_q + i).
    """
    q8 = _c(q8, np.uint8)
    k8 = _c(k8, np.uint8)
    n_q, H_I, d_I = q8.shape
    n_k = k8.shape[0]
    rows = _rows(rows, n_q)
    out = np.full((len(rows), n_k), np.nan, dtype=np.float64)
    rc = _load().oracle_indexer(_ptr(q8), _ptr(_c(q_scale, np.float32)), _ptr(_c(w, np.float32)),
                                _ptr(k8), _ptr(_c(k_scale, np.float32)), n_q, n_k, H_I, d_I,
                                _ptr(rows), len(rows), _ptr(out), n_k)
    _check(rc, "oracle_indexer")
    return out


def topk(scores, n_q, k, rows=None) -> np.ndarray:
    """Top-k for one sequence: scores float64 [len(rows), n_k] (candidates of
    row r at 0..p_r).  Returns int32 [len(rows), k], ascending, -1 padded."""
    scores = _c(scores, np.float64)
    n_k = scores.shape[1]
    rows = _rows(rows, n_q)
    assert scores.shape[0] == len(rows)
    idx = np.empty((len(rows), k), dtype=np.int32)
    rc = _load().oracle_topk(_ptr(scores), n_k, n_q, n_k, _ptr(rows), len(rows), k, _ptr(idx))
    if rc != 0:
        raise ValueError("oracle_topk: bad arguments")
    return idx


def sparse_mla(q_bits, kv_bits, idx, n_k, scale, d_v=512, rows=None):
    """Sparse MQA-mode attention for one sequence.

    q_bits: uint16 [n_q, H, d_qk] (bf16 bit patterns); kv_bits: uint16
    [n_k, d_qk]; idx: int32 [len(rows), k].  Returns (out float64
    [len(rows), H, d_v], lse float64 [len(rows), H]).
    """
    q_bits = _c(q_bits, np.uint16)
    kv_bits = _c(kv_bits, np.uint16)
    idx = _c(idx, np.int32)
    n_q, H, d_qk = q_bits.shape
    assert kv_bits.shape == (n_k, d_qk)
    rows = _rows(rows, n_q)
    k = idx.shape[1]
    out = np.empty((len(rows), H, d_v), dtype=np.float64)
    lse = np.empty((len(rows), H), dtype=np.float64)
    rc = _load().oracle_sparse_mla(_ptr(q_bits), _ptr(kv_bits), _ptr(idx), n_q, n_k, H, d_qk, d_v,
                                   k, float(scale), _ptr(rows), len(rows), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_sparse_mla: bad arguments")
    return out, lse


def forward(q8, q_scale, w, k8, k_scale, q_bits, kv_bits, k, scale, d_v=512, rows=None):
    """indexer -> top-k -> sparse attention for the listed rows of one
    sequence.  Returns (idx int32 [R, k], out float64 [R, H, d_v], lse [R, H])."""
    q8 = _c(q8, np.uint8)
    k8 = _c(k8, np.uint8)
    q_bits = _c(q_bits, np.uint16)
    kv_bits = _c(kv_bits, np.uint16)
    n_q, H_I, d_I = q8.shape
    n_k = k8.shape[0]
    _, H, d_qk = q_bits.shape
    rows = _rows(rows, n_q)
    R = len(rows)
    idx = np.empty((R, k), dtype=np.int32)
    out = np.empty((R, H, d_v), dtype=np.float64)
    lse = np.empty((R, H), dtype=np.float64)
    rc = _load().oracle_forward(_ptr(q8), _ptr(_c(q_scale, np.float32)), _ptr(_c(w, np.float32)),
                                _ptr(k8), _ptr(_c(k_scale, np.float32)), _ptr(q_bits),
                                _ptr(kv_bits), n_q, n_k, H_I, d_I, H, d_qk, d_v, k, float(scale),
                                _ptr(rows), R, _ptr(idx), _ptr(out), _ptr(lse))
    _check(rc, "oracle_forward")
    return idx, out, lse


def forward_at(q8, q_scale, w, k8, k_scale, q_bits, kv_bits, pos, k, scale, d_v=512):
    """The whole path for query rows given with their positions: row r of the
    query-side arrays sits at position pos[r] of the sequence whose keys are
    k8 / k_scale / kv_bits.  Returns (idx [R, k], out [R, H, d_v], lse [R, H])."""
    q8 = _c(q8, np.uint8)
    k8 = _c(k8, np.uint8)
    q_bits = _c(q_bits, np.uint16)
    kv_bits = _c(kv_bits, np.uint16)
    pos = _c(pos, np.int64)
    R, H_I, d_I = q8.shape
    n_k = k8.shape[0]
    _, H, d_qk = q_bits.shape
    idx = np.empty((R, k), dtype=np.int32)
    out = np.empty((R, H, d_v), dtype=np.float64)
    lse = np.empty((R, H), dtype=np.float64)
    rc = _load().oracle_forward_at(_ptr(q8), _ptr(_c(q_scale, np.float32)), _ptr(_c(w, np.float32)),
                                   _ptr(k8), _ptr(_c(k_scale, np.float32)), _ptr(q_bits),
                                   _ptr(kv_bits), _ptr(pos), R, n_k, H_I, d_I, H, d_qk, d_v, k,
                                   float(scale), _ptr(idx), _ptr(out), _ptr(lse))
    _check(rc, "oracle_forward_at")
    return idx, out, lse


def indexer_at(q8, q_scale, w, k8, k_scale, pos):
    """Indexer scores of query rows at explicit positions: row r of q8 /
    q_scale / w sits at position pos[r].  Returns float64 [R, n_k], NaN where
    s > pos[r]."""
    q8 = _c(q8, np.uint8)
    k8 = _c(k8, np.uint8)
    pos = _c(pos, np.int64)
    R, H_I, d_I = q8.shape
    n_k = k8.shape[0]
    out = np.full((R, n_k), np.nan, dtype=np.float64)
    rc = _load().oracle_indexer_at(_ptr(q8), _ptr(_c(q_scale, np.float32)), _ptr(_c(w, np.float32)),
                                   _ptr(k8), _ptr(_c(k_scale, np.float32)), _ptr(pos), R, n_k, H_I,
                                   d_I, _ptr(out), n_k)
    _check(rc, "oracle_indexer_at")
    return out


def sparse_mla_at(q_bits, kv_bits, idx, pos, scale, d_v=512):
    """Sparse attention of query rows at explicit positions pos[r] (idx row r
    is row r's selection).  Returns (out [R, H, d_v], lse [R, H])."""
    q_bits = _c(q_bits, np.uint16)
    kv_bits = _c(kv_bits, np.uint16)
    idx = _c(idx, np.int32)
    pos = _c(pos, np.int64)
    R, H, d_qk = q_bits.shape
    n_k = kv_bits.shape[0]
    k = idx.shape[1]
    out = np.empty((R, H, d_v), dtype=np.float64)
    lse = np.empty((R, H), dtype=np.float64)
    rc = _load().oracle_sparse_mla_at(_ptr(q_bits), _ptr(kv_bits), _ptr(idx), _ptr(pos), R, n_k, H,
                                      d_qk, d_v, k, float(scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_sparse_mla_at: bad arguments")
    return out, lse


def indexer_kl_at(q_bits, kv_bits, idx, pos, logits, scale):
    """KL alignment of the indexer to the main attention over each row's
    selection ("DeepSeek V3.2 and the lightning indexer", "Teaching a dense
    model to be sparse"; "DeepSeek-V3.2" atlas entry, "Design overview"): row r
    (query at position pos[r], index row idx[r], indexer scores logits[r, :])
    gets the target p = head-averaged attention distribution over its valid
    selected entries, the loss KL(p || softmax(I)) and the gradient
    softmax(I) - p.  Returns (kl [R], grad [R, k], target [R, k]) in fp64, the
    last two in index-row order with zeros at invalid entries."""
    q_bits = _c(q_bits, np.uint16)
    kv_bits = _c(kv_bits, np.uint16)
    idx = _c(idx, np.int32)
    pos = _c(pos, np.int64)
    logits = _c(logits, np.float32)
    R, H, d_qk = q_bits.shape
    n_k = kv_bits.shape[0]
    k = idx.shape[1]
    kl = np.empty((R,), dtype=np.float64)
    grad = np.empty((R, k), dtype=np.float64)
    target = np.empty((R, k), dtype=np.float64)
    rc = _load().oracle_indexer_kl_at(_ptr(q_bits), _ptr(kv_bits), _ptr(idx), _ptr(pos),
                                      _ptr(logits), int(logits.shape[1]), R, n_k, H, d_qk, k,
                                      float(scale), _ptr(kl), _ptr(grad), _ptr(target))
    if rc != 0:
        raise ValueError("oracle_indexer_kl_at: bad arguments")
    return kl, grad, target


def indexer_backward(q_hat, w, k_hat, g, pos):
    """The indexer's backward ("DeepSeek V3.2 and the lightning indexer",
    "Teaching a dense model to be sparse": the warm-up trains the indexer
    alone on the KL signal): for scores I[t,s] = sum_j w[t,j] *
    ReLU(q_hat[t,j] . k_hat[s]) over s <= pos[t] and an upstream gradient g
    [n_q, n_k] (dense; entries past pos[t] are ignored), returns (dq [n_q, H,
    d], dw [n_q, H], dk [n_k, d]) in fp64; the ReLU's derivative is 0 at 0."""
    q_hat = _c(q_hat, np.float64)
    w = _c(w, np.float64)
    k_hat = _c(k_hat, np.float64)
    g = _c(g, np.float64)
    pos = _c(pos, np.int64)
    n_q, H, d = q_hat.shape
    n_k = k_hat.shape[0]
    if w.shape != (n_q, H) or k_hat.shape != (n_k, d) or g.shape != (n_q, n_k) or pos.shape != (n_q,):
        raise ValueError("indexer_backward: shape mismatch")
    dq = np.empty_like(q_hat)
    dw = np.empty_like(w)
    dk = np.empty_like(k_hat)
    rc = _load().oracle_indexer_backward(_ptr(q_hat), _ptr(w), _ptr(k_hat), _ptr(g), _ptr(pos),
                                         n_q, n_k, H, d, _ptr(dq), _ptr(dw), _ptr(dk))
    if rc != 0:
        raise ValueError("oracle_indexer_backward: bad arguments")
    return dq, dw, dk


def masked_mha_at(q_bits, k_bits, v_bits, idx, pos, scale):
    """The masked MHA mode ("DeepSeek-V3.2" atlas entry, "Design overview":
    short prompts are prefilled with a masked MHA standing in for DSA): per-head dense
    attention of query row r (position pos[r]) over the set of its valid
    selected keys.  q_bits [R, H, d_qk], k_bits [n_k, H, d_qk], v_bits
    [n_k, H, d_v] (bf16 bits), idx [R, topk].  Returns (out [R, H, d_v],
    lse [R, H]) in fp64."""
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    v_bits = _c(v_bits, np.uint16)
    idx = _c(idx, np.int32)
    pos = _c(pos, np.int64)
    R, H, d_qk = q_bits.shape
    n_k = k_bits.shape[0]
    d_v = v_bits.shape[2]
    if k_bits.shape != (n_k, H, d_qk) or v_bits.shape[:2] != (n_k, H) or idx.shape[0] != R:
        raise ValueError("masked_mha_at: shape mismatch")
    out = np.empty((R, H, d_v), dtype=np.float64)
    lse = np.empty((R, H), dtype=np.float64)
    rc = _load().oracle_masked_mha_at(_ptr(q_bits), _ptr(k_bits), _ptr(v_bits), _ptr(idx), _ptr(pos),
                                      R, n_k, H, d_qk, d_v, int(idx.shape[1]), float(scale),
                                      _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_masked_mha_at: bad arguments")
    return out, lse
