"""GPU parity of the indexer's backward (dsa_indexer_backward) against the
fp64 oracle (oracle.indexer_backward, pinned in test_oracle_pins.py).

Two regimes:
* integer-valued inputs (e4m3 codes of the integers -4..4, scales 1, head
  weights -2..2, gradients in multiples of 1/8): every gate is exact (the FP8
  dot products are small integers), every bf16 operand is exact, and every
  fp32 partial sum is an exact multiple of 1/8, so the three gradients must
  match the oracle bit for bit, whatever the order of the additions;
* real-valued inputs: one operand of each gated sum is rounded to bf16 once
  (relative error 2^-9 per product, the other operand being an exact e4m3
  code) and the sums run in fp32, so each gradient tensor must lie within a
  relative L2 error of 5e-3 (2.5x 2^-9) of the oracle.  A gate whose FP8 dot
  product is within fp32 rounding of 0 may flip; such terms are rare and
  small, and the L2 bar absorbs them.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_08_b200 as dsa
from sparse_attention_08_b200 import workloads as W
from tests import dsa_cases as C

pytestmark = pytest.mark.gpu

BWD_REL_L2 = 5e-3


def _hat(b8, scale):
    f = torch.from_numpy(C.np_(b8).copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return f * scale


def _run(wl, g):
    gpu = wl.to("cuda")
    dq = torch.full((wl.T_q, 64, 128), float("nan"), device="cuda")
    dw = torch.full((wl.T_q, 64), float("nan"), device="cuda")
    dk = torch.full((wl.T_k, 128), float("nan"), device="cuda")
    dsa.dsa_indexer_backward(gpu.q8, gpu.q_scale, gpu.w, gpu.k8, gpu.k_scale, g.cuda(), gpu.cu_q,
                             gpu.cu_k, wl.B, wl.max_len_q, wl.max_len_k, dq, dw, dk)
    C.assert_no_device_error()
    return C.np_(dq), C.np_(dw), C.np_(dk)


def _oracle(wl, g, b):
    q0, q1, k0, k1 = C.seq_slices(wl, b)
    qh = _hat(wl.q8[q0:q1], C.np_(wl.q_scale[q0:q1])[:, :, None])
    kh = _hat(wl.k8[k0:k1], C.np_(wl.k_scale[k0:k1])[:, None])
    pos = (k1 - k0) - (q1 - q0) + np.arange(q1 - q0)
    return oracle.indexer_backward(qh, C.np_(wl.w[q0:q1]), kh,
                                   C.np_(g[q0:q1, :k1 - k0]).astype(np.float64), pos)


CASES = [
    ([300], None),                     # one prefill, a ragged last key tile
    ([700, 300], [700, 45]),           # a prefill and a chunk at the end of a cache
    ([5, 260, 1000], [1, 1, 1]),       # one-query rows (decode shape)
]


@pytest.mark.parametrize("lens,lens_q", CASES)
def test_indexer_backward_integer_inputs_exact(lens, lens_q):
    wl = W.make_small(H_I=64, d_I=128, H=16, lens=lens, lens_q=lens_q, k=64, integer=True,
                      seed=141)
    gen = torch.Generator().manual_seed(5)
    ld = (wl.max_len_k + 3) // 4 * 4
    g = torch.randint(-4, 5, (wl.T_q, ld), generator=gen).float() / 8.0
    dq, dw, dk = _run(wl, g)
    for b in range(wl.B):
        q0, q1, k0, k1 = C.seq_slices(wl, b)
        o_dq, o_dw, o_dk = _oracle(wl, g, b)
        assert np.array_equal(dq[q0:q1].astype(np.float64), o_dq), f"dq, sequence {b}"
        assert np.array_equal(dw[q0:q1].astype(np.float64), o_dw), f"dw, sequence {b}"
        assert np.array_equal(dk[k0:k1].astype(np.float64), o_dk), f"dk, sequence {b}"


@pytest.mark.parametrize("lens,lens_q", CASES)
def test_indexer_backward_real_inputs(lens, lens_q):
    wl = W.make_small(H_I=64, d_I=128, H=16, lens=lens, lens_q=lens_q, k=64, seed=142)
    gen = torch.Generator().manual_seed(6)
    ld = (wl.max_len_k + 3) // 4 * 4
    # a KL-like gradient: small values of both signs on every causal key
    g = torch.randn((wl.T_q, ld), generator=gen) * 1e-2
    dq, dw, dk = _run(wl, g)
    for b in range(wl.B):
        q0, q1, k0, k1 = C.seq_slices(wl, b)
        o_dq, o_dw, o_dk = _oracle(wl, g, b)
        for name, got, ref in (("dq", dq[q0:q1], o_dq), ("dw", dw[q0:q1], o_dw),
                               ("dk", dk[k0:k1], o_dk)):
            rel = np.linalg.norm(got.astype(np.float64) - ref) / max(np.linalg.norm(ref), 1e-300)
            assert rel <= BWD_REL_L2, f"{name}, sequence {b}: relative L2 {rel:.2e}"


def test_indexer_backward_config1_rows():
    # the L = 8192 workload, at full size in one call.  The gradients are
    # linear in g, so g is non-zero only on a set of rows R (the first rows,
    # rows around k, and the last 64): dq and dw of R, and dk of every key,
    # are then the oracle's over R alone (and dq, dw of the other rows are 0)
    wl = W.make_prefill(1)
    gen = torch.Generator().manual_seed(7)
    L = wl.T_q
    rows = np.concatenate([[0, 1, 2047, 2048, 4000], np.arange(L - 64, L)])
    g = torch.zeros((L, L))
    g[torch.as_tensor(rows)] = torch.randn((len(rows), L), generator=gen) * 1e-3
    dq, dw, dk = _run(wl, g)
    rt = torch.as_tensor(rows)
    qh = _hat(wl.q8[rt], C.np_(wl.q_scale[rt])[:, :, None])
    kh = _hat(wl.k8, C.np_(wl.k_scale)[:, None])
    o_dq, o_dw, o_dk = oracle.indexer_backward(qh, C.np_(wl.w[rt]), kh,
                                               C.np_(g[rt]).astype(np.float64), rows)
    for name, got, ref in (("dq", dq[rows], o_dq), ("dw", dw[rows], o_dw), ("dk", dk, o_dk)):
        rel = np.linalg.norm(got.astype(np.float64) - ref) / max(np.linalg.norm(ref), 1e-300)
        assert rel <= BWD_REL_L2, f"{name}: relative L2 {rel:.2e}"
    others = np.setdiff1d(np.arange(L), rows)
    assert np.all(dq[others] == 0) and np.all(dw[others] == 0)
