"""GPU parity of the masked MHA mode ("DeepSeek-V3.2" atlas entry, "Design
overview": short prompts are prefilled with a masked MHA standing in for DSA): the CUDA path
through the C ABI against the fp64 oracle on the same seeded inputs.  Small
cases are compared over every query row (several query and key tiles, ragged
tails, varlen chunks); the benchmark's workload runs in the launch the
benchmark times and is compared on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_08_b200 as dsa
from sparse_attention_08_b200 import workloads as W
from tests import dsa_cases as C

pytestmark = pytest.mark.gpu


def _gpu(m, idx=None):
    dev = "cuda"
    T_q, H = m.T_q, m.q.shape[1]
    out = torch.full((T_q, H, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((T_q, H), float("nan"), dtype=torch.float32, device=dev)
    ix = (m.idx if idx is None else idx).to(dev).contiguous()
    dsa.dsa_masked_mha_fwd(m.q.to(dev), m.k.to(dev), m.v.to(dev), ix, m.cu_q.to(dev),
                           m.cu_k.to(dev), m.B, m.max_len_q, m.max_len_k, ix.shape[1], m.scale,
                           out, lse)
    C.assert_no_device_error()
    return C.np_(out.float()).astype(np.float64), C.np_(lse).astype(np.float64)


def _oracle(m, idx, b, rows):
    q0 = int(m.cu_q[b])
    k0, k1 = int(m.cu_k[b]), int(m.cu_k[b + 1])
    lq, lk = m.lens_q[b], m.lens_k[b]
    rows = np.asarray(rows)
    pos = lk - lq + rows
    sel = torch.from_numpy(q0 + rows)
    return oracle.masked_mha_at(C.bits(m.q[sel]), C.bits(m.k[k0:k1]), C.bits(m.v[k0:k1]),
                                np.ascontiguousarray(idx[q0 + rows]), pos, m.scale)


def _check(g_out, g_lse, o_out, o_lse):
    C.check_attention(g_out, o_out)
    fin = np.isfinite(o_lse)
    assert np.array_equal(np.isneginf(g_lse), ~fin), "rows with an empty selection"
    if fin.any():
        assert float(np.max(np.abs(g_lse[fin] - o_lse[fin]))) <= C.LSE_ABS
    assert np.all(g_out[~fin] == 0.0)


def _compare_all(m, idx=None):
    g_out, g_lse = _gpu(m, idx)
    ix = C.np_(m.idx if idx is None else idx)
    o_all, ol_all = [], []
    for b in range(m.B):
        o, ol = _oracle(m, ix, b, np.arange(m.lens_q[b]))
        o_all.append(o)
        ol_all.append(ol)
    _check(g_out, g_lse, np.concatenate(o_all), np.concatenate(ol_all))


@pytest.mark.parametrize("lens,lens_q,H,topk", [
    ([300], None, 2, 64),                 # sparse selections, ragged third query tile
    ([300, 200], [300, 50], 3, 64),       # varlen, the second sequence a chunk
    ([260], None, 1, 512),                # every causal key selected: causal attention
    ([129, 1, 400], [129, 1, 7], 4, 32),  # a one-key sequence, a 129-row sequence
])
def test_masked_mha_small(lens, lens_q, H, topk):
    m = W.make_mha(lens, lens_q, H=H, topk=topk, seed=301)
    _compare_all(m)


def test_masked_mha_repeats_holes_and_empty_rows():
    m = W.make_mha([280], None, H=2, topk=96, seed=302)
    idx = m.idx.clone()
    idx[:, 1] = idx[:, 0]                     # a repeated entry counts once
    idx[40:, 5] = -5                          # holes
    idx[60:, 7] = 100000                      # past p: skipped
    idx[9, :] = -1                            # an empty selection: out 0, lse -inf
    idx[200, :] = 150                         # one key, repeated
    _compare_all(m, idx)


def test_masked_mha_sharp_softmax_rescales():
    # q / 2 instead of q / sqrt(192): scores of several units, and keys whose
    # scale ramps up along the sequence, so the running maximum jumps by more
    # than the lazy-rescale threshold within rows
    m = W.make_mha([520], None, H=2, topk=256, seed=303, q_div=2.0)
    ramp = (1.0 + torch.arange(520, dtype=torch.float32) / 60.0)[:, None, None]
    m.k = (m.k.float() * ramp).to(torch.bfloat16)
    _compare_all(m)


def test_masked_mha_short_prefill_sampled():
    """The workload the benchmark times (L = 4096, H = 128, topk = 2048: the
    second half of the queries attend to a strict subset), on sampled rows."""
    m = W.make_mha([4096], None, H=128, topk=2048, seed=W.BASE_SEED + 900, device="cuda")
    g_out, g_lse = _gpu(m)
    rows = np.array([0, 1, 127, 128, 1000, 2046, 2047, 2048, 3001, 4094, 4095])
    ix = C.np_(m.idx)
    sel = torch.from_numpy(rows).to(m.q.device)
    o, ol = oracle.masked_mha_at(C.bits(m.q[sel].cpu()), C.bits(m.k.cpu()), C.bits(m.v.cpu()),
                                 np.ascontiguousarray(ix[rows]), rows, m.scale)
    _check(g_out[rows], g_lse[rows], o, ol)
