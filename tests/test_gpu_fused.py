"""The fused indexer + top-k (dsa_forward_fused) against the oracle and
against the unfused composition.

The fused path computes every score with the same arithmetic as
dsa_indexer_logits and selects from a candidate list that holds every score
at or above the row's threshold; a row whose list is short, full or all ties
goes through the unfused kernels.  Its indices, outputs and lse must
therefore equal dsa_forward's bit for bit on every input, and through those
they meet the oracle under the end-to-end rules (the near-cut rule for the
selection, the attention bars for out and lse), which the small case also
checks against the oracle directly.
"""
import numpy as np
import pytest
import torch

import sparse_attention_08_b200 as dsa
from sparse_attention_08_b200 import workloads as W
from tests import dsa_cases as C
from tests.test_gpu_parity import _sampled_parity

pytestmark = pytest.mark.gpu


def _fused(wl):
    H = wl.q.shape[1]
    out = torch.full((wl.T_q, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.T_q, H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((wl.T_q, wl.k), -7, dtype=torch.int32, device="cuda")
    nbytes = dsa.dsa_forward_fused_workspace_size(wl.T_q, wl.T_k, wl.B, wl.max_len_k, wl.k,
                                                  wl.q8.shape[2])
    assert nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dsa.dsa_forward_fused(wl.q8, wl.q_scale, wl.w, wl.k8, wl.k_scale, wl.q, wl.kv, wl.cu_q,
                          wl.cu_k, wl.B, wl.max_len_q, wl.max_len_k, wl.k, wl.scale, out, lse, ws,
                          idx_out=idx)
    C.assert_no_device_error()
    return idx, out, lse


def _same_as_unfused(wl):
    f_idx, f_out, f_lse = _fused(wl)
    u_idx, u_out, u_lse = C.gpu_forward(wl)
    C.assert_no_device_error()
    assert torch.equal(f_idx, u_idx), "indices differ from dsa_forward"
    assert np.array_equal(C.bits(f_out), C.bits(u_out)), "outputs differ from dsa_forward"
    assert np.array_equal(C.np_(f_lse).view(np.uint32), C.np_(u_lse).view(np.uint32)), "lse"
    return f_idx, f_out, f_lse


def test_fused_small_against_oracle():
    # one prefill past the all-pass limit (rows beyond 4096 scores use the
    # sampled threshold), a chunk at the end of a cache, and a decode row;
    # the oracle evaluates sampled rows of each at their own positions
    wl = W.make_small(H_I=64, d_I=128, H=64, lens=[6500, 9000, 7000], lens_q=[6500, 300, 1],
                      k=256, seed=151, device="cuda")
    idx, out, lse = _same_as_unfused(wl)
    for b, rows in enumerate(([0, 1, 255, 256, 4095, 4096, 4097, 5000, 6499],
                              [0, 150, 299], [0])):
        _sampled_parity(wl, b, rows, idx, out, lse)


@pytest.mark.parametrize("k", [64, 2048])
def test_fused_equals_unfused_varlen(k):
    wl = W.make_small(H_I=64, d_I=128, H=16, lens=[12000, 5000, 4100, 300],
                      lens_q=[12000, 2000, 4100, 1], k=k, seed=152, device="cuda")
    _same_as_unfused(wl)


def test_fused_equals_unfused_decode_batch():
    wl = W.make_decode(3, device="cuda", B=16, seed=153)
    _same_as_unfused(wl)


def test_fused_falls_back_on_massive_ties():
    # every key of the long sequence is the same FP8 row with the same scale,
    # so every causal score of a query is equal: the candidate lists overflow
    # and those rows must go through the unfused path, with the same result
    wl = W.make_small(H_I=64, d_I=128, H=16, lens=[9000, 2000], lens_q=[9000, 2000], k=512,
                      seed=154, device="cuda")
    k0, k1 = 0, 9000
    wl.k8[k0:k1] = wl.k8[k0:k0 + 1].clone()
    wl.k_scale[k0:k1] = wl.k_scale[k0]
    _same_as_unfused(wl)


def test_fused_equals_unfused_config1():
    _same_as_unfused(W.make_prefill(1, device="cuda"))


def test_fused_equals_unfused_config4_chunks():
    full = W.make_prefill(4, device="cuda")
    C_ = full.T_q // full.cfg.chunks
    for c in (0, 3, 7):
        _same_as_unfused(W.chunk_of(full, c, C_))
        torch.cuda.empty_cache()


def test_fused_equals_unfused_config2_bench_size():
    # the L = 32768 prefill, the size the bench measures the fused path at
    _same_as_unfused(W.make_prefill(2, device="cuda"))


def test_fused_equals_unfused_config3_all_rows():
    _same_as_unfused(W.make_decode(3, device="cuda"))
