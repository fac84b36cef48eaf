"""dsa_forward_noalloc: the whole path for callers that cannot allocate device
memory (a serving engine whose pool already owns the device, a latency-critical
loop that cannot take an allocation's device synchronisation).  Its scratch
lives in a fixed 48 MiB device array inside the library instead of a caller
workspace.

The GPU test calls the entry point through the C ABI twice in a row, on two
different batches, and checks each result against dsa_forward (the existing
entry point, given a caller workspace) on the same inputs: identical indices,
and outputs within the attention tolerance the parity tests use.  The second
call runs over the scratch the first one left behind.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_08_b200 as dsa
from sparse_attention_08_b200 import workloads as W
from tests import dsa_cases as C

SCRATCH_BYTES = 48 << 20
WORKSPACE = 4


def _call_noalloc(wl, out, lse, idx):
    lib = dsa.load()
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    H = wl.q.shape[1]
    return lib.dsa_forward_noalloc(P(wl.q8), P(wl.q_scale), P(wl.w), P(wl.k8), P(wl.k_scale),
                                   P(wl.q), P(wl.kv), P(wl.cu_q), P(wl.cu_k), wl.B, wl.max_len_q,
                                   wl.max_len_k, wl.T_q, wl.T_k, wl.q8.shape[1], wl.q8.shape[2], H,
                                   576, 512, wl.k, ctypes.c_float(wl.scale), P(out), P(lse),
                                   P(idx), stream)


def _outputs(wl):
    H = wl.q.shape[1]
    return (torch.full((wl.T_q, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda"),
            torch.full((wl.T_q, H), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((wl.T_q, wl.k), -7, dtype=torch.int32, device="cuda"))


@pytest.mark.gpu
def test_noalloc_matches_dsa_forward_on_two_calls_in_a_row():
    batches = [
        # varlen decode: four sequences, one new query each
        W.make_small(H_I=64, d_I=128, H=128, lens=[5000, 3000, 2049, 700], lens_q=[1, 1, 1, 1],
                     k=2048, seed=41),
        # a prefill and a chunk, smaller k
        W.make_small(H_I=64, d_I=128, H=128, lens=[900, 1300], lens_q=[900, 300], k=512,
                     seed=42),
    ]
    for cpu in batches:
        wl = cpu.to("cuda")
        assert dsa.dsa_forward_workspace_size(wl.T_q, wl.max_len_k, wl.k) <= SCRATCH_BYTES
        ref_idx, ref_out, ref_lse = C.gpu_forward(wl)        # existing entry point
        out, lse, idx = _outputs(wl)
        rc = _call_noalloc(wl, out, lse, idx)
        assert rc == 0, dsa.dsa_status_string(rc)
        C.assert_no_device_error()
        assert torch.equal(idx, ref_idx)
        C.check_attention(C.np_(out.float()), C.np_(ref_out.float()).astype(np.float64),
                          C.np_(lse), C.np_(ref_lse).astype(np.float64))


def test_noalloc_refuses_problems_beyond_its_scratch():
    # a 32768-token prefill needs ~4.5 GB of scores: refused before any launch
    lib = dsa.load()
    p = ctypes.c_void_p(0x10000)
    rc = lib.dsa_forward_noalloc(p, p, p, p, p, p, p, p, p, 1, 32768, 32768, 32768, 32768, 64, 128,
                                 128, 576, 512, 2048, ctypes.c_float(1 / 24), p, None, None, None)
    assert rc == WORKSPACE
    assert dsa.dsa_forward_workspace_size(32768, 32768, 2048) > SCRATCH_BYTES
