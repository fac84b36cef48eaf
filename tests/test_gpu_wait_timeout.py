"""Failure detection on the device, without a fault.

Every wait inside the kernels is bounded: a wait that runs out records
DSA_ERR_TIMEOUT in the device error word and the kernel winds down and
returns, so the CUDA context stays usable.  This test makes one wait run out
on purpose through the library's test hook: with a 20 ms wait limit, the next
indexer launch leaves out the first key-tile load of every CTA, so the MMA
issuer's wait for it gives up.  Nothing traps, faults or hangs; the host reads
the status, and the next ordinary call must be exact again.
"""
import time

import numpy as np
import pytest
import torch

import sparse_attention_08_b200 as dsa
from sparse_attention_08_b200 import workloads as W
from tests import dsa_cases as C

pytestmark = pytest.mark.gpu

DSA_ERR_TIMEOUT = 6


def test_timed_out_wait_is_reported_and_the_next_call_is_exact():
    cpu = W.make_small(H_I=4, d_I=64, H=16, L=1500, k=64, integer=True, seed=131)
    gpu = cpu.to("cuda")
    C.assert_no_device_error()
    torch.cuda.synchronize()
    dsa.dsa_debug_fault_injection(20_000_000, True)
    try:
        t0 = time.perf_counter()
        C.gpu_indexer(gpu)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        st = dsa.dsa_get_device_error()
    finally:
        dsa.dsa_debug_fault_injection(0, False)
    assert st == DSA_ERR_TIMEOUT, f"status {st}"
    # the launch gave up after a few 20 ms limits, not the default 2 s
    assert elapsed < 1.5, elapsed
    # the word was read and cleared; the context is usable and the next
    # ordinary call gives the exact scores
    assert dsa.dsa_get_device_error() == 0
    g = C.np_(C.gpu_indexer(gpu))
    C.assert_no_device_error()
    o = C.oracle_scores(cpu, 0)
    C.check_indexer(g, o, None, list(range(cpu.T_q)), exact=True)
