"""The C ABI on the host (no GPU needed): the library loads, exports every
symbol include/dsa.h declares, and rejects bad arguments with the documented
status before touching the device."""
import ctypes
import os
import re

import pytest

import sparse_attention_08_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")

OK, INVALID, UNSUPPORTED, ALIGN, WORKSPACE, CUDA = 0, 1, 2, 3, 4, 5


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^DSA_API\s+[\w\*\s]+?\b(dsa_\w+)\s*\(", text, flags=re.M)))


def test_header_declarations_are_exported():
    names = _declared()
    assert names == sorted(dsa.EXPORTED)
    lib = dsa.load()
    for n in names:
        assert hasattr(lib, n), n
    # nothing but the ABI is exported from the C side
    assert dsa.dsa_version() == "0.1.0"


def test_status_strings():
    for s in range(8):
        assert dsa.dsa_status_string(s)
    assert dsa.dsa_status_string(99) == "unknown status"


def test_workspace_size():
    T, L, k = 1000, 1001, 64
    ld = 1004
    expect = (T * ld * 4 + 255) // 256 * 256 + (T * k * 4 + 255) // 256 * 256
    assert dsa.dsa_forward_workspace_size(T, L, k) == expect
    assert dsa.dsa_forward_workspace_size(-1, L, k) == 0


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_indexer_argument_checks_before_device():
    lib = dsa.load()
    p = _fake()
    args = dict(q=p, qs=p, w=p, k=p, ks=p, cq=p, ck=p, B=1, mlq=64, mlk=64, tq=64, tk=64, H_I=64,
                d_I=128, lg=p, ld=64)

    def call(**kw):
        a = dict(args, **kw)
        return lib.dsa_indexer_logits(a["q"], a["qs"], a["w"], a["k"], a["ks"], a["cq"], a["ck"],
                                      a["B"], a["mlq"], a["mlk"], a["tq"], a["tk"], a["H_I"],
                                      a["d_I"], a["lg"], a["ld"], None)
    assert call(q=None) == INVALID
    assert call(cq=None) == INVALID
    assert call(H_I=48) == UNSUPPORTED
    assert call(d_I=96) == UNSUPPORTED
    assert call(ld=32) == INVALID                  # ld < max_len_k
    assert call(ld=66) == ALIGN                    # row stride not 16-byte
    assert call(lg=_fake(0x10004)) == ALIGN
    assert call(mlq=65, mlk=64) == INVALID         # more queries than keys
    assert call(tq=65) == INVALID                  # total beyond B * max_len
    assert call(tq=0) == OK                        # nothing to do, no launch
    if not _have_gpu():
        assert call() == CUDA                      # no device: fails loudly


def test_indexer_backward_argument_checks_before_device():
    lib = dsa.load()
    p = _fake()
    args = dict(q=p, qs=p, w=p, k=p, ks=p, g=p, ldg=64, cq=p, ck=p, B=1, mlq=64, mlk=64, tq=64,
                tk=64, H_I=64, d_I=128, dq=p, dw=p, dk=p)

    def call(**kw):
        a = dict(args, **kw)
        return lib.dsa_indexer_backward(a["q"], a["qs"], a["w"], a["k"], a["ks"], a["g"], a["ldg"],
                                        a["cq"], a["ck"], a["B"], a["mlq"], a["mlk"], a["tq"],
                                        a["tk"], a["H_I"], a["d_I"], a["dq"], a["dw"], a["dk"],
                                        None)
    assert call(g=None) == INVALID
    assert call(dk=None) == INVALID
    assert call(H_I=32) == UNSUPPORTED
    assert call(d_I=64) == UNSUPPORTED
    assert call(ldg=32) == INVALID                 # ld_g < max_len_k
    assert call(ldg=66) == ALIGN
    assert call(dq=_fake(0x10004)) == ALIGN
    assert call(tq=0) == OK
    if not _have_gpu():
        assert call() == CUDA


def test_topk_and_attention_argument_checks():
    lib = dsa.load()
    p = _fake()
    assert lib.dsa_topk(p, 64, p, p, 1, 64, 64, 64, 0, p, None, None) == UNSUPPORTED
    assert lib.dsa_topk(p, 64, p, p, 1, 64, 64, 64, 5000, p, None, None) == UNSUPPORTED
    assert lib.dsa_topk(None, 64, p, p, 1, 64, 64, 64, 16, p, None, None) == INVALID
    assert lib.dsa_topk(p, 64, p, p, 1, 64, 64, 64, 16, _fake(0x10008), None, None) == ALIGN
    assert lib.dsa_topk(p, 66, p, p, 1, 64, 64, 64, 16, p, None, None) == ALIGN
    f = ctypes.c_float(1.0 / 24)
    mla = lib.dsa_sparse_mla_fwd
    assert mla(p, p, p, p, p, 1, 64, 64, 64, 64, 128, 512, 512, 64, f, p, None, None) == UNSUPPORTED
    assert mla(p, p, p, p, p, 1, 64, 64, 64, 64, 48, 576, 512, 64, f, p, None, None) == UNSUPPORTED
    assert mla(p, p, p, p, p, 1, 64, 64, 64, 64, 128, 576, 512, 64, ctypes.c_float(-1.0), p, None,
               None) == INVALID
    assert mla(p, None, p, p, p, 1, 64, 64, 64, 64, 128, 576, 512, 64, f, p, None, None) == INVALID
    assert mla(p, p, p, p, p, 1, 64, 64, 64, 64, 128, 576, 512, 64, f, _fake(0x10002), None,
               None) == ALIGN


def test_forward_workspace_checks():
    lib = dsa.load()
    p = _fake()
    f = ctypes.c_float(1.0 / 24)
    need = dsa.dsa_forward_workspace_size(64, 64, 16)

    def fwd(ws, nbytes):
        return lib.dsa_forward(p, p, p, p, p, p, p, p, p, 1, 64, 64, 64, 64, 64, 128, 128, 576, 512,
                               16, f, p, None, None, ws, nbytes, None)
    assert fwd(None, need) == WORKSPACE
    assert fwd(p, need - 1) == WORKSPACE
    assert fwd(_fake(0x10001), need) == ALIGN


def test_forward_host_checks_before_any_device_call():
    """Argument checks of the host-buffer entry point run on the host: each of
    these returns its status without touching a device."""
    import numpy as np
    lib = dsa.load()
    f = ctypes.c_float(1.0 / 24)
    cu_q = np.array([0, 64], dtype=np.int32)
    cu_k = np.array([0, 64], dtype=np.int32)
    bad_k = np.array([0, 32], dtype=np.int32)          # fewer keys than queries
    p = _fake()
    need = dsa.dsa_forward_host_workspace_size(64, 64, 1, 64, 128, 128, 16, 32, 2)
    assert need > 0
    # one more stream costs one more chunk region
    assert dsa.dsa_forward_host_workspace_size(64, 64, 1, 64, 128, 128, 16, 32, 3) > need
    assert dsa.dsa_forward_host_workspace_size(64, 64, 1, 64, 128, 128, 16, 0, 2) == 0
    streams = (ctypes.c_void_p * 2)(_fake().value, _fake().value)

    def host(cq, ck, chunk=32, ws=p, nbytes=need, st=streams, n=2, d_qk=576):
        return lib.dsa_forward_host(p, p, p, p, p, p, p, cq.ctypes.data, ck.ctypes.data, 1, 64, 64,
                                    64, int(ck[-1]), 64, 128, 128, d_qk, 512, 16, f, p, None,
                                    chunk, ws, nbytes, st, n)
    assert host(cu_q, cu_k, chunk=0) == INVALID
    assert host(cu_q, cu_k, st=None) == INVALID
    assert host(cu_q, cu_k, n=0) == INVALID
    assert host(cu_q, bad_k) == INVALID
    assert host(cu_q, cu_k, d_qk=512) == UNSUPPORTED
    assert host(cu_q, cu_k, ws=None) == WORKSPACE
    assert host(cu_q, cu_k, nbytes=need - 1) == WORKSPACE
    assert host(cu_q, cu_k, ws=_fake(0x10010)) == ALIGN


def _have_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.gpu
def test_device_error_word_starts_clear():
    import torch
    torch.zeros(1, device="cuda")
    assert dsa.dsa_get_device_error() == OK


def test_masked_mha_checks_before_any_device_call():
    """Argument checks of the masked MHA mode run on the host."""
    lib = dsa.load()
    p = _fake()
    f = ctypes.c_float(1.0 / 192 ** 0.5)
    need = dsa.dsa_masked_mha_workspace_size(256, 256)
    assert need == 256 * 8 * 4                       # 8 words of 32 keys per row
    assert dsa.dsa_masked_mha_workspace_size(256, 0) == 0
    assert dsa.dsa_masked_mha_workspace_size(256, 131073) == 0

    def call(d_qk=192, d_v=128, H=4, topk=64, ws=p, nbytes=need, scale=f, q=p):
        return lib.dsa_masked_mha_fwd(q, p, p, p, p, p, 1, 256, 256, 256, 256, H, d_qk, d_v, topk,
                                      scale, p, None, ws, nbytes, None)
    assert call(d_qk=576) == UNSUPPORTED
    assert call(d_v=512) == UNSUPPORTED
    assert call(topk=0) == UNSUPPORTED
    assert call(scale=ctypes.c_float(-1.0)) == INVALID
    assert call(q=None) == INVALID
    assert call(ws=None) == WORKSPACE
    assert call(nbytes=need - 1) == WORKSPACE
    assert call(q=_fake(0x10008)) == ALIGN


def test_forward_fused_checks_before_any_device_call():
    lib = dsa.load()
    p = _fake()
    T, Tk, B, L, k, d_I = 64, 64, 1, 64, 32, 128
    need = dsa.dsa_forward_fused_workspace_size(T, Tk, B, L, k, d_I)
    assert need > dsa.dsa_forward_workspace_size(T, L, k)
    # sizes it does not support
    assert dsa.dsa_forward_fused_workspace_size(T, Tk, B, L, 4096, d_I) == 0
    assert dsa.dsa_forward_fused_workspace_size(T, Tk, B, 131073, k, d_I) == 0
    assert dsa.dsa_forward_fused_workspace_size(T, Tk, B, L, k, 96) == 0

    def call(ws=p, nbytes=need, k=k, H_I=64, mlk=L):
        return lib.dsa_forward_fused(p, p, p, p, p, p, p, p, p, B, L, mlk, T, Tk, H_I, d_I, 128,
                                     576, 512, k, 0.05, p, p, None, ws, nbytes, None)
    assert call(ws=None) == WORKSPACE
    assert call(nbytes=need - 1) == WORKSPACE
    assert call(ws=_fake(0x10008)) == ALIGN
    assert call(k=4096) == UNSUPPORTED               # the candidate lists hold 5120 entries
    assert call(H_I=48) == UNSUPPORTED
    assert call(H_I=32) == UNSUPPORTED               # the compact read-out is 64-head only
    if not _have_gpu():
        assert call() == CUDA                        # no device: fails loudly
