"""B200-native DeepSeek Sparse Attention (DSA) hot path.

The compute lives in ``libdsa.so`` (CUDA for sm_100a, C ABI in
``include/dsa.h``); this module only marshals torch tensors into that ABI.
Every function has the name of its C entry point and takes device tensors
plus the stream it should run on (default: torch's current stream).  There is
no CPU path: if the library is missing, importing the binding fails.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "DSAError", "lib_path", "load", "dsa_version", "dsa_status_string",
    "dsa_indexer_logits", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_forward",
    "dsa_forward_workspace_size", "dsa_get_device_error", "dsa_forward_noalloc",
    "dsa_forward_host", "dsa_forward_host_workspace_size", "dsa_indexer_kl",
    "dsa_indexer_kl_workspace_size", "dsa_masked_mha_fwd", "dsa_masked_mha_workspace_size",
    "dsa_debug_fault_injection", "dsa_indexer_backward", "dsa_forward_fused",
    "dsa_forward_fused_workspace_size", "EXPORTED",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdsa.so")
_lib = None

# Every symbol include/dsa.h declares.
EXPORTED = (
    "dsa_indexer_logits", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_forward",
    "dsa_forward_workspace_size", "dsa_status_string", "dsa_get_device_error", "dsa_version",
    "dsa_forward_noalloc", "dsa_forward_host", "dsa_forward_host_workspace_size",
    "dsa_indexer_kl", "dsa_indexer_kl_workspace_size", "dsa_masked_mha_fwd",
    "dsa_masked_mha_workspace_size", "dsa_debug_fault_injection", "dsa_indexer_backward",
    "dsa_forward_fused", "dsa_forward_fused_workspace_size",
)

STATUS = {
    0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_ALIGNMENT",
    4: "DSA_ERR_WORKSPACE", 5: "DSA_ERR_CUDA", 6: "DSA_ERR_TIMEOUT", 7: "DSA_ERR_BOUNDS",
}


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS.get(self.status, self.status)} "
                         f"({dsa_status_string(self.status)})")


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Loads libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m sparse_attention_08_b200._build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, I64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.dsa_indexer_logits.argtypes = [P, P, P, P, P, P, P, I, I, I, I64, I64, I, I, P, I64, P]
    lib.dsa_topk.argtypes = [P, I64, P, P, I, I, I, I64, I, P, P, P]
    lib.dsa_sparse_mla_fwd.argtypes = [P, P, P, P, P, I, I, I, I64, I64, I, I, I, I, F, P, P, P]
    lib.dsa_forward.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I64, I64, I, I, I, I, I, I, F,
                                P, P, P, P, ctypes.c_size_t, P]
    lib.dsa_forward_fused.argtypes = lib.dsa_forward.argtypes
    lib.dsa_forward_fused_workspace_size.argtypes = [I64, I64, I, I, I, I]
    lib.dsa_forward_fused_workspace_size.restype = ctypes.c_size_t
    lib.dsa_forward_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I64, I64, I, I, I, I,
                                        I, I, F, P, P, P, P]
    lib.dsa_forward_host.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I64, I64, I, I, I, I, I,
                                     I, F, P, P, I, P, ctypes.c_size_t, P, I]
    lib.dsa_indexer_kl.argtypes = [P, P, P, P, P, I64, P, P, I, I, I, I64, I64, I, I, I, F, P, P,
                                   P, P, ctypes.c_size_t, P]
    lib.dsa_indexer_kl.restype = I
    lib.dsa_indexer_kl_workspace_size.argtypes = [I64, I, I]
    lib.dsa_indexer_kl_workspace_size.restype = ctypes.c_size_t
    lib.dsa_masked_mha_fwd.argtypes = [P, P, P, P, P, P, I, I, I, I64, I64, I, I, I, I, F, P, P, P,
                                       ctypes.c_size_t, P]
    lib.dsa_masked_mha_fwd.restype = I
    lib.dsa_masked_mha_workspace_size.argtypes = [I64, I]
    lib.dsa_masked_mha_workspace_size.restype = ctypes.c_size_t
    lib.dsa_forward_host_workspace_size.argtypes = [I64, I, I, I, I, I, I, I, I]
    lib.dsa_forward_host_workspace_size.restype = ctypes.c_size_t
    for name in ("dsa_indexer_logits", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_forward",
                 "dsa_forward_noalloc", "dsa_forward_host", "dsa_forward_fused"):
        getattr(lib, name).restype = I
    lib.dsa_forward_workspace_size.argtypes = [I64, I, I]
    lib.dsa_forward_workspace_size.restype = ctypes.c_size_t
    lib.dsa_status_string.argtypes = [I]
    lib.dsa_status_string.restype = ctypes.c_char_p
    lib.dsa_get_device_error.argtypes = [P]
    lib.dsa_get_device_error.restype = I
    lib.dsa_indexer_backward.argtypes = [P, P, P, P, P, P, I64, P, P, I, I, I, I64, I64, I, I, P,
                                         P, P, P]
    lib.dsa_indexer_backward.restype = I
    lib.dsa_debug_fault_injection.argtypes = [ctypes.c_uint64, I]
    lib.dsa_debug_fault_injection.restype = None
    lib.dsa_version.argtypes = []
    lib.dsa_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def dsa_debug_fault_injection(wait_limit_ns: int = 0, drop_first_key_load: bool = False):
    """Test hook: the wait limit of later launches (0 = the default 2 s) and a
    one-shot request that the next dsa_indexer_logits launch leave out its
    first key-tile load, so a bounded wait runs out (DSA_ERR_TIMEOUT)."""
    load().dsa_debug_fault_injection(int(wait_limit_ns), 1 if drop_first_key_load else 0)


def dsa_version() -> str:
    return load().dsa_version().decode()


def dsa_status_string(status: int) -> str:
    return load().dsa_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, where: str):
    if rc != 0:
        raise DSAError(rc, where)


def _need(t, dtype, name, ndim=None):
    import torch
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    del torch


def dsa_indexer_logits(q_fp8, q_scale, w, k_fp8, k_scale, cu_seqlens_q, cu_seqlens_k, B,
                       max_len_q, max_len_k, logits, ld_logits=None, stream=None):
    """Indexer scores into logits (f32, row stride ld_logits).  q_fp8 / k_fp8
    are uint8 (or float8_e4m3fn) tensors [T_q, H_I, d_I] / [T_k, d_I]."""
    import torch
    q8 = q_fp8.view(torch.uint8) if q_fp8.dtype == torch.float8_e4m3fn else q_fp8
    k8 = k_fp8.view(torch.uint8) if k_fp8.dtype == torch.float8_e4m3fn else k_fp8
    _need(q8, torch.uint8, "q_fp8", 3)
    _need(k8, torch.uint8, "k_fp8", 2)
    _need(q_scale, torch.float32, "q_scale")
    _need(w, torch.float32, "w")
    _need(k_scale, torch.float32, "k_scale")
    _need(cu_seqlens_q, torch.int32, "cu_seqlens_q")
    _need(cu_seqlens_k, torch.int32, "cu_seqlens_k")
    if ld_logits is None:
        ld_logits = logits.stride(0)
    T_q, H_I, d_I = q8.shape
    rc = load().dsa_indexer_logits(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale),
                                   _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(B), int(max_len_q),
                                   int(max_len_k), int(T_q), int(k8.shape[0]), int(H_I), int(d_I),
                                   _ptr(logits), int(ld_logits), _stream(stream))
    _check(rc, "dsa_indexer_logits")


def dsa_indexer_backward(q_fp8, q_scale, w, k_fp8, k_scale, g, cu_seqlens_q, cu_seqlens_k, B,
                         max_len_q, max_len_k, dq, dw, dk, ld_g=None, stream=None):
    """The indexer's backward: dq [T_q, 64, 128], dw [T_q, 64], dk [T_k, 128]
    (f32) from the upstream score gradient g (f32, row stride ld_g)."""
    import torch
    q8 = q_fp8.view(torch.uint8) if q_fp8.dtype == torch.float8_e4m3fn else q_fp8
    k8 = k_fp8.view(torch.uint8) if k_fp8.dtype == torch.float8_e4m3fn else k_fp8
    _need(q8, torch.uint8, "q_fp8", 3)
    _need(k8, torch.uint8, "k_fp8", 2)
    for t, n in ((q_scale, "q_scale"), (w, "w"), (k_scale, "k_scale"), (dw, "dw")):
        _need(t, torch.float32, n)
    _need(dq, torch.float32, "dq", 3)
    _need(dk, torch.float32, "dk", 2)
    _need(cu_seqlens_q, torch.int32, "cu_seqlens_q")
    _need(cu_seqlens_k, torch.int32, "cu_seqlens_k")
    if g.dtype != torch.float32 or not g.is_cuda or g.stride(1) != 1:
        raise ValueError("g must be a CUDA float32 tensor with contiguous rows")
    if ld_g is None:
        ld_g = g.stride(0)
    T_q, H_I, d_I = q8.shape
    rc = load().dsa_indexer_backward(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale),
                                     _ptr(g), int(ld_g), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                     int(B), int(max_len_q), int(max_len_k), int(T_q),
                                     int(k8.shape[0]), int(H_I), int(d_I), _ptr(dq), _ptr(dw),
                                     _ptr(dk), _stream(stream))
    _check(rc, "dsa_indexer_backward")


def dsa_topk(logits, cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, k, idx_out,
             val_out=None, ld_logits=None, total_q=None, stream=None):
    import torch
    _need(idx_out, torch.int32, "idx_out", 2)
    _need(val_out, torch.float32, "val_out", 2)
    if logits.dtype != torch.float32 or not logits.is_cuda:
        raise ValueError("logits must be a CUDA float32 tensor")
    if ld_logits is None:
        ld_logits = logits.stride(0)
    if total_q is None:
        total_q = idx_out.shape[0]
    rc = load().dsa_topk(_ptr(logits), int(ld_logits), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                         int(B), int(max_len_q), int(max_len_k), int(total_q), int(k),
                         _ptr(idx_out), _ptr(val_out), _stream(stream))
    _check(rc, "dsa_topk")


def dsa_sparse_mla_fwd(q, kv, idx, cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k,
                       sm_scale, out, lse=None, stream=None):
    import torch
    _need(q, torch.bfloat16, "q", 3)
    _need(kv, torch.bfloat16, "kv", 2)
    _need(idx, torch.int32, "idx", 2)
    _need(out, torch.bfloat16, "out", 3)
    _need(lse, torch.float32, "lse", 2)
    T_q, H, d_qk = q.shape
    rc = load().dsa_sparse_mla_fwd(_ptr(q), _ptr(kv), _ptr(idx), _ptr(cu_seqlens_q),
                                   _ptr(cu_seqlens_k), int(B), int(max_len_q), int(max_len_k),
                                   int(T_q), int(kv.shape[0]), int(H), int(d_qk),
                                   int(out.shape[2]), int(idx.shape[1]), float(sm_scale),
                                   _ptr(out), _ptr(lse), _stream(stream))
    _check(rc, "dsa_sparse_mla_fwd")


def dsa_forward_workspace_size(total_q, max_len_k, k) -> int:
    return int(load().dsa_forward_workspace_size(int(total_q), int(max_len_k), int(k)))


def dsa_forward(q_fp8, q_scale, w, k_fp8, k_scale, q, kv, cu_seqlens_q, cu_seqlens_k, B,
                max_len_q, max_len_k, k, sm_scale, out, lse, workspace, idx_out=None,
                stream=None):
    import torch
    q8 = q_fp8.view(torch.uint8) if q_fp8.dtype == torch.float8_e4m3fn else q_fp8
    k8 = k_fp8.view(torch.uint8) if k_fp8.dtype == torch.float8_e4m3fn else k_fp8
    _need(q8, torch.uint8, "q_fp8", 3)
    _need(k8, torch.uint8, "k_fp8", 2)
    _need(q, torch.bfloat16, "q", 3)
    _need(kv, torch.bfloat16, "kv", 2)
    _need(out, torch.bfloat16, "out", 3)
    _need(lse, torch.float32, "lse", 2)
    _need(idx_out, torch.int32, "idx_out", 2)
    T_q, H_I, d_I = q8.shape
    _, H, d_qk = q.shape
    rc = load().dsa_forward(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), _ptr(q),
                            _ptr(kv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(B),
                            int(max_len_q), int(max_len_k), int(T_q), int(k8.shape[0]), int(H_I),
                            int(d_I), int(H), int(d_qk), int(out.shape[2]), int(k),
                            float(sm_scale), _ptr(out), _ptr(lse), _ptr(idx_out),
                            _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                            _stream(stream))
    _check(rc, "dsa_forward")


def dsa_forward_fused_workspace_size(total_q, total_k, B, max_len_k, k, d_I) -> int:
    return int(load().dsa_forward_fused_workspace_size(int(total_q), int(total_k), int(B),
                                                       int(max_len_k), int(k), int(d_I)))


def dsa_forward_fused(q_fp8, q_scale, w, k_fp8, k_scale, q, kv, cu_seqlens_q, cu_seqlens_k, B,
                      max_len_q, max_len_k, k, sm_scale, out, lse, workspace, idx_out=None,
                      stream=None):
    """dsa_forward with the indexer and top-k fused into two passes over the
    keys (the score matrix stays out of HBM); same results, bit for bit.  The
    workspace holds dsa_forward_fused_workspace_size bytes."""
    import torch
    q8 = q_fp8.view(torch.uint8) if q_fp8.dtype == torch.float8_e4m3fn else q_fp8
    k8 = k_fp8.view(torch.uint8) if k_fp8.dtype == torch.float8_e4m3fn else k_fp8
    _need(q8, torch.uint8, "q_fp8", 3)
    _need(k8, torch.uint8, "k_fp8", 2)
    _need(q, torch.bfloat16, "q", 3)
    _need(kv, torch.bfloat16, "kv", 2)
    _need(out, torch.bfloat16, "out", 3)
    _need(lse, torch.float32, "lse", 2)
    _need(idx_out, torch.int32, "idx_out", 2)
    T_q, H_I, d_I = q8.shape
    _, H, d_qk = q.shape
    rc = load().dsa_forward_fused(
        _ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), _ptr(q), _ptr(kv),
        _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(B), int(max_len_q), int(max_len_k), int(T_q),
        int(k8.shape[0]), int(H_I), int(d_I), int(H), int(d_qk), int(out.shape[2]), int(k),
        float(sm_scale), _ptr(out), _ptr(lse), _ptr(idx_out), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _stream(stream))
    _check(rc, "dsa_forward_fused")


def dsa_forward_noalloc(q_fp8, q_scale, w, k_fp8, k_scale, q, kv, cu_seqlens_q, cu_seqlens_k, B,
                        max_len_q, max_len_k, k, sm_scale, out, lse, idx_out=None, stream=None):
    """dsa_forward without a workspace, for callers that cannot allocate device
    memory: the scratch lives in a fixed 48 MiB device array inside the
    library (see include/dsa.h).  Raises DSAError(DSA_ERR_WORKSPACE) when the
    problem's scratch exceeds it."""
    import torch
    q8 = q_fp8.view(torch.uint8) if q_fp8.dtype == torch.float8_e4m3fn else q_fp8
    k8 = k_fp8.view(torch.uint8) if k_fp8.dtype == torch.float8_e4m3fn else k_fp8
    _need(q8, torch.uint8, "q_fp8", 3)
    _need(k8, torch.uint8, "k_fp8", 2)
    _need(q, torch.bfloat16, "q", 3)
    _need(kv, torch.bfloat16, "kv", 2)
    _need(out, torch.bfloat16, "out", 3)
    _need(lse, torch.float32, "lse", 2)
    _need(idx_out, torch.int32, "idx_out", 2)
    T_q, H_I, d_I = q8.shape
    _, H, d_qk = q.shape
    rc = load().dsa_forward_noalloc(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale),
                                    _ptr(q), _ptr(kv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                    int(B), int(max_len_q), int(max_len_k), int(T_q),
                                    int(k8.shape[0]), int(H_I), int(d_I), int(H), int(d_qk),
                                    int(out.shape[2]), int(k), float(sm_scale), _ptr(out),
                                    _ptr(lse), _ptr(idx_out), _stream(stream))
    _check(rc, "dsa_forward_noalloc")


def _need_host(t, dtype, name, ndim=None):
    if t is None:
        return
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def dsa_forward_host_workspace_size(total_k, max_len_k, B, H_I, d_I, H, k, chunk_q,
                                    n_streams) -> int:
    return int(load().dsa_forward_host_workspace_size(int(total_k), int(max_len_k), int(B),
                                                      int(H_I), int(d_I), int(H), int(k),
                                                      int(chunk_q), int(n_streams)))


def dsa_forward_host(q_fp8, q_scale, w, k_fp8, k_scale, q, kv, cu_seqlens_q, cu_seqlens_k, B,
                     max_len_q, max_len_k, k, sm_scale, out, lse, chunk_q, workspace, streams):
    """dsa_forward over host tensors (pin them for the copies to overlap):
    the library uploads the key side once and the query rows in chunks of
    chunk_q rows spread over `streams` (torch.cuda.Stream objects), and returns
    with `out` / `lse` (host tensors) filled.  `workspace` is a uint8 CUDA
    tensor of dsa_forward_host_workspace_size(...) bytes."""
    import torch
    q8 = q_fp8.view(torch.uint8) if q_fp8.dtype == torch.float8_e4m3fn else q_fp8
    k8 = k_fp8.view(torch.uint8) if k_fp8.dtype == torch.float8_e4m3fn else k_fp8
    for t, dt, name, nd in ((q8, torch.uint8, "q_fp8", 3), (k8, torch.uint8, "k_fp8", 2),
                            (q_scale, torch.float32, "q_scale", 2), (w, torch.float32, "w", 2),
                            (k_scale, torch.float32, "k_scale", 1),
                            (q, torch.bfloat16, "q", 3), (kv, torch.bfloat16, "kv", 2),
                            (cu_seqlens_q, torch.int32, "cu_seqlens_q", 1),
                            (cu_seqlens_k, torch.int32, "cu_seqlens_k", 1),
                            (out, torch.bfloat16, "out", 3), (lse, torch.float32, "lse", 2)):
        _need_host(t, dt, name, nd)
    _need(workspace, torch.uint8, "workspace", 1)
    T_q, H_I, d_I = q8.shape
    _, H, d_qk = q.shape
    arr = (ctypes.c_void_p * len(streams))(*[s.cuda_stream for s in streams])
    rc = load().dsa_forward_host(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale),
                                 _ptr(q), _ptr(kv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                 int(B), int(max_len_q), int(max_len_k), int(T_q),
                                 int(k8.shape[0]), int(H_I), int(d_I), int(H), int(d_qk),
                                 int(out.shape[2]), int(k), float(sm_scale), _ptr(out),
                                 _ptr(lse), int(chunk_q), _ptr(workspace),
                                 int(workspace.numel()), arr, len(streams))
    _check(rc, "dsa_forward_host")


def dsa_indexer_kl_workspace_size(total_q, H, k) -> int:
    return int(load().dsa_indexer_kl_workspace_size(int(total_q), int(H), int(k)))


def dsa_indexer_kl(q, kv, idx, lse, logits, cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k,
                   k, sm_scale, kl_out, grad_out=None, target_out=None, workspace=None,
                   ld_logits=None, stream=None):
    """The indexer's KL training signal over each query's selection (see
    include/dsa.h): kl_out [T_q], and optionally the gradient with respect to
    the selected indexer scores and the head-averaged attention target, both
    [T_q, k] in index-row order.  `workspace` (uint8 CUDA tensor) is allocated
    here when not given."""
    import torch
    _need(q, torch.bfloat16, "q", 3)
    _need(kv, torch.bfloat16, "kv", 2)
    _need(idx, torch.int32, "idx", 2)
    _need(lse, torch.float32, "lse", 2)
    _need(kl_out, torch.float32, "kl_out", 1)
    _need(grad_out, torch.float32, "grad_out", 2)
    _need(target_out, torch.float32, "target_out", 2)
    T_q, H, d_qk = q.shape
    nbytes = dsa_indexer_kl_workspace_size(T_q, H, k)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    ld = logits.stride(0) if ld_logits is None else ld_logits
    rc = load().dsa_indexer_kl(_ptr(q), _ptr(kv), _ptr(idx), _ptr(lse), _ptr(logits), int(ld),
                               _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(B), int(max_len_q),
                               int(max_len_k), int(T_q), int(kv.shape[0]), int(H), int(d_qk),
                               int(k), float(sm_scale), _ptr(kl_out), _ptr(grad_out),
                               _ptr(target_out), _ptr(workspace), int(workspace.numel()),
                               _stream(stream))
    _check(rc, "dsa_indexer_kl")


def dsa_masked_mha_workspace_size(total_q, max_len_k) -> int:
    return int(load().dsa_masked_mha_workspace_size(int(total_q), int(max_len_k)))


def dsa_masked_mha_fwd(q, k, v, idx, cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k,
                       topk, sm_scale, out, lse=None, workspace=None, stream=None):
    """The masked MHA mode (see include/dsa.h): dense per-head attention of
    q [T_q, H, 192] over k [T_k, H, 192], v [T_k, H, 128], restricted to each
    query's selected set idx [T_q, topk]; writes out [T_q, H, 128] (bf16) and
    lse [T_q, H] (fp32, optional).  `workspace` (uint8 CUDA tensor) is
    allocated here when not given."""
    import torch
    _need(q, torch.bfloat16, "q", 3)
    _need(k, torch.bfloat16, "k", 3)
    _need(v, torch.bfloat16, "v", 3)
    _need(idx, torch.int32, "idx", 2)
    _need(out, torch.bfloat16, "out", 3)
    _need(lse, torch.float32, "lse", 2)
    T_q, H, d_qk = q.shape
    nbytes = dsa_masked_mha_workspace_size(T_q, max_len_k)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    rc = load().dsa_masked_mha_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cu_seqlens_q),
                                   _ptr(cu_seqlens_k), int(B), int(max_len_q), int(max_len_k),
                                   int(T_q), int(k.shape[0]), int(H), int(d_qk), int(v.shape[2]),
                                   int(topk), float(sm_scale), _ptr(out), _ptr(lse),
                                   _ptr(workspace), int(workspace.numel()), _stream(stream))
    _check(rc, "dsa_masked_mha_fwd")


def dsa_get_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error
    status: 0 = DSA_OK, 6 = DSA_ERR_TIMEOUT, 7 = DSA_ERR_BOUNDS."""
    return int(load().dsa_get_device_error(_stream(stream)))
