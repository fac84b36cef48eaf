"""Shared helpers for the parity tests: run the CUDA path through the C ABI,
run the oracle on the same inputs, and compare under the parity rules.

Parity rules (kernel vs oracle on the same seeded inputs):
* indexer: integer-valued inputs must match exactly; real-valued inputs must
  satisfy |g - o| <= 2^-16 * B, with B = k_scale * sum_j |w q_scale| |q8|.|k8|
  the sum of the magnitudes the fp32 arithmetic touches (a few hundred fp32
  ulps of B);
* top-k on the SAME fp32 scores: bit-exact index sets and order;
* end-to-end top-k (GPU fp32 scores vs oracle fp64 scores): the sets agree
  except for entries whose oracle score lies within 1e-3 * |k-th score| of the
  cut, and both sides keep the same count;
* attention (oracle fed the GPU's indices): relative L2 error <= 5e-3 and max
  abs error <= 2e-2 over the output; lse within 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_attention_08_b200 as dsa

ATT_REL_L2 = 5e-3
ATT_MAX_ABS = 2e-2
LSE_ABS = 1e-3
NEAR_CUT_REL = 1e-3
IDX_TOL = 2.0 ** -16


def np_(t):
    return t.detach().cpu().numpy()


def bits(t_bf16):
    return np_(t_bf16.contiguous().view(torch.int16)).view(np.uint16)


def seq_slices(wl, b):
    q0, q1 = int(wl.cu_q[b]), int(wl.cu_q[b + 1])
    k0, k1 = int(wl.cu_k[b]), int(wl.cu_k[b + 1])
    return q0, q1, k0, k1


def ld_of(wl):
    return (wl.max_len_k + 3) // 4 * 4


# ---------------------------------------------------------------------------
# GPU side (through the C ABI)
# ---------------------------------------------------------------------------

def gpu_indexer(wl, fill=float("nan")):
    ld = ld_of(wl)
    logits = torch.full((wl.T_q, ld), fill, dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_logits(wl.q8, wl.q_scale, wl.w, wl.k8, wl.k_scale, wl.cu_q, wl.cu_k, wl.B,
                           wl.max_len_q, wl.max_len_k, logits, ld)
    return logits


def gpu_topk(wl, logits, with_val=True):
    idx = torch.full((wl.T_q, wl.k), -7, dtype=torch.int32, device="cuda")
    val = torch.empty((wl.T_q, wl.k), dtype=torch.float32, device="cuda") if with_val else None
    dsa.dsa_topk(logits, wl.cu_q, wl.cu_k, wl.B, wl.max_len_q, wl.max_len_k, wl.k, idx, val,
                 ld_logits=logits.stride(0))
    return idx, val


def gpu_attention(wl, idx):
    out = torch.full((wl.T_q, wl.q.shape[1], 512), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    lse = torch.full((wl.T_q, wl.q.shape[1]), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_mla_fwd(wl.q, wl.kv, idx, wl.cu_q, wl.cu_k, wl.B, wl.max_len_q, wl.max_len_k,
                           wl.scale, out, lse)
    return out, lse


def gpu_forward(wl):
    H = wl.q.shape[1]
    out = torch.empty((wl.T_q, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.T_q, H), dtype=torch.float32, device="cuda")
    idx = torch.empty((wl.T_q, wl.k), dtype=torch.int32, device="cuda")
    nbytes = dsa.dsa_forward_workspace_size(wl.T_q, wl.max_len_k, wl.k)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dsa.dsa_forward(wl.q8, wl.q_scale, wl.w, wl.k8, wl.k_scale, wl.q, wl.kv, wl.cu_q, wl.cu_k,
                    wl.B, wl.max_len_q, wl.max_len_k, wl.k, wl.scale, out, lse, ws, idx_out=idx)
    return idx, out, lse


def assert_no_device_error():
    torch.cuda.synchronize()            # surfaces a CUDA fault with its message
    st = dsa.dsa_get_device_error()
    assert st == 0, f"device error status {st}"


# ---------------------------------------------------------------------------
# Oracle side (CPU, fp64)
# ---------------------------------------------------------------------------

def oracle_scores(wl_cpu, b, rows=None, abs_bound=False):
    """Oracle indexer scores for sequence b (rows = local query rows)."""
    q0, q1, k0, k1 = seq_slices(wl_cpu, b)
    q8, k8 = np_(wl_cpu.q8[q0:q1]), np_(wl_cpu.k8[k0:k1])
    w = np_(wl_cpu.w[q0:q1])
    if abs_bound:
        q8 = q8 & 0x7F
        k8 = k8 & 0x7F
        w = np.abs(w)
    return oracle.indexer(q8, np_(wl_cpu.q_scale[q0:q1]), w, k8, np_(wl_cpu.k_scale[k0:k1]),
                          rows=rows)


def oracle_attention(wl_cpu, b, idx_rows, rows):
    q0, q1, k0, k1 = seq_slices(wl_cpu, b)
    return oracle.sparse_mla(bits(wl_cpu.q[q0:q1]), bits(wl_cpu.kv[k0:k1]), idx_rows, k1 - k0,
                             wl_cpu.scale, rows=rows)


# ---------------------------------------------------------------------------
# Comparisons
# ---------------------------------------------------------------------------

def check_indexer(g_rows, o_rows, bound_rows, p_of_row, exact=False):
    for r in range(g_rows.shape[0]):
        p = p_of_row[r]
        g = g_rows[r, : p + 1].astype(np.float64)
        o = o_rows[r, : p + 1]
        if exact:
            assert np.array_equal(g, o), f"row {r}: first diff at " \
                f"{int(np.flatnonzero(g != o)[0]) if np.any(g != o) else -1}"
        else:
            tol = IDX_TOL * bound_rows[r, : p + 1] + 1e-30
            bad = np.abs(g - o) > tol
            assert not np.any(bad), (f"row {r}: {int(bad.sum())} scores out of tolerance; "
                                     f"worst {np.max(np.abs(g - o) - tol)}")


def check_topk_near_cut(g_idx, o_idx, o_scores, p_of_row, k):
    """North-star rule: equal sets except near-cut entries; same counts."""
    for r in range(g_idx.shape[0]):
        p = p_of_row[r]
        m = min(k, p + 1)
        G = set(int(x) for x in g_idx[r] if x >= 0)
        O = set(int(x) for x in o_idx[r] if x >= 0)
        assert len(G) == len(O) == m, (r, len(G), len(O), m)
        assert list(g_idx[r, :m]) == sorted(G) and np.all(g_idx[r, m:] == -1)
        if G == O:
            continue
        sc = o_scores[r, : p + 1]
        vk = np.sort(sc)[::-1][m - 1]
        band = NEAR_CUT_REL * abs(vk)
        for s in G ^ O:
            assert abs(sc[s] - vk) <= band, (r, s, sc[s], vk)


def check_attention(g_out, o_out, g_lse=None, o_lse=None):
    g = g_out.astype(np.float64)
    diff = g - o_out
    rel = np.linalg.norm(diff) / max(np.linalg.norm(o_out), 1e-300)
    mx = float(np.max(np.abs(diff))) if diff.size else 0.0
    assert rel <= ATT_REL_L2, f"relative L2 {rel:.3e} > {ATT_REL_L2}"
    assert mx <= ATT_MAX_ABS, f"max abs {mx:.3e} > {ATT_MAX_ABS}"
    if g_lse is not None:
        d = np.abs(g_lse.astype(np.float64) - o_lse)
        assert float(np.max(d)) <= LSE_ABS, f"lse max abs {float(np.max(d)):.3e}"
    return rel, mx
