"""Host logic of bench.py on CPU: the work counts behind every roofline
fraction, the stage bounds, the oracle's row sampling and cost model, and
the reported fused entry.  The counts are checked against brute-force loops
over the causal pairs, so a wrong term in the formulas would show here."""
import numpy as np
import pytest

import bench
from sparse_attention_08_b200 import workloads as W


def _brute_counts(lens_q, lens_k, k):
    causal = attended = 0
    for nq, nk in zip(lens_q, lens_k):
        for i in range(nq):
            p = nk - nq + i
            causal += p + 1
            attended += min(k, p + 1)
    return causal, attended


@pytest.mark.parametrize("lens,lens_q,k", [([300], None, 64), ([700, 300], [700, 45], 128),
                                           ([5, 260, 1000], [1, 1, 1], 64)])
def test_counts_match_brute_force(lens, lens_q, k):
    wl = W.make_small(H_I=64, d_I=128, H=16, lens=lens, lens_q=lens_q, k=k, seed=1)
    c = bench.counts(wl)
    causal, attended = _brute_counts(wl.lens_q, wl.lens_k, k)
    assert c["causal_pairs"] == causal
    assert c["attended_pairs"] == attended
    assert c["indexer_flops"] == 2 * 64 * 128 * causal
    assert c["attention_flops"] == attended * 16 * (2 * 576 + 2 * 512)
    # top-k reads every causal score once and writes k indices per query
    assert c["topk_bytes"] == 4 * causal + 4 * k * wl.T_q
    assert c["topk_flops"] == 0


def test_counts_add_over_chunks():
    wl = W.make_small(H_I=64, d_I=128, H=16, lens=[1200], k=64, seed=2)
    a = W.make_small(H_I=64, d_I=128, H=16, lens=[1200], lens_q=[600], k=64, seed=2)
    whole = bench.counts(wl)
    # the first 600 queries as a chunk of a 600-key cache, then the rest
    first = W.make_small(H_I=64, d_I=128, H=16, lens=[600], k=64, seed=2)
    both = bench.add_counts(bench.counts(first), bench.counts(a))
    assert both["causal_pairs"] == whole["causal_pairs"]
    assert both["attended_pairs"] == whole["attended_pairs"]


def test_stage_rooflines_pick_the_slower_bound():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    c = {"indexer_flops": 2e12, "indexer_bytes": 1e9,       # 10 ms of FP8 vs 1 ms of HBM
         "topk_flops": 0, "topk_bytes": 2e9,                # 2 ms of HBM
         "attention_flops": 1e12, "attention_bytes": 2e10}  # 10 ms of bf16 vs 20 ms of HBM
    out, t_roof = bench.stage_rooflines(c, [20.0, 4.0, 40.0], peaks)
    assert out["indexer_kernel"]["bound"] == "tensor"
    assert out["indexer_kernel"]["peak"] == 200.0             # FP8 at twice bf16
    assert out["indexer_kernel"]["frac"] == pytest.approx(0.5)
    assert out["topk_kernel"]["bound"] == "hbm"
    assert out["topk_kernel"]["frac"] == pytest.approx(0.5)
    assert out["sparse_mla_kernel"]["bound"] == "hbm"
    assert out["sparse_mla_kernel"]["frac"] == pytest.approx(0.5)
    assert t_roof == pytest.approx(0.010 + 0.002 + 0.020)


def test_oracle_rows_are_stratified():
    L, k = 32768, 2048
    rows = bench.oracle_rows(L, k, 512, seed=3)
    assert rows.dtype == np.int64
    assert np.all(np.diff(rows) > 0) and rows[0] >= 0 and rows[-1] < L
    for p in (0, k - 1, k, L - 1):
        assert p in rows
    # at least one row in each of the equal-width strata [floor(e_i), floor(e_i+1))
    edges = np.floor(np.linspace(0, L, 512 - 4 + 1)).astype(np.int64)
    for lo, hi in zip(edges[:-1], edges[1:]):
        assert np.any((rows >= lo) & (rows < max(hi, lo + 1))), (lo, hi)
    assert len(rows) <= 512
    assert np.array_equal(rows, bench.oracle_rows(L, k, 512, seed=3))


def test_oracle_row_cost_model():
    k, H_I, d_I, H = 2048, 64, 128, 128
    p = np.array([0, k - 1, k, 32767])
    got = bench.oracle_row_cost(p, k, H_I, d_I, H)
    for pi, g in zip(p, got):
        assert g == (pi + 1) * 2 * H_I * d_I + min(pi + 1, k) * H * (2 * 576 + 2 * 512)


def test_fused_entry_reports_the_ratio():
    e = bench.fused_entry(30.0, 9, 33.0)
    assert e["ms"] == 30.0 and e["unfused_ms"] == 33.0
    assert e["speedup"] == pytest.approx(1.1)
    assert e["gpu_launches_per_step"] == 9


def test_every_config_has_a_metric():
    for cid in W.CONFIGS:
        assert cid in bench.METRICS
    for cid in bench.EXTRA_CONFIGS + bench.FUSED_CONFIGS:
        assert cid in W.CONFIGS
