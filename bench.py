#!/usr/bin/env python
"""Benchmark of the DSA hot path: lightning indexer (FP8) -> top-2048 ->
sparse MQA-mode MLA attention, on synthetic data shaped like the headline
workload (one 32768-token prefill, H_I=64, d_I=128, H=128, 576-d latents).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole path over one batch (one sequence per GPU).
Prints ONE JSON line on rank 0.  With --gpus N > 1 it runs under torchrun,
one rank per GPU; every rank runs its own sequence (data-parallel, no
collective on the data path) and the step time is the maximum over ranks.
``--impl reference`` times the CPU oracle (oracle/, fp64, host cores) on a
bounded sample of the same workload.  ``--split-sequence`` instead splits ONE
sequence over the ranks (strong scaling): every rank holds a position shard
of the key-side cache, gathers the whole cache with one all-gather per
tensor, and runs its two zig-zag query blocks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DSA query-tokens/s (indexer+top-2048+sparse MLA) at L=32K; % roofline"
METRICS = {
    0: "DSA query-tokens/s (indexer+top-128+sparse MLA, 16 heads) at L=1K; % roofline",
    1: "DSA query-tokens/s (indexer+top-2048+sparse MLA) at L=8K; % roofline",
    2: METRIC,
    3: "DSA query-tokens/s (indexer+top-2048+sparse MLA), decode batch of 64 over 4K-131K "
       "caches; % roofline",
    4: "DSA query-tokens/s (indexer+top-2048+sparse MLA), L=128K prefill in 8 chunks of 16K; "
       "% roofline",
}
UNIT = "query-tokens/s"
EXTRA_CONFIGS = (1, 3, 4)      # measured beside the headline on the default line
L2_FLUSH_BYTES = 256 << 20
KERNEL_FILES = {
    "indexer_kernel": "sparse_attention_08_b200/csrc/indexer.cu",
    "topk_kernel": "sparse_attention_08_b200/csrc/topk.cu",
    "sparse_mla_kernel": "sparse_attention_08_b200/csrc/sparse_mla.cu",
    "attn_target_kernel": "sparse_attention_08_b200/csrc/indexer_kl.cu",
    "masked_mha_kernel": "sparse_attention_08_b200/csrc/masked_mha.cu",
}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kl", action="store_true")
    ap.add_argument("--no-mha", action="store_true")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-fused", action="store_true")
    ap.add_argument("--rows", type=int, default=0,
                    help="reference arm: query rows the oracle runs per step (default: one "
                         "per host core, at least 8)")
    ap.add_argument("--split-sequence", action="store_true")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="measure only --config, not the other full-size configs")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(cfg_id, rank):
    """Each rank runs its own sequence: rank 0 uses the workload's seed."""
    from sparse_attention_08_b200 import workloads as W
    return W.seed_of(cfg_id) + 1000 * rank


def max_over_ranks(x: float) -> float:
    """Maximum of a per-rank float over the process group (identity alone)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world: int, queries_per_rank: int, step_ms: float) -> float:
    """Whole-job query-tokens/s: every rank's queries over the slowest rank's step."""
    return world * queries_per_rank / (step_ms / 1e3)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def source_sha(kernel):
    with open(os.path.join(ROOT, KERNEL_FILES[kernel]), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """Per-launch DRAM bytes from profiles/traffic.txt, if the capture was taken
    on the current source of the kernel (null otherwise)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and \
                parts[1] == workload and parts[3] == source_sha(kernel):
            return float(parts[2])
    return None


def counts(wl):
    """Algorithmic work of one pass over the workload (one call of each stage):
    flops on the tensor cores and the bytes that must cross HBM at least once."""
    causal, attended, lat_rows = 0, 0, 0
    for nq, nk in zip(wl.lens_q, wl.lens_k):
        causal += nq * (nk - nq) + nq * (nq + 1) // 2
        for i in range(nq):
            attended += min(wl.k, nk - nq + i + 1)
        # distinct latent rows the sequence's selections can touch
        lat_rows += min(nk, nq * wl.k)
    H_I, d_I = wl.q8.shape[1], wl.q8.shape[2]
    H = wl.q.shape[1]
    T_q, T_k = wl.T_q, wl.T_k
    return {
        "causal_pairs": causal,
        "attended_pairs": attended,
        # FP8 products of the indexer contraction (2 flops per MAC)
        "indexer_flops": 2 * H_I * d_I * causal,
        # indexer queries, weights and scales in; keys and their scales in
        # once; every causal score written once
        "indexer_bytes": T_q * H_I * (d_I + 8) + T_k * (d_I + 4) + 4 * causal,
        "topk_flops": 0,
        # top-k: read every causal score once, write k indices per query
        "topk_bytes": 4 * causal + 4 * wl.k * T_q,
        # QK^T over 576 dims + PV over 512 dims for every head and attended pair
        "attention_flops": attended * H * (2 * 576 + 2 * 512),
        # queries in, outputs and lse out, indices in, every distinct latent
        # row the selections touch once (L2 serves the repeats)
        "attention_bytes": (T_q * H * (576 + 512) * 2 + T_q * H * 4 + 4 * wl.k * T_q
                            + lat_rows * 576 * 2),
    }


def add_counts(a, b):
    return {n: a[n] + b[n] for n in a}


def stage_rooflines(c, stage_ms, peaks):
    """Per stage: the bound is whichever of (tensor flops / tensor peak) and
    (HBM bytes / HBM bandwidth) takes longer; achieved is the work of that
    bound over the measured time.  Peaks are the burst figures (the kernels
    run at 1.8-1.97 GHz, as the cuBLAS burst did), FP8 at twice bf16."""
    tens = {"indexer_kernel": 2.0 * peaks["bf16_tflops"], "topk_kernel": None,
            "sparse_mla_kernel": peaks["bf16_tflops"]}
    keys = {"indexer_kernel": "indexer", "topk_kernel": "topk",
            "sparse_mla_kernel": "attention"}
    out, t_roof = {}, 0.0
    for i, n in enumerate(("indexer_kernel", "topk_kernel", "sparse_mla_kernel")):
        fl, by = c[keys[n] + "_flops"], c[keys[n] + "_bytes"]
        t_t = fl / (tens[n] * 1e12) if tens[n] else 0.0
        t_m = by / (peaks["hbm_gbs"] * 1e9)
        ms = float(stage_ms[i])
        if t_t >= t_m:
            ach, peak, unit, bound = fl / (ms / 1e3) / 1e12, tens[n], "TFLOP/s", "tensor"
        else:
            ach, peak, unit, bound = by / (ms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
        t_roof += max(t_t, t_m)
        out[n] = {"ms": round(ms, 4), "bound": bound, "achieved": round(ach, 2),
                  "peak": peak, "unit": unit, "frac": round(ach / peak, 4),
                  "roof_ms": round(max(t_t, t_m) * 1e3, 4)}
    return out, t_roof


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = f"/tmp/dsa_clocks_{os.getpid()}.csv"
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[3]) if v.lower() == "active"})
        pmax = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "power_w_max": pmax}


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def oracle_rows(L, k, n_rows, seed):
    """A stratified sample of positions of one causal prefill of length L:
    the edge positions 0, k-1, k and L-1, and one position drawn uniformly
    from each of the remaining equal-width strata of [0, L)."""
    rng = np.random.default_rng(seed)
    fixed = sorted({p for p in (0, k - 1, k, L - 1) if 0 <= p < L})
    m = max(0, n_rows - len(fixed))
    edges = np.linspace(0, L, m + 1)
    drawn = [int(rng.integers(int(edges[i]), max(int(edges[i]) + 1, int(edges[i + 1]))))
             for i in range(m)]
    return np.array(sorted(set(fixed) | set(drawn)), dtype=np.int64)


def oracle_row_cost(p, k, H_I, d_I, H):
    """Per-row work of the oracle at position p: p+1 indexer pairs and
    min(p+1, k) attended pairs, in flops."""
    p = np.asarray(p, dtype=np.float64)
    return (p + 1) * 2 * H_I * d_I + np.minimum(p + 1, k) * H * (2 * 576 + 2 * 512)


def oracle_sample(wl, n_rows, seed):
    """Runs the oracle (all host cores, one OpenMP region) on a stratified
    sample of the query rows of a one-sequence prefill and extrapolates the
    time of the whole workload with the per-row cost model.  Returns (sample
    seconds, extrapolated query-tokens/s, description)."""
    import oracle
    from tests import dsa_cases as C
    n_k = wl.lens_k[0]
    L = wl.T_q
    rows = oracle_rows(L, wl.k, n_rows, seed)
    k8, ks, kvb = C.np_(wl.k8[:n_k]), C.np_(wl.k_scale[:n_k]), C.bits(wl.kv[:n_k])
    rt = torch.as_tensor(rows, device=wl.q8.device)
    q8, qs, w = C.np_(wl.q8[rt]), C.np_(wl.q_scale[rt]), C.np_(wl.w[rt])
    qb = C.bits(wl.q[rt])
    pos = rows + (n_k - L)
    t0 = time.perf_counter()
    oracle.forward_at(q8, qs, w, k8, ks, qb, kvb, pos, wl.k, wl.scale)
    dt = time.perf_counter() - t0
    H_I, d_I, H = wl.q8.shape[1], wl.q8.shape[2], wl.q.shape[1]
    all_pos = np.arange(n_k - L, n_k)
    full = float(oracle_row_cost(all_pos, wl.k, H_I, d_I, H).sum())
    part = float(oracle_row_cost(pos, wl.k, H_I, d_I, H).sum())
    full_s = dt * full / part
    desc = (f"{len(rows)} query rows, stratified over positions 0..{L - 1} (0, k-1, k, L-1 "
            f"and one per stratum); the whole workload's time extrapolated from the sample by "
            f"the per-row flop model (p+1 indexer pairs, min(p+1,k) attended pairs): "
            f"{full_s:.0f} s")
    return dt, L / full_s, desc


def oracle_sample_decode(wl, n_rows, seed):
    """Runs the oracle on a sample of the rows of a one-query-per-sequence
    batch (each row against its own cache) and extrapolates the time of the
    whole batch with the per-row cost model.  The sample is stratified by
    cache length: the shortest and the longest row and evenly spaced ranks
    between (the seed is unused: the choice is deterministic)."""
    import oracle
    from tests import dsa_cases as C
    lens = np.array([int(wl.cu_k[b + 1]) - int(wl.cu_k[b]) for b in range(wl.B)])
    order = np.argsort(lens, kind="stable")
    pick = sorted({int(i) for i in np.linspace(0, wl.B - 1, min(n_rows, wl.B)).round()})
    rows = order[pick]
    dt = 0.0
    for b in rows:
        q0, q1, k0, k1 = C.seq_slices(wl, int(b))
        args = (C.np_(wl.q8[q0:q1]), C.np_(wl.q_scale[q0:q1]), C.np_(wl.w[q0:q1]),
                C.np_(wl.k8[k0:k1]), C.np_(wl.k_scale[k0:k1]), C.bits(wl.q[q0:q1]),
                C.bits(wl.kv[k0:k1]), np.array([k1 - k0 - 1], dtype=np.int64))
        t0 = time.perf_counter()
        oracle.forward_at(*args, wl.k, wl.scale)
        dt += time.perf_counter() - t0
    H_I, d_I, H = wl.q8.shape[1], wl.q8.shape[2], wl.q.shape[1]
    full = float(oracle_row_cost(lens - 1, wl.k, H_I, d_I, H).sum())
    part = float(oracle_row_cost(lens[rows] - 1, wl.k, H_I, d_I, H).sum())
    full_s = dt * full / part
    desc = (f"{len(rows)} of {wl.B} decode rows, stratified by cache length (shortest, longest "
            f"and evenly spaced ranks); the whole batch's time extrapolated from the sample by "
            f"the per-row flop model (n indexer pairs, min(n,k) attended pairs): "
            f"{full_s:.1f} s")
    return dt, wl.T_q / full_s, desc


def oracle_threads():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def make_workload(cfg_id, seed):
    from sparse_attention_08_b200 import workloads as W
    if W.CONFIGS[cfg_id].decode:
        return W.make_decode(cfg_id, device="cuda", seed=seed)
    return W.make_prefill(cfg_id, device="cuda", seed=seed)


class Stepper:
    """One step of the path over a workload: the three stages on one stream,
    once per chunk of a chunked prefill (each chunk's queries against the
    cache up to its end), else once over the whole batch."""

    def __init__(self, dsa, wl, stream):
        from sparse_attention_08_b200 import workloads as W
        self.dsa, self.wl, self.stream = dsa, wl, stream
        if wl.cfg.chunks > 1:
            C = wl.T_q // wl.cfg.chunks
            self.parts = [(c * C, W.chunk_of(wl, c, C)) for c in range(wl.cfg.chunks)]
        else:
            self.parts = [(0, wl)]
        H = wl.q.shape[1]
        self.ld = (wl.max_len_k + 3) // 4 * 4
        rows = max(p.T_q for _, p in self.parts)
        self.logits = torch.empty((rows, self.ld), dtype=torch.float32, device="cuda")
        self.idx = torch.empty((wl.T_q, wl.k), dtype=torch.int32, device="cuda")
        self.out = torch.empty((wl.T_q, H, 512), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((wl.T_q, H), dtype=torch.float32, device="cuda")

    def launches(self):
        return 3 * len(self.parts)

    def step(self, ev=None):
        """ev: None, or per part a list of 4 events around the three stages."""
        dsa, s = self.dsa, self.stream
        for pi, (r0, p) in enumerate(self.parts):
            e = ev[pi] if ev is not None else None
            r1 = r0 + p.T_q
            if e is not None:
                e[0].record(s)
            dsa.dsa_indexer_logits(p.q8, p.q_scale, p.w, p.k8, p.k_scale, p.cu_q, p.cu_k, p.B,
                                   p.max_len_q, p.max_len_k, self.logits, self.ld, stream=s)
            if e is not None:
                e[1].record(s)
            dsa.dsa_topk(self.logits, p.cu_q, p.cu_k, p.B, p.max_len_q, p.max_len_k, p.k,
                         self.idx[r0:r1], ld_logits=self.ld, stream=s)
            if e is not None:
                e[2].record(s)
            dsa.dsa_sparse_mla_fwd(p.q, p.kv, self.idx[r0:r1], p.cu_q, p.cu_k, p.B, p.max_len_q,
                                   p.max_len_k, p.scale, self.out[r0:r1], self.lse[r0:r1],
                                   stream=s)
            if e is not None:
                e[3].record(s)

    def counts(self):
        c = None
        for _, p in self.parts:
            c = counts(p) if c is None else add_counts(c, counts(p))
        return c


FUSED_CONFIGS = (2, 4)   # where the fused indexer + top-k is measured beside the step


def measure_fused(dsa, st, steps, warmup, flush):
    """The same step through dsa_forward_fused (indexer and top-k fused into
    two passes over the keys; results equal the step's bit for bit), once per
    chunk on the Stepper's buffers.  Returns (mean ms per step, launches per
    step)."""
    wl, s = st.wl, st.stream
    d_I = wl.q8.shape[2]
    need = max(dsa.dsa_forward_fused_workspace_size(p.T_q, p.T_k, p.B, p.max_len_k, p.k, d_I)
               for _, p in st.parts)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")

    def step():
        for r0, p in st.parts:
            r1 = r0 + p.T_q
            dsa.dsa_forward_fused(p.q8, p.q_scale, p.w, p.k8, p.k_scale, p.q, p.kv, p.cu_q,
                                  p.cu_k, p.B, p.max_len_q, p.max_len_k, p.k, p.scale,
                                  st.out[r0:r1], st.lse[r0:r1], ws, idx_out=st.idx[r0:r1],
                                  stream=s)
    for _ in range(warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        ev[i][0].record(s)
        step()
        ev[i][1].record(s)
    torch.cuda.synchronize()
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error in the fused measurement")
    del ws
    # per chunk: sample offsets, sample gather, three indexer launches (sampled,
    # compact, recompute), threshold, candidate top-k, recompute top-k, attention
    return float(np.mean([e[0].elapsed_time(e[1]) for e in ev])), 9 * len(st.parts)


def fused_entry(ms, launches, unfused_ms):
    return {"ms": round(ms, 4), "unfused_ms": round(unfused_ms, 4),
            "speedup": round(unfused_ms / ms, 4), "gpu_launches_per_step": launches,
            "what": "dsa_forward_fused: the indexer scores a 1/32 key sample for per-row "
                    "thresholds, then appends only scores above them to candidate lists that "
                    "top-k selects from; indices, outputs and lse equal the step's bit for bit"}


def measure(dsa, st, steps, warmup, flush, clocks=None, barrier=None):
    """Warm-up, then `steps` timed steps with L2 flushed before each (outside
    the events).  Returns (mean ms per step, mean ms per stage [3], clocks)."""
    for _ in range(warmup):
        flush.fill_(1.0)
        st.step()
    torch.cuda.synchronize()
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    n = len(st.parts)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
           for _ in range(steps)]
    if barrier:
        barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    for i in range(steps):
        flush.fill_(float(i))           # evicts L2 between steps (outside the events)
        st.step(evs[i])
    torch.cuda.synchronize()
    if barrier:
        barrier()
    clk = clocks.stop() if clocks else None
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error during the timed region")
    per = np.array([[sum(evs[i][pi][j].elapsed_time(evs[i][pi][j + 1]) for pi in range(n))
                     for j in range(3)] for i in range(steps)])      # ms per stage per step
    return float(per.sum(axis=1).mean()), per.mean(axis=0), clk


def config_line(cfg_id, st, step_ms, stage_ms, peaks, world):
    """Throughput and rooflines of one measured configuration."""
    c = st.counts()
    stages, t_roof = stage_rooflines(c, stage_ms, peaks)
    return c, stages, t_roof, aggregate_value(world, st.wl.T_q, step_ms)


def run_ours(args):
    import sparse_attention_08_b200 as dsa
    from sparse_attention_08_b200 import workloads as W
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dsa.load()
    cfg = W.CONFIGS[args.config]
    seed = rank_seed(args.config, rank)
    wl = make_workload(args.config, seed)
    st = Stepper(dsa, wl, torch.cuda.current_stream())
    H_I, d_I, H = wl.q8.shape[1], wl.q8.shape[2], wl.q.shape[1]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = st.stream

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    step_ms, stage_ms, clk = measure(dsa, st, args.steps, args.warmup, flush,
                                     clocks=ClockSampler(local), barrier=barrier)
    step_ms = max_over_ranks(step_ms)
    peaks = measured_peaks()
    c, stages, t_roof, value = config_line(args.config, st, step_ms, stage_ms, peaks, world)

    # ---- roofline of the dominant kernel and of the whole step
    names = ("indexer_kernel", "topk_kernel", "sparse_mla_kernel")
    dom = names[int(np.argmax(stage_ms))]
    d = stages[dom]
    sustained = peaks["bf16_tflops_sustained"]
    roofline = {"kernel": dom, "bound": d["bound"], "achieved": d["achieved"],
                "peak": d["peak"], "unit": d["unit"], "frac": d["frac"],
                "traffic": ncu_traffic(dom, cfg.name) if len(st.parts) == 1 else None,
                "peak_source": f"{peaks['source']}: burst bf16 (x2 for fp8) and HBM copy",
                "step_frac": round(t_roof * 1e3 / step_ms, 4),
                "step_roof_ms": round(t_roof * 1e3, 4),
                "stages": stages}
    if d["unit"] == "TFLOP/s":
        roofline["frac_of_sustained"] = round(
            d["achieved"] / (sustained * (2.0 if dom == "indexer_kernel" else 1.0)), 4)

    # ---- the indexer's KL training signal on the same workload (not part of
    # the step): its score products are the attention's S half, M = 128
    kl_extra = None
    bf16_peak = peaks["bf16_tflops"]
    if not args.no_kl and world == 1 and len(st.parts) == 1:
        kl = torch.empty((wl.T_q,), dtype=torch.float32, device="cuda")
        grad = torch.empty((wl.T_q, wl.k), dtype=torch.float32, device="cuda")
        ws_kl = torch.empty(max(16, dsa.dsa_indexer_kl_workspace_size(wl.T_q, H, wl.k)),
                            dtype=torch.uint8, device="cuda")

        def kl_call():
            dsa.dsa_indexer_kl(wl.q, wl.kv, st.idx, st.lse, st.logits, wl.cu_q, wl.cu_k, wl.B,
                               wl.max_len_q, wl.max_len_k, wl.k, wl.scale, kl, grad,
                               workspace=ws_kl, ld_logits=st.ld, stream=stream)
        for _ in range(3):
            kl_call()
        kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
        for e in kev:
            flush.fill_(2.0)
            e[0].record(stream)
            kl_call()
            e[1].record(stream)
        torch.cuda.synchronize()
        if dsa.dsa_get_device_error() != 0:
            raise RuntimeError("device error in the KL measurement")
        kl_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in kev]))
        s_flops = c["attended_pairs"] * H * 2 * 576
        kl_tf = s_flops / (kl_ms / 1e3) / 1e12
        kl_extra = {"ms": round(kl_ms, 4), "bound": "tensor", "achieved": round(kl_tf, 2),
                    "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(kl_tf / bf16_peak, 4),
                    "work": "S = Q K^T of every head and selected entry (2*576 flops each)",
                    "traffic": ncu_traffic("attn_target_kernel", f"{cfg.name}")}
        del ws_kl, grad

    # ---- the indexer's backward on the same workload (not part of the step):
    # dq, dw, dk of a dense score-space gradient over every causal pair (the
    # dense warm-up's case); the step's score buffer serves as that gradient
    bwd_extra = None
    if not args.no_bwd and world == 1 and len(st.parts) == 1 and H_I == 64 and d_I == 128:
        dq = torch.empty((wl.T_q, H_I, d_I), dtype=torch.float32, device="cuda")
        dw = torch.empty((wl.T_q, H_I), dtype=torch.float32, device="cuda")
        dk = torch.empty((wl.T_k, d_I), dtype=torch.float32, device="cuda")

        def bwd_call():
            dsa.dsa_indexer_backward(wl.q8, wl.q_scale, wl.w, wl.k8, wl.k_scale, st.logits,
                                     wl.cu_q, wl.cu_k, wl.B, wl.max_len_q, wl.max_len_k, dq, dw,
                                     dk, ld_g=st.ld, stream=stream)
        for _ in range(3):
            bwd_call()
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
        for e in bev:
            flush.fill_(4.0)
            e[0].record(stream)
            bwd_call()
            e[1].record(stream)
        torch.cuda.synchronize()
        if dsa.dsa_get_device_error() != 0:
            raise RuntimeError("device error in the indexer backward measurement")
        b_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in bev]))
        # per causal pair: the FP8 gates twice (dq/dw pass and dk pass) and two
        # bf16 gated sums, each 2*H_I*d_I flops; FP8 counted at half weight
        # against the bf16 peak (it runs at twice the rate)
        b_flops = c["causal_pairs"] * 2 * H_I * d_I * (1 + 2)
        b_tf = b_flops / (b_ms / 1e3) / 1e12
        bwd_extra = {"ms": round(b_ms, 4), "bound": "tensor", "achieved": round(b_tf, 2),
                     "peak": bf16_peak, "unit": "TFLOP/s (bf16-equivalent)",
                     "frac": round(b_tf / bf16_peak, 4),
                     "work": "per causal pair: two FP8 gate products (half weight) and two "
                             "bf16 gated sums, 2*H_I*d_I flops each",
                     "traffic": None}
        del dq, dw, dk

    # ---- the masked MHA short-prefill mode (not part of the step): dense
    # per-head attention over the selection, on its own short-prefill workload
    mha_extra = None
    if not args.no_mha and world == 1:
        L_m = 4096
        mh = W.make_mha([L_m], None, H=128, topk=2048, device="cuda")
        m_out = torch.empty((mh.T_q, 128, W.D_V_MHA), dtype=torch.bfloat16, device="cuda")
        m_lse = torch.empty((mh.T_q, 128), dtype=torch.float32, device="cuda")
        m_ws = torch.empty(dsa.dsa_masked_mha_workspace_size(mh.T_q, L_m), dtype=torch.uint8,
                           device="cuda")

        def mha_call():
            dsa.dsa_masked_mha_fwd(mh.q, mh.k, mh.v, mh.idx, mh.cu_q, mh.cu_k, 1, L_m, L_m,
                                   mh.topk, mh.scale, m_out, m_lse, workspace=m_ws, stream=stream)
        for _ in range(3):
            mha_call()
        mev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(5)]
        for e in mev:
            flush.fill_(3.0)
            e[0].record(stream)
            mha_call()
            e[1].record(stream)
        torch.cuda.synchronize()
        if dsa.dsa_get_device_error() != 0:
            raise RuntimeError("device error in the masked MHA measurement")
        m_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in mev]))
        # dense causal attention: every (query, earlier key) pair of every head
        m_flops = L_m * (L_m + 1) / 2 * 128 * 2 * (W.D_QK_MHA + W.D_V_MHA)
        m_tf = m_flops / (m_ms / 1e3) / 1e12
        mha_extra = {"workload": f"short prefill L={L_m}, H=128, d_qk=192, d_v=128, topk=2048",
                     "ms": round(m_ms, 4), "bound": "tensor", "achieved": round(m_tf, 2),
                     "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(m_tf / bf16_peak, 4),
                     "work": "causal pairs x heads x 2*(192+128) flops",
                     "traffic": ncu_traffic("masked_mha_kernel", f"mha-L{L_m}")}
        del mh, m_out, m_lse, m_ws

    # ---- end to end through the host-buffer entry point
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0 and len(st.parts) == 1:
        e2e = run_e2e(dsa, wl, args, world, local, stream)

    # ---- CPU baseline: the oracle, rank 0 at N=1 only
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline and not cfg.decode:
        n_rows = max(20, min(64, 2 * oracle_threads()))
        dt, v, desc = oracle_sample(wl, n_rows, seed=99)
        cpu = {"value": round(v, 4), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
               "sample": desc, "seconds": round(dt, 2)}

    line = {
        "metric": METRICS[args.config], "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8e4m3+bf16", "data": "synthetic",
        "config": {"workload": f"{cfg.name} (" + ("one varlen decode batch" if cfg.decode else
                                                  "one causal prefill") + " per GPU)",
                   "L": cfg.L, "H_I": H_I, "d_I": d_I, "H": H, "d_qk": 576, "d_v": 512,
                   "k": wl.k, "chunks": cfg.chunks, "global_batch_sequences": world * wl.B,
                   "parallelism": f"dp{world}",
                   "l2": "flushed between steps (256 MiB write outside the timed events)"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": st.launches() * args.steps, "clocks": clk,
        "indexer_kl": kl_extra,
        "indexer_backward": bwd_extra,
        "masked_mha": mha_extra,
    }
    if not args.no_fused and world == 1 and args.config in FUSED_CONFIGS:
        f_steps = max(3, min(args.steps, 5))
        f_ms, f_l = measure_fused(dsa, st, f_steps, 3, flush)
        line["fused_indexer_topk"] = fused_entry(f_ms, f_l, step_ms)
        line["gpu_launches"] += f_l * f_steps
    del st, wl

    # ---- the other full-size configurations at one GPU, each with its own
    # metric and per-stage rooflines (fewer timed steps; same timing rules)
    if world == 1 and not args.no_extra_configs:
        extra = {}
        for cid in EXTRA_CONFIGS:
            if cid == args.config:
                continue
            torch.cuda.empty_cache()
            xw = make_workload(cid, rank_seed(cid, rank))
            xs = Stepper(dsa, xw, stream)
            x_steps = max(3, min(args.steps, 5))
            xms, xstage, xclk = measure(dsa, xs, x_steps, 3, flush, clocks=ClockSampler(local))
            xc, xstages, xroof, xval = config_line(cid, xs, xms, xstage, peaks, 1)
            xcfg = W.CONFIGS[cid]
            extra[xcfg.name] = {
                "metric": METRICS[cid], "value": round(xval, 1), "unit": UNIT,
                "ms_per_step": round(xms, 4), "steps": x_steps, "warmup": 3,
                "queries_per_step": xw.T_q, "chunks": xcfg.chunks,
                "step_frac": round(xroof * 1e3 / xms, 4), "step_roof_ms": round(xroof * 1e3, 4),
                "stages": xstages, "gpu_launches": xs.launches() * x_steps, "clocks": xclk}
            if not args.no_fused and cid in FUSED_CONFIGS:
                f_ms, f_l = measure_fused(dsa, xs, x_steps, 3, flush)
                extra[xcfg.name]["fused_indexer_topk"] = fused_entry(f_ms, f_l, xms)
                extra[xcfg.name]["gpu_launches"] += f_l * x_steps
            del xs, xw
        line["configs"] = extra
        line["gpu_launches"] += sum(v["gpu_launches"] for v in extra.values())

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


E2E_CHUNK = 1024        # query rows per chunk of the host-buffer pipeline
E2E_STREAMS = 3


def run_e2e(dsa, wl, args, world, local, stream):
    """The same step through dsa_forward_host: inputs in pinned host memory,
    outputs back in pinned host memory, every copy inside the timed region
    (the call returns once the outputs are in host memory)."""
    names = ("q8", "q_scale", "w", "k8", "k_scale", "q", "kv", "cu_q", "cu_k")
    host = {n: getattr(wl, n).cpu().contiguous().pin_memory() for n in names}
    H = wl.q.shape[1]
    H_I, d_I = wl.q8.shape[1], wl.q8.shape[2]
    out_h = torch.empty((wl.T_q, H, 512), dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty((wl.T_q, H), dtype=torch.float32).pin_memory()
    nbytes = dsa.dsa_forward_host_workspace_size(wl.T_k, wl.max_len_k, wl.B, H_I, d_I, H, wl.k,
                                                 E2E_CHUNK, E2E_STREAMS)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    streams = [torch.cuda.Stream() for _ in range(E2E_STREAMS)]
    h2d = sum(t.numel() * t.element_size() for n, t in host.items())
    d2h = out_h.numel() * 2 + lse_h.numel() * 4

    def one(ev=None):
        if ev is not None:
            ev[0].record(streams[0])
        dsa.dsa_forward_host(host["q8"], host["q_scale"], host["w"], host["k8"],
                             host["k_scale"], host["q"], host["kv"], host["cu_q"], host["cu_k"],
                             wl.B, wl.max_len_q, wl.max_len_k, wl.k, wl.scale, out_h, lse_h,
                             E2E_CHUNK, ws, streams)
        if ev is not None:
            ev[1].record(streams[0])

    one()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.e2e_steps)]
    for i in range(args.e2e_steps):
        one(evs[i])
    torch.cuda.synchronize()
    ms = max_over_ranks(float(np.mean([e[0].elapsed_time(e[1]) for e in evs])))
    return {"value": round(aggregate_value(world, wl.T_q, ms), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms, 3), "steps": args.e2e_steps, "api": "dsa_forward_host",
            "chunk_rows": E2E_CHUNK, "streams": E2E_STREAMS}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------

def run_split(args):
    """One prefill split over the ranks by zig-zag query blocks (strong
    scaling); the key-side cache arrives sharded by position and is gathered
    inside the timed step."""
    import sparse_attention_08_b200 as dsa
    from sparse_attention_08_b200 import sharding as S
    from sparse_attention_08_b200 import workloads as W
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dsa.load()
    cfg = W.CONFIGS[args.config]
    if cfg.decode or cfg.B != 1:
        raise SystemExit("--split-sequence splits one prefill sequence")
    wl = W.make_prefill(args.config, device="cuda", seed=W.seed_of(args.config))
    L, H = wl.T_q, wl.q.shape[1]
    k0, k1 = S.key_shard(L, world, rank)
    shard = [wl.k8[k0:k1].clone(), wl.k_scale[k0:k1].clone(), wl.kv[k0:k1].clone()]
    full = [torch.empty_like(wl.k8), torch.empty_like(wl.k_scale), torch.empty_like(wl.kv)]
    blocks = S.zigzag_blocks(L, world, rank)
    args_b = [S.block_args(q0, q1) for q0, q1 in blocks]
    cus = [(torch.tensor(a["cu_q"], dtype=torch.int32, device="cuda"),
            torch.tensor(a["cu_k"], dtype=torch.int32, device="cuda")) for a in args_b]
    ws = torch.empty(max(dsa.dsa_forward_workspace_size(a["max_len_q"], a["max_len_k"], wl.k)
                         for a in args_b), dtype=torch.uint8, device="cuda")
    out = torch.empty((L, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((L, H), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        if world > 1:
            for loc, dst in zip(shard, full):
                dst.copy_(S.all_gather_rows(loc))
        else:
            for loc, dst in zip(shard, full):
                dst.copy_(loc)
        for a, (cq, ck) in zip(args_b, cus):
            r, kr = a["q_rows"], a["key_rows"]
            dsa.dsa_forward(wl.q8[r], wl.q_scale[r], wl.w[r], full[0][kr], full[1][kr], wl.q[r],
                            full[2][kr], cq, ck, 1, a["max_len_q"], a["max_len_k"], wl.k, wl.scale,
                            out[r], lse[r], ws, stream=stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error during the timed region")
    step_ms = max_over_ranks(float(np.mean([e[0].elapsed_time(e[1]) for e in evs])))
    value = L / (step_ms / 1e3)
    if rank == 0:
        print(json.dumps({
            "metric": METRICS[args.config], "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "fp8e4m3+bf16", "data": "synthetic",
            "config": {"workload": f"{cfg.name} (one causal prefill split over the GPUs)",
                       "L": L, "parallelism": f"zigzag{world}",
                       "exchange": "one all-gather per key-side tensor inside the step",
                       "l2": "flushed between steps (256 MiB write outside the timed events)"},
            "gpu_launches": 3 * len(blocks) * args.steps, "clocks": clk}), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    from sparse_attention_08_b200 import workloads as W
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cfg = W.CONFIGS[args.config]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if cfg.decode:
        wl = W.make_decode(args.config, device=dev)
        sample = oracle_sample_decode
    else:
        wl = W.make_prefill(args.config, device=dev)
        sample = oracle_sample
    n_rows = args.rows if args.rows else max(8, oracle_threads())
    for i in range(args.warmup):
        sample(wl, max(4, n_rows // 4), seed=1000 + i)
    secs, vals = [], []
    for i in range(args.steps):
        dt, v, desc = sample(wl, n_rows, seed=i)
        secs.append(dt)
        vals.append(v)
    step_s = float(np.mean(secs))
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRICS[args.config], "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name} (" + ("one varlen decode batch" if cfg.decode else
                                                  "one causal prefill") + ")",
                   "L": cfg.L, "k": cfg.k,
                   "H": cfg.H, "H_I": cfg.H_I, "d_I": cfg.d_I,
                   "step": f"{n_rows} stratified query rows per step; value extrapolated to "
                           f"the whole workload by the per-row flop model"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.split_sequence:
        run_split(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
