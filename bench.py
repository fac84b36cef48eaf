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
UNIT = "query-tokens/s"
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
    ap.add_argument("--split-sequence", action="store_true")
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
    """Algorithmic work of one pass over the workload."""
    causal, attended = 0, 0
    for nq, nk in zip(wl.lens_q, wl.lens_k):
        causal += nq * (nk - nq) + nq * (nq + 1) // 2
        for i in range(nq):
            attended += min(wl.k, nk - nq + i + 1)
    H_I, d_I = wl.q8.shape[1], wl.q8.shape[2]
    H = wl.q.shape[1]
    return {
        "causal_pairs": causal,
        "attended_pairs": attended,
        # FP8 products of the indexer contraction (2 flops per MAC)
        "indexer_flops": 2 * H_I * d_I * causal,
        # QK^T over 576 dims + PV over 512 dims for every head and attended pair
        "attention_flops": attended * H * (2 * 576 + 2 * 512),
        # top-k: read every causal score once, write k indices per query
        "topk_bytes": 4 * causal + 4 * wl.k * sum(wl.lens_q),
    }


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

def oracle_sample(wl, n_rows, seed):
    """Runs the oracle on n_rows query rows drawn uniformly over positions (all
    host cores, one OpenMP region); returns (elapsed seconds, description)."""
    import oracle
    from tests import dsa_cases as C
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(wl.T_q, size=n_rows, replace=False)).astype(np.int64)
    n_k = wl.lens_k[0]
    k8, ks, kvb = C.np_(wl.k8[:n_k]), C.np_(wl.k_scale[:n_k]), C.bits(wl.kv[:n_k])
    rt = torch.as_tensor(rows, device=wl.q8.device)
    q8, qs, w = C.np_(wl.q8[rt]), C.np_(wl.q_scale[rt]), C.np_(wl.w[rt])
    qb = C.bits(wl.q[rt])
    pos = rows + (n_k - wl.T_q)
    t0 = time.perf_counter()
    oracle.forward_at(q8, qs, w, k8, ks, qb, kvb, pos, wl.k, wl.scale)
    dt = time.perf_counter() - t0
    return dt, f"{n_rows} query rows drawn uniformly over positions 0..{wl.T_q - 1}"


def oracle_threads():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

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
    if cfg.decode:
        # a varlen decode batch (not the headline; a measurement of that shape)
        wl = W.make_decode(args.config, device="cuda", seed=seed)
    else:
        wl = W.make_prefill(args.config, device="cuda", seed=seed)
    H_I, d_I, H = wl.q8.shape[1], wl.q8.shape[2], wl.q.shape[1]
    ld = (wl.max_len_k + 3) // 4 * 4
    logits = torch.empty((wl.T_q, ld), dtype=torch.float32, device="cuda")
    idx = torch.empty((wl.T_q, wl.k), dtype=torch.int32, device="cuda")
    out = torch.empty((wl.T_q, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.T_q, H), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dsa.dsa_indexer_logits(wl.q8, wl.q_scale, wl.w, wl.k8, wl.k_scale, wl.cu_q, wl.cu_k, wl.B,
                               wl.max_len_q, wl.max_len_k, logits, ld, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        dsa.dsa_topk(logits, wl.cu_q, wl.cu_k, wl.B, wl.max_len_q, wl.max_len_k, wl.k, idx,
                     ld_logits=ld, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        dsa.dsa_sparse_mla_fwd(wl.q, wl.kv, idx, wl.cu_q, wl.cu_k, wl.B, wl.max_len_q,
                               wl.max_len_k, wl.scale, out, lse, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.fill_(float(i))           # evicts L2 between steps (outside the events)
        step(evs[i])
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error during the timed region")
    st = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)]
                   for i in range(args.steps)])             # ms per stage per step
    step_ms = float(st.sum(axis=1).mean())
    stage_ms = st.mean(axis=0)
    step_ms = max_over_ranks(step_ms)
    value = aggregate_value(world, wl.T_q, step_ms)

    # ---- roofline of the dominant kernel and of the whole step
    peaks = measured_peaks()
    c = counts(wl)
    fp8_peak = 2.0 * peaks["bf16_tflops_sustained"]     # nominal fp8:bf16 ratio 2
    bf16_peak = peaks["bf16_tflops_sustained"]
    names = ("indexer_kernel", "topk_kernel", "sparse_mla_kernel")
    per = {
        "indexer_kernel": ("tensor", c["indexer_flops"] / (stage_ms[0] / 1e3) / 1e12, fp8_peak,
                           "TFLOP/s"),
        "topk_kernel": ("hbm", c["topk_bytes"] / (stage_ms[1] / 1e3) / 1e9, peaks["hbm_gbs"],
                        "GB/s"),
        "sparse_mla_kernel": ("tensor", c["attention_flops"] / (stage_ms[2] / 1e3) / 1e12,
                              bf16_peak, "TFLOP/s"),
    }
    dom = names[int(np.argmax(stage_ms))]
    bound, ach, peak, unit = per[dom]
    workload_name = f"{cfg.name}"
    roofline = {"kernel": dom, "bound": bound, "achieved": round(ach, 2), "peak": peak,
                "unit": unit, "frac": round(ach / peak, 4),
                "traffic": ncu_traffic(dom, workload_name),
                "peak_source": f"{peaks['source']} (sustained bf16" +
                               (", x2 for fp8)" if dom == "indexer_kernel" else ")")}
    t_roof = (c["indexer_flops"] / (fp8_peak * 1e12) + c["topk_bytes"] / (peaks["hbm_gbs"] * 1e9)
              + c["attention_flops"] / (bf16_peak * 1e12))
    roofline["step_frac"] = round(t_roof * 1e3 / step_ms, 4)
    roofline["stages"] = {n: {"ms": round(float(stage_ms[i]), 4), "bound": per[n][0],
                              "achieved": round(per[n][1], 2), "peak": per[n][2],
                              "unit": per[n][3], "frac": round(per[n][1] / per[n][2], 4)}
                          for i, n in enumerate(names)}

    # ---- the indexer's KL training signal on the same workload (not part of
    # the step): its score products are the attention's S half, M = 128
    kl_extra = None
    if not args.no_kl and world == 1:
        kl = torch.empty((wl.T_q,), dtype=torch.float32, device="cuda")
        grad = torch.empty((wl.T_q, wl.k), dtype=torch.float32, device="cuda")
        ws_kl = torch.empty(max(16, dsa.dsa_indexer_kl_workspace_size(wl.T_q, H, wl.k)),
                            dtype=torch.uint8, device="cuda")

        def kl_call():
            dsa.dsa_indexer_kl(wl.q, wl.kv, idx, lse, logits, wl.cu_q, wl.cu_k, wl.B,
                               wl.max_len_q, wl.max_len_k, wl.k, wl.scale, kl, grad,
                               workspace=ws_kl, ld_logits=ld, stream=stream)
        for _ in range(2):
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
        kl_extra = {"ms": round(kl_ms, 4), "bound": "tensor",
                    "achieved": round(s_flops / (kl_ms / 1e3) / 1e12, 2), "peak": bf16_peak,
                    "unit": "TFLOP/s", "frac": round(s_flops / (kl_ms / 1e3) / 1e12 / bf16_peak, 4),
                    "work": "S = Q K^T of every head and selected entry (2*576 flops each)",
                    "traffic": ncu_traffic("attn_target_kernel", f"{cfg.name}")}
        del ws_kl, grad

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

    # ---- end to end through dsa_forward with host buffers
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        e2e = run_e2e(dsa, wl, args, world, local, stream)

    # ---- CPU baseline: the oracle, rank 0 at N=1 only
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline and not cfg.decode:
        n_rows = max(8, min(64, 2 * oracle_threads()))
        dt, desc = oracle_sample(wl, n_rows, seed=99)
        cpu = {"value": round(n_rows / dt, 4), "unit": UNIT, "cores": oracle_threads(),
               "kind": "oracle", "sample": desc, "seconds": round(dt, 2)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8e4m3+bf16", "data": "synthetic",
            "config": {"workload": f"{cfg.name} (" + ("one varlen decode batch" if cfg.decode else "one causal prefill") + " per GPU)", "L": cfg.L,
                       "H_I": H_I, "d_I": d_I, "H": H, "d_qk": 576, "d_v": 512, "k": wl.k,
                       "global_batch_sequences": world, "parallelism": f"dp{world}",
                       "l2": "flushed between steps (256 MiB write outside the timed events)"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 3 * args.steps, "clocks": clk,
            "indexer_kl": kl_extra,
            "masked_mha": mha_extra,
        }
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
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
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
    wl = W.make_prefill(args.config, device=dev)
    n_rows = max(4, oracle_threads())
    for i in range(args.warmup):
        oracle_sample(wl, max(1, n_rows // 4), seed=1000 + i)
    secs = []
    for i in range(args.steps):
        dt, desc = oracle_sample(wl, n_rows, seed=i)
        secs.append(dt)
    step_s = float(np.mean(secs))
    value = n_rows / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name} (one causal prefill)", "L": cfg.L, "k": cfg.k,
                   "H": cfg.H, "H_I": cfg.H_I, "d_I": cfg.d_I,
                   "step": f"{n_rows} sampled query rows per step"},
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
