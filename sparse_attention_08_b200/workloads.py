"""Seeded synthetic workloads for the DSA hot path.

This module only draws inputs.  It holds none of the method's arithmetic (no
indexer score, selection or attention); the CUDA library and the CPU oracle
both consume what it produces.  The one numeric step besides drawing random
numbers is the FP8 quantisation of the indexer queries and keys, which the
workload definition itself prescribes (per-token absmax scale, e4m3 bytes);
it uses torch's own float32 -> float8_e4m3fn conversion, and the bytes it
yields are shared inputs, read identically by both sides.

Shapes follow the DSA setting of the pages ("DeepSeek V3.2 and the lightning
indexer", section "How the lightning indexer works": FP8 indexer, top 2,048
per query, MQA-mode MLA latents shared by all heads).  The latent width
(512 content + 64 RoPE), the head counts and the distributions are the
workload definitions of this project:

=====  =================================================================
cfg    shape / distribution
=====  =================================================================
0      B=1, L=1024, H_I=4, d_I=64, k=128, H=16.  q_I, k_I: integers in
       [-4, 4] held exactly in e4m3, scale 1; w: integers in [-2, 2].
1      B=1, L=8192, H_I=64, d_I=128, k=2048, H=128.  q_I, k_I ~ N(0,1)
       with 32 planted positions per query, per-token absmax e4m3;
       w ~ N(0, variance 1/64).
2      as 1 with L=32768 (headline).
3      decode: B=64 sequences, one query each, cache length
       U{4096..131072}; 32 plants per query.
4      L=131072 as 8 chunks of 16384 queries against the growing cache.
=====  =================================================================

Every config: latents c ~ N(0,1) bf16 [T_k, 576]; queries q ~ N(0,1)/24 bf16
[T_q, H, 576]; softmax scale 1/sqrt(576).  Seeds: 20251202 + 100*cfg + chunk.
Draw order: q_I, k_I, w, plants, latents, q.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

D_QK = 576
D_V = 512
E4M3_MAX = 448.0
BASE_SEED = 20251202


@dataclass(frozen=True)
class Config:
    """One workload shape."""
    name: str
    B: int
    L: int                 # prefill length (or max cache length for decode)
    H_I: int
    d_I: int
    H: int
    k: int
    integer: bool = False  # integer-valued FP8 indexer inputs (exact scores)
    decode: bool = False
    chunks: int = 1        # chunked prefill: L split into this many chunks
    plants: int = 32
    min_len: int = 4096    # decode cache lengths are U{min_len..L}


CONFIGS = {
    0: Config("tiny-prefill-L1024", B=1, L=1024, H_I=4, d_I=64, H=16, k=128, integer=True,
              plants=0),
    1: Config("prefill-L8192", B=1, L=8192, H_I=64, d_I=128, H=128, k=2048),
    2: Config("prefill-L32768", B=1, L=32768, H_I=64, d_I=128, H=128, k=2048),
    3: Config("decode-B64-L4k-131k", B=64, L=131072, H_I=64, d_I=128, H=128, k=2048,
              decode=True),
    4: Config("chunked-prefill-L131072", B=1, L=131072, H_I=64, d_I=128, H=128, k=2048,
              chunks=8),
}


@dataclass
class Workload:
    """Inputs of one call of the path, all on one device.

    Varlen convention: sequence b owns query rows cu_q[b]..cu_q[b+1]-1 and key
    rows cu_k[b]..cu_k[b+1]-1; its queries are the last len_q positions of
    the sequence, so local query i sits at p = len_k - len_q + i.
    """
    cfg: Config
    q8: torch.Tensor        # uint8 [T_q, H_I, d_I]   e4m3 bytes
    q_scale: torch.Tensor   # f32   [T_q, H_I]
    w: torch.Tensor         # f32   [T_q, H_I]
    k8: torch.Tensor        # uint8 [T_k, d_I]        e4m3 bytes
    k_scale: torch.Tensor   # f32   [T_k]
    q: torch.Tensor         # bf16  [T_q, H, 576]
    kv: torch.Tensor        # bf16  [T_k, 576]
    cu_q: torch.Tensor      # int32 [B+1]
    cu_k: torch.Tensor      # int32 [B+1]
    lens_q: list = field(default_factory=list)
    lens_k: list = field(default_factory=list)
    k: int = 2048
    scale: float = 1.0 / math.sqrt(D_QK)
    plants_kept: int = 0

    @property
    def B(self) -> int:
        return len(self.lens_q)

    @property
    def max_len_q(self) -> int:
        return max(self.lens_q) if self.lens_q else 0

    @property
    def max_len_k(self) -> int:
        return max(self.lens_k) if self.lens_k else 0

    @property
    def T_q(self) -> int:
        return int(self.q8.shape[0])

    @property
    def T_k(self) -> int:
        return int(self.k8.shape[0])

    def to(self, device) -> "Workload":
        t = {n: getattr(self, n).to(device) for n in
             ("q8", "q_scale", "w", "k8", "k_scale", "q", "kv", "cu_q", "cu_k")}
        return Workload(cfg=self.cfg, lens_q=list(self.lens_q), lens_k=list(self.lens_k),
                        k=self.k, scale=self.scale, plants_kept=self.plants_kept, **t)


def seed_of(cfg_id: int, chunk: int = 0) -> int:
    return BASE_SEED + 100 * cfg_id + chunk


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device, rows_per_draw: int | None = None) -> torch.Tensor:
    """N(0,1) float32, drawn in row blocks so huge tensors need little scratch."""
    if rows_per_draw is None or shape[0] <= rows_per_draw:
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    out = torch.empty(shape, device=device, dtype=torch.float32)
    for r0 in range(0, shape[0], rows_per_draw):
        r1 = min(shape[0], r0 + rows_per_draw)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device,
                                 dtype=torch.float32)
    return out


def _bf16_normal(shape, g, device, div: float = 1.0, rows_per_draw: int = 2048) -> torch.Tensor:
    out = torch.empty(shape, device=device, dtype=torch.bfloat16)
    for r0 in range(0, shape[0], rows_per_draw):
        r1 = min(shape[0], r0 + rows_per_draw)
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device,
                        dtype=torch.float32)
        if div != 1.0:
            x = x / div
        out[r0:r1] = x.to(torch.bfloat16)
    return out


def quantize_e4m3_per_row(x: torch.Tensor):
    """Per-row absmax quantisation onto e4m3 (input preparation).

    Row r is divided by scale[r] = max|x[r]| / 448 (1 for an all-zero row) and
    rounded to the nearest e4m3 value by torch's conversion.  Returns
    (uint8 bytes shaped like x, float32 scale [rows]).
    """
    rows = x.shape[0]
    flat = x.reshape(rows, -1)
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).to(torch.float32)
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    q = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return q.contiguous(), scale


def _int_e4m3(shape, lo, hi, g, device) -> torch.Tensor:
    v = torch.randint(lo, hi + 1, shape, generator=g, device=device).to(torch.float32)
    return v.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()


def _plant(k_I: torch.Tensor, q_I: torch.Tensor, p_of_query: torch.Tensor,
           key_base_of_query: torch.Tensor, n_plants: int, g, device) -> int:
    """Planted structure: for each query t at position p, n_plants draws (with
    replacement) of an earlier position s in [0, p) receive
    k_I[s] = 0.7 * q_I[t, j*] + 0.3 * N(0,1), j* uniform over indexer heads.
    Keys are shared, so the largest t that planted s wins.  Returns the number
    of keys that carry a plant."""
    T, H_I, d_I = q_I.shape
    if n_plants == 0 or T == 0:
        return 0
    jstar = torch.randint(0, H_I, (T,), generator=g, device=device)
    u = torch.rand((T, n_plants), generator=g, device=device, dtype=torch.float64)
    p = p_of_query.to(torch.float64)[:, None]
    s_local = torch.floor(u * p).to(torch.int64)              # in [0, p)
    ok = (p_of_query > 0)[:, None].expand(T, n_plants)
    t_idx = torch.arange(T, device=device)[:, None].expand(T, n_plants)
    s_glob = s_local + key_base_of_query[:, None]
    s_glob, t_idx = s_glob[ok], t_idx[ok]
    noise = torch.randn((int(s_glob.numel()), d_I), generator=g, device=device)
    if s_glob.numel() == 0:
        return 0
    # last writer (largest t) wins for each key
    winner = torch.full((k_I.shape[0],), -1, dtype=torch.int64, device=device)
    winner.scatter_reduce_(0, s_glob, t_idx, reduce="amax")
    keep = winner[s_glob] == t_idx
    # among duplicate draws of the same (t, s), the last draw wins
    s_k, t_k, n_k = s_glob[keep], t_idx[keep], noise[keep]
    order = torch.arange(s_k.numel(), device=device)
    last = torch.full((k_I.shape[0],), -1, dtype=torch.int64, device=device)
    last.scatter_reduce_(0, s_k, order, reduce="amax")
    fin = last[s_k] == order
    s_f, t_f, n_f = s_k[fin], t_k[fin], n_k[fin]
    k_I[s_f] = 0.7 * q_I[t_f, jstar[t_f]] + 0.3 * n_f
    return int(s_f.numel())


def make_prefill(cfg_id: int, device="cpu", L: int | None = None, chunk: int | None = None,
                 seed: int | None = None) -> Workload:
    """Prefill workload for config cfg_id (optionally with a smaller L).

    For a chunked config, ``chunk`` selects chunk c: queries c*C..(c+1)*C-1
    against keys 0..(c+1)*C-1 (C = L / chunks).  All keys are drawn up front
    from one seed, so every chunk sees the same cache.
    """
    cfg = CONFIGS[cfg_id]
    L = cfg.L if L is None else L
    g = _gen(device, seed_of(cfg_id) if seed is None else seed)
    T = L
    if cfg.integer:
        q8 = _int_e4m3((T, cfg.H_I, cfg.d_I), -4, 4, g, device)
        k8 = _int_e4m3((T, cfg.d_I), -4, 4, g, device)
        w = torch.randint(-2, 3, (T, cfg.H_I), generator=g, device=device).to(torch.float32)
        q_scale = torch.ones((T, cfg.H_I), device=device, dtype=torch.float32)
        k_scale = torch.ones((T,), device=device, dtype=torch.float32)
        kept = 0
    else:
        q_I = _randn((T, cfg.H_I, cfg.d_I), g, device, rows_per_draw=4096)
        k_I = _randn((T, cfg.d_I), g, device)
        w = torch.randn((T, cfg.H_I), generator=g, device=device) * 0.125
        pos = torch.arange(T, device=device)
        kept = _plant(k_I, q_I, pos, torch.zeros_like(pos), cfg.plants, g, device)
        q8, qs = quantize_e4m3_per_row(q_I)
        del q_I
        q_scale = qs[:, None].expand(T, cfg.H_I).contiguous()
        k8, k_scale = quantize_e4m3_per_row(k_I)
        del k_I
    kv = _bf16_normal((T, D_QK), g, device)
    q = _bf16_normal((T, cfg.H, D_QK), g, device, div=math.sqrt(D_QK), rows_per_draw=256)
    wl = Workload(cfg=cfg, q8=q8, q_scale=q_scale, w=w.contiguous(), k8=k8, k_scale=k_scale,
                  q=q, kv=kv,
                  cu_q=torch.tensor([0, T], dtype=torch.int32, device=device),
                  cu_k=torch.tensor([0, T], dtype=torch.int32, device=device),
                  lens_q=[T], lens_k=[T], k=cfg.k, plants_kept=kept)
    if chunk is not None:
        wl = chunk_of(wl, chunk, L // cfg.chunks)
    return wl


def chunk_of(wl: Workload, c: int, C: int) -> Workload:
    """Chunk c of a one-sequence prefill: queries c*C..(c+1)*C-1, keys
    0..(c+1)*C-1 (views, no copies)."""
    q0, q1 = c * C, (c + 1) * C
    dev = wl.q8.device
    return Workload(cfg=wl.cfg, q8=wl.q8[q0:q1], q_scale=wl.q_scale[q0:q1], w=wl.w[q0:q1],
                    k8=wl.k8[:q1], k_scale=wl.k_scale[:q1], q=wl.q[q0:q1], kv=wl.kv[:q1],
                    cu_q=torch.tensor([0, C], dtype=torch.int32, device=dev),
                    cu_k=torch.tensor([0, q1], dtype=torch.int32, device=dev),
                    lens_q=[C], lens_k=[q1], k=wl.k, scale=wl.scale, plants_kept=wl.plants_kept)


def make_decode(cfg_id: int = 3, device="cpu", B: int | None = None, min_len: int | None = None,
                max_len: int | None = None, seed: int | None = None) -> Workload:
    """Varlen decode: B sequences, one new query each, cache lengths drawn
    uniformly from [min_len, max_len]; the new token is already in the cache,
    so the query sits at p = n_b - 1 and its plants come from [0, n_b - 1)."""
    cfg = CONFIGS[cfg_id]
    B = cfg.B if B is None else B
    lo = cfg.min_len if min_len is None else min_len
    hi = cfg.L if max_len is None else max_len
    g = _gen(device, seed_of(cfg_id) if seed is None else seed)
    lens = torch.randint(lo, hi + 1, (B,), generator=g, device=device)
    lens_k = [int(x) for x in lens.cpu()]
    T_k = sum(lens_k)
    cu_k = [0]
    for n in lens_k:
        cu_k.append(cu_k[-1] + n)
    q_I = _randn((B, cfg.H_I, cfg.d_I), g, device)
    k_I = _randn((T_k, cfg.d_I), g, device, rows_per_draw=1 << 20)
    w = torch.randn((B, cfg.H_I), generator=g, device=device) * 0.125
    p = torch.tensor([n - 1 for n in lens_k], device=device)
    base = torch.tensor(cu_k[:-1], device=device)
    kept = _plant(k_I, q_I, p, base, cfg.plants, g, device)
    q8, qs = quantize_e4m3_per_row(q_I)
    q_scale = qs[:, None].expand(B, cfg.H_I).contiguous()
    k8, k_scale = quantize_e4m3_per_row(k_I)
    del k_I
    kv = _bf16_normal((T_k, D_QK), g, device, rows_per_draw=1 << 16)
    q = _bf16_normal((B, cfg.H, D_QK), g, device, div=math.sqrt(D_QK))
    return Workload(cfg=cfg, q8=q8, q_scale=q_scale, w=w.contiguous(), k8=k8, k_scale=k_scale,
                    q=q, kv=kv,
                    cu_q=torch.arange(B + 1, dtype=torch.int32, device=device),
                    cu_k=torch.tensor(cu_k, dtype=torch.int32, device=device),
                    lens_q=[1] * B, lens_k=lens_k, k=cfg.k, plants_kept=kept)


def make_small(H_I=4, d_I=64, H=16, L=300, k=64, seed=7, integer=False, device="cpu",
               lens=None, lens_q=None, q_div=None) -> Workload:
    """A small free-form workload (tests): one or more sequences, prefill or
    chunked depending on lens_q.  q_div scales the attention queries
    (default sqrt(576)); a small divisor gives sharp softmaxes."""
    g = _gen(device, seed)
    lens_k = [L] if lens is None else list(lens)
    lens_qq = list(lens_k) if lens_q is None else list(lens_q)
    B = len(lens_k)
    T_q, T_k = sum(lens_qq), sum(lens_k)
    if integer:
        q8 = _int_e4m3((T_q, H_I, d_I), -4, 4, g, device)
        k8 = _int_e4m3((T_k, d_I), -4, 4, g, device)
        w = torch.randint(-2, 3, (T_q, H_I), generator=g, device=device).to(torch.float32)
        q_scale = torch.ones((T_q, H_I), device=device)
        k_scale = torch.ones((T_k,), device=device)
    else:
        q_I = _randn((T_q, H_I, d_I), g, device)
        k_I = _randn((T_k, d_I), g, device)
        w = torch.randn((T_q, H_I), generator=g, device=device) * (1.0 / math.sqrt(H_I))
        q8, qs = quantize_e4m3_per_row(q_I)
        q_scale = qs[:, None].expand(T_q, H_I).contiguous()
        k8, k_scale = quantize_e4m3_per_row(k_I)
    kv = _bf16_normal((T_k, D_QK), g, device)
    q = _bf16_normal((T_q, H, D_QK), g, device, div=math.sqrt(D_QK) if q_div is None else q_div)
    cu_q, cu_k = [0], [0]
    for a, b in zip(lens_qq, lens_k):
        cu_q.append(cu_q[-1] + a)
        cu_k.append(cu_k[-1] + b)
    return Workload(cfg=Config("small", B=B, L=max(lens_k), H_I=H_I, d_I=d_I, H=H, k=k,
                               integer=integer),
                    q8=q8, q_scale=q_scale.contiguous(), w=w.contiguous(), k8=k8,
                    k_scale=k_scale.contiguous(), q=q, kv=kv,
                    cu_q=torch.tensor(cu_q, dtype=torch.int32, device=device),
                    cu_k=torch.tensor(cu_k, dtype=torch.int32, device=device),
                    lens_q=lens_qq, lens_k=lens_k, k=k)


# ---------------------------------------------------------------------------
# Masked MHA mode ("DeepSeek-V3.2" atlas entry, "Design overview" and
# "Inference efficiency": for short prompts the prefill runs a masked form of
# MHA as a stand-in for DSA).  Per-head queries and keys of 192 dims (128 + 64
# RoPE) and values of 128 dims, the MHA form of MLA.

D_QK_MHA = 192
D_V_MHA = 128


@dataclass
class MhaInputs:
    q: torch.Tensor        # bf16 [T_q, H, 192]
    k: torch.Tensor        # bf16 [T_k, H, 192]
    v: torch.Tensor        # bf16 [T_k, H, 128]
    idx: torch.Tensor      # int32 [T_q, topk]: a drawn selection, ascending, -1 padded
    cu_q: torch.Tensor
    cu_k: torch.Tensor
    lens_q: list
    lens_k: list
    topk: int
    scale: float

    @property
    def B(self):
        return len(self.lens_k)

    @property
    def T_q(self):
        return int(sum(self.lens_q))

    @property
    def max_len_q(self):
        return max(self.lens_q)

    @property
    def max_len_k(self):
        return max(self.lens_k)


def make_mha(lens, lens_q=None, H=128, topk=2048, seed=BASE_SEED + 900, device="cpu",
             q_div=None) -> MhaInputs:
    """Inputs of the masked MHA mode: q ~ N(0,1)/q_div (default sqrt(192)),
    k, v ~ N(0,1), all bf16, and a selection per query row at position p:
    min(topk, p+1) distinct keys of [0, p] drawn uniformly at random (every
    key when p+1 <= topk), ascending, padded with -1.  Queries of a sequence
    are its last len_q positions.  Softmax scale 1/sqrt(192).  Draw order:
    q, k, v, selection noise."""
    g = _gen(device, seed)
    lens_k = list(lens)
    lens_qq = list(lens_k) if lens_q is None else list(lens_q)
    T_q, T_k = sum(lens_qq), sum(lens_k)
    q = _bf16_normal((T_q, H, D_QK_MHA), g, device,
                     div=math.sqrt(D_QK_MHA) if q_div is None else q_div, rows_per_draw=256)
    k = _bf16_normal((T_k, H, D_QK_MHA), g, device, rows_per_draw=256)
    v = _bf16_normal((T_k, H, D_V_MHA), g, device, rows_per_draw=256)
    idx = torch.full((T_q, topk), -1, dtype=torch.int32, device=device)
    q_row = 0
    for lq, lk in zip(lens_qq, lens_k):
        pos = torch.arange(lk - lq, lk, device=device)
        for r0 in range(0, lq, 1024):
            r1 = min(lq, r0 + 1024)
            # uniform noise over the keys; keys past a row's position get +inf,
            # the topk smallest are a uniform random subset of [0, p]
            noise = torch.rand((r1 - r0, lk), generator=g, device=device)
            noise.masked_fill_(torch.arange(lk, device=device)[None, :] > pos[r0:r1, None], 2.0)
            n = min(topk, lk)
            sel = torch.topk(noise, n, dim=1, largest=False).indices
            sel = torch.where(torch.gather(noise, 1, sel) < 2.0, sel, torch.full_like(sel, lk))
            sel = torch.sort(sel, dim=1).values
            sel = torch.where(sel >= lk, torch.full_like(sel, -1), sel)
            idx[q_row + r0:q_row + r1, :n] = sel.to(torch.int32)
        q_row += lq
    cu_q, cu_k = [0], [0]
    for a, b in zip(lens_qq, lens_k):
        cu_q.append(cu_q[-1] + a)
        cu_k.append(cu_k[-1] + b)
    return MhaInputs(q=q, k=k, v=v, idx=idx,
                     cu_q=torch.tensor(cu_q, dtype=torch.int32, device=device),
                     cu_k=torch.tensor(cu_k, dtype=torch.int32, device=device),
                     lens_q=lens_qq, lens_k=lens_k, topk=topk,
                     scale=1.0 / math.sqrt(D_QK_MHA))
