"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Small cases are compared element by element over whole
tensors (several tiles plus ragged tails); the full-size configurations run in
the launch configuration the benchmark times and are compared on sampled
query rows, which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_08_b200 as dsa
from sparse_attention_08_b200 import workloads as W
from tests import dsa_cases as C

pytestmark = pytest.mark.gpu


def _small(**kw):
    wl = W.make_small(**kw)
    return wl, wl.to("cuda")


def _p_rows(wl, b, rows):
    q0, q1, k0, k1 = C.seq_slices(wl, b)
    return [(k1 - k0) - (q1 - q0) + int(i) for i in rows]


# --------------------------------------------------------------------------
# Indexer
# --------------------------------------------------------------------------

@pytest.mark.parametrize("H_I,d_I", [(4, 64), (64, 128), (16, 128), (8, 64)])
def test_indexer_integer_inputs_exact(H_I, d_I):
    cpu, gpu = _small(H_I=H_I, d_I=d_I, H=16, L=333, k=64, integer=True, seed=101)
    g = C.np_(C.gpu_indexer(gpu))
    C.assert_no_device_error()
    o = C.oracle_scores(cpu, 0)
    rows = np.arange(cpu.T_q)
    C.check_indexer(g, o, None, _p_rows(cpu, 0, rows), exact=True)


@pytest.mark.parametrize("H_I,d_I", [(64, 128), (32, 64)])
def test_indexer_real_varlen_and_chunk(H_I, d_I):
    # two sequences: a 700-token prefill and a 150-query chunk at the end of
    # a 520-token cache (positions 370..519)
    cpu, gpu = _small(H_I=H_I, d_I=d_I, H=16, lens=[700, 520], lens_q=[700, 150], k=64, seed=102)
    g = C.np_(C.gpu_indexer(gpu))
    C.assert_no_device_error()
    for b in range(2):
        q0, q1, _, _ = C.seq_slices(cpu, b)
        rows = np.arange(q1 - q0)
        o = C.oracle_scores(cpu, b)
        bound = C.oracle_scores(cpu, b, abs_bound=True)
        C.check_indexer(g[q0:q1], o, bound, _p_rows(cpu, b, rows))
        # entries beyond the causal limit stay untouched
        for r in (0, len(rows) // 2):
            p = _p_rows(cpu, b, [r])[0]
            assert np.all(np.isnan(g[q0 + r, p + 1:cpu.max_len_k]))


@pytest.mark.parametrize("H_I,d_I,integer", [(64, 128, True), (128, 64, True), (32, 128, False),
                                              (64, 64, False)])
def test_indexer_decode_batch(H_I, d_I, integer):
    # one query per sequence (the decode shape: one-query tiles) over caches
    # of ragged lengths, several key tiles and chunks each
    lens = [1, 130, 700, 2100, 257]
    cpu, gpu = _small(H_I=H_I, d_I=d_I, H=16, lens=lens, lens_q=[1] * len(lens), k=64,
                      integer=integer, seed=108)
    g = C.np_(C.gpu_indexer(gpu))
    C.assert_no_device_error()
    for b in range(len(lens)):
        q0, q1, _, _ = C.seq_slices(cpu, b)
        o = C.oracle_scores(cpu, b)
        bound = None if integer else C.oracle_scores(cpu, b, abs_bound=True)
        C.check_indexer(g[q0:q1], o, bound, _p_rows(cpu, b, [0]), exact=integer)


# --------------------------------------------------------------------------
# Top-k (same fp32 scores on both sides -> bit-exact)
# --------------------------------------------------------------------------

def _topk_vs_oracle(cpu, gpu, logits_gpu, check_val=True):
    idx, val = C.gpu_topk(gpu, logits_gpu)
    C.assert_no_device_error()
    g_idx, g_val = C.np_(idx), C.np_(val)
    L = C.np_(logits_gpu).astype(np.float64)
    for b in range(cpu.B):
        q0, q1, _, k1k = C.seq_slices(cpu, b)
        n_q, n_k = q1 - q0, cpu.lens_k[b]
        sc = np.nan_to_num(L[q0:q1, :n_k], nan=0.0)
        o_idx = oracle.topk(sc, n_q, cpu.k)
        assert np.array_equal(g_idx[q0:q1], o_idx), f"seq {b}: top-k differs"
        if check_val:
            for r in range(n_q):
                sel = o_idx[r][o_idx[r] >= 0]
                assert np.array_equal(g_val[q0 + r, : len(sel)].astype(np.float64), sc[r, sel])
                assert np.all(np.isnan(g_val[q0 + r, len(sel):]))


def test_topk_exact_integer_scores_with_ties():
    cpu, gpu = _small(H_I=4, d_I=64, H=16, lens=[900, 400], lens_q=[900, 77], k=128, integer=True,
                      seed=103)
    _topk_vs_oracle(cpu, gpu, C.gpu_indexer(gpu))


def test_topk_exact_real_scores():
    cpu, gpu = _small(H_I=64, d_I=128, H=16, L=1500, k=256, seed=104)
    _topk_vs_oracle(cpu, gpu, C.gpu_indexer(gpu))


@pytest.mark.parametrize("k", [1, 7, 2048, 4096])
def test_topk_exact_adversarial_rows(k):
    # hand-made score rows: constant rows, signed zeros, heavy ties, huge
    # magnitudes, a long row (50000 > the shared-memory-sized rows)
    n = 50000
    lens = [n, 3000, 5000]
    g = torch.Generator().manual_seed(k)
    rows = []
    rows.append(torch.zeros(n))
    r = torch.randint(-3, 4, (n,), generator=g).float()
    r[torch.rand(n, generator=g) < 0.3] = -0.0
    rows.append(r)
    rows.append(torch.randn(n, generator=g) * 1e30)
    rows.append(torch.where(torch.rand(n, generator=g) < 0.5, torch.tensor(-1.0),
                            torch.tensor(1.0)))
    logits = torch.full((len(rows) + 2, n), float("nan"))
    for i, rr in enumerate(rows):
        logits[i] = rr
    T_q = logits.shape[0]
    # sequence 0: the 4 hand rows are its last 4 queries of a length-n
    # sequence; sequences 1 and 2: single decode rows
    lens_q = [len(rows), 1, 1]
    logits[len(rows), :3000] = torch.randn(3000, generator=g)
    logits[len(rows) + 1, :5000] = torch.randint(0, 2, (5000,), generator=g).float()
    cu_q = torch.tensor([0, len(rows), len(rows) + 1, len(rows) + 2], dtype=torch.int32)
    cu_k = torch.tensor([0, n, n + 3000, n + 8000], dtype=torch.int32)
    lg = logits.cuda()
    idx = torch.full((T_q, k), -7, dtype=torch.int32, device="cuda")
    val = torch.empty((T_q, k), dtype=torch.float32, device="cuda")
    from sparse_attention_08_b200 import dsa_topk
    dsa_topk(lg, cu_q.cuda(), cu_k.cuda(), 3, len(rows), n, k, idx, val)
    C.assert_no_device_error()
    gi = C.np_(idx)
    L = logits.numpy().astype(np.float64)
    for b in range(3):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        n_k = lens[b]
        o = oracle.topk(np.nan_to_num(L[q0:q1, :n_k], nan=0.0), q1 - q0, k)
        assert np.array_equal(gi[q0:q1], o), f"sequence {b}"


def test_topk_exact_few_long_rows():
    # a batch of one-query sequences with a long cache (the shape that splits
    # each row over several CTAs whose candidates are merged): random rows of
    # many lengths around k, the no-threshold limit and the merge capacity;
    # a rising row (all candidates in the last segment); a row with 8000
    # evenly spread ties at the top (more candidates than one merged list
    # holds); a row of two values
    k = 2048
    g = torch.Generator().manual_seed(808)
    lens = [1, 2047, 2048, 2049, 4095, 4160, 4161, 5000, 5121, 9000, 16385, 30000, 65536,
            70001, 131072]
    rows = [torch.randn(n, generator=g) for n in lens]
    lens.append(60000)
    rows.append(torch.linspace(-1.0, 1.0, 60000))
    lens.append(60000)
    r = -torch.rand(60000, generator=g)
    r[::7][:8000] = 1.0
    rows.append(r)
    lens.append(100000)
    rows.append(torch.where(torch.rand(100000, generator=g) < 0.01, torch.tensor(2.0),
                            torch.tensor(-2.0)))
    B = len(rows)
    ld = (max(lens) + 3) // 4 * 4
    logits = torch.full((B, ld), float("nan"))
    for i, rr in enumerate(rows):
        logits[i, :lens[i]] = rr
    cu_q = torch.arange(B + 1, dtype=torch.int32)
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    val = torch.empty((B, k), dtype=torch.float32, device="cuda")
    dsa.dsa_topk(logits.cuda(), cu_q.cuda(), cu_k.cuda(), B, 1, max(lens), k, idx, val,
                 ld_logits=ld)
    C.assert_no_device_error()
    gi, gv = C.np_(idx), C.np_(val)
    L = logits.numpy().astype(np.float64)
    for b, n in enumerate(lens):
        o = oracle.topk(L[b:b + 1, :n], 1, k)[0]
        assert np.array_equal(gi[b], o), f"row {b} (n = {n})"
        kept = o >= 0
        assert np.array_equal(gv[b][kept], logits[b].numpy()[o[kept]]), f"values, row {b}"


# --------------------------------------------------------------------------
# Sparse attention (oracle fed the GPU's indices)
# --------------------------------------------------------------------------

def _attention_vs_oracle(cpu, gpu, idx_gpu):
    out, lse = C.gpu_attention(gpu, idx_gpu)
    C.assert_no_device_error()
    g_out, g_lse, g_idx = C.np_(out.float()), C.np_(lse), C.np_(idx_gpu)
    o_all, ol_all, g_all, gl_all = [], [], [], []
    for b in range(cpu.B):
        q0, q1, _, _ = C.seq_slices(cpu, b)
        rows = np.arange(q1 - q0)
        o, ol = C.oracle_attention(cpu, b, g_idx[q0:q1], rows)
        o_all.append(o)
        ol_all.append(ol)
        g_all.append(g_out[q0:q1])
        gl_all.append(g_lse[q0:q1])
    return C.check_attention(np.concatenate(g_all), np.concatenate(o_all),
                             np.concatenate(gl_all), np.concatenate(ol_all))


# Every work item is (query, group of 64 heads): H = 16 and 32 fill part of
# one group, 128 is two groups, 192 three and 256 four.
@pytest.mark.parametrize("H,k", [(16, 64), (128, 100), (64, 256), (32, 130), (192, 128),
                                 (256, 64)])
def test_attention_small(H, k):
    cpu, gpu = _small(H_I=8, d_I=64, H=H, lens=[400, 300], lens_q=[400, 90], k=k, seed=105)
    idx, _ = C.gpu_topk(gpu, C.gpu_indexer(gpu), with_val=False)
    _attention_vs_oracle(cpu, gpu, idx)


def test_attention_rescales_when_the_maximum_jumps():
    # The RoPE dims (512..575) of later keys are scaled up, so the logits grow
    # along the key index and the running softmax maximum jumps by far more
    # than the lazy-rescale threshold several times per row, while the value
    # dims keep the workload's N(0,1) scale.
    cpu, gpu = _small(H_I=8, d_I=64, H=128, L=700, k=512, seed=106, q_div=0.5)
    ramp = (1.0 + torch.arange(cpu.T_k, dtype=torch.float32) / 40.0)[:, None]
    kv = cpu.kv.float()
    kv[:, 512:] *= ramp
    cpu.kv = kv.to(torch.bfloat16)
    gpu.kv = cpu.kv.cuda()
    idx, _ = C.gpu_topk(gpu, C.gpu_indexer(gpu), with_val=False)
    _attention_vs_oracle(cpu, gpu, idx)


@pytest.mark.parametrize("H", [64, 128])
def test_attention_skips_invalid_entries(H):
    cpu, gpu = _small(H_I=8, d_I=64, H=H, L=300, k=128, seed=107)
    idx, _ = C.gpu_topk(gpu, C.gpu_indexer(gpu), with_val=False)
    bad = idx.clone()
    bad[5:, 3] = -1                 # holes inside the valid prefix
    bad[200:, 10] = 100000          # beyond p: skipped
    _attention_vs_oracle(cpu, gpu, bad)


# --------------------------------------------------------------------------
# End to end
# --------------------------------------------------------------------------

def test_forward_end_to_end_small_varlen():
    cpu, gpu = _small(H_I=64, d_I=128, H=128, lens=[1100, 700, 300], lens_q=[1100, 1, 45], k=256,
                      seed=108)
    idx, out, lse = C.gpu_forward(gpu)
    C.assert_no_device_error()
    g_idx, g_out, g_lse = C.np_(idx), C.np_(out.float()), C.np_(lse)
    for b in range(cpu.B):
        q0, q1, _, _ = C.seq_slices(cpu, b)
        rows = np.arange(q1 - q0)
        sc = C.oracle_scores(cpu, b)
        o_idx = oracle.topk(np.nan_to_num(sc, nan=0.0), q1 - q0, cpu.k)
        C.check_topk_near_cut(g_idx[q0:q1], o_idx, sc, _p_rows(cpu, b, rows), cpu.k)
        o, ol = C.oracle_attention(cpu, b, g_idx[q0:q1], rows)
        C.check_attention(g_out[q0:q1], o, g_lse[q0:q1], ol)


# --------------------------------------------------------------------------
# The indexer's KL training signal (oracle fed the GPU's scores and indices;
# the kernel uses the attention's lse, whose parity bar is 1e-3, so the
# per-head probabilities may differ by that much relatively: 2e-3)
# --------------------------------------------------------------------------

KL_RTOL = 2e-3


def _gpu_kl(gpu, logits, idx, lse):
    T_q, k = idx.shape
    kl = torch.full((T_q,), float("nan"), device="cuda")
    grad = torch.full((T_q, k), float("nan"), device="cuda")
    tgt = torch.full((T_q, k), float("nan"), device="cuda")
    dsa.dsa_indexer_kl(gpu.q, gpu.kv, idx, lse, logits, gpu.cu_q, gpu.cu_k, gpu.B, gpu.max_len_q,
                       gpu.max_len_k, gpu.k, gpu.scale, kl, grad, tgt)
    C.assert_no_device_error()
    return C.np_(kl), C.np_(grad), C.np_(tgt)


def _kl_vs_oracle(cpu, logits, idx, kl, grad, tgt, rows_of=None):
    lg = C.np_(logits)
    gi = C.np_(idx)
    for b in range(cpu.B):
        q0, q1, k0, k1 = C.seq_slices(cpu, b)
        rows = np.arange(q1 - q0) if rows_of is None else rows_of(b)
        if len(rows) == 0:
            continue
        pos = np.array(_p_rows(cpu, b, rows), dtype=np.int64)
        r_abs = q0 + rows
        o_kl, o_grad, o_tgt = oracle.indexer_kl_at(
            C.bits(cpu.q[torch.as_tensor(r_abs)]), C.bits(cpu.kv[k0:k1]), gi[r_abs], pos,
            lg[r_abs], cpu.scale)
        scale = np.abs(o_tgt).max(axis=1, keepdims=True) + 1e-12
        assert np.all(np.abs(tgt[r_abs] - o_tgt) <= KL_RTOL * scale), f"target, sequence {b}"
        qprob = o_grad + o_tgt
        gscale = (np.abs(qprob) + np.abs(o_tgt)).max(axis=1, keepdims=True) + 1e-12
        assert np.all(np.abs(grad[r_abs] - o_grad) <= KL_RTOL * gscale), f"grad, sequence {b}"
        assert np.all(np.abs(kl[r_abs] - o_kl) <= KL_RTOL * np.abs(o_kl) + 1e-5), f"kl, sequence {b}"
        invalid = ~((gi[r_abs] >= 0) & (gi[r_abs] <= pos[:, None]))
        assert np.all(grad[r_abs][invalid] == 0) and np.all(tgt[r_abs][invalid] == 0)


@pytest.mark.parametrize("H,k", [(128, 100), (16, 64), (192, 256), (64, 130)])
def test_indexer_kl_small(H, k):
    cpu, gpu = _small(H_I=8, d_I=64, H=H, lens=[400, 300], lens_q=[400, 90], k=k, seed=121,
                      q_div=3.0)
    logits = C.gpu_indexer(gpu, fill=0.0)
    idx, _ = C.gpu_topk(gpu, logits, with_val=False)
    if k >= 100:
        idx[5:, 3] = -1                  # holes inside the valid prefix
    _, lse = C.gpu_attention(gpu, idx)
    kl, grad, tgt = _gpu_kl(gpu, logits, idx, lse)
    _kl_vs_oracle(cpu, logits, idx, kl, grad, tgt)


def test_indexer_kl_dense_warmup_all_keys():
    # k >= every p + 1: the selection is every causal key (the dense warm-up)
    cpu, gpu = _small(H_I=8, d_I=64, H=128, L=300, k=320, seed=122, q_div=3.0)
    logits = C.gpu_indexer(gpu, fill=0.0)
    idx, _ = C.gpu_topk(gpu, logits, with_val=False)
    _, lse = C.gpu_attention(gpu, idx)
    kl, grad, tgt = _gpu_kl(gpu, logits, idx, lse)
    _kl_vs_oracle(cpu, logits, idx, kl, grad, tgt)


def test_indexer_kl_config1_sampled():
    cpu = W.make_prefill(1)
    gpu = cpu.to("cuda")
    logits = C.gpu_indexer(gpu, fill=0.0)
    idx, _ = C.gpu_topk(gpu, logits, with_val=False)
    _, lse = C.gpu_attention(gpu, idx)
    kl, grad, tgt = _gpu_kl(gpu, logits, idx, lse)
    L, k = cpu.T_q, cpu.k
    rows = np.array([0, 1, k - 2, k - 1, k, k + 1, 4000, L - 1])
    lg = torch.zeros(logits.shape, dtype=torch.float32)
    lg[torch.as_tensor(rows)] = logits[torch.as_tensor(rows, device="cuda")].cpu()
    del logits
    _kl_vs_oracle(cpu, lg, idx, kl, grad, tgt, rows_of=lambda b: rows)


# Host-buffer entry point: the batch goes through in chunks of query rows on
# several streams; each row's arithmetic is unchanged, so the results are
# bitwise those of dsa_forward.  The chunk sizes cut sequences in the middle
# and put several sequences (one without queries) into one chunk.
@pytest.mark.parametrize("chunk,n_streams", [(64, 3), (333, 2), (5000, 1)])
def test_forward_host_matches_forward(chunk, n_streams):
    cpu, gpu = _small(H_I=64, d_I=128, H=128, lens=[1100, 200, 700, 300],
                      lens_q=[1100, 0, 1, 45], k=256, seed=111)
    _, out_ref, lse_ref = C.gpu_forward(gpu)
    names = ("q8", "q_scale", "w", "k8", "k_scale", "q", "kv", "cu_q", "cu_k")
    h = {n: getattr(cpu, n).contiguous().pin_memory() for n in names}
    H = cpu.q.shape[1]
    out = torch.full((cpu.T_q, H, 512), float("nan"), dtype=torch.bfloat16).pin_memory()
    lse = torch.full((cpu.T_q, H), float("nan"), dtype=torch.float32).pin_memory()
    nbytes = dsa.dsa_forward_host_workspace_size(cpu.T_k, cpu.max_len_k, cpu.B, 64, 128, H,
                                                 cpu.k, chunk, n_streams)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    streams = [torch.cuda.Stream() for _ in range(n_streams)]
    torch.cuda.synchronize()
    dsa.dsa_forward_host(h["q8"], h["q_scale"], h["w"], h["k8"], h["k_scale"], h["q"], h["kv"],
                         h["cu_q"], h["cu_k"], cpu.B, cpu.max_len_q, cpu.max_len_k, cpu.k,
                         cpu.scale, out, lse, chunk, ws, streams)
    C.assert_no_device_error()
    assert np.array_equal(C.bits(out), C.bits(out_ref.cpu()))
    assert np.array_equal(C.np_(lse).view(np.uint32), C.np_(lse_ref).view(np.uint32))


def test_config0_full_exact():
    cpu = W.make_prefill(0)
    gpu = cpu.to("cuda")
    logits = C.gpu_indexer(gpu)
    idx, out, lse = C.gpu_forward(gpu)
    C.assert_no_device_error()
    o_sc = C.oracle_scores(cpu, 0)
    rows = np.arange(cpu.T_q)
    C.check_indexer(C.np_(logits), o_sc, None, _p_rows(cpu, 0, rows), exact=True)
    # scores are exact, so the selection must be bit-exact end to end
    o_idx = oracle.topk(np.nan_to_num(o_sc, nan=0.0), cpu.T_q, cpu.k)
    assert np.array_equal(C.np_(idx), o_idx)
    o, ol = C.oracle_attention(cpu, 0, o_idx, rows)
    C.check_attention(C.np_(out.float()), o, C.np_(lse), ol)


# --------------------------------------------------------------------------
# Full-size configurations, sampled rows
# --------------------------------------------------------------------------

def _sample_rows(n_q, n_k, k, extra, seed):
    rng = np.random.default_rng(seed)
    base = {0, min(n_q - 1, 1), n_q - 1}
    off = n_k - n_q
    for p in (k - 2, k - 1, k, k + 1):
        if 0 <= p - off < n_q:
            base.add(p - off)
    base.update(int(x) for x in rng.integers(0, n_q, size=extra))
    return np.array(sorted(base), dtype=np.int64)


def _sampled_parity(wl_gpu, b, rows, idx, out, lse, logits=None):
    """Oracle on sampled query rows of sequence b, each at its own position
    (the oracle evaluates exactly those rows of the full problem)."""
    q0, q1, k0, k1 = C.seq_slices(wl_gpu, b)
    n_q, n_k = q1 - q0, k1 - k0
    rows = np.asarray(rows, dtype=np.int64)
    pos = rows + (n_k - n_q)
    t = torch.as_tensor(q0 + rows, device=wl_gpu.q8.device)
    k8 = C.np_(wl_gpu.k8[k0:k1])
    ks = C.np_(wl_gpu.k_scale[k0:k1])
    q8, qs, w = C.np_(wl_gpu.q8[t]), C.np_(wl_gpu.q_scale[t]), C.np_(wl_gpu.w[t])
    sc = oracle.indexer_at(q8, qs, w, k8, ks, pos)
    if logits is not None:
        bound = oracle.indexer_at(q8 & 0x7F, qs, np.abs(w), k8 & 0x7F, ks, pos)
        C.check_indexer(C.np_(logits[t]), sc, bound, list(pos))
    o_idx = np.stack([oracle.topk(sc[r:r + 1, : p + 1], 1, wl_gpu.k)[0]
                      for r, p in enumerate(pos)])
    g_idx = C.np_(idx[t])
    C.check_topk_near_cut(g_idx, o_idx, sc, list(pos), wl_gpu.k)
    o, ol = oracle.sparse_mla_at(C.bits(wl_gpu.q[t]), C.bits(wl_gpu.kv[k0:k1]), g_idx, pos,
                                 wl_gpu.scale)
    return C.check_attention(C.np_(out[t].float()), o, C.np_(lse[t]), ol)


def test_config1_sampled():
    wl = W.make_prefill(1, device="cuda")
    logits = C.gpu_indexer(wl)
    idx, out, lse = C.gpu_forward(wl)
    C.assert_no_device_error()
    rows = _sample_rows(wl.T_q, wl.T_k, wl.k, 12, seed=1)
    _sampled_parity(wl, 0, rows, idx, out, lse, logits=logits)


def test_config2_sampled_bench_launch():
    wl = W.make_prefill(2, device="cuda")
    idx, out, lse = C.gpu_forward(wl)
    C.assert_no_device_error()
    rows = _sample_rows(wl.T_q, wl.T_k, wl.k, 6, seed=2)
    _sampled_parity(wl, 0, rows, idx, out, lse)
    # properties that hold at any size, checked on every row
    g = C.np_(idx)
    n = np.minimum(np.arange(wl.T_q) + 1, wl.k)
    assert np.array_equal((g >= 0).sum(axis=1), n)
    valid = g >= 0
    assert np.all(np.diff(g, axis=1)[valid[:, 1:]] > 0)
    assert torch.isfinite(out.float()).all()


def _attention_compact(q_rows_bits, kv_of_row, g_idx, pos, scale):
    """Oracle attention of rows from different sequences in one call: row r's
    valid selected latents (0 <= s <= pos[r]) are copied, in its index-row
    order, into a compact latent array at rows r*k + j, and its index row is
    renumbered to point there.  The oracle then sums exactly the same latents
    in the same order (a relabelling of rows, no arithmetic)."""
    R, k = g_idx.shape
    d = q_rows_bits.shape[2]
    kvc = np.zeros((R * k, d), dtype=np.uint16)
    idxc = np.full((R, k), -1, dtype=np.int32)
    for r in range(R):
        valid = (g_idx[r] >= 0) & (g_idx[r] <= pos[r])
        j = np.flatnonzero(valid)
        kvc[r * k + j] = kv_of_row(r, g_idx[r, j])
        idxc[r, j] = r * k + j
    pos_c = np.array([r * k + k - 1 for r in range(R)], dtype=np.int64)
    return oracle.sparse_mla_at(q_rows_bits, kvc, idxc, pos_c, scale)


def test_config3_decode_all_rows():
    # every one of the 64 decode rows (ragged caches of 4K..131K keys), in the
    # launch configuration the bench times
    wl = W.make_decode(3, device="cuda")
    idx, out, lse = C.gpu_forward(wl)
    C.assert_no_device_error()
    g_idx = C.np_(idx)
    q8, qs, w = C.np_(wl.q8), C.np_(wl.q_scale), C.np_(wl.w)
    k8_all, ks_all = C.np_(wl.k8), C.np_(wl.k_scale)
    cu_k = C.np_(wl.cu_k).astype(np.int64)
    pos = []
    for b in range(wl.B):
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        p = k1 - k0 - 1
        pos.append(p)
        sc = oracle.indexer_at(q8[b:b + 1], qs[b:b + 1], w[b:b + 1], k8_all[k0:k1],
                               ks_all[k0:k1], np.array([p]))
        o_idx = oracle.topk(sc, 1, wl.k)
        C.check_topk_near_cut(g_idx[b:b + 1], o_idx, sc, [p], wl.k)

    def kv_of_row(r, s):
        rows = torch.as_tensor(cu_k[r] + s, device="cuda")
        return C.bits(wl.kv[rows])

    o, ol = _attention_compact(C.bits(wl.q), kv_of_row, g_idx, np.array(pos), wl.scale)
    C.check_attention(C.np_(out.float()), o, C.np_(lse), ol)


def test_config4_every_chunk_sampled():
    # the 131072-token prefill as 8 chunks of 16384 queries against the
    # growing cache, each chunk through dsa_forward as the bench runs it;
    # sampled rows of every chunk (its first and last query and one drawn
    # row, plus positions k-2..k+1 in chunk 0) go to the oracle together
    full = W.make_prefill(4, device="cuda")
    n_ch = full.cfg.chunks
    C_ = full.cfg.L // n_ch
    rng = np.random.default_rng(4)
    rows, g_idx, g_out, g_lse = [], [], [], []
    for c in range(n_ch):
        wl = W.chunk_of(full, c, C_)
        idx, out, lse = C.gpu_forward(wl)
        C.assert_no_device_error()
        # properties that hold at any size, on every row of the chunk
        g = C.np_(idx)
        p_all = np.arange(c * C_, (c + 1) * C_)
        assert np.array_equal((g >= 0).sum(axis=1), np.minimum(p_all + 1, wl.k))
        assert np.all(np.diff(g, axis=1)[(g >= 0)[:, 1:]] > 0)
        assert torch.isfinite(out.float()).all()
        loc = {0, C_ - 1, int(rng.integers(1, C_ - 1))}
        if c == 0:
            loc |= {wl.k - 2, wl.k - 1, wl.k, wl.k + 1}
        loc = np.array(sorted(loc), dtype=np.int64)
        t = torch.as_tensor(loc, device="cuda")
        rows.append(c * C_ + loc)
        g_idx.append(g[loc])
        g_out.append(C.np_(out[t].float()))
        g_lse.append(C.np_(lse[t]))
        del idx, out, lse, wl
        torch.cuda.empty_cache()
    rows = np.concatenate(rows)
    g_idx, g_out, g_lse = np.concatenate(g_idx), np.concatenate(g_out), np.concatenate(g_lse)
    t = torch.as_tensor(rows, device="cuda")
    sc = oracle.indexer_at(C.np_(full.q8[t]), C.np_(full.q_scale[t]), C.np_(full.w[t]),
                           C.np_(full.k8), C.np_(full.k_scale), rows)
    o_idx = np.stack([oracle.topk(sc[r:r + 1, : p + 1], 1, full.k)[0]
                      for r, p in enumerate(rows)])
    C.check_topk_near_cut(g_idx, o_idx, sc, list(rows), full.k)
    o, ol = oracle.sparse_mla_at(C.bits(full.q[t]), C.bits(full.kv), g_idx, rows, full.scale)
    C.check_attention(g_out, o, g_lse, ol)
