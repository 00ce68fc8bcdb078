"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs.  Small cases span several tiles plus ragged tails;
the five long-context workloads run at full size with sampled outputs."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_attn, assert_mostly_exact, check_topk, dev, f64, score_eps

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_kv_03_b200 as csa
    csa.load()
    yield csa
    torch.cuda.synchronize()


class LazySeq:
    """Per-sequence float64 views of a device/host tensor, made on demand."""

    def __init__(self, fn):
        self.fn = fn

    def __getitem__(self, b):
        return self.fn(b)


def _csa():
    import compressed_sparse_kv_03_b200 as csa
    return csa


def test_auto_attention_kernel_choice(cuda_lib):
    """The automatic choice runs the mma.sync kernel when a query's row list
    holds at most 256 rows (top_k + window) or when at most 16 heads cover at
    least 2048 queries, and the tensor-core kernel otherwise: its output
    equals, bit for bit, that of the kernel it names, and matches the
    oracle."""
    csa = _csa()
    g = synth.generator(777)
    m = 4
    cases = [(300, 64, 64, 8, "mma_sync"), (300, 64, 64, 64, "mma_sync"),
             (300, 128, 128, 64, "mma_sync"), (300, 129, 128, 8, "tcgen05"),
             (300, 512, 64, 64, "tcgen05"), (2048, 512, 64, 8, "mma_sync"),
             (2048, 512, 64, 16, "mma_sync"), (2048, 512, 64, 17, "tcgen05"),
             (2047, 512, 64, 8, "tcgen05")]
    try:
        for L, k, W, H, named in cases:
            kv_comp, kv_raw = synth.normal(g, (L // m, 128)), synth.normal(g, (L, 128))
            idx, cnt = synth.random_topk_lists(g, L, k, [t // m for t in range(L)])
            q = synth.normal(g, (L, H, 128))
            outs = {}
            for kern in ("auto", named):
                csa.set_attention_kernel(kern)
                outs[kern] = csa.sparse_attn_prefill(dev(q), dev(kv_comp), dev(kv_raw), dev(idx), dev(cnt),
                                                     W, 0.088)
            assert torch.equal(outs["auto"], outs[named]), (L, k, W, H)
            ref, _ = oracle.csa_prefill_attention(f64(q), f64(kv_comp), f64(kv_raw), idx.numpy(),
                                                  cnt.numpy(), W, 0.088)
            assert_close_attn(outs["auto"], ref, f"auto kernel L={L} k={k} W={W} H={H}")
    finally:
        csa.set_attention_kernel("auto")


@pytest.fixture(params=["tcgen05", "mma_sync"])
def attn_kernel(request):
    """Run an attention test once per attention kernel."""
    csa = _csa()
    csa.set_attention_kernel(request.param)
    yield request.param
    csa.set_attention_kernel("auto")


# ---------------------------------------------------------------------------
# step 1: compression
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,dim,m,bias", [(1000, 128, 4, False), (1003, 64, 4, True),
                                          (517, 512, 5, True), (4096, 128, 128, True),
                                          (37, 8, 1, False), (3, 128, 4, False)])
def test_compress_block(N, dim, m, bias):
    csa = _csa()
    g = synth.generator(10 + N + m)
    Cc, Z = synth.normal(g, (N, dim)), synth.normal(g, (N, dim))
    B = synth.normal(g, (m, dim), dtype=torch.float32) if bias else None
    out = csa.compress_kv(dev(Cc), dev(Z), m, bias=dev(B))
    assert out.shape == (N // m, dim)
    ref = oracle.pool_block(f64(Cc), f64(Z), m, None if B is None else f64(B))
    assert_close_attn(out, ref, "compress block")


@pytest.mark.parametrize("N,dim,m,bias,separate", [(1000, 128, 4, True, True),
                                                   (999, 64, 4, False, False),
                                                   (260, 128, 2, True, True),
                                                   (300, 256, 16, True, True)])
def test_compress_overlap(N, dim, m, bias, separate):
    csa = _csa()
    g = synth.generator(20 + N)
    Ca, Za = synth.normal(g, (N, dim)), synth.normal(g, (N, dim))
    Cb, Zb = (synth.normal(g, (N, dim)), synth.normal(g, (N, dim))) if separate else (None, None)
    B = synth.normal(g, (2, m, dim), dtype=torch.float32) if bias else None
    out = csa.compress_kv(dev(Ca), dev(Za), m, C_b=dev(Cb), Z_b=dev(Zb), bias=dev(B), overlap=True)
    ref = oracle.pool_overlap(f64(Ca), f64(Za), f64(Cb if separate else Ca),
                              f64(Zb if separate else Za), m,
                              None if B is None else f64(B[0]), None if B is None else f64(B[1]))
    assert_close_attn(out, ref, "compress overlap")


@pytest.mark.parametrize("T,H,dim,rope,gain", [(300, 64, 128, 64, True), (1000, 1, 128, 64, False),
                                               (77, 8, 64, 32, True), (50, 4, 256, 64, True)])
def test_norm_rope_prologue(T, H, dim, rope, gain):
    """Query / KV prologue: RMSNorm with a gain, then partial RoPE at large
    positions; compressed entries at position i*m."""
    csa = _csa()
    g = synth.generator(160 + T + dim)
    x = synth.normal(g, (T, H, dim), 2.5)
    gn = (1.0 + 0.2 * synth.normal(g, (dim,), dtype=torch.float32)) if gain else None
    pos = torch.randint(0, 1 << 20, (T,), generator=g, dtype=torch.int64)
    use_pos = H > 1
    out = csa.norm_rope(dev(x), gain=dev(gn), pos=dev(pos) if use_pos else None, pos_mul=1 if use_pos else 4,
                        rope_dims=rope)
    p = f64(pos) if use_pos else np.arange(T) * 4.0
    ref = oracle.rope_rotate(oracle.rmsnorm(f64(x), None if gn is None else f64(gn)),
                             p[:, None] if H > 1 else p[:, None], rope_dims=rope)
    assert_close_attn(out, ref, "norm + rope")


def test_norm_rope_output_derotation_in_place():
    csa = _csa()
    g = synth.generator(170)
    T, H = 200, 64
    o = synth.normal(g, (T, H, 128))
    pos = torch.randint(0, 1 << 22, (T,), generator=g, dtype=torch.int64)
    od = dev(o)
    got = csa.norm_rope(od, eps=None, pos=dev(pos), inverse=True, out=od)
    assert got.data_ptr() == od.data_ptr()
    ref = oracle.rope_rotate(f64(o), f64(pos)[:, None], inverse=True)
    assert_close_attn(got, ref, "de-rotation")
    # the content coordinates pass through unchanged
    assert torch.equal(got[:, :, :64].cpu(), o[:, :, :64])


@pytest.mark.parametrize("overlap,paged,dim", [(True, False, 128), (False, True, 128), (True, True, 64),
                                              (True, True, 512), (False, False, 512)])
def test_cache_append_matches_bulk_compression(overlap, paged, dim):
    """Decode-time appends, one token per sequence per call: entry for entry the
    bits of csa_compress_kv on the whole sequence, within tolerance of the
    oracle's DecodeCacheState, and the window ring holds the last W raw rows.
    dim 512 is the pages' compressed-entry width c."""
    csa = _csa()
    g = synth.generator(140 + dim + int(overlap) + 2 * int(paged))
    B, N, m, W = 3, 37, 4, 16
    S = N // m
    Ca, Za, Cb, Zb = (synth.normal(g, (B, N, dim)) for _ in range(4))
    bias = synth.normal(g, ((2, m, dim) if overlap else (m, dim)), dtype=torch.float32)
    if paged:
        pool, table = synth.paged_pool(g, [S + 3] * B, dim, 4)
        cache = csa.Cache(dev(torch.zeros_like(pool)), page_table=dev(table), page_size=4)
        read = lambda b: oracle.unpage(cache.data.cpu(), table[b], S, 4)
    else:
        buf = torch.zeros((B, S + 3, dim), dtype=torch.bfloat16)
        cache = csa.Cache.contiguous(dev(buf))
        read = lambda b: cache.data.cpu().reshape(B, S + 3, dim)[b, :S]
    st = csa.AppendState.new(B, dim, m, W, overlap)
    ws = csa.Workspace()
    for t in range(N):
        pos = torch.full((B,), t, dtype=torch.int64, device="cuda")
        csa.cache_append(dev(Ca[:, t].contiguous()), dev(Za[:, t].contiguous()), pos, cache, m, st,
                         S + 3, C_b=dev(Cb[:, t].contiguous()) if overlap else None,
                         Z_b=dev(Zb[:, t].contiguous()) if overlap else None, bias=dev(bias),
                         overlap=overlap, ws=ws)
    ws.check()
    for b in range(B):
        got = read(b)
        bulk = csa.compress_kv(dev(Ca[b]), dev(Za[b]), m, C_b=dev(Cb[b]) if overlap else None,
                               Z_b=dev(Zb[b]) if overlap else None, bias=dev(bias), overlap=overlap).cpu()
        assert torch.equal(got, bulk), f"seq {b}: append differs from csa_compress_kv"
        ref = oracle.DecodeCacheState(m, W, overlap, f64(bias[0] if overlap else bias),
                                      f64(bias[1]) if overlap else None)
        for t in range(N):
            ref.append(f64(Ca[b, t]), f64(Za[b, t]), f64(Cb[b, t]), f64(Zb[b, t]))
        assert_close_attn(got, np.array(ref.entries), f"cache append seq {b}")
        ring = st.win[b].cpu()
        for t in range(N - W, N):
            assert torch.equal(ring[t % W], Ca[b, t]), (b, t)


def test_cache_append_reports_full_cache():
    """A block completed past max_entries is skipped and recorded."""
    csa = _csa()
    g = synth.generator(150)
    B, dim, m = 2, 64, 2
    cache = csa.Cache.contiguous(dev(torch.zeros((B, 1, dim), dtype=torch.bfloat16)))
    st = csa.AppendState.new(B, dim, m, 0, False)
    ws = csa.Workspace()
    for t in range(4):   # blocks 0 and 1; only entry 0 fits
        x = dev(synth.normal(g, (B, dim)))
        csa.cache_append(x, x, torch.full((B,), t, dtype=torch.int64, device="cuda"), cache, m, st, 1, ws=ws)
    with pytest.raises(csa.CsaError, match="device check"):
        ws.check()


# ---------------------------------------------------------------------------
# steps 2-3: indexer + top-k
# ---------------------------------------------------------------------------
def _check_queries(idx, cnt, qI, w, key_of_query, elig_of_query, k, queries, scores=None):
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    sc = scores.cpu().numpy() if scores is not None else None
    stats = {"exact": 0, "near-tie": 0}
    for t in queries:
        n = elig_of_query(t)
        KI = key_of_query(t)[:n]
        s = oracle.indexer_scores(f64(qI[t]), f64(w[t]), KI)
        eps = score_eps(f64(qI[t]), f64(w[t]), KI)
        stats[check_topk(idx[t], cnt[t], s, k, eps)] += 1
        if sc is not None and cnt[t]:
            sel = idx[t, :cnt[t]]
            np.testing.assert_allclose(sc[t, :cnt[t]], s[sel], rtol=1e-5, atol=10 * eps + 1e-6)
    assert_mostly_exact(stats, len(queries))
    return stats


@pytest.mark.parametrize("H_I,c_I,wdist", [(8, 64, "uniform"), (4, 64, "normal"),
                                           (16, 128, "uniform"), (1, 64, "uniform"),
                                           (12, 64, "normal"), (64, 128, "uniform")])
def test_indexer_topk_decode_ragged(H_I, c_I, wdist):
    csa = _csa()
    g = synth.generator(30 + H_I + c_I)
    m, k = 4, 64
    pos = torch.tensor([0, 3, 4, 100, 257, 259, 1000, 9001], dtype=torch.int64)
    B, S = pos.shape[0], int(pos.max()) // m
    qI = synth.normal(g, (B, H_I, c_I))
    w = synth.head_weights(g, (B, H_I), wdist)
    KI = synth.normal(g, (B, S, c_I))
    seq = torch.arange(B, dtype=torch.int32)
    idx, cnt, sc = csa.indexer_topk(dev(qI), dev(w), csa.Cache.contiguous(dev(KI)), m, k,
                                    seq_id=dev(seq), q_pos=dev(pos), max_entries=S,
                                    return_scores=True)
    _check_queries(idx, cnt, qI, w, lambda t: f64(KI[t]), lambda t: int(pos[t]) // m, k,
                   range(B), sc)


@pytest.mark.parametrize("H_I,c_I,k", [(8, 64, 512), (64, 128, 256), (12, 64, 2048), (4, 64, 64),
                                       (64, 128, 512), (64, 128, 1024), (32, 128, 2048)])
def test_indexer_topk_decode_sampled_threshold(H_I, c_I, k):
    """Contexts long enough (more than 4096 eligible entries) for the sampled
    threshold: the selection comes from the candidate lists; scores too.
    H_I = 64 heads of c_I = 128 with k in {512, 1024} is the pages' indexer."""
    csa = _csa()
    g = synth.generator(35 + H_I + c_I + k)
    m = 4
    pos = torch.tensor([20000, 40001, 65537, 131072, 77777], dtype=torch.int64)
    B, S = pos.shape[0], int(pos.max()) // m
    qI = synth.normal(g, (B, H_I, c_I))
    w = synth.uniform(g, (B, H_I))
    KI = synth.normal(g, (B, S, c_I))
    idx, cnt, sc = csa.indexer_topk(dev(qI), dev(w), csa.Cache.contiguous(dev(KI)), m, k,
                                    seq_id=dev(torch.arange(B, dtype=torch.int32)), q_pos=dev(pos),
                                    max_entries=S, return_scores=True)
    _check_queries(idx, cnt, qI, w, lambda t: f64(KI[t]), lambda t: int(pos[t]) // m, k,
                   range(B), sc)


@pytest.mark.parametrize("H_I,c_I", [(8, 64), (16, 128)])
def test_indexer_topk_decode_long_context_clustered_sample(H_I, c_I):
    """More than 32768 eligible entries for some query: the sample of each
    query is scored by a cluster of CTAs and gathered through distributed
    shared memory before the threshold is set."""
    csa = _csa()
    g = synth.generator(38 + H_I)
    m, k = 4, 2048
    pos = torch.tensor([4 * 70000, 4 * 33000 + 3, 50000], dtype=torch.int64)
    B, S = pos.shape[0], int(pos.max()) // m
    qI = synth.normal(g, (B, H_I, c_I))
    w = synth.uniform(g, (B, H_I))
    KI = synth.normal(g, (B, S, c_I))
    idx, cnt, sc = csa.indexer_topk(dev(qI), dev(w), csa.Cache.contiguous(dev(KI)), m, k,
                                    seq_id=dev(torch.arange(B, dtype=torch.int32)), q_pos=dev(pos),
                                    max_entries=S, return_scores=True)
    _check_queries(idx, cnt, qI, w, lambda t: f64(KI[t]), lambda t: int(pos[t]) // m, k,
                   range(B), sc)


@pytest.mark.parametrize("return_scores", [False, True])
def test_indexer_topk_all_equal_scores_beyond_the_candidate_slots(return_scores):
    """20000 eligible entries whose scores are all exactly 0 (every head
    negative): every key reaches any threshold, more than the candidate slots
    hold, so the selection falls back to recomputing the keys.  The first k
    entries must win (ties to the lower index), bit-exactly."""
    csa = _csa()
    T, S, k, m = 3, 20000, 300, 4
    qI = torch.ones((T, 2, 64), dtype=torch.bfloat16)
    KI = -torch.ones((S, 64), dtype=torch.bfloat16)
    w = torch.rand((T, 2), generator=synth.generator(36))
    pos = torch.tensor([4 * S, 4 * S - 1, 4 * 1000 + 3], dtype=torch.int64)
    out = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), m, k, q_pos=dev(pos),
                           max_entries=S, return_scores=return_scores)
    idx, cnt = out[0].cpu(), out[1].cpu()
    assert torch.equal(idx, torch.arange(k, dtype=torch.int32).expand(T, k))
    assert torch.all(cnt == k)
    if return_scores:
        assert torch.all(out[2].cpu() == 0)


@pytest.mark.parametrize("H_I,c_I", [(8, 64), (16, 128)])
def test_indexer_topk_sample_misled_by_structure(H_I, c_I):
    """A cache whose every 32nd row (the sample's stride at this length)
    scores far above the rest: the threshold drawn from the sample is then too
    high (fewer than k keys reach it) and the selection recomputes.  Whatever
    path it takes, the result must be the oracle's."""
    csa = _csa()
    g = synth.generator(37 + H_I)
    B, m, k = 2, 4, 2048
    S = 40960                               # a multiple of 32: the sample hits rows 0 mod 32
    qI = synth.normal(g, (B, H_I, c_I))
    w = synth.uniform(g, (B, H_I))
    KI = synth.normal(g, (B, S, c_I), 0.05)
    for b in range(B):                      # rows 0 mod 32 aligned with the query's heads
        KI[b, ::32] = (qI[b].float().sum(0) / H_I).to(torch.bfloat16)
    pos = torch.full((B,), S * m, dtype=torch.int64)
    idx, cnt, sc = csa.indexer_topk(dev(qI), dev(w), csa.Cache.contiguous(dev(KI)), m, k,
                                    seq_id=dev(torch.arange(B, dtype=torch.int32)), q_pos=dev(pos),
                                    max_entries=S, return_scores=True)
    _check_queries(idx, cnt, qI, w, lambda t: f64(KI[t]), lambda t: S, k, range(B), sc)


@pytest.mark.parametrize("T,m,k,H_I", [(700, 4, 32, 4), (1500, 2, 100, 8), (300, 1, 300, 8)])
def test_indexer_topk_prefill_causal(T, m, k, H_I):
    csa = _csa()
    g = synth.generator(40 + T)
    S = (T - 1) // m
    qI = synth.normal(g, (T, H_I, 64))
    w = synth.uniform(g, (T, H_I))
    KI = synth.normal(g, (S, 64))
    idx, cnt = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), m, k)
    KI64 = f64(KI)
    stats = _check_queries(idx, cnt, qI, w, lambda t: KI64, lambda t: t // m, k, range(T))
    assert stats["exact"] >= 0.99 * T, stats


@pytest.mark.parametrize("T,m,k,H_I,scores", [(6000, 1, 256, 8, False), (9000, 2, 128, 4, True),
                                              (5000, 1, 1024, 16, False), (4500, 1, 200, 12, True)])
def test_indexer_topk_many_queries(T, m, k, H_I, scores):
    """More than 2048 queries on one sequence (prefill mode): with H_I in
    {4, 8, 16} the tcgen05 scorer's own sample pass, per-warp thresholds,
    candidate lists and a per-warp finish; H_I = 12 takes the per-query
    sample and finish launches.  Contexts pass the 4096 entries from which a
    threshold is sampled, and T = 9000 spans two chunks of 7680 queries.
    Checked on the first and last queries, both sides of the sampling and
    chunk boundaries, and 240 random queries."""
    csa = _csa()
    g = synth.generator(45 + T + H_I)
    S = (T - 1) // m
    qI = synth.normal(g, (T, H_I, 64))
    w = synth.uniform(g, (T, H_I))
    KI = synth.normal(g, (S, 64))
    out = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), m, k, return_scores=scores)
    idx, cnt, sc = out if scores else (out[0], out[1], None)
    picks = {0, 1, T - 2, T - 1} | set(range(4090 * m, 4102 * m)) | set(range(7676, 7685))
    picks |= set(torch.randint(0, T, (240,), generator=g).tolist())
    queries = sorted(t for t in picks if t < T)
    KI64 = f64(KI)
    stats = _check_queries(idx, cnt, qI, w, lambda t: KI64, lambda t: t // m, k, queries, sc)
    assert stats["exact"] >= 0.99 * len(queries), stats


def test_indexer_topk_many_queries_all_equal_scores():
    """9000 queries whose scores are all exactly 0: below 4097 entries every
    key is a candidate, up to 8192 the sampled threshold admits every key, and
    beyond 8192 entries the count passes the candidate slots so the query is
    listed for the exact recompute.  Every query must select its first k
    entries (ties to the lower index), bit for bit."""
    csa = _csa()
    T, k, m = 9000, 64, 1
    S = T - 1
    qI = torch.ones((T, 8, 64), dtype=torch.bfloat16)
    KI = -torch.ones((S, 64), dtype=torch.bfloat16)
    w = torch.rand((T, 8), generator=synth.generator(46))
    idx, cnt = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), m, k)
    idx, cnt = idx.cpu(), cnt.cpu()
    n = torch.clamp(torch.arange(T), max=k)
    assert torch.equal(cnt, n.to(torch.int32))
    want = torch.where(torch.arange(k)[None, :] < n[:, None], torch.arange(k)[None, :], -1)
    assert torch.equal(idx, want.to(torch.int32))


@pytest.mark.parametrize("T,m,k,H_I,scores", [(4096, 4, 64, 4, True), (3000, 3, 256, 8, False),
                                              (2500, 4, 600, 16, True)])
def test_indexer_topk_many_queries_short_lists(T, m, k, H_I, scores):
    """More than 2048 queries whose entry lists hold at most 1024 entries:
    every key is a candidate and the per-warp finish selects among them in
    registers (exact k-th key by a bitwise radix select, ties to the lower
    index).  Checked on the first and last queries, the k boundary and 240
    random queries, with the scores when returned."""
    csa = _csa()
    g = synth.generator(61 + T + k)
    S = (T - 1) // m
    qI = synth.normal(g, (T, H_I, 64))
    w = synth.uniform(g, (T, H_I))
    KI = synth.normal(g, (S, 64))
    out = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), m, k, return_scores=scores)
    idx, cnt, sc = out if scores else (out[0], out[1], None)
    picks = {0, 1, T - 2, T - 1} | set(range(k * m - 3, k * m + 4))
    picks |= set(torch.randint(0, T, (240,), generator=g).tolist())
    queries = sorted(t for t in picks if t < T)
    KI64 = f64(KI)
    stats = _check_queries(idx, cnt, qI, w, lambda t: KI64, lambda t: t // m, k, queries, sc)
    assert stats["exact"] >= 0.99 * len(queries), stats


def test_indexer_topk_many_queries_short_lists_exact_ties():
    """Integer-valued keys and queries over 3000 queries with at most 749
    entries each (the register finish): integer scores with many exact ties,
    the lower index winning, bit for bit on 200 queries; and all-zero scores,
    where every query takes its first k entries."""
    csa = _csa()
    g = synth.generator(62)
    T, m, k, H_I = 3000, 4, 100, 8
    S = (T - 1) // m
    qI = torch.randint(-1, 2, (T, H_I, 64), generator=g).to(torch.bfloat16)
    KI = torch.randint(-1, 2, (S, 64), generator=g).to(torch.bfloat16)
    w = torch.ones((T, H_I), dtype=torch.float32)
    idx, cnt = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), m, k)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for t in sorted({0, 5, k * m, k * m + 1, T - 1} | set(torch.randint(0, T, (195,), generator=g).tolist())):
        n = t // m
        s = oracle.indexer_scores(f64(qI[t]), f64(w[t]), f64(KI[:n]))
        ref = oracle.topk_select(s, k)
        assert cnt[t] == ref.shape[0], t
        np.testing.assert_array_equal(idx[t, :cnt[t]], ref)
    qz = torch.ones((T, H_I, 64), dtype=torch.bfloat16)
    kz = -torch.ones((S, 64), dtype=torch.bfloat16)
    idx, cnt = csa.indexer_topk(dev(qz), dev(w), csa.Cache(dev(kz)), m, k)
    idx, cnt = idx.cpu(), cnt.cpu()
    nn = torch.clamp(torch.arange(T) // m, max=k)
    assert torch.equal(cnt, nn.to(torch.int32))
    want = torch.where(torch.arange(k)[None, :] < nn[:, None], torch.arange(k)[None, :], -1)
    assert torch.equal(idx, want.to(torch.int32))


def test_indexer_topk_exact_ties():
    """Integer-valued keys and queries make integer scores with many exact
    ties: the lower index must win, bit-exactly."""
    csa = _csa()
    g = synth.generator(50)
    T, S, H_I, k, m = 64, 3000, 4, 200, 4
    qI = torch.randint(-1, 2, (T, H_I, 64), generator=g).to(torch.bfloat16)
    KI = torch.randint(-1, 2, (S, 64), generator=g).to(torch.bfloat16)
    w = torch.ones((T, H_I), dtype=torch.float32)
    pos = torch.randint(0, S * m, (T,), generator=g, dtype=torch.int64)
    idx, cnt = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), m, k, q_pos=dev(pos),
                                seq_id=dev(torch.zeros(T, dtype=torch.int32)), max_entries=S)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for t in range(T):
        n = int(pos[t]) // m
        s = oracle.indexer_scores(f64(qI[t]), f64(w[t]), f64(KI[:n]))
        ref = oracle.topk_select(s, k)
        assert cnt[t] == ref.shape[0]
        np.testing.assert_array_equal(idx[t, :cnt[t]], ref)


def test_indexer_topk_all_zero_scores():
    """Every head negative -> every score is exactly 0: the first k win."""
    csa = _csa()
    T, S, k = 4, 500, 37
    qI = torch.ones((T, 2, 64), dtype=torch.bfloat16)
    KI = -torch.ones((S, 64), dtype=torch.bfloat16)
    w = torch.rand((T, 2))
    pos = torch.full((T,), 4 * S, dtype=torch.int64)
    idx, cnt = csa.indexer_topk(dev(qI), dev(w), csa.Cache(dev(KI)), 4, k, q_pos=dev(pos),
                                max_entries=S)
    assert torch.equal(idx.cpu(), torch.arange(k, dtype=torch.int32).expand(T, k))
    assert torch.all(cnt.cpu() == k)


@pytest.mark.parametrize("page_size", [64, 16])
def test_indexer_topk_paged(page_size):
    csa = _csa()
    g = synth.generator(60 + page_size)
    m, k, H_I = 4, 128, 8
    pos = torch.tensor([77, 2048, 4097, 30000, 12345], dtype=torch.int64)
    S = [int(p) // m for p in pos]
    pool, table = synth.paged_pool(g, S, 64, page_size)
    B = len(S)
    qI, w = synth.normal(g, (B, H_I, 64)), synth.uniform(g, (B, H_I))
    cache = csa.Cache(dev(pool), page_table=dev(table), page_size=page_size)
    idx, cnt = csa.indexer_topk(dev(qI), dev(w), cache, m, k, seq_id=dev(torch.arange(B, dtype=torch.int32)),
                                q_pos=dev(pos), max_entries=max(S))
    _check_queries(idx, cnt, qI, w,
                   lambda b: f64(oracle.unpage(pool, table[b], S[b], page_size)),
                   lambda b: S[b], k, range(B))


# ---------------------------------------------------------------------------
# step 4: attention
# ---------------------------------------------------------------------------
@pytest.mark.usefixtures("attn_kernel")
@pytest.mark.parametrize("L,H,W,k,sink", [(300, 64, 128, 64, False), (257, 8, 16, 40, True),
                                          (130, 20, 1, 33, False), (200, 128, 64, 100, True)])
def test_sparse_attn_prefill(L, H, W, k, sink):
    csa = _csa()
    g = synth.generator(70 + L + H)
    m = 4
    S = max(L // m, 1)
    q = synth.normal(g, (L, H, 128), 1 / math.sqrt(128))
    kv_comp, kv_raw = synth.normal(g, (S, 128)), synth.normal(g, (L, 128))
    idx, cnt = synth.random_topk_lists(g, L, k, [t // m for t in range(L)])
    z = synth.normal(g, (H,), dtype=torch.float32) if sink else None
    out, lse = csa.sparse_attn_prefill(dev(q), dev(kv_comp), dev(kv_raw), dev(idx), dev(cnt), W,
                                       1.0, sink=dev(z), return_lse=True)
    ref, ref_lse = oracle.csa_prefill_attention(f64(q), f64(kv_comp), f64(kv_raw), idx.numpy(),
                                                cnt.numpy(), W, 1.0, None if z is None else f64(z))
    assert_close_attn(out, ref, "sparse prefill")
    np.testing.assert_allclose(f64(lse), ref_lse, atol=1e-3, rtol=1e-4)


@pytest.mark.usefixtures("attn_kernel")
@pytest.mark.parametrize("B,H,k,paged,sink", [(5, 64, 2048, False, False), (3, 64, 300, True, True),
                                              (7, 16, 100, False, True), (2, 128, 513, True, False)])
def test_sparse_attn_decode(B, H, k, paged, sink):
    csa = _csa()
    g = synth.generator(80 + B + k)
    W = 128
    S = [5000 + 977 * b for b in range(B)]
    q = synth.normal(g, (B, H, 128))
    win = synth.normal(g, (B, W, 128))
    win_len = torch.tensor([W, 1, 77, W, 5, 128, 0][:B], dtype=torch.int32)
    cnt_want = [min(k, s) for s in S]
    cnt_want[0] = 0 if B > 2 else cnt_want[0]          # an empty selection
    idx = torch.full((B, k), -1, dtype=torch.int32)
    for b in range(B):
        c = cnt_want[b]
        idx[b, :c] = torch.randperm(S[b], generator=g)[:c].sort().values.to(torch.int32)
    cnt = torch.tensor(cnt_want, dtype=torch.int32)
    if paged:
        pool, table = synth.paged_pool(g, S, 128, 64)
        cache = csa.Cache(dev(pool), page_table=dev(table), page_size=64)
        logical = lambda b: f64(oracle.unpage(pool, table[b], S[b], 64))
    else:
        Smax = max(S)
        kvc = synth.normal(g, (B, Smax, 128))
        cache = csa.Cache.contiguous(dev(kvc))
        logical = lambda b: f64(kvc[b])
    z = synth.normal(g, (H,), dtype=torch.float32) if sink else None
    lam = 1 / math.sqrt(128)
    out, lse = csa.sparse_attn_decode(dev(q), cache, dev(win), dev(win_len), dev(idx), dev(cnt), lam,
                                      sink=dev(z), return_lse=True)
    out = f64(out)
    for b in range(B):
        rows = np.concatenate([logical(b)[idx[b, :cnt[b]].numpy()], f64(win[b, :win_len[b]])])
        if rows.shape[0] == 0 and z is None:
            assert np.all(out[b] == 0)
            continue
        ref, ref_lse = oracle.attend_shared_kv(f64(q[b]), rows, lam, None if z is None else f64(z))
        assert_close_attn(out[b], ref, f"decode seq {b}")
        np.testing.assert_allclose(f64(lse[b]), ref_lse, atol=1e-3, rtol=1e-4)


@pytest.mark.usefixtures("attn_kernel")
@pytest.mark.parametrize("B,H,m,paged", [(3, 64, 128, False), (4, 24, 4, True), (1, 64, 16, False)])
def test_hca_decode(B, H, m, paged):
    csa = _csa()
    g = synth.generator(90 + B + m)
    W = 128
    pos = torch.tensor([70000, 127, 128, 5000][:B], dtype=torch.int64)
    S = [int(p) // m for p in pos]
    q = synth.normal(g, (B, H, 128))
    win = synth.normal(g, (B, W, 128))
    win_len = torch.clamp(pos + 1, max=W).to(torch.int32)
    if paged:
        pool, table = synth.paged_pool(g, [max(s, 1) for s in S], 128, 64)
        cache = csa.Cache(dev(pool), page_table=dev(table), page_size=64)
        logical = lambda b: f64(oracle.unpage(pool, table[b], S[b], 64))
    else:
        kvc = synth.normal(g, (B, max(S), 128))
        cache = csa.Cache.contiguous(dev(kvc))
        logical = lambda b: f64(kvc[b])
    lam = 1 / math.sqrt(128)
    out = csa.hca_attn(dev(q), cache, dev(win), m, W, lam, win_len=dev(win_len), q_pos=dev(pos),
                       max_entries=max(S))
    ref, _ = oracle.hca_decode(f64(q), LazySeq(logical), f64(win), win_len.numpy(), pos.numpy(), m,
                               lam)
    assert_close_attn(out, ref, "hca decode")


@pytest.mark.usefixtures("attn_kernel")
def test_hca_prefill():
    csa = _csa()
    g = synth.generator(95)
    L, H, m, W = 1100, 64, 16, 128
    q = synth.normal(g, (L, H, 128), 1 / math.sqrt(128))
    kv_raw, Z = synth.normal(g, (L, 128)), synth.normal(g, (L, 128))
    kv_comp = csa.compress_kv(dev(kv_raw), dev(Z), m)
    out = csa.hca_attn(dev(q), csa.Cache(kv_comp), dev(kv_raw), m, W, 1.0)
    ref, _ = oracle.hca_prefill(f64(q), oracle.bf16_round(oracle.pool_block(f64(kv_raw), f64(Z), m)),
                                f64(kv_raw), m, W, 1.0)
    assert_close_attn(out, ref, "hca prefill")


@pytest.mark.usefixtures("attn_kernel")
@pytest.mark.parametrize("paged", [False, True])
def test_hca_prefill_packed_sequences(paged):
    """Three sequences of 300, 517 and 1 tokens laid end to end: query i
    reads the compressed entries of sequence seq_id[i] and its window from the
    packed raw rows; each sequence must equal its own single-sequence HCA
    prefill in the oracle."""
    csa = _csa()
    g = synth.generator(96 + int(paged))
    lens, H, m, W = [300, 517, 1], 20, 8, 64
    T = sum(lens)
    q = synth.normal(g, (T, H, 128), 1 / math.sqrt(128))
    kv_raw = synth.normal(g, (T, 128))
    seq_id = torch.cat([torch.full((n,), b, dtype=torch.int32) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n, dtype=torch.int64) for n in lens])
    S = [max(n // m, 1) for n in lens]
    if paged:
        pool, table = synth.paged_pool(g, S, 128, 16)
        cache = csa.Cache(dev(pool), page_table=dev(table), page_size=16)
        logical = lambda b: f64(oracle.unpage(pool, table[b], S[b], 16))
    else:
        kvc = synth.normal(g, (len(lens), max(S), 128))
        cache = csa.Cache.contiguous(dev(kvc))
        logical = lambda b: f64(kvc[b])
    out, lse = csa.hca_attn(dev(q), cache, dev(kv_raw), m, W, 1.0, seq_id=dev(seq_id),
                            q_pos=dev(pos), max_entries=max(S), return_lse=True)
    off = 0
    for b, n in enumerate(lens):
        ref, ref_lse = oracle.hca_prefill(f64(q[off:off + n]), logical(b), f64(kv_raw[off:off + n]),
                                          m, W, 1.0)
        assert_close_attn(out[off:off + n], ref, f"packed hca prefill, sequence {b}")
        np.testing.assert_allclose(f64(lse[off:off + n]), ref_lse, atol=1e-3, rtol=1e-4)
        off += n


@pytest.mark.usefixtures("attn_kernel")
def test_attention_device_check_reports_bad_index():
    """An entry id outside the cache is skipped and reported through the
    workspace header; the other queries are unaffected."""
    csa = _csa()
    g = synth.generator(99)
    B, H, k, S = 3, 16, 8, 100
    q, win = synth.normal(g, (B, H, 128)), synth.normal(g, (B, 4, 128))
    kvc = synth.normal(g, (B, S, 128))
    idx = torch.arange(k, dtype=torch.int32).repeat(B, 1)
    idx[1, 3] = S + 5                          # outside sequence 1's rows
    cnt = torch.full((B,), k, dtype=torch.int32)
    wl = torch.full((B,), 4, dtype=torch.int32)
    ws = csa.Workspace()
    out = csa.sparse_attn_decode(dev(q), csa.Cache(dev(kvc.reshape(-1, 128)), seq_stride=S),
                                 dev(win), dev(wl), dev(idx), dev(cnt), 0.1, ws=ws)
    with pytest.raises(csa.CsaError, match="device check"):
        ws.check()
    ws.check()                                   # the record was cleared
    out = f64(out)
    for b in (0, 2):
        rows = np.concatenate([f64(kvc[b, :k]), f64(win[b])])
        ref, _ = oracle.attend_shared_kv(f64(q[b]), rows, 0.1)
        assert_close_attn(out[b], ref, "unaffected query")


def test_bounded_wait_timeout_is_reported_and_the_device_stays_usable():
    """Failure detection without a fault: the self-test withholds the first
    query tile of one tensor-core attention launch, so its bounded pipeline
    waits (about 1 ms each) run out.  The launch must end by itself, the
    workspace header must report the timeout, and the next call must give the
    same bits as before the test."""
    import time
    csa = _csa()
    g = synth.generator(97)
    B, H, k, W, S = 4, 64, 256, 128, 5000
    q = synth.normal(g, (B, H, 128))
    kvc = synth.normal(g, (B, S, 128))
    win = synth.normal(g, (B, W, 128))
    win_len = torch.full((B,), W, dtype=torch.int32)
    idx = torch.stack([torch.randperm(S, generator=g)[:k].sort().values for _ in range(B)]).to(torch.int32)
    cnt = torch.full((B,), k, dtype=torch.int32)
    args = (dev(q), csa.Cache.contiguous(dev(kvc)), dev(win), dev(win_len), dev(idx), dev(cnt), 0.088)
    csa.set_attention_kernel("tcgen05")
    ws = csa.Workspace()
    try:
        ref = csa.sparse_attn_decode(*args, ws=ws)
        ws.check()
        csa.test_attention_timeout(True)
        t0 = time.time()
        csa.sparse_attn_decode(*args, ws=ws)
        torch.cuda.synchronize()
        took = time.time() - t0
        with pytest.raises(csa.CsaError, match="timed out"):
            ws.check()
        assert took < 30, took
        again = csa.sparse_attn_decode(*args, ws=ws)
        ws.check()
        assert torch.equal(again, ref)
    finally:
        csa.test_attention_timeout(False)
        csa.set_attention_kernel("auto")


@pytest.mark.usefixtures("attn_kernel")
def test_decode_is_deterministic():
    csa = _csa()
    g = synth.generator(101)
    cfg = synth.CsaDecode("t", B=4, N=40000, H=64, d=128, H_I=8, c_I=64, m=4, k=512, W=128,
                          lam=1 / math.sqrt(128))
    x = {k_: dev(v) for k_, v in synth.csa_decode_inputs(cfg).items()}
    S = cfg.N // cfg.m

    def run():
        idx, cnt = csa.indexer_topk(x["qI"], x["w"], csa.Cache.contiguous(x["kI_comp"]), cfg.m, cfg.k,
                                    seq_id=torch.arange(cfg.B, dtype=torch.int32, device="cuda"),
                                    q_pos=x["pos"], max_entries=S)
        return idx, csa.sparse_attn_decode(x["q"], csa.Cache.contiguous(x["kv_comp"]), x["win"],
                                           x["win_len"], idx, cnt, cfg.lam)
    i1, o1 = run()
    i2, o2 = run()
    assert torch.equal(i1, i2) and torch.equal(o1, o2)


@pytest.mark.usefixtures("attn_kernel")
@pytest.mark.parametrize("paged", [False, True])
def test_batch_invariant_decode(paged):
    """In batch-invariant mode a sequence's decode step (indexer, top-k and
    attention) gives the same bits alone, in the full batch and in a
    reordered sub-batch; the outputs still match the oracle."""
    csa = _csa()
    g = synth.generator(120 + int(paged))
    B, H, k, W, m = 6, 64, 300, 128, 4
    S = [900 + 517 * b for b in range(B)]
    q = synth.normal(g, (B, H, 128))
    qI = synth.normal(g, (B, 8, 64))
    w = synth.uniform(g, (B, 8))
    win = synth.normal(g, (B, W, 128))
    win_len = torch.tensor([W, 40, 1, W, 77, W], dtype=torch.int32)
    pos = torch.tensor([s * m + 3 for s in S], dtype=torch.int64)
    if paged:
        pool, table = synth.paged_pool(g, S, 128, 64)
        kpool = synth.normal(g, (pool.shape[0], 64))
        cache = lambda sel: csa.Cache(dev(pool), page_table=dev(table[sel]), page_size=64)
        kcache = lambda sel: csa.Cache(dev(kpool), page_table=dev(table[sel]), page_size=64)
        logical = lambda b: f64(oracle.unpage(pool, table[b], S[b], 64))
    else:
        kvc, kI = synth.normal(g, (B, max(S), 128)), synth.normal(g, (B, max(S), 64))
        cache = lambda sel: csa.Cache.contiguous(dev(kvc[sel]))
        kcache = lambda sel: csa.Cache.contiguous(dev(kI[sel]))
        logical = lambda b: f64(kvc[b])
    lam = 1 / math.sqrt(128)

    def step(sel):
        n = len(sel)
        idx, cnt = csa.indexer_topk(dev(qI[sel]), dev(w[sel]), kcache(sel), m, k,
                                    seq_id=torch.arange(n, dtype=torch.int32, device="cuda"),
                                    q_pos=dev(pos[sel]), max_entries=max(S))
        out, lse = csa.sparse_attn_decode(dev(q[sel]), cache(sel), dev(win[sel]), dev(win_len[sel]),
                                          idx, cnt, lam, return_lse=True)
        return idx.cpu(), out.cpu(), lse.cpu()

    csa.set_batch_invariant(True)
    try:
        full = step(list(range(B)))
        subsets = [[b] for b in range(B)] + [[4, 1, 3]]
        for sel in subsets:
            part = step(sel)
            for j, b in enumerate(sel):
                assert torch.equal(part[0][j], full[0][b]), ("idx", sel, b)
                assert torch.equal(part[1][j], full[1][b]), ("out", sel, b)
                assert torch.equal(part[2][j], full[2][b]), ("lse", sel, b)
    finally:
        csa.set_batch_invariant(False)
    idx, out = full[0], f64(full[1])
    for b in range(B):
        c = int((idx[b] >= 0).sum())
        rows = np.concatenate([logical(b)[idx[b, :c].numpy()], f64(win[b, :win_len[b]])])
        ref, _ = oracle.attend_shared_kv(f64(q[b]), rows, lam)
        assert_close_attn(out[b], ref, f"batch-invariant decode seq {b}")


@pytest.mark.usefixtures("attn_kernel")
def test_batch_invariant_hca_decode():
    csa = _csa()
    g = synth.generator(125)
    B, H, m, W = 5, 64, 16, 128
    pos = torch.tensor([20000, 130, 9000, 4097, 16], dtype=torch.int64)
    S = [int(p) // m for p in pos]
    q = synth.normal(g, (B, H, 128))
    kvc = synth.normal(g, (B, max(S), 128))
    win = synth.normal(g, (B, W, 128))
    win_len = torch.clamp(pos + 1, max=W).to(torch.int32)
    lam = 1 / math.sqrt(128)

    def step(sel):
        return csa.hca_attn(dev(q[sel]), csa.Cache.contiguous(dev(kvc[sel])), dev(win[sel]), m, W, lam,
                            win_len=dev(win_len[sel]), q_pos=dev(pos[sel]), max_entries=max(S)).cpu()

    csa.set_batch_invariant(True)
    try:
        full = step(list(range(B)))
        for sel in [[b] for b in range(B)] + [[3, 0]]:
            part = step(sel)
            for j, b in enumerate(sel):
                assert torch.equal(part[j], full[b]), (sel, b)
    finally:
        csa.set_batch_invariant(False)
    ref, _ = oracle.hca_decode(f64(q), LazySeq(lambda b: f64(kvc[b])), f64(win), win_len.numpy(),
                               pos.numpy(), m, lam)
    assert_close_attn(full, ref, "batch-invariant hca decode")
