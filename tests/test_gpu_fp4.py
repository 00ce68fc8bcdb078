"""GPU parity of the 4-bit indexer (E2M1 codes with one power-of-two scale
byte per 32 elements): the quantizer bit-exactly against the oracle's, and the
4-bit scorer + top-k against the oracle's scores of the same key codes and of
the oracle's quantization of the same bf16 queries (the scorer quantizes its
queries itself, with the quantizer checked bit-exact here)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_mostly_exact, check_topk, dev, f64, score_eps
from oracle import mxfp4 as ofp4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_kv_03_b200 as csa
    csa.load()
    yield csa
    torch.cuda.synchronize()


def _csa():
    import compressed_sparse_kv_03_b200 as csa
    return csa


# ---------------------------------------------------------------------------
# quantization
# ---------------------------------------------------------------------------
def _quant_inputs(g, rows, dim):
    """Normal rows at binades from 2^-40 to 2^40, plus rows that reach the
    format's edges: all zero, signed zeros, subnormal bf16 values, exact
    midpoints of the E2M1 grid, values just above 6 * 2^X (saturation)."""
    x = synth.normal(g, (rows, dim), dtype=torch.float32)
    x *= 2.0 ** torch.randint(-40, 41, (rows, 1), generator=g).float()
    mags = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mids = (mags[1:] + mags[:-1]) / 2
    x[0] = 0.0
    x[1] = -0.0
    x[2] = torch.tensor(2.0 ** -130) * torch.sign(torch.randn(dim, generator=g))
    for r, X in ((3, 0), (4, -5), (5, 7)):
        row = mids[torch.randint(0, 7, (dim,), generator=g)] * 2.0 ** X
        row[0] = 7.0 * 2.0 ** X          # amax in [4, 8) * 2^X fixes the scale
        row *= torch.where(torch.rand(dim, generator=g) < 0.5, -1.0, 1.0)
        x[r] = row
    x[6] = 6.0 * 1.0625                    # everything saturates to 6
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,dim", [(1000, 64), (37, 128), (8, 32)])
def test_quantize_mxfp4_matches_oracle(rows, dim):
    csa = _csa()
    g = synth.generator(900 + rows + dim)
    x = _quant_inputs(g, rows, dim)
    codes, scales = csa.quantize_mxfp4(dev(x))
    want_c, want_s = ofp4.mxfp4_quantize(f64(x))
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)


def test_quantize_mxfp4_keeps_leading_shape():
    csa = _csa()
    g = synth.generator(950)
    x = synth.normal(g, (3, 5, 64))
    codes, scales = csa.quantize_mxfp4(dev(x))
    assert codes.shape == (3, 5, 32) and scales.shape == (3, 5, 2)
    want_c, want_s = ofp4.mxfp4_quantize(f64(x))
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)


# ---------------------------------------------------------------------------
# 4-bit scorer + top-k
# ---------------------------------------------------------------------------
def _check_fp4_queries(idx, cnt, sc, q, w, keys_of, elig_of, k, queries):
    """q[t] = (codes, scales) of query t; keys_of(t) = (codes, scales) of its
    sequence's logical entries."""
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    sc = sc.cpu().numpy() if sc is not None else None
    stats = {"exact": 0, "near-tie": 0}
    for t in queries:
        n = elig_of(t)
        kc, ks = keys_of(t)
        qc, qs = q(t)
        s = ofp4.indexer_scores_mxfp4(qc, qs, f64(w[t]), kc[:n], ks[:n])
        eps = score_eps(ofp4.mxfp4_dequantize(qc, qs), f64(w[t]),
                        ofp4.mxfp4_dequantize(kc[:n], ks[:n]))
        stats[check_topk(idx[t], cnt[t], s, k, eps)] += 1
        if sc is not None and cnt[t]:
            sel = idx[t, :cnt[t]]
            np.testing.assert_allclose(sc[t, :cnt[t]], s[sel], rtol=1e-5, atol=10 * eps + 1e-6)
    assert_mostly_exact(stats, len(queries))
    return stats


@pytest.mark.parametrize("H_I,c_I", [(8, 64), (16, 128), (1, 64), (12, 64), (64, 128), (40, 64), (24, 64)])
def test_indexer_topk_mxfp4_decode_ragged(H_I, c_I):
    """Few-query (histogram + bitmap select) mode, one sequence per query,
    ragged eligible counts; the codes are the oracle's quantization of normal
    vectors."""
    csa = _csa()
    g = synth.generator(960 + H_I + c_I)
    m, k = 4, 64
    pos = torch.tensor([0, 3, 4, 100, 257, 259, 1000, 9001], dtype=torch.int64)
    B, S = pos.shape[0], int(pos.max()) // m
    qI = synth.normal(g, (B, H_I, c_I))
    qc, qs = ofp4.mxfp4_quantize(f64(qI))
    kc, ks = ofp4.mxfp4_quantize(f64(synth.normal(g, (B * S, c_I))))
    w = synth.uniform(g, (B, H_I))
    seq = torch.arange(B, dtype=torch.int32)
    cache = csa.Cache(dev(torch.from_numpy(kc)), seq_stride=S)
    idx, cnt, sc = csa.indexer_topk_mxfp4(dev(qI), dev(w), cache, dev(torch.from_numpy(ks)), m, k,
                                          seq_id=dev(seq), q_pos=dev(pos), max_entries=S,
                                          return_scores=True)
    kc3, ks3 = kc.reshape(B, S, -1), ks.reshape(B, S, -1)
    stats = _check_fp4_queries(idx, cnt, sc, lambda t: (qc[t], qs[t]), w,
                               lambda t: (kc3[t], ks3[t]), lambda t: int(pos[t]) // m, k, range(B))
    assert stats["exact"] >= B - 1, stats


@pytest.mark.parametrize("T,m,k,H_I", [(700, 4, 32, 4), (1500, 2, 100, 8)])
def test_indexer_topk_mxfp4_prefill_causal(T, m, k, H_I):
    """Many-query (radix select) mode on one sequence."""
    csa = _csa()
    g = synth.generator(970 + T)
    S = (T - 1) // m
    qI = synth.normal(g, (T, H_I, 64))
    qc, qs = ofp4.mxfp4_quantize(f64(qI))
    kc, ks = ofp4.mxfp4_quantize(f64(synth.normal(g, (S, 64))))
    w = synth.uniform(g, (T, H_I))
    idx, cnt = csa.indexer_topk_mxfp4(dev(qI), dev(w), csa.Cache(dev(torch.from_numpy(kc))),
                                      dev(torch.from_numpy(ks)), m, k)
    stats = _check_fp4_queries(idx, cnt, None, lambda t: (qc[t], qs[t]), w, lambda t: (kc, ks),
                               lambda t: t // m, k, range(T))
    assert stats["exact"] >= 0.99 * T, stats


def test_indexer_topk_mxfp4_identical_keys_tie_to_lower_index():
    """Keys that repeat the same codes score identically: the lower entry
    index must win, bit-exactly."""
    csa = _csa()
    g = synth.generator(980)
    T, S, H_I, k, m = 16, 2000, 4, 150, 4
    base_c, base_s = synth.fp4_codes(g, (50,), 64)
    pick = torch.randint(0, 50, (S,), generator=g)
    kc, ks = base_c[pick].numpy(), base_s[pick].numpy()
    qI = synth.normal(g, (T, H_I, 64))
    qc, qs = ofp4.mxfp4_quantize(f64(qI))
    w = synth.uniform(g, (T, H_I))
    pos = torch.randint(0, S * m, (T,), generator=g, dtype=torch.int64)
    idx, cnt = csa.indexer_topk_mxfp4(dev(qI), dev(w), csa.Cache(dev(torch.from_numpy(kc))),
                                      dev(torch.from_numpy(ks)), m, k, q_pos=dev(pos),
                                      seq_id=dev(torch.zeros(T, dtype=torch.int32)), max_entries=S)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for t in range(T):
        n = int(pos[t]) // m
        s = ofp4.indexer_scores_mxfp4(qc[t], qs[t], f64(w[t]), kc[:n], ks[:n])
        ref = oracle.topk_select(s, k)
        assert cnt[t] == ref.shape[0]
        np.testing.assert_array_equal(idx[t, :cnt[t]], ref)


@pytest.mark.parametrize("page_size", [64, 16])
def test_indexer_topk_mxfp4_paged(page_size):
    """Codes and scale bytes paged through one page table (same physical rows)."""
    csa = _csa()
    g = synth.generator(990 + page_size)
    m, k, H_I = 4, 128, 8
    pos = torch.tensor([77, 2048, 4097, 30000, 12345], dtype=torch.int64)
    S = [int(p) // m for p in pos]
    pages = [-(-n // page_size) for n in S]
    perm = torch.randperm(sum(pages), generator=g).to(torch.int32)
    table = torch.full((len(S), max(pages)), -1, dtype=torch.int32)
    off = 0
    for b, p in enumerate(pages):
        table[b, :p] = perm[off:off + p]
        off += p
    pool_c, pool_s = synth.fp4_codes(g, (sum(pages) * page_size,), 64)
    B = len(S)
    qI = synth.normal(g, (B, H_I, 64))
    qc, qs = ofp4.mxfp4_quantize(f64(qI))
    w = synth.uniform(g, (B, H_I))
    cache = csa.Cache(dev(pool_c), page_table=dev(table), page_size=page_size)
    idx, cnt = csa.indexer_topk_mxfp4(dev(qI), dev(w), cache, dev(pool_s), m, k,
                                      seq_id=dev(torch.arange(B, dtype=torch.int32)),
                                      q_pos=dev(pos), max_entries=max(S))
    _check_fp4_queries(idx, cnt, None, lambda b: (qc[b], qs[b]), w,
                       lambda b: (oracle.unpage(pool_c, table[b], S[b], page_size).numpy(),
                                  oracle.unpage(pool_s, table[b], S[b], page_size).numpy()),
                       lambda b: S[b], k, range(B))


def test_indexer_topk_mxfp4_decode_full_size_sampled():
    """The 64-sequence, 131072-token decode shape (32768 entries per sequence,
    H_I = 8, c_I = 64, k = 2048) on random codes, with the launch the
    benchmark times; a sample of queries is checked against the oracle."""
    csa = _csa()
    g = synth.generator(999)
    B, S, H_I, k, m = 64, 32768, 8, 2048, 4
    kc, ks = synth.fp4_codes(g, (B * S,), 64)
    qI = synth.normal(g, (B, H_I, 64))
    qc, qs = ofp4.mxfp4_quantize(f64(qI))
    w = synth.uniform(g, (B, H_I))
    pos = torch.full((B,), S * m, dtype=torch.int64)
    idx, cnt = csa.indexer_topk_mxfp4(dev(qI), dev(w), csa.Cache(dev(kc), seq_stride=S), dev(ks),
                                      m, k, seq_id=dev(torch.arange(B, dtype=torch.int32)),
                                      q_pos=dev(pos), max_entries=S)
    kc3, ks3 = kc.view(B, S, -1).numpy(), ks.view(B, S, -1).numpy()
    _check_fp4_queries(idx, cnt, None, lambda b: (qc[b], qs[b]), w,
                       lambda b: (kc3[b], ks3[b]), lambda b: S, k, [0, 17, 40, 63])


def test_indexer_topk_mxfp4_all_equal_scores_beyond_the_candidate_slots():
    """4-bit keys that all score exactly 0 (every code -1 against positive
    queries) on 20000 entries: more keys reach the threshold than the
    candidate slots hold, so the selection recomputes from the codes; the
    first k entries win, bit-exactly."""
    csa = _csa()
    T, S, k, m = 2, 20000, 500, 4
    qI = torch.ones((T, 8, 64), dtype=torch.bfloat16)
    codes = torch.full((S, 32), 0xAA, dtype=torch.uint8)        # every nibble -1.0
    scales = torch.full((S, 2), 127, dtype=torch.uint8)
    w = torch.rand((T, 8), generator=synth.generator(990))
    pos = torch.full((T,), 4 * S, dtype=torch.int64)
    idx, cnt = csa.indexer_topk_mxfp4(dev(qI), dev(w), csa.Cache(dev(codes)), dev(scales), m, k,
                                      q_pos=dev(pos), max_entries=S)
    assert torch.equal(idx.cpu(), torch.arange(k, dtype=torch.int32).expand(T, k))
    assert torch.all(cnt.cpu() == k)
