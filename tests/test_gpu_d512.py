"""GPU parity of the attention calls at the pages' entry width, head dim 512
(DeepSeek-V4 book, Ch.5 "Decode-time cache state": c = 512; Ch.6 "Shared
key-value MQA"; Ch.7 "The 128-token uncompressed sliding window", "Dense
attention over heavily compressed history").  Every case runs through the C
ABI against the fp64 oracle, which is written for any head dim; top-k sizes
are the pages' k in {512, 1024}.  Decode cases are long enough that the row
list is split across CTAs and the partials meet in the merge kernel."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_attn, dev, f64

pytestmark = pytest.mark.gpu
D = 512


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_kv_03_b200 as csa
    csa.load()
    yield csa
    torch.cuda.synchronize()


@pytest.mark.parametrize("k,H,paged,sink", [(512, 64, False, False), (1024, 16, True, True),
                                            (1024, 20, False, True)])
def test_decode_d512(cuda_lib, k, H, paged, sink):
    csa = cuda_lib
    g = synth.generator(900 + k + H)
    B, W = 3, 128
    S = [k + 700, 3000, 40 + k // 4]
    q = synth.normal(g, (B, H, D))
    win = synth.normal(g, (B, W, D))
    win_len = torch.tensor([W, 77, 1], dtype=torch.int32)
    idx = torch.full((B, k), -1, dtype=torch.int32)
    cnt = torch.tensor([min(k, s) for s in S], dtype=torch.int32)
    for b in range(B):
        idx[b, :cnt[b]] = torch.randperm(S[b], generator=g)[:cnt[b]].sort().values.to(torch.int32)
    if paged:
        pool, table = synth.paged_pool(g, S, D, 64)
        cache = csa.Cache(dev(pool), page_table=dev(table), page_size=64)
        logical = lambda b: f64(oracle.unpage(pool, table[b], S[b], 64))
    else:
        kvc = synth.normal(g, (B, max(S), D))
        cache = csa.Cache.contiguous(dev(kvc))
        logical = lambda b: f64(kvc[b])
    z = (0.5 * synth.normal(g, (H,), dtype=torch.float32)) if sink else None
    lam = 1 / math.sqrt(D)
    out, lse = csa.sparse_attn_decode(dev(q), cache, dev(win), dev(win_len), dev(idx), dev(cnt), lam,
                                      sink=dev(z), return_lse=True)
    for b in range(B):
        rows = np.concatenate([logical(b)[idx[b, :cnt[b]].numpy()], f64(win[b, :win_len[b]])])
        o, l = oracle.attend_shared_kv(f64(q[b]), rows, lam, None if z is None else f64(z))
        assert_close_attn(out[b], o, f"d=512 decode seq {b}")
        np.testing.assert_allclose(f64(lse[b]), l, atol=2e-3, rtol=1e-4)


def test_prefill_d512(cuda_lib):
    csa = cuda_lib
    g = synth.generator(930)
    L, H, W, k, m = 300, 16, 64, 512, 4
    S = L // m
    q = synth.normal(g, (L, H, D))
    kv_comp, kv_raw = synth.normal(g, (S, D)), synth.normal(g, (L, D))
    idx, cnt = synth.random_topk_lists(g, L, k, [t // m for t in range(L)])
    lam = 1 / math.sqrt(D)
    out, lse = csa.sparse_attn_prefill(dev(q), dev(kv_comp), dev(kv_raw), dev(idx), dev(cnt), W, lam,
                                       return_lse=True)
    ref, ref_lse = oracle.csa_prefill_attention(f64(q), f64(kv_comp), f64(kv_raw), idx.numpy(),
                                                cnt.numpy(), W, lam)
    assert_close_attn(out, ref, "d=512 prefill")
    np.testing.assert_allclose(f64(lse), ref_lse, atol=2e-3, rtol=1e-4)


def test_hca_decode_d512(cuda_lib):
    csa = cuda_lib
    g = synth.generator(940)
    B, H, m, W = 2, 16, 128, 128
    pos = torch.tensor([70000, 3000], dtype=torch.int64)
    S = [int(p) // m for p in pos]
    q = synth.normal(g, (B, H, D))
    win = synth.normal(g, (B, W, D))
    win_len = torch.clamp(pos + 1, max=W).to(torch.int32)
    kvc = synth.normal(g, (B, max(S), D))
    lam = 1 / math.sqrt(D)
    out = csa.hca_attn(dev(q), csa.Cache.contiguous(dev(kvc)), dev(win), m, W, lam,
                       win_len=dev(win_len), q_pos=dev(pos), max_entries=max(S))
    ref, _ = oracle.hca_decode(f64(q), [f64(kvc[b]) for b in range(B)], f64(win), win_len.numpy(),
                               pos.numpy(), m, lam)
    assert_close_attn(out, ref, "d=512 hca decode")


def test_d512_refuses_what_runs_at_128_only(cuda_lib):
    """Mixed-precision entries and the fused query prologue are built for
    head dim 128; at 512 the calls are refused before anything runs."""
    csa = cuda_lib
    q = torch.zeros((2, 16, D), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((64, D), dtype=torch.bfloat16, device="cuda")
    win = torch.zeros((2, 8, D), dtype=torch.bfloat16, device="cuda")
    wl = torch.ones(2, dtype=torch.int32, device="cuda")
    idx = torch.zeros((2, 8), dtype=torch.int32, device="cuda")
    cnt = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError, match="tensor-core"):
        csa.sparse_attn_decode(q, csa.Cache.contiguous(kv.view(1, 64, D)), win, wl, idx, cnt, 0.05,
                               qrope=csa.QRope(pos=torch.zeros(2, dtype=torch.int64, device="cuda")))
    codes = torch.zeros((64, D - 64), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((64, (D - 64) // 32), dtype=torch.uint8, device="cuda")
    rope = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(csa.CsaError, match="head dim 128"):
        csa.sparse_attn_decode_fp8(q, csa.Cache(codes), scales, rope, win, wl, idx, cnt, 0.05)
