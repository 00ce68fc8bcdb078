"""GPU parity of the mixed-precision compressed entries (E4M3 content with a
power-of-two scale byte per 32, bf16 rotary part): the quantizer bit-exactly
against the oracle's, and the decode attention over such entries against the
oracle's attention over its own dequantization of the same bf16 entries."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_attn, dev, f64
from oracle import fp8_entry as ofp8

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


def _entries(g, rows, dim, rope):
    """Normal rows over 80 binades plus rows at the format's edges: all zero,
    signed zeros, subnormal bf16 values, exact E4M3 midpoints, saturation."""
    x = synth.normal(g, (rows, dim), dtype=torch.float32)
    x *= 2.0 ** torch.randint(-40, 41, (rows, 1), generator=g).float()
    dc = dim - rope
    mags = torch.from_numpy(ofp8.e4m3_value(np.arange(0x7F))).float()
    mids = (mags[1:] + mags[:-1]) / 2
    x[0] = 0.0
    x[1] = -0.0
    x[2] = torch.tensor(2.0 ** -130) * torch.sign(torch.randn(dim, generator=g))
    for r, X in ((3, 0), (4, -9), (5, 6)):
        row = mids[torch.randint(0, mids.numel(), (dim,), generator=g)] * 2.0 ** X
        for b in range(dc // 32):
            row[32 * b] = 300.0 * 2.0 ** X         # block max in [256, 512) * 2^X fixes X
        row *= torch.where(torch.rand(dim, generator=g) < 0.5, -1.0, 1.0)
        x[r] = row
    x[6] = 500.0 * torch.where(torch.rand(dim, generator=g) < 0.5, -1.0, 1.0)   # saturates
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,dim,rope", [(500, 128, 64), (37, 128, 0), (20, 512, 64), (9, 128, 96)])
def test_quantize_entries_fp8_matches_oracle(rows, dim, rope):
    csa = _csa()
    g = synth.generator(700 + rows + dim + rope)
    x = _entries(g, rows, dim, rope)
    codes, scales, rp = csa.quantize_entries_fp8(dev(x), rope)
    want_c, want_s, want_r = ofp8.entry_quantize(f64(x), rope)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(f64(rp), want_r)


def _decode_case(g, B, H, k, paged, rope):
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
        seq_rows = lambda b: oracle.unpage(pool, table[b], S[b], 64)   # noqa: E731
        store = dict(data=pool, page_table=table, page_size=64)
    else:
        Smax = max(S)
        kvc = synth.normal(g, (B, Smax, 128))
        seq_rows = lambda b: kvc[b]   # noqa: E731
        store = dict(data=kvc.reshape(B * Smax, 128), seq_stride=Smax)
    return q, win, win_len, idx, cnt, seq_rows, store


@pytest.fixture(params=["tcgen05", "mma_sync"])
def attn_kernel(request):
    """Run an attention test once per attention kernel."""
    csa = _csa()
    csa.set_attention_kernel(request.param)
    yield request.param
    csa.set_attention_kernel("auto")


@pytest.mark.usefixtures("attn_kernel")
@pytest.mark.parametrize("B,H,k,paged,sink,rope", [(5, 64, 2048, False, False, 64),
                                                   (3, 64, 300, True, True, 64),
                                                   (2, 20, 500, False, True, 32),
                                                   (4, 64, 700, True, False, 0)])
def test_sparse_attn_decode_fp8(B, H, k, paged, sink, rope):
    csa = _csa()
    g = synth.generator(720 + B + k + rope)
    q, win, win_len, idx, cnt, seq_rows, store = _decode_case(g, B, H, k, paged, rope)
    codes, scales, rp = csa.quantize_entries_fp8(dev(store["data"]), rope)
    cache = csa.Cache(codes, seq_stride=store.get("seq_stride", 0),
                      page_table=dev(store.get("page_table")), page_size=store.get("page_size", 0))
    z = synth.normal(g, (H,), dtype=torch.float32) if sink else None
    lam = 1 / math.sqrt(128)
    out, lse = csa.sparse_attn_decode_fp8(dev(q), cache, scales, rp, dev(win), dev(win_len),
                                          dev(idx), dev(cnt), lam, sink=dev(z), return_lse=True)
    out = f64(out)
    for b in range(B):
        sel = f64(seq_rows(b)[idx[b, :cnt[b]].long()]) if cnt[b] else np.zeros((0, 128))
        ent = ofp8.entry_dequantize(*ofp8.entry_quantize(sel, rope)) if sel.shape[0] else sel
        rows = np.concatenate([ent, f64(win[b, :win_len[b]])])
        if rows.shape[0] == 0 and z is None:
            assert np.all(out[b] == 0)
            continue
        ref, ref_lse = oracle.attend_shared_kv(f64(q[b]), rows, lam, None if z is None else f64(z))
        assert_close_attn(out[b], ref, f"fp8 decode seq {b}")
        np.testing.assert_allclose(f64(lse[b]), ref_lse, atol=1e-3, rtol=1e-4)


@pytest.mark.parametrize("paged", [False, True])
def test_sparse_attn_decode_fp8_equals_bf16_on_dequantized_cache(attn_kernel, paged):
    """The expansion is exact: attention over the stored entries equals the
    same kernel's over a bf16 cache holding the dequantized entries, bit for
    bit (tcgen05: expanded by its producer warps; mma.sync: by its gather)."""
    csa = _csa()
    g = synth.generator(760)
    B, H, k = 4, 64, 600
    q, win, win_len, idx, cnt, seq_rows, store = _decode_case(g, B, H, k, paged, 64)
    c_np, s_np, r_np = ofp8.entry_quantize(f64(store["data"]), 64)   # the oracle's storage
    deq = ofp8.entry_dequantize(c_np, s_np, r_np)
    deq_bf16 = torch.from_numpy(deq).to(torch.bfloat16)
    assert np.array_equal(f64(deq_bf16), deq)          # dequantized values are bf16 numbers
    codes = dev(torch.from_numpy(c_np))
    scales = dev(torch.from_numpy(s_np))
    rp = dev(torch.from_numpy(r_np).to(torch.bfloat16))
    lam = 1 / math.sqrt(128)
    lay = dict(seq_stride=store.get("seq_stride", 0), page_table=dev(store.get("page_table")),
               page_size=store.get("page_size", 0))
    a = csa.sparse_attn_decode_fp8(dev(q), csa.Cache(codes, **lay), scales, rp, dev(win), dev(win_len),
                                   dev(idx), dev(cnt), lam)
    b_ = csa.sparse_attn_decode(dev(q), csa.Cache(dev(deq_bf16), **lay), dev(win), dev(win_len),
                                dev(idx), dev(cnt), lam)
    assert torch.equal(a, b_)


def test_sparse_attn_decode_fp8_full_size_sampled():
    """The 64-sequence, 32768-entry decode shape with k = 2048 and a full
    window, in the configuration the benchmark times; two sequences are
    checked against the oracle."""
    csa = _csa()
    cfg = synth.CFG_DECODE_128K
    host = synth.csa_decode_inputs(cfg)
    S = cfg.N // cfg.m
    kv = host["kv_comp"].cuda()
    codes, scales, rp = csa.quantize_entries_fp8(kv.reshape(-1, 128), 64)
    g = synth.generator(770)
    idx, cnt = synth.random_topk_lists(g, cfg.B, cfg.k, [S] * cfg.B)
    out = csa.sparse_attn_decode_fp8(host["q"].cuda(), csa.Cache(codes, seq_stride=S), scales, rp,
                                     host["win"].cuda(), host["win_len"].cuda(), dev(idx), dev(cnt),
                                     cfg.lam)
    out = f64(out)
    for b in (0, 63):
        sel = f64(host["kv_comp"][b][idx[b, :cnt[b]].long()])
        ent = ofp8.entry_dequantize(*ofp8.entry_quantize(sel, 64))
        rows = np.concatenate([ent, f64(host["win"][b, :host["win_len"][b]])])
        ref, _ = oracle.attend_shared_kv(f64(host["q"][b]), rows, cfg.lam)
        assert_close_attn(out[b], ref, f"fp8 decode full-size seq {b}")
