"""GPU parity of the attention calls' fused query prologue and output
epilogue (csa_qrope_t; DeepSeek-V4 Ch.7 "Query and KV RMSNorm", "Partial RoPE
and output de-rotation"): the raw queries go in, and the kernel applies
RMSNorm with a gain, rounds to bf16 after the rotation R_t of the last
rope_dims coordinates, attends, and rotates each output head back by R_{-t}.

The expected values chain the oracle's own steps in fp64: rmsnorm ->
rope_rotate -> bf16 rounding -> attention -> rope_rotate(inverse).  Positions
reach 2^22 so that the angle reduction is exercised, and the decode cases run
with enough rows per query that the split-KV partials path is taken (the
de-rotation is applied to the partials before the merge)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_attn, dev, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_kv_03_b200 as csa
    csa.load()
    csa.set_attention_kernel("auto")
    yield csa
    torch.cuda.synchronize()


def _prologue(q, pos, gain, eps, rope_dims, base):
    """The oracle's query prologue, rounded to bf16 like the kernel's operand."""
    x = f64(q)
    if eps is not None:
        x = oracle.rmsnorm(x, None if gain is None else f64(gain), eps)
    if rope_dims:
        x = oracle.rope_rotate(x, np.asarray(pos, dtype=np.float64)[:, None], rope_dims, base)
    return oracle.bf16_round(x)


def _epilogue(o, pos, rope_dims, base, derotate):
    if not (rope_dims and derotate):
        return o
    return oracle.rope_rotate(o, np.asarray(pos, dtype=np.float64)[:, None], rope_dims, base,
                              inverse=True)


@pytest.mark.parametrize("H,rope_dims,eps,gain,derotate", [
    (64, 64, 1e-6, True, True),       # the DeepSeek-V4 layout: 64 rotary coordinates of 128
    (20, 64, 1e-6, False, True),      # a partial head group (the tile holds other rows too)
    (64, 128, -1.0, False, False),    # rotation of the whole head, no RMSNorm, no de-rotation
    (8, 0, 1e-5, True, False),        # RMSNorm alone
])
def test_prefill_with_fused_query_prologue(cuda_lib, H, rope_dims, eps, gain, derotate):
    csa = cuda_lib
    g = synth.generator(400 + H + rope_dims)
    L, W, k, m = 300, 128, 64, 4
    S = L // m
    q = synth.normal(g, (L, H, 128), 3.0)       # raw: the prologue normalises it
    kv_comp, kv_raw = synth.normal(g, (S, 128)), synth.normal(g, (L, 128))
    idx, cnt = synth.random_topk_lists(g, L, k, [t // m for t in range(L)])
    gn = (1.0 + 0.25 * synth.normal(g, (128,), dtype=torch.float32)) if gain else None
    lam = 1 / math.sqrt(128)
    qr = csa.QRope(gain=dev(gn), eps=eps, rope_dims=rope_dims, derotate=derotate)
    out, lse = csa.sparse_attn_prefill(dev(q), dev(kv_comp), dev(kv_raw), dev(idx), dev(cnt), W, lam,
                                       qrope=qr, return_lse=True)
    pos = np.arange(L)
    qn = _prologue(q, pos, gn, eps if eps >= 0 else None, rope_dims, 10000.0)
    ref, ref_lse = oracle.csa_prefill_attention(qn, f64(kv_comp), f64(kv_raw), idx.numpy(),
                                                cnt.numpy(), W, lam)
    ref = _epilogue(ref, pos, rope_dims, 10000.0, derotate)
    assert_close_attn(out, ref, "prefill with the fused prologue")
    np.testing.assert_allclose(f64(lse), ref_lse, atol=2e-3, rtol=1e-4)


@pytest.mark.parametrize("paged,base", [(False, 10000.0), (True, 50000.0)])
def test_decode_with_fused_query_prologue_and_derotation(cuda_lib, paged, base):
    csa = cuda_lib
    g = synth.generator(430 + paged)
    B, H, k, W = 5, 64, 2048, 128
    S = [5000 + 977 * b for b in range(B)]
    q = synth.normal(g, (B, H, 128), 2.0)
    win = synth.normal(g, (B, W, 128))
    win_len = torch.tensor([W, 1, 77, W, 5], dtype=torch.int32)
    idx = torch.full((B, k), -1, dtype=torch.int32)
    cnt = torch.tensor([min(k, s) for s in S], dtype=torch.int32)
    for b in range(B):
        idx[b, :cnt[b]] = torch.randperm(S[b], generator=g)[:cnt[b]].sort().values.to(torch.int32)
    if paged:
        pool, table = synth.paged_pool(g, S, 128, 64)
        cache = csa.Cache(dev(pool), page_table=dev(table), page_size=64)
        logical = lambda b: f64(oracle.unpage(pool, table[b], S[b], 64))
    else:
        kvc = synth.normal(g, (B, max(S), 128))
        cache = csa.Cache.contiguous(dev(kvc))
        logical = lambda b: f64(kvc[b])
    pos = torch.randint(1 << 20, 1 << 22, (B,), generator=g, dtype=torch.int64)
    gn = 1.0 + 0.25 * synth.normal(g, (128,), dtype=torch.float32)
    lam = 1 / math.sqrt(128)
    qr = csa.QRope(gain=dev(gn), eps=1e-6, rope_dims=64, rope_base=base, derotate=True, pos=dev(pos))
    out, lse = csa.sparse_attn_decode(dev(q), cache, dev(win), dev(win_len), dev(idx), dev(cnt), lam,
                                      qrope=qr, return_lse=True)
    qn = _prologue(q, pos.numpy(), gn, 1e-6, 64, base)
    for b in range(B):
        rows = np.concatenate([logical(b)[idx[b, :cnt[b]].numpy()], f64(win[b, :win_len[b]])])
        o, l = oracle.attend_shared_kv(qn[b], rows, lam)
        o = _epilogue(o[None], pos.numpy()[b:b + 1], 64, base, True)[0]
        assert_close_attn(out[b], o, f"decode seq {b}")
        np.testing.assert_allclose(f64(lse[b]), l, atol=2e-3, rtol=1e-4)
    # the fused form equals the unfused chain on the device: the library's own
    # norm_rope on the queries, plain attention, then norm_rope's de-rotation
    qd = csa.norm_rope(dev(q), gain=dev(gn), eps=1e-6, pos=dev(pos), rope_dims=64, rope_base=base)
    o2 = csa.sparse_attn_decode(qd, cache, dev(win), dev(win_len), dev(idx), dev(cnt), lam)
    o2 = csa.norm_rope(o2, eps=None, pos=dev(pos), rope_dims=64, rope_base=base, inverse=True)
    assert (out.float() - o2.float()).abs().max().item() <= 2e-2


def test_hca_with_fused_query_prologue(cuda_lib):
    """HCA decode takes q_pos as the rotary position, HCA prefill the row index."""
    csa = cuda_lib
    g = synth.generator(450)
    B, H, m, W = 3, 64, 128, 128
    pos = torch.tensor([70000, 127, 3000000], dtype=torch.int64)
    S = [int(p) // m for p in pos]
    q = synth.normal(g, (B, H, 128), 2.0)
    win = synth.normal(g, (B, W, 128))
    win_len = torch.clamp(pos + 1, max=W).to(torch.int32)
    kvc = synth.normal(g, (B, max(S), 128))
    lam = 1 / math.sqrt(128)
    qr = csa.QRope(eps=1e-6, rope_dims=64, derotate=True)
    out = csa.hca_attn(dev(q), csa.Cache.contiguous(dev(kvc)), dev(win), m, W, lam,
                       win_len=dev(win_len), q_pos=dev(pos), max_entries=max(S), qrope=qr)
    qn = _prologue(q, pos.numpy(), None, 1e-6, 64, 10000.0)
    ref, _ = oracle.hca_decode(qn, [f64(kvc[b]) for b in range(B)], f64(win), win_len.numpy(),
                               pos.numpy(), m, lam)
    ref = _epilogue(ref, pos.numpy(), 64, 10000.0, True)
    assert_close_attn(out, ref, "hca decode with the fused prologue")

    L, mp = 700, 16
    qp = synth.normal(g, (L, H, 128), 2.0)
    kv_raw, Z = synth.normal(g, (L, 128)), synth.normal(g, (L, 128))
    kv_comp = csa.compress_kv(dev(kv_raw), dev(Z), mp)
    outp = csa.hca_attn(dev(qp), csa.Cache(kv_comp), dev(kv_raw), mp, W, lam, qrope=qr)
    qn = _prologue(qp, np.arange(L), None, 1e-6, 64, 10000.0)
    ref, _ = oracle.hca_prefill(qn, f64(kv_comp), f64(kv_raw), mp, W, lam)
    ref = _epilogue(ref, np.arange(L), 64, 10000.0, True)
    assert_close_attn(outp, ref, "hca prefill with the fused prologue")


def test_prologue_needs_the_tensor_core_kernel(cuda_lib):
    csa = cuda_lib
    q = torch.zeros((4, 64, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((16, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((4, 8), dtype=torch.int32, device="cuda")
    cnt = torch.ones(4, dtype=torch.int32, device="cuda")
    csa.set_attention_kernel("mma_sync")
    try:
        with pytest.raises(csa.CsaError, match="tensor-core"):
            csa.sparse_attn_prefill(q, kv, kv[:4], idx, cnt, 4, 0.1, qrope=csa.QRope())
    finally:
        csa.set_attention_kernel("auto")
