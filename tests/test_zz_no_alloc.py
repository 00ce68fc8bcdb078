"""csa_sparse_attn_decode_noalloc: the decode attention form for callers that
cannot allocate device memory (it keeps its split-KV partials in a fixed array
inside the library).  Called through the C ABI and checked against
csa_sparse_attn_decode on the same inputs, on two calls in a row.

This file is named so that pytest collects it last."""
import ctypes as C
import math

import pytest
import torch

import synth
from helpers import ATTN_MAX_ABS, ATTN_MEAN_ABS

pytestmark = pytest.mark.gpu


def _inputs(seed, B=8, H=64, k=512, S=20000, W=128):
    g = synth.generator(seed)
    q = synth.normal(g, (B, H, 128)).cuda()
    kvc = synth.normal(g, (B, S, 128)).cuda()
    win = synth.normal(g, (B, W, 128)).cuda()
    win_len = torch.tensor([W, 1, 77, W, 5, 128, 64, 33][:B], dtype=torch.int32).cuda()
    idx = torch.full((B, k), -1, dtype=torch.int32)
    cnt = torch.zeros(B, dtype=torch.int32)
    for b in range(B):
        c = k - 13 * b
        idx[b, :c] = torch.randperm(S, generator=g)[:c].sort().values.to(torch.int32)
        cnt[b] = c
    return q, kvc, win, win_len, idx.cuda(), cnt.cuda()


def test_noalloc_matches_workspace_form_on_two_calls():
    assert torch.cuda.is_available(), "GPU test"
    import compressed_sparse_kv_03_b200 as csa
    from compressed_sparse_kv_03_b200._lib import CacheT, check, load
    lib = load()
    lam = 1 / math.sqrt(128)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (11, 12):                       # two calls in a row, different inputs
        q, kvc, win, win_len, idx, cnt = _inputs(seed)
        B, H, d = q.shape
        k, W = idx.shape[1], win.shape[1]
        cache = csa.Cache.contiguous(kvc)
        want = csa.sparse_attn_decode(q, cache, win, win_len, idx, cnt, lam)
        got = torch.empty_like(q)
        kc = cache.c()
        check(lib.csa_sparse_attn_decode_noalloc(
            C.c_void_p(q.data_ptr()), C.byref(kc), C.c_void_p(win.data_ptr()),
            C.c_void_p(win_len.data_ptr()), C.c_void_p(idx.data_ptr()), C.c_void_p(cnt.data_ptr()),
            B, H, d, k, W, lam, None, C.c_void_p(got.data_ptr()), None, stream))
        torch.cuda.synchronize()
        err = (got.float() - want.float()).abs()
        assert torch.isfinite(got.float()).all()
        assert err.max().item() <= ATTN_MAX_ABS and err.mean().item() <= ATTN_MEAN_ABS, \
            (seed, err.max().item(), err.mean().item())


def test_noalloc_rejects_calls_beyond_its_scratch():
    """295 queries x 64 heads split in two need about 19.6 MB of partials, more
    than the static scratch: the call must fail before enqueueing anything.
    Every pointer is a real device buffer of the right size regardless."""
    import compressed_sparse_kv_03_b200 as csa
    from compressed_sparse_kv_03_b200._lib import load
    lib = load()
    B, H, k, W, S = 295, 64, 2048, 128, 4096
    need = lib.csa_sparse_attn_decode_workspace_size(B, H, 128, k, W)
    assert need > (16 << 20)
    q = torch.zeros((B, H, 128), dtype=torch.bfloat16, device="cuda")
    kvc = torch.zeros((B, S, 128), dtype=torch.bfloat16, device="cuda")
    win = torch.zeros((B, W, 128), dtype=torch.bfloat16, device="cuda")
    win_len = torch.ones(B, dtype=torch.int32, device="cuda")
    idx = torch.zeros((B, k), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    kc = csa.Cache.contiguous(kvc).c()
    before = lib.csa_launch_count()
    st = lib.csa_sparse_attn_decode_noalloc(
        C.c_void_p(q.data_ptr()), C.byref(kc), C.c_void_p(win.data_ptr()),
        C.c_void_p(win_len.data_ptr()), C.c_void_p(idx.data_ptr()), C.c_void_p(cnt.data_ptr()),
        B, H, 128, k, W, 0.1, None, C.c_void_p(out.data_ptr()), None,
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 5 and b"static scratch" in lib.csa_last_error()
    assert lib.csa_launch_count() == before
