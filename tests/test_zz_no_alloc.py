"""csa_sparse_attn_decode_noalloc: the decode attention form for callers that
cannot allocate device memory, such as a plugin inside a serving engine that
owns every allocation and hands it only a stream.  That form keeps its split-KV
partials in a fixed array inside the library.

Called through the C ABI and checked on two calls in a row against
csa_sparse_attn_decode on the same inputs.  Both forms run the same kernels
with the same split, so outputs and log-sum-exps must agree bit for bit, for
contiguous and paged caches and with batch-invariant mode off and on.  The
scratch-free form is also checked against the oracle.

This file is named so that pytest collects it last."""
import ctypes as C
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_attn, f64

pytestmark = pytest.mark.gpu


def _inputs(seed, paged, B=8, H=64, k=512, S=20000, W=128, page=64):
    g = synth.generator(seed)
    q = synth.normal(g, (B, H, 128))
    if paged:
        pool, table = synth.paged_pool(g, [S] * B, 128, page)
        logical = [oracle.unpage(pool, table[b], S, page) for b in range(B)]
    else:
        kvc = synth.normal(g, (B, S, 128))
        logical = [kvc[b] for b in range(B)]
    win = synth.normal(g, (B, W, 128))
    win_len = torch.tensor([W, 1, 77, W, 5, 128, 64, 33][:B], dtype=torch.int32)
    idx = torch.full((B, k), -1, dtype=torch.int32)
    cnt = torch.zeros(B, dtype=torch.int32)
    for b in range(B):
        c = k - 13 * b
        idx[b, :c] = torch.randperm(S, generator=g)[:c].sort().values.to(torch.int32)
        cnt[b] = c
    import compressed_sparse_kv_03_b200 as csa
    cache = (csa.Cache(pool.cuda(), page_table=table.cuda(), page_size=page) if paged
             else csa.Cache.contiguous(kvc.cuda()))
    host = dict(q=q, win=win, win_len=win_len, idx=idx, cnt=cnt, logical=logical)
    return cache, q.cuda(), win.cuda(), win_len.cuda(), idx.cuda(), cnt.cuda(), host


def _call_noalloc(lib, cache, q, win, win_len, idx, cnt, lam, out, lse):
    from compressed_sparse_kv_03_b200._lib import check
    B, H, d = q.shape
    kc = cache.c()
    check(lib.csa_sparse_attn_decode_noalloc(
        C.c_void_p(q.data_ptr()), C.byref(kc), C.c_void_p(win.data_ptr()),
        C.c_void_p(win_len.data_ptr()), C.c_void_p(idx.data_ptr()), C.c_void_p(cnt.data_ptr()),
        B, H, d, idx.shape[1], win.shape[1], lam, None, C.c_void_p(out.data_ptr()),
        C.c_void_p(lse.data_ptr()), C.c_void_p(torch.cuda.current_stream().cuda_stream)))


@pytest.mark.parametrize("invariant", [False, True], ids=["split", "batch_invariant"])
@pytest.mark.parametrize("paged", [False, True], ids=["contiguous", "paged"])
def test_noalloc_matches_workspace_form_on_two_calls(paged, invariant):
    assert torch.cuda.is_available(), "GPU test"
    import compressed_sparse_kv_03_b200 as csa
    from compressed_sparse_kv_03_b200._lib import load
    lib = load()
    lam = 1 / math.sqrt(128)
    csa.set_batch_invariant(invariant)
    try:
        for call, seed in enumerate((11, 12)):    # two calls in a row, different inputs
            cache, q, win, win_len, idx, cnt, host = _inputs(seed + 10 * paged, paged)
            want, want_lse = csa.sparse_attn_decode(q, cache, win, win_len, idx, cnt, lam,
                                                    return_lse=True)
            got = torch.empty_like(q)
            got_lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
            _call_noalloc(lib, cache, q, win, win_len, idx, cnt, lam, got, got_lse)
            torch.cuda.synchronize()
            assert torch.equal(got, want), (paged, invariant, call, "outputs differ in bits")
            assert torch.equal(got_lse, want_lse), (paged, invariant, call, "lse differs in bits")
            if call == 0:
                # and the scratch-free form against the oracle, query by query
                for b in range(q.shape[0]):
                    c = int(host["cnt"][b])
                    rows = np.concatenate([f64(host["logical"][b][host["idx"][b, :c].long()]),
                                           f64(host["win"][b, :int(host["win_len"][b])])])
                    o, l = oracle.attend_shared_kv(f64(host["q"][b]), rows, lam)
                    assert_close_attn(got[b], o, f"noalloc query {b}")
                    assert np.abs(f64(got_lse[b]) - l).max() <= 1e-3
    finally:
        csa.set_batch_invariant(False)


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
