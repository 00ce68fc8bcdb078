"""CPU-side checks of the C-ABI library: it loads, exports every symbol the
header declares, and its host-side validation and workspace sizing behave
(no kernel is launched; nothing here needs a GPU)."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "csa.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while", "for", "sizeof")))


@pytest.fixture(scope="module")
def lib():
    from compressed_sparse_kv_03_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from compressed_sparse_kv_03_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_the_five_calls():
    fns = header_functions()
    for name in ("csa_compress_kv", "csa_indexer_topk", "csa_sparse_attn_prefill",
                 "csa_sparse_attn_decode", "hca_attn"):
        assert name in fns


def test_library_exports_every_declared_symbol(lib):
    from compressed_sparse_kv_03_b200 import _lib
    fns = header_functions()
    assert fns, "no declarations parsed"
    for name in fns:
        assert hasattr(lib, name), f"{name} declared in csa.h but not exported"
    assert set(fns) == set(_lib.SIGNATURES), "binding signatures differ from the header"


def test_version_and_last_error(lib):
    assert b"sm_100a" in lib.csa_version()
    assert lib.csa_launch_count() == 0


def test_compress_rejects_bad_arguments_without_launching(lib):
    from compressed_sparse_kv_03_b200._lib import STATUS_NAMES
    buf = (C.c_uint8 * 64)()
    p = C.cast(buf, C.c_void_p)
    # m = 0
    st = lib.csa_compress_kv(p, p, None, None, None, 16, 8, 0, 0, p, None)
    assert STATUS_NAMES[st] == "CSA_ERR_INVALID_ARG"
    assert b"m >= 1" in lib.csa_last_error()
    # dim not a multiple of 8
    assert lib.csa_compress_kv(p, p, None, None, None, 16, 12, 4, 0, p, None) == 1
    # missing output
    assert lib.csa_compress_kv(p, p, None, None, None, 16, 8, 4, 0, None, None) == 1
    # overlap flag out of range
    assert lib.csa_compress_kv(p, p, None, None, None, 16, 8, 4, 2, p, None) == 1
    assert lib.csa_launch_count() == 0


def test_attention_rejects_unsupported_dims(lib):
    from compressed_sparse_kv_03_b200._lib import CacheT
    buf = (C.c_uint8 * 4096)()
    p = C.cast(C.addressof(buf) + (-C.addressof(buf)) % 16, C.c_void_p)
    cache = CacheT(p.value, 16, 16, None, 0, 0)
    ws = (C.c_uint8 * 1024)()
    wsp = C.cast(C.addressof(ws) + (-C.addressof(ws)) % 256, C.c_void_p)
    # head dim 256 is a legal size the library does not build (128 and 512 are)
    st = lib.csa_sparse_attn_decode(p, C.byref(cache), p, p, p, p, 1, 8, 256, 4, 8, 1.0, None, p,
                                    None, wsp, 512, None, None)
    assert st == 2 and b"head dim" in lib.csa_last_error()
    # indexer key dim 96
    st = lib.csa_indexer_topk(p, p, C.byref(cache), None, None, 4, 2, 96, 4, 16, 2, p, p, None,
                              wsp, 512, None)
    assert st == 2
    # null cache data
    bad = CacheT(None, 16, 16, None, 0, 0)
    st = lib.hca_attn(p, C.byref(bad), p, None, None, None, 4, 8, 128, 4, 16, 8, 1.0, None, p,
                      None, wsp, 512, None, None)
    assert st == 1
    # decode with a window needs the window buffer
    st = lib.csa_sparse_attn_decode(p, C.byref(cache), None, None, p, p, 1, 8, 128, 4, 8, 1.0,
                                    None, p, None, wsp, 512, None, None)
    assert st == 1
    assert lib.csa_launch_count() == 0


def test_qrope_arguments_are_checked_before_any_launch(lib):
    """The fused query prologue's arguments (csa_qrope_t) are validated on the
    host: rotary width a multiple of 8 up to the head dim, a base above 1, a
    0/1 de-rotation flag, an aligned gain, and a position array on the decode
    call, which has no other source of positions."""
    from compressed_sparse_kv_03_b200._lib import CacheT, QRopeT
    buf = (C.c_uint8 * 4096)()
    p = C.cast(C.addressof(buf) + (-C.addressof(buf)) % 16, C.c_void_p)
    cache = CacheT(p.value, 16, 16, None, 0, 0)
    ws = (C.c_uint8 * 1024)()
    wsp = C.cast(C.addressof(ws) + (-C.addressof(ws)) % 256, C.c_void_p)
    odd_gain = C.c_void_p(p.value + 4)
    bad = [QRopeT(None, 1e-6, 60, 1e4, 1, p.value),        # rope_dims not a multiple of 8
           QRopeT(None, 1e-6, 136, 1e4, 1, p.value),       # wider than the head
           QRopeT(None, 1e-6, 64, 1.0, 1, p.value),        # base must exceed 1
           QRopeT(None, 1e-6, 64, 1e4, 2, p.value),        # derotate not 0/1
           QRopeT(None, float("nan"), 64, 1e4, 1, p.value),
           QRopeT(odd_gain, 1e-6, 64, 1e4, 1, p.value),    # misaligned gain
           QRopeT(None, 1e-6, 64, 1e4, 1, None)]           # decode without positions
    for r in bad:
        st = lib.csa_sparse_attn_decode(p, C.byref(cache), p, p, p, p, 1, 8, 128, 4, 8, 1.0, None,
                                        p, None, wsp, 512, None, C.byref(r))
        assert st == 1 and b"qrope" in lib.csa_last_error(), (r.rope_dims, lib.csa_last_error())
    # prefill takes the row index as the position: no pos needed, but the
    # other checks hold there too
    st = lib.csa_sparse_attn_prefill(p, p, 16, p, p, p, 4, 8, 128, 4, 8, 1.0, None, p, None, wsp,
                                     512, None, C.byref(bad[0]))
    assert st == 1 and b"qrope" in lib.csa_last_error()
    assert lib.csa_launch_count() == 0


def test_workspace_sizes(lib):
    hdr = 256
    # decode split-KV: 64 queries x 2176 rows -> partials are needed
    n = lib.csa_sparse_attn_decode_workspace_size(64, 64, 128, 2048, 128)
    assert n > hdr and n % 256 == 0
    # prefill never splits
    assert lib.csa_sparse_attn_prefill_workspace_size(65536, 64, 128) == hdr
    # decode-mode indexer scratch is O(queries x top_k): a threshold, a count, a
    # fallback slot, 4 top_k (at least 8192) candidate (key, entry) pairs and
    # 1024 sampled keys per query -- no score matrix, and independent of the
    # number of entries
    n = lib.csa_indexer_topk_workspace_size(64, 32768, 2048)
    per_query = 8192 * 8 + 1024 * 4
    assert hdr + 64 * per_query <= n <= hdr + 64 * (per_query + 12) + 4 * 256
    assert lib.csa_indexer_topk_workspace_size(64, 1 << 19, 2048) == n
    assert lib.csa_indexer_topk_workspace_size(64, 32768, 4096) > n
    # many-query (prefill) mode: the same O(top_k) candidate lists plus 1024
    # sampled keys per query, in chunks of a multiple of 256 queries within
    # about 512 MB -- no score per eligible entry
    n = lib.csa_indexer_topk_workspace_size(65536, 16384, 2048)
    per_query = 8192 * 8 + 1024 * 4
    assert hdr + 256 * per_query <= n <= (520 << 20)
    assert lib.csa_indexer_topk_workspace_size(65536, 40000, 2048) == n   # independent of the entries
    # too small a workspace is refused before anything runs
    from compressed_sparse_kv_03_b200._lib import CacheT
    buf = (C.c_uint8 * 4096)()
    p = C.cast(C.addressof(buf) + (-C.addressof(buf)) % 256, C.c_void_p)
    cache = CacheT(p.value, 16, 16, None, 0, 0)
    st = lib.csa_indexer_topk(p, p, C.byref(cache), None, None, 64, 8, 64, 4, 32768, 2048, p, p,
                              None, p, 1024, None)
    assert st == 5 and b"workspace" in lib.csa_last_error()


def test_timing_event_hook_validation(lib):
    assert lib.csa_set_timing_events(99, None, None) == 1
    assert lib.csa_set_timing_events(0, C.c_void_p(1), None) == 1
    assert lib.csa_set_timing_events(0, None, None) == 0


def test_attention_kernel_choice_validation(lib):
    assert lib.csa_set_attention_kernel(3) == 1 and b"out of range" in lib.csa_last_error()
    assert lib.csa_set_attention_kernel(-1) == 1
    for choice in (1, 2, 0):
        assert lib.csa_set_attention_kernel(choice) == 0


def test_timeout_self_test_validation(lib):
    assert lib.csa_test_attention_timeout(2) == 1 and b"0 or 1" in lib.csa_last_error()
    assert lib.csa_test_attention_timeout(-1) == 1
    assert lib.csa_test_attention_timeout(1) == 0
    assert lib.csa_test_attention_timeout(0) == 0   # cleared before any launch


def test_batch_invariant_mode_validation_and_sizing(lib):
    assert lib.csa_set_batch_invariant(2) == 1 and b"0 or 1" in lib.csa_last_error()
    # B=400 queries fill the GPU without splitting; fixed 512-row slices need partials
    plain = lib.csa_sparse_attn_decode_workspace_size(400, 64, 128, 2048, 128)
    assert lib.csa_set_batch_invariant(1) == 0
    try:
        inv = lib.csa_sparse_attn_decode_workspace_size(400, 64, 128, 2048, 128)
    finally:
        assert lib.csa_set_batch_invariant(0) == 0
    n = (2048 + 128 + 511) // 512
    assert inv >= 400 * n * 64 * (128 + 2) * 4 > plain


def test_product_path_does_not_import_the_oracle():
    """The package and the bench's timed path never touch oracle/."""
    pkg = os.path.join(ROOT, "compressed_sparse_kv_03_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_mxfp4_calls_reject_bad_arguments_without_launching(lib):
    from compressed_sparse_kv_03_b200._lib import CacheT
    before = lib.csa_launch_count()
    buf = (C.c_uint8 * 4096)()
    p = C.c_void_p((C.addressof(buf) + 255) // 256 * 256)
    # quantize: dim not a multiple of 32, missing output, misaligned codes
    assert lib.csa_quantize_mxfp4(p, 4, 48, p, p, None) == 1
    assert b"multiple of 32" in lib.csa_last_error()
    assert lib.csa_quantize_mxfp4(p, 4, 64, None, p, None) == 1
    assert lib.csa_quantize_mxfp4(p, 4, 64, C.c_void_p(p.value + 4), p, None) == 1
    assert lib.csa_quantize_mxfp4(p, 0, 64, None, None, None) == 0   # nothing to do
    cache = CacheT(p.value, 16, 16, None, 0, 0)
    # q_idx, w, k_codes, k_scales, seq_id, q_pos, T, H_I, c_I, m, max_entries, top_k,
    # idx_out, count_out, score_out, ws, ws_bytes, stream
    args = [p, p, C.byref(cache), p, None, None, 8, 8, 64, 4, 16, 4, p, p, None, p, 1 << 20, None]
    # c_I not built
    a = list(args); a[8] = 96
    assert lib.csa_indexer_topk_mxfp4(*a) == 2
    # missing scales
    a = list(args); a[3] = None
    assert lib.csa_indexer_topk_mxfp4(*a) == 1 and b"k_scales" in lib.csa_last_error()
    # misaligned queries
    a = list(args); a[0] = C.c_void_p(p.value + 2)
    assert lib.csa_indexer_topk_mxfp4(*a) == 1 and b"aligned" in lib.csa_last_error()
    # H_I above 64
    a = list(args); a[7] = 65
    assert lib.csa_indexer_topk_mxfp4(*a) == 2
    # workspace too small
    a = list(args); a[16] = 256
    assert lib.csa_indexer_topk_mxfp4(*a) == 5
    assert lib.csa_launch_count() == before


def test_fp8_entry_calls_reject_bad_arguments_without_launching(lib):
    from compressed_sparse_kv_03_b200._lib import CacheT
    before = lib.csa_launch_count()
    buf = (C.c_uint8 * 4096)()
    p = C.c_void_p((C.addressof(buf) + 255) // 256 * 256)
    # content part not a multiple of 32, rope not below dim, missing rotary output
    assert lib.csa_quantize_entries_fp8(p, 4, 128, 48, p, p, p, None) == 1
    assert b"multiple of 32" in lib.csa_last_error()
    assert lib.csa_quantize_entries_fp8(p, 4, 128, 128, p, p, p, None) == 1
    assert lib.csa_quantize_entries_fp8(p, 4, 128, 64, p, p, None, None) == 1
    assert lib.csa_quantize_entries_fp8(p, 0, 128, 64, None, None, None, None) == 0
    cache = CacheT(p.value, 16, 16, None, 0, 0)
    # q, kv_codes, kv_scales, kv_rope, rope_dims, win, win_len, idx, count, B, H, d,
    # top_k, window, sm_scale, sink, out, lse, ws, ws_bytes, stream
    args = [p, C.byref(cache), p, p, 64, p, p, p, p, 2, 8, 128, 16, 4, 0.1, None, p, None, p,
            1 << 20, None]
    a = list(args); a[4] = 40            # 128 - 40 not a multiple of 32
    assert lib.csa_sparse_attn_decode_fp8(*a) == 1 and b"rope_dims" in lib.csa_last_error()
    a = list(args); a[11] = 64           # head dim not built
    assert lib.csa_sparse_attn_decode_fp8(*a) == 2
    a = list(args); a[2] = None          # scales missing
    assert lib.csa_sparse_attn_decode_fp8(*a) == 1 and b"kv_scales" in lib.csa_last_error()
    # workspace too small: a shape whose split needs partials (so that the
    # check, not a launch, ends the call)
    a = list(args); a[10], a[12], a[13], a[19] = 64, 2048, 128, 256
    assert lib.csa_sparse_attn_decode_workspace_size(2, 64, 128, 2048, 128) > 256
    assert lib.csa_sparse_attn_decode_fp8(*a) == 5
    assert lib.csa_launch_count() == before


def test_noalloc_rejects_bad_arguments_before_touching_its_scratch(lib):
    """The scratch-free decode form runs the decode call's argument checks
    before it looks up or clears its static scratch: on a host without a GPU a
    bad call still returns CSA_ERR_INVALID_ARG / CSA_ERR_UNSUPPORTED (not
    CSA_ERR_CUDA), and B == 0 returns CSA_OK without loading anything."""
    from compressed_sparse_kv_03_b200._lib import CacheT
    before = lib.csa_launch_count()
    buf = (C.c_uint8 * 4096)()
    p = C.c_void_p((C.addressof(buf) + 255) // 256 * 256)
    cache = CacheT(p.value, 16, 16, None, 0, 0)
    # q, kv_comp, win, win_len, idx, count, B, H, d, top_k, window, sm_scale, sink, out, lse, stream
    args = [p, C.byref(cache), p, p, p, p, 2, 8, 128, 16, 4, 0.1, None, p, None, None]
    a = list(args); a[0] = None                  # no queries
    assert lib.csa_sparse_attn_decode_noalloc(*a) == 1
    assert b"csa_sparse_attn_decode_noalloc" in lib.csa_last_error()
    a = list(args); a[4] = None                  # no selection
    assert lib.csa_sparse_attn_decode_noalloc(*a) == 1
    a = list(args); a[2] = None                  # window rows missing with window > 0
    assert lib.csa_sparse_attn_decode_noalloc(*a) == 1
    a = list(args); a[8] = 64                    # head dim not built
    assert lib.csa_sparse_attn_decode_noalloc(*a) == 2
    a = list(args); a[0] = C.c_void_p(p.value + 2)   # misaligned queries
    assert lib.csa_sparse_attn_decode_noalloc(*a) == 1
    a = list(args); a[6] = 0                     # nothing to do
    assert lib.csa_sparse_attn_decode_noalloc(*a) == 0
    assert lib.csa_launch_count() == before
