"""Python entry points with the names of the C ABI (include/csa.h).

Arguments are torch CUDA tensors; results are written by the CUDA library on
the current torch stream.  Shapes follow the header:

    compress_kv          (step 1)    C, Z [N, dim] -> [N // m, dim]
    indexer_topk         (steps 2-3) q_idx [T, H_I, c_I], w [T, H_I], keys -> idx [T, k], count [T]
    quantize_mxfp4       x [..., dim] bf16 -> 4-bit codes [..., dim/2] + scale bytes [..., dim/32]
    indexer_topk_mxfp4   (steps 2-3) on 4-bit queries and keys
    quantize_entries_fp8 entries [..., dim] bf16 -> E4M3 content + scale bytes + bf16 rotary part
    sparse_attn_decode_fp8 (step 4)  decode over those mixed-precision entries
    sparse_attn_prefill  (step 4)    q [L, H, d] over kv_comp[idx] + raw window
    sparse_attn_decode   (step 4)    q [B, H, d] over cache[idx] + window buffer
    hca_attn             (step 4)    q [T, H, d] over all eligible entries + window
                                     (d = 128, or 512: the pages' entry width)
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import CacheT, QRopeT, check, load


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need(t, name, dtype, ndim=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t


@dataclass
class Cache:
    """A compressed cache: ``data`` [rows, dim] bf16, contiguous per sequence
    (``seq_stride`` rows apart) or paged through ``page_table`` [n_seq,
    max_pages] int32 with ``page_size`` rows per page."""
    data: torch.Tensor
    seq_stride: int = 0
    page_table: Optional[torch.Tensor] = None
    page_size: int = 0

    @staticmethod
    def contiguous(t):
        """[n_seq, S, dim] -> one contiguous cache per sequence."""
        return Cache(t.reshape(-1, t.shape[-1]), seq_stride=t.shape[-2] if t.dim() == 3 else 0)

    @property
    def dim(self):
        return self.data.shape[-1]

    def c(self, dtype=torch.bfloat16):
        _need(self.data, "cache.data", dtype, 2)
        if self.page_table is not None:
            _need(self.page_table, "cache.page_table", torch.int32, 2)
            return CacheT(self.data.data_ptr(), self.data.shape[0], 0, self.page_table.data_ptr(),
                          self.page_size, self.page_table.shape[1])
        return CacheT(self.data.data_ptr(), self.data.shape[0], self.seq_stride, None, 0, 0)


class Workspace:
    """Device scratch for the calls that take one; grows on demand.  The
    header is zeroed at allocation (csa_workspace_init)."""

    def __init__(self, device=None):
        self.device = torch.device(device if device is not None else "cuda")
        self.buf = None

    def get(self, nbytes):
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes + 256:
            self.buf = torch.zeros(nbytes + 256, dtype=torch.uint8, device=self.device)
        base = self.buf.data_ptr()
        off = (-base) % 256
        return C.c_void_p(base + off), self.buf.numel() - off

    def check(self, stream=None):
        """Synchronise and raise CsaError if a kernel recorded a device check."""
        if self.buf is None:
            return
        ptr, _ = self.get(256)
        check(load().csa_workspace_check(ptr, _stream(stream)))


_default_ws = {}


def _ws(ws, device):
    if ws is not None:
        return ws
    key = torch.device(device).index
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


# ---------------------------------------------------------------------------
def compress_kv(C_a, Z_a, m, *, C_b=None, Z_b=None, bias=None, overlap=False, out=None,
                stream=None):
    """Step 1: coordinate-wise softmax pooling of [N, dim] into [N // m, dim]."""
    _need(C_a, "C_a", torch.bfloat16, 2)
    _need(Z_a, "Z_a", torch.bfloat16, 2, C_a.device)
    if Z_a.shape != C_a.shape:
        raise ValueError("C_a and Z_a shapes differ")
    N, dim = C_a.shape
    for name, t in (("C_b", C_b), ("Z_b", Z_b)):
        if t is not None:
            _need(t, name, torch.bfloat16, 2, C_a.device)
            if t.shape != C_a.shape:
                raise ValueError(f"{name} shape differs from C_a")
    if bias is not None:
        _need(bias, "bias", torch.float32, None, C_a.device)
        want = (2, m, dim) if overlap else (m, dim)
        if tuple(bias.shape) != want:
            raise ValueError(f"bias must be {want}")
    if out is None:
        out = torch.empty((N // m, dim), dtype=torch.bfloat16, device=C_a.device)
    _need(out, "out", torch.bfloat16, 2, C_a.device)
    check(load().csa_compress_kv(_ptr(C_a), _ptr(Z_a), _ptr(C_b), _ptr(Z_b), _ptr(bias), N, dim,
                                 m, int(bool(overlap)), _ptr(out), _stream(stream)))
    return out


def norm_rope(x, *, gain=None, eps=1e-6, pos=None, pos_mul=1, rope_dims=64, rope_base=10000.0,
              inverse=False, out=None, stream=None):
    """RMSNorm (eps >= 0; eps=None skips it) and partial RoPE (rope_dims > 0)
    of [T, H, dim] or [T, dim] bf16 vectors at positions (pos or row) * pos_mul;
    inverse=True applies the output de-rotation R_{-t} (use eps=None)."""
    _need(x, "x", torch.bfloat16)
    dev = x.device
    if x.dim() not in (2, 3):
        raise ValueError("x must be [T, dim] or [T, H, dim]")
    T, dim = x.shape[0], x.shape[-1]
    H = x.shape[1] if x.dim() == 3 else 1
    if gain is not None:
        _need(gain, "gain", torch.float32, 1, dev)
    if pos is not None:
        _need(pos, "pos", torch.int64, 1, dev)
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", torch.bfloat16, None, dev)
    check(load().csa_norm_rope(_ptr(x), _ptr(out), T, H, dim, _ptr(gain),
                               -1.0 if eps is None else float(eps), _ptr(pos), int(pos_mul),
                               int(rope_dims), float(rope_base), int(bool(inverse)), _stream(stream)))
    return out


@dataclass
class AppendState:
    """Per-sequence decode-time cache state for `cache_append`: the unfinished
    block's a-branch rows, the b-branch rows by block parity (overlap mode) and
    the window ring."""
    blk_c: torch.Tensor
    blk_z: torch.Tensor
    bb_c: Optional[torch.Tensor]
    bb_z: Optional[torch.Tensor]
    win: Optional[torch.Tensor]

    @staticmethod
    def new(B, dim, m, window, overlap, device="cuda"):
        z = lambda *shape: torch.zeros(shape, dtype=torch.bfloat16, device=device)
        return AppendState(z(B, m, dim), z(B, m, dim), z(B, 2, m, dim) if overlap else None,
                           z(B, 2, m, dim) if overlap else None,
                           z(B, window, dim) if window > 0 else None)


def cache_append(C_a, Z_a, pos, cache: Cache, m, state: AppendState, max_entries, *, C_b=None,
                 Z_b=None, bias=None, overlap=False, ws=None, stream=None):
    """Decode-time cache maintenance: append one token per sequence (C_a, Z_a
    [B, dim] at positions pos [B]); every m-th token completes a block, whose
    entry is written into `cache`.  `state` persists between calls."""
    _need(C_a, "C_a", torch.bfloat16, 2)
    dev = C_a.device
    B, dim = C_a.shape
    _need(Z_a, "Z_a", torch.bfloat16, 2, dev)
    _need(pos, "pos", torch.int64, 1, dev)
    for name, t in (("C_b", C_b), ("Z_b", Z_b)):
        if t is not None:
            _need(t, name, torch.bfloat16, 2, dev)
    if bias is not None:
        _need(bias, "bias", torch.float32, None, dev)
    window = state.win.shape[1] if state.win is not None else 0
    lib = load()
    wsp, wsb = _ws(ws, dev).get(256)
    kc = cache.c()
    check(lib.csa_cache_append(_ptr(C_a), _ptr(Z_a), _ptr(C_b), _ptr(Z_b), _ptr(bias), _ptr(pos), B,
                               dim, m, int(bool(overlap)), _ptr(state.blk_c), _ptr(state.blk_z),
                               _ptr(state.bb_c), _ptr(state.bb_z), _ptr(state.win), window,
                               C.byref(kc), max_entries, wsp, wsb, _stream(stream)))


def indexer_topk(q_idx, w, keys: Cache, m, top_k, *, seq_id=None, q_pos=None, max_entries=None,
                 return_scores=False, ws=None, stream=None, out=None):
    """Steps 2-3: lightning-indexer scores and exact top-k per query.
    Returns (idx [T, top_k] int32, count [T] int32[, scores [T, top_k] fp32])."""
    _need(q_idx, "q_idx", torch.bfloat16, 3)
    T, H_I, c_I = q_idx.shape
    dev = q_idx.device
    _need(w, "w", torch.float32, 2, dev)
    if tuple(w.shape) != (T, H_I):
        raise ValueError("w must be [T, H_I]")
    if keys.dim != c_I:
        raise ValueError("indexer keys dim differs from c_I")
    if seq_id is not None:
        _need(seq_id, "seq_id", torch.int32, 1, dev)
    if q_pos is not None:
        _need(q_pos, "q_pos", torch.int64, 1, dev)
    if max_entries is None:
        if q_pos is None:
            max_entries = max(T - 1, 0) // m
        else:
            raise ValueError("max_entries is required with q_pos")
    if out is None:
        idx = torch.empty((T, top_k), dtype=torch.int32, device=dev)
        cnt = torch.empty((T,), dtype=torch.int32, device=dev)
        sco = torch.empty((T, top_k), dtype=torch.float32, device=dev) if return_scores else None
    else:
        idx, cnt, sco = out
    lib = load()
    wsp, wsb = _ws(ws, dev).get(lib.csa_indexer_topk_workspace_size(T, max_entries, top_k))
    kc = keys.c()
    check(lib.csa_indexer_topk(_ptr(q_idx), _ptr(w), C.byref(kc), _ptr(seq_id), _ptr(q_pos), T,
                               H_I, c_I, m, max_entries, top_k, _ptr(idx), _ptr(cnt), _ptr(sco),
                               wsp, wsb, _stream(stream)))
    return (idx, cnt, sco) if return_scores else (idx, cnt)


def quantize_mxfp4(x, *, stream=None, out=None):
    """4-bit storage of bf16 vectors (E2M1 codes, one power-of-two scale byte
    per 32 elements; see include/csa.h): x [..., dim] -> (codes [..., dim/2]
    uint8, scales [..., dim/32] uint8)."""
    _need(x, "x", torch.bfloat16)
    dim = x.shape[-1]
    if dim % 32 != 0 or dim == 0:
        raise ValueError("the last dim must be a positive multiple of 32")
    n = x.numel() // dim
    if out is None:
        codes = torch.empty(x.shape[:-1] + (dim // 2,), dtype=torch.uint8, device=x.device)
        scales = torch.empty(x.shape[:-1] + (dim // 32,), dtype=torch.uint8, device=x.device)
    else:
        codes, scales = out
    check(load().csa_quantize_mxfp4(_ptr(x), n, dim, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def indexer_topk_mxfp4(q_idx, w, keys: Cache, k_scales, m, top_k, *, seq_id=None, q_pos=None,
                       max_entries=None, return_scores=False, ws=None, stream=None, out=None):
    """Steps 2-3 with the indexer keys in 4-bit storage: keys.data [rows,
    c_I/2] uint8 codes with k_scales [rows, c_I/32] uint8 (same rows, same
    paging), e.g. from quantize_mxfp4; the bf16 queries q_idx [T, H_I, c_I]
    are quantized to the same format inside the call.
    Returns (idx [T, top_k] int32, count [T] int32[, scores [T, top_k] fp32])."""
    _need(q_idx, "q_idx", torch.bfloat16, 3)
    T, H_I, c_I = q_idx.shape
    dev = q_idx.device
    _need(w, "w", torch.float32, 2, dev)
    if tuple(w.shape) != (T, H_I):
        raise ValueError("w must be [T, H_I]")
    if keys.dim * 2 != c_I:
        raise ValueError("key code rows must hold c_I/2 bytes")
    _need(k_scales, "k_scales", torch.uint8, 2, dev)
    if tuple(k_scales.shape) != (keys.data.shape[0], c_I // 32):
        raise ValueError("k_scales must be [rows of keys.data, c_I/32]")
    if seq_id is not None:
        _need(seq_id, "seq_id", torch.int32, 1, dev)
    if q_pos is not None:
        _need(q_pos, "q_pos", torch.int64, 1, dev)
    if max_entries is None:
        if q_pos is None:
            max_entries = max(T - 1, 0) // m
        else:
            raise ValueError("max_entries is required with q_pos")
    if out is None:
        idx = torch.empty((T, top_k), dtype=torch.int32, device=dev)
        cnt = torch.empty((T,), dtype=torch.int32, device=dev)
        sco = torch.empty((T, top_k), dtype=torch.float32, device=dev) if return_scores else None
    else:
        idx, cnt, sco = out
    lib = load()
    wsp, wsb = _ws(ws, dev).get(lib.csa_indexer_topk_workspace_size(T, max_entries, top_k))
    kc = keys.c(torch.uint8)
    check(lib.csa_indexer_topk_mxfp4(_ptr(q_idx), _ptr(w), C.byref(kc), _ptr(k_scales),
                                     _ptr(seq_id), _ptr(q_pos), T, H_I, c_I, m, max_entries, top_k,
                                     _ptr(idx), _ptr(cnt), _ptr(sco), wsp, wsb, _stream(stream)))
    return (idx, cnt, sco) if return_scores else (idx, cnt)


@dataclass
class QRope:
    """The attention calls' fused query prologue / output epilogue
    (csa_qrope_t): every query head becomes R_t . RMSNorm(q) * gain, rounded to
    bf16, before the dot products; with `derotate` each output head's last
    rope_dims coordinates are rotated back by R_{-t}.  eps < 0 skips the
    RMSNorm, rope_dims = 0 the rotation.  pos: int64 [T] query positions
    (required on decode calls; default: the row index, or q_pos for HCA)."""
    gain: "torch.Tensor | None" = None
    eps: float = 1e-6
    rope_dims: int = 64
    rope_base: float = 10000.0
    derotate: bool = True
    pos: "torch.Tensor | None" = None


def _qrope_c(qr, dev):
    if qr is None:
        return None
    if qr.gain is not None:
        _need(qr.gain, "qrope.gain", torch.float32, 1, dev)
    if qr.pos is not None:
        _need(qr.pos, "qrope.pos", torch.int64, 1, dev)
    return C.byref(QRopeT(_ptr(qr.gain), float(qr.eps), int(qr.rope_dims), float(qr.rope_base),
                          int(bool(qr.derotate)), _ptr(qr.pos)))


def sparse_attn_prefill(q, kv_comp, kv_raw, idx, count, window, sm_scale, *, sink=None,
                        qrope=None, return_lse=False, ws=None, stream=None, out=None):
    """Step 4 (CSA prefill): query t attends to kv_comp[idx[t, :count[t]]]
    and the raw window rows max(0, t-W+1) .. t; `qrope` (QRope) fuses the
    query RMSNorm / RoPE and the output de-rotation."""
    _need(q, "q", torch.bfloat16, 3)
    L, H, d = q.shape
    dev = q.device
    _need(kv_comp, "kv_comp", torch.bfloat16, 2, dev)
    _need(kv_raw, "kv_raw", torch.bfloat16, 2, dev)
    _need(idx, "idx", torch.int32, 2, dev)
    _need(count, "count", torch.int32, 1, dev)
    if sink is not None:
        _need(sink, "sink", torch.float32, 1, dev)
    top_k = idx.shape[1]
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((L, H), dtype=torch.float32, device=dev) if return_lse else None
    lib = load()
    wsp, wsb = _ws(ws, dev).get(lib.csa_sparse_attn_prefill_workspace_size(L, H, d))
    check(lib.csa_sparse_attn_prefill(_ptr(q), _ptr(kv_comp), kv_comp.shape[0], _ptr(kv_raw),
                                      _ptr(idx), _ptr(count), L, H, d, top_k, window,
                                      float(sm_scale), _ptr(sink), _ptr(out), _ptr(lse), wsp, wsb,
                                      _stream(stream), _qrope_c(qrope, dev)))
    return (out, lse) if return_lse else out


def sparse_attn_decode(q, kv: Cache, win, win_len, idx, count, sm_scale, *, sink=None,
                       qrope=None, return_lse=False, ws=None, stream=None, out=None):
    """Step 4 (CSA decode): query b attends to entries idx[b, :count[b]] of
    sequence b of `kv` and its window buffer win[b, :win_len[b]]; `qrope`
    (QRope, pos required) fuses the query prologue / output de-rotation."""
    _need(q, "q", torch.bfloat16, 3)
    B, H, d = q.shape
    dev = q.device
    _need(win, "win", torch.bfloat16, 3, dev)
    _need(win_len, "win_len", torch.int32, 1, dev)
    _need(idx, "idx", torch.int32, 2, dev)
    _need(count, "count", torch.int32, 1, dev)
    if sink is not None:
        _need(sink, "sink", torch.float32, 1, dev)
    top_k, window = idx.shape[1], win.shape[1]
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev) if return_lse else None
    lib = load()
    wsp, wsb = _ws(ws, dev).get(
        lib.csa_sparse_attn_decode_workspace_size(B, H, d, top_k, window))
    kc = kv.c()
    check(lib.csa_sparse_attn_decode(_ptr(q), C.byref(kc), _ptr(win), _ptr(win_len), _ptr(idx),
                                     _ptr(count), B, H, d, top_k, window, float(sm_scale),
                                     _ptr(sink), _ptr(out), _ptr(lse), wsp, wsb, _stream(stream),
                                     _qrope_c(qrope, dev)))
    return (out, lse) if return_lse else out


def quantize_entries_fp8(x, rope_dims=64, *, stream=None, out=None):
    """Mixed-precision storage of compressed entries x [..., dim] bf16 (E4M3
    content with a scale byte per 32, the last rope_dims coordinates kept in
    bf16; see include/csa.h): returns (codes [..., dim - rope_dims] uint8,
    scales [..., (dim - rope_dims)/32] uint8, rope [..., rope_dims] bf16)."""
    _need(x, "x", torch.bfloat16)
    dim = x.shape[-1]
    dc = dim - rope_dims
    if rope_dims < 0 or rope_dims % 8 or dc <= 0 or dc % 32:
        raise ValueError("need rope_dims a multiple of 8 below dim, dim - rope_dims a multiple of 32")
    n = x.numel() // dim
    lead = x.shape[:-1]
    if out is None:
        codes = torch.empty(lead + (dc,), dtype=torch.uint8, device=x.device)
        scales = torch.empty(lead + (dc // 32,), dtype=torch.uint8, device=x.device)
        rope = torch.empty(lead + (rope_dims,), dtype=torch.bfloat16, device=x.device)
    else:
        codes, scales, rope = out
    check(load().csa_quantize_entries_fp8(_ptr(x), n, dim, rope_dims, _ptr(codes), _ptr(scales),
                                          _ptr(rope) if rope_dims else None, _stream(stream)))
    return codes, scales, rope


def sparse_attn_decode_fp8(q, codes: Cache, scales, rope, win, win_len, idx, count, sm_scale, *,
                           sink=None, return_lse=False, ws=None, stream=None, out=None):
    """Step 4 (CSA decode) over mixed-precision entries: codes.data [rows,
    128 - r] uint8 (contiguous or paged), scales [rows, (128 - r)/32] uint8,
    rope [rows, r] bf16 (same rows), from quantize_entries_fp8; the window
    rows stay bf16.  Arguments otherwise as sparse_attn_decode."""
    _need(q, "q", torch.bfloat16, 3)
    B, H, d = q.shape
    dev = q.device
    rows = codes.data.shape[0]
    _need(scales, "scales", torch.uint8, 2, dev)
    _need(rope, "rope", torch.bfloat16, 2, dev)
    r = rope.shape[1]
    if codes.data.shape[1] != d - r or tuple(scales.shape) != (rows, (d - r) // 32) or rope.shape[0] != rows:
        raise ValueError("codes / scales / rope shapes do not describe the same entries")
    _need(win, "win", torch.bfloat16, 3, dev)
    _need(win_len, "win_len", torch.int32, 1, dev)
    _need(idx, "idx", torch.int32, 2, dev)
    _need(count, "count", torch.int32, 1, dev)
    if sink is not None:
        _need(sink, "sink", torch.float32, 1, dev)
    top_k, window = idx.shape[1], win.shape[1]
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev) if return_lse else None
    lib = load()
    wsp, wsb = _ws(ws, dev).get(lib.csa_sparse_attn_decode_workspace_size(B, H, d, top_k, window))
    kc = codes.c(torch.uint8)
    check(lib.csa_sparse_attn_decode_fp8(_ptr(q), C.byref(kc), _ptr(scales), _ptr(rope) if r else None,
                                         r, _ptr(win), _ptr(win_len), _ptr(idx), _ptr(count), B, H,
                                         d, top_k, window, float(sm_scale), _ptr(sink), _ptr(out),
                                         _ptr(lse), wsp, wsb, _stream(stream)))
    return (out, lse) if return_lse else out

def hca_attn(q, kv: Cache, kv_win, m, window, sm_scale, *, win_len=None, q_pos=None,
             seq_id=None, max_entries=None, sink=None, qrope=None, return_lse=False, ws=None,
             stream=None, out=None):
    """Step 4 (HCA): dense attention over every entry s < floor(t/m) plus the
    window.  Decode when `win_len` is given (kv_win [T, window, d]; query i
    reads sequence seq_id[i], default i); prefill otherwise: of sequence 0
    (kv_win = its raw tokens [*, d]), or, with `seq_id` and `q_pos`, of packed
    sequences whose raw rows kv_win [T, d] line up with the queries."""
    _need(q, "q", torch.bfloat16, 3)
    T, H, d = q.shape
    dev = q.device
    if win_len is not None:
        _need(win_len, "win_len", torch.int32, 1, dev)
        _need(kv_win, "kv_win", torch.bfloat16, 3, dev)
    else:
        _need(kv_win, "kv_win", torch.bfloat16, 2, dev)
    if q_pos is not None:
        _need(q_pos, "q_pos", torch.int64, 1, dev)
    if seq_id is not None:
        _need(seq_id, "seq_id", torch.int32, 1, dev)
        if win_len is None and q_pos is None:
            raise ValueError("packed prefill (seq_id without win_len) needs q_pos")
    if sink is not None:
        _need(sink, "sink", torch.float32, 1, dev)
    if max_entries is None:
        if q_pos is None:
            max_entries = max(T - 1, 0) // m
        else:
            raise ValueError("max_entries is required with q_pos")
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((T, H), dtype=torch.float32, device=dev) if return_lse else None
    lib = load()
    wsp, wsb = _ws(ws, dev).get(lib.hca_attn_workspace_size(T, H, d, max_entries, window))
    kc = kv.c()
    check(lib.hca_attn(_ptr(q), C.byref(kc), _ptr(kv_win), _ptr(win_len), _ptr(seq_id), _ptr(q_pos),
                       T, H, d, m,
                       max_entries, window, float(sm_scale), _ptr(sink), _ptr(out), _ptr(lse), wsp,
                       wsb, _stream(stream), _qrope_c(qrope, dev)))
    return (out, lse) if return_lse else out


def launch_count():
    """Kernels launched by the library since it was loaded."""
    return int(load().csa_launch_count())


ATTENTION_KERNELS = {"auto": 0, "tcgen05": 1, "mma_sync": 2}


def set_attention_kernel(name):
    """Choose the attention kernel: "auto" (default), "tcgen05" or "mma_sync"."""
    check(load().csa_set_attention_kernel(ATTENTION_KERNELS[name]))


def set_batch_invariant(on):
    """Batch-invariant decode attention on or off (see csa_set_batch_invariant)."""
    check(load().csa_set_batch_invariant(1 if on else 0))


def test_attention_timeout(on=True):
    """Failure-detection self-test (see csa_test_attention_timeout): the next
    tensor-core attention launch lets its bounded pipeline waits run out and
    records the timeout in its workspace header."""
    check(load().csa_test_attention_timeout(1 if on else 0))


def set_timing_events(kernel_id, begin=None, end=None):
    """Attach torch.cuda.Event objects (enable_timing=True) around every launch
    of one library kernel; pass None to detach."""
    b = C.c_void_p(begin.cuda_event) if begin is not None else None
    e = C.c_void_p(end.cuda_event) if end is not None else None
    check(load().csa_set_timing_events(kernel_id, b, e))
