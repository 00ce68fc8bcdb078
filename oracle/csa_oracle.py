"""fp64 reference definitions of the CSA / HCA hot path.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Source pages (cited by chapter and section):
  * "DeepSeek-V4" book (slop-6tp.pages.dev/papers-html-argon/dsv4.html),
    Ch.5 "How CSA Compresses Memory", Ch.6 "How CSA Selects and Reads Memory",
    Ch.7 "HCA, Local Attention, and Position".

Everything is computed in float64 from inputs that the caller has already
rounded to bf16 (the bytes the GPU sees, widened).  No blocking, fusion or
reordering beyond the definitions: each function is the formula written out,
with numpy's matmul / sort as the only library steps.

Readings taken where the pages are silent:
  R1  causal rule with 0-based positions: query t may use entry s iff
      s < floor(t/m) (Ch.5 "Causal availability and the local sliding window").
  R2  the window holds the raw tokens max(0, t-W+1) .. t, the current token
      included; entries that also sit in the window are not de-duplicated
      (Ch.7 "The 128-token uncompressed sliding window").
  R3  top-k ranks the indexer scores after rounding them to fp32 (the kernel's
      precision decides the integer result, as it would on the GPU); equal
      scores go to the lower entry index; with fewer than k eligible entries all
      of them are taken; indices are reported in ascending order.
  R4  compressed entries are stored in bf16, so the pipelines round the pooled
      entries to bf16 (round-to-nearest-even) before the indexer and the
      attention read them.
  R5  the optional sink adds exp(z'_h) to each head's softmax denominator; the
      reported log-sum-exp is the log of that full denominator.
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------
def bf16_round(x):
    """Round to the nearest bf16 value (ties to even), returned as float64.

    Goes through float32 (numpy's own round-to-nearest), then keeps the top
    16 bits of the float32 pattern with round-to-nearest-even on the rest.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# paged compressed caches
# ---------------------------------------------------------------------------
def page_rows(table_row, n_entries, page_size):
    """Physical rows of logical entries 0 .. n_entries-1 of one sequence of a
    paged compressed cache: entry s sits in the page table_row[s // page_size]
    at offset s % page_size, i.e. at physical row
    table_row[s // page_size] * page_size + s % page_size.

    The DeepSeek-V4 infrastructure transcript ("KV cache management": the
    classical KV cache holds the CSA / HCA compressed entries, managed in
    blocks) leaves the block addressing open; this is the plainest reading,
    the usual block-table mapping of a paged cache.  Returns int64 [n_entries].
    """
    table = np.asarray(table_row, dtype=np.int64)
    s = np.arange(int(n_entries), dtype=np.int64)
    return table[s // page_size] * page_size + s % page_size


def unpage(pool, table_row, n_entries, page_size):
    """Logical [n_entries, dim] view of one sequence of a paged pool: the rows
    page_rows(...) of `pool` (a numpy array or a CPU torch tensor)."""
    return pool[page_rows(table_row, n_entries, page_size)]


# ---------------------------------------------------------------------------
# step 1: block compression by coordinate-wise softmax pooling
# ---------------------------------------------------------------------------
def _softmax_pool(content, logits):
    """One compressed entry: for every coordinate r, a softmax over the source
    positions j of logits[j, r], used to weight content[j, r]
    (Ch.5 "Coordinate-wise softmax pooling")."""
    top = logits.max(axis=0)
    e = np.exp(logits - top)
    return (e * content).sum(axis=0) / e.sum(axis=0)


def pool_block(C, Z, m, B=None):
    """Non-overlapping pooling: entry i pools tokens m*i .. m*(i+1)-1 with
    logits Z[j] + B[j - m*i] (Ch.7 "HCA's 128:1 non-overlapping compressor").

    C, Z: [N, c]; B: [m, c] or None.  Returns [floor(N/m), c]; trailing tokens
    that do not fill a block produce no entry.
    """
    C = np.asarray(C, dtype=np.float64)
    Z = np.asarray(Z, dtype=np.float64)
    N, c = C.shape
    S = N // m
    out = np.empty((S, c))
    bias = 0.0 if B is None else np.asarray(B, dtype=np.float64)
    for i in range(S):
        rows = slice(m * i, m * (i + 1))
        out[i] = _softmax_pool(C[rows], Z[rows] + bias)
    return out


def pool_overlap(Ca, Za, Cb, Zb, m, Ba=None, Bb=None):
    """Overlapping CSA pooling (Ch.5 "Coordinate-wise softmax pooling").

    Entry i pools 2m positions: the a branch is block i (tokens m*i ..
    m*(i+1)-1, content Ca, logits Za + Ba), the b branch is block i-1 (tokens
    m*(i-1) .. m*i-1, content Cb, logits Zb + Bb).  For i = 0 there is no
    previous block: its b-branch content is zero and its logits are -inf, so
    all weight falls on tokens 0 .. m-1 ("Receptive field versus compression
    stride").
    """
    Ca, Za, Cb, Zb = (np.asarray(a, dtype=np.float64) for a in (Ca, Za, Cb, Zb))
    N, c = Ca.shape
    S = N // m
    ba = 0.0 if Ba is None else np.asarray(Ba, dtype=np.float64)
    bb = 0.0 if Bb is None else np.asarray(Bb, dtype=np.float64)
    out = np.empty((S, c))
    for i in range(S):
        a = slice(m * i, m * (i + 1))
        ua = Za[a] + ba
        if i == 0:
            ub = np.full((m, c), -np.inf)
            cb = np.zeros((m, c))
        else:
            b = slice(m * (i - 1), m * i)
            ub = Zb[b] + bb
            cb = Cb[b]
        out[i] = _softmax_pool(np.concatenate([Ca[a], cb]), np.concatenate([ua, ub]))
    return out


class DecodeCacheState:
    """Decode-time cache state of one sequence (Ch.5 "Decode-time cache state";
    Ch.8 "Quantization scales and bounded tail buffers"): the growing list of
    compressed entries, the window of the last W raw rows, the rows of the
    unfinished block and, in overlap mode, the b-branch rows of the last
    completed block.  `append` takes one decode token; the entry of a block is
    made when its last token arrives, from the block (and the previous block's
    b-branch rows) alone, with the same pooling definition as the bulk
    compressor."""

    def __init__(self, m, W, overlap, Ba=None, Bb=None):
        self.m, self.W, self.overlap = int(m), int(W), bool(overlap)
        self.Ba, self.Bb = Ba, Bb
        self.t = 0
        self.entries = []
        self.window = []        # raw rows, oldest first, at most W
        self.block = []         # (c_a, z_a, c_b, z_b) of the unfinished block
        self.prev_b = None      # (C_b rows, Z_b rows) of the last completed block

    def append(self, c_a, z_a, c_b=None, z_b=None):
        c_a, z_a = np.asarray(c_a, dtype=np.float64), np.asarray(z_a, dtype=np.float64)
        c_b = c_a if c_b is None else np.asarray(c_b, dtype=np.float64)
        z_b = z_a if z_b is None else np.asarray(z_b, dtype=np.float64)
        if self.W > 0:
            self.window = (self.window + [c_a])[-self.W:]
        self.block.append((c_a, z_a, c_b, z_b))
        self.t += 1
        if len(self.block) == self.m:
            Ca, Za, Cb, Zb = (np.stack([r[k] for r in self.block]) for k in range(4))
            if not self.overlap:
                self.entries.append(pool_block(Ca, Za, self.m, self.Ba)[0])
            elif self.prev_b is None:        # block 0: no previous block
                self.entries.append(pool_overlap(Ca, Za, Cb, Zb, self.m, self.Ba, self.Bb)[0])
            else:                            # blocks i-1 (b branch only) and i
                pCb, pZb = self.prev_b
                two = lambda p, q: np.concatenate([p, q])
                self.entries.append(pool_overlap(two(Ca, Ca), two(Za, Za), two(pCb, Cb), two(pZb, Zb),
                                                 self.m, self.Ba, self.Bb)[1])
            self.prev_b = (Cb, Zb)
            self.block = []


# ---------------------------------------------------------------------------
# attention prologue / epilogue: RMSNorm, partial RoPE, output de-rotation
# ---------------------------------------------------------------------------
def rmsnorm(x, gain=None, eps=1e-6):
    """RMSNorm over the last axis (Ch.2 "Normalization and rotary position
    embeddings"; Ch.7 "Query and KV RMSNorm"): x / sqrt(mean(x^2) + eps),
    times a per-coordinate gain.  eps is not printed; 1e-6 is the reading."""
    x = np.asarray(x, dtype=np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if gain is None else y * np.asarray(gain, dtype=np.float64)


def rope_rotate(x, pos, rope_dims=64, base=10000.0, inverse=False):
    """Partial RoPE (Ch.7 "Partial RoPE and output de-rotation"): the last
    `rope_dims` coordinates of every vector are rotated by R_t, block-diagonal
    with 2x2 rotations of the pairs (2j, 2j+1) of the rotary slice by angle
    t * base^(-2j / rope_dims); inverse applies R_{-t} = R_t^T.  The pairing
    and the base are not printed; interleaved pairs and base 10000 are the
    reading.  x: [..., d]; pos: broadcastable to x.shape[:-1]."""
    x = np.array(x, dtype=np.float64)
    d = x.shape[-1]
    r0 = d - rope_dims
    j = np.arange(rope_dims // 2)
    theta = base ** (-2.0 * j / rope_dims)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    if inverse:
        ang = -ang
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., r0::2].copy(), x[..., r0 + 1::2].copy()
    x[..., r0::2] = a * c - b * s
    x[..., r0 + 1::2] = a * s + b * c
    return x


# ---------------------------------------------------------------------------
# steps 2-3: lightning indexer and top-k
# ---------------------------------------------------------------------------
def eligible_entries(t, m):
    """Number of compressed entries query position t may read: s < floor(t/m)
    (Ch.5 "Causal availability and the local sliding window"; Ch.6 "The
    lightning indexer")."""
    return int(t) // int(m)


def indexer_scores(qI, w, KI):
    """I_s = sum_h w_h * ReLU(qI_h . KI_s) for every row s of KI
    (Ch.6 "The lightning indexer").  qI: [H_I, c_I]; w: [H_I]; KI: [n, c_I]."""
    qI = np.asarray(qI, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    KI = np.asarray(KI, dtype=np.float64)
    dots = KI @ qI.T                      # [n, H_I]
    return np.maximum(dots, 0.0) @ w      # [n]


def topk_select(scores, k):
    """Indices of the k highest scores (Ch.6 "Top-k selection and asymptotic
    scaling"), under reading R3: ranked on fp32-rounded scores, ties to the
    lower index, all entries if fewer than k, ascending order."""
    s32 = np.asarray(scores, dtype=np.float32).astype(np.float64)
    n = s32.shape[0]
    if n <= k:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((np.arange(n), -s32))   # primary: score desc; then index asc
    return np.sort(order[:k])


# ---------------------------------------------------------------------------
# step 4: shared-KV softmax attention
# ---------------------------------------------------------------------------
def attend_shared_kv(q, rows, lam, sink=None):
    """All query heads attend to the same rows, each row serving as both key
    and value (Ch.6 "Shared key-value MQA"), in one softmax over every row
    given (Ch.7 "The 128-token uncompressed sliding window"); an optional
    per-head sink logit adds exp(z'_h) to the denominator (Ch.7 "Learned
    attention sinks").

    q: [H, d]; rows: [n, d]; returns (o [H, d], lse [H]).
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    logits = lam * (q @ rows.T)                       # [H, n]
    top = logits.max(axis=1) if rows.shape[0] else np.full(q.shape[0], -np.inf)
    if sink is not None:
        top = np.maximum(top, np.asarray(sink, dtype=np.float64))
    e = np.exp(logits - top[:, None])
    den = e.sum(axis=1)
    if sink is not None:
        den = den + np.exp(np.asarray(sink, dtype=np.float64) - top)
    o = (e @ rows) / den[:, None]
    return o, top + np.log(den)


def prefill_window_rows(t, W):
    """Raw-token rows in query t's window: max(0, t-W+1) .. t (reading R2)."""
    return np.arange(max(0, t - W + 1), t + 1)


# ---------------------------------------------------------------------------
# pipelines
# ---------------------------------------------------------------------------
def csa_prefill_topk(qI, w, KI, m, k, rows=None):
    """Top-k entry lists for prefill queries t (all rows, or the given ones).
    Returns (idx [n_rows, k] padded with -1, count [n_rows])."""
    L = qI.shape[0]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    idx = np.full((rows.shape[0], k), -1, dtype=np.int64)
    cnt = np.zeros(rows.shape[0], dtype=np.int64)
    for r, t in enumerate(rows):
        n = eligible_entries(t, m)
        sel = topk_select(indexer_scores(qI[t], w[t], KI[:n]), k)
        idx[r, :sel.shape[0]] = sel
        cnt[r] = sel.shape[0]
    return idx, cnt


def csa_prefill_attention(q, kv_comp, kv_raw, idx, count, W, lam, sink=None, rows=None):
    """CSA attention for prefill queries: selected compressed entries plus the
    raw window, one softmax (Ch.6 "Shared key-value MQA"; Ch.7 "The 128-token
    uncompressed sliding window").  idx/count are indexed like `rows`."""
    L, H, d = q.shape
    rows = np.arange(L) if rows is None else np.asarray(rows)
    out = np.empty((rows.shape[0], H, d))
    lse = np.empty((rows.shape[0], H))
    for r, t in enumerate(rows):
        sel = np.asarray(idx[r][: int(count[r])], dtype=np.int64)
        kv = np.concatenate([kv_comp[sel], kv_raw[prefill_window_rows(t, W)]])
        out[r], lse[r] = attend_shared_kv(q[t], kv, lam, sink)
    return out, lse


def csa_prefill(q, kv_raw, Z, kI_raw, ZI, qI, w, m, k, W, lam, sink=None,
                B=None, BI=None, rows=None):
    """Whole CSA prefill of one sequence from raw inputs, block pooling
    (the configured "softmaxed within each block" compressor): compress the
    main KV and the indexer keys, round them to bf16 storage (R4), score,
    select, attend.  Returns (out, lse, idx, count, kv_comp, kI_comp)."""
    kv_comp = bf16_round(pool_block(kv_raw, Z, m, B))
    kI_comp = bf16_round(pool_block(kI_raw, ZI, m, BI))
    idx, cnt = csa_prefill_topk(qI, w, kI_comp, m, k, rows)
    out, lse = csa_prefill_attention(q, kv_comp, kv_raw, idx, cnt, W, lam, sink, rows)
    return out, lse, idx, cnt, kv_comp, kI_comp


def csa_decode(q, kv_comp, kI_comp, qI, w, win, win_len, pos, m, k, lam, sink=None,
               seqs=None):
    """One decode step of CSA for a batch: sequence b's new token sits at
    position pos[b], so floor(pos[b]/m) entries are eligible (R1); the window
    buffer win[b, :win_len[b]] holds its recent raw tokens, oldest first,
    the new token last (R2).  kv_comp / kI_comp are per-sequence logical
    arrays [S_b, d] / [S_b, c_I].  Returns (out, lse, idx, count)."""
    B, H, d = q.shape
    seqs = np.arange(B) if seqs is None else np.asarray(seqs)
    out = np.empty((seqs.shape[0], H, d))
    lse = np.empty((seqs.shape[0], H))
    idx = np.full((seqs.shape[0], k), -1, dtype=np.int64)
    cnt = np.zeros(seqs.shape[0], dtype=np.int64)
    for r, b in enumerate(seqs):
        n = eligible_entries(pos[b], m)
        sel = topk_select(indexer_scores(qI[b], w[b], kI_comp[b][:n]), k)
        idx[r, :sel.shape[0]] = sel
        cnt[r] = sel.shape[0]
        kv = np.concatenate([kv_comp[b][sel], win[b][: int(win_len[b])]])
        out[r], lse[r] = attend_shared_kv(q[b], kv, lam, sink)
    return out, lse, idx, cnt


def hca_decode(q, kv_comp, win, win_len, pos, m, lam, sink=None, seqs=None):
    """One HCA decode step: dense attention over every eligible heavily
    compressed entry s < floor(pos/m) plus the window (Ch.7 "Dense attention
    over heavily compressed history")."""
    B, H, d = q.shape
    seqs = np.arange(B) if seqs is None else np.asarray(seqs)
    out = np.empty((seqs.shape[0], H, d))
    lse = np.empty((seqs.shape[0], H))
    for r, b in enumerate(seqs):
        n = eligible_entries(pos[b], m)
        kv = np.concatenate([kv_comp[b][:n], win[b][: int(win_len[b])]])
        out[r], lse[r] = attend_shared_kv(q[b], kv, lam, sink)
    return out, lse


def hca_prefill(q, kv_comp, kv_raw, m, W, lam, sink=None, rows=None):
    """HCA for prefill queries t: all entries s < floor(t/m) plus the raw
    window max(0, t-W+1) .. t."""
    L, H, d = q.shape
    rows = np.arange(L) if rows is None else np.asarray(rows)
    out = np.empty((rows.shape[0], H, d))
    lse = np.empty((rows.shape[0], H))
    for r, t in enumerate(rows):
        n = eligible_entries(t, m)
        kv = np.concatenate([kv_comp[:n], kv_raw[prefill_window_rows(t, W)]])
        out[r], lse[r] = attend_shared_kv(q[t], kv, lam, sink)
    return out, lse
