"""Seeded synthetic inputs for the CSA / HCA hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Tests feed the same tensors to the CUDA library and to
the oracle; ``bench.py`` feeds them to the library (and to the oracle for its
CPU-baseline leg).  Every tensor is drawn in float32 on the CPU from a seeded
``torch.Generator`` and rounded once to bf16 where the path stores bf16.

Workloads (shapes of the DeepSeek-V4 long-context configurations):
  csa_prefill   one sequence, L tokens: raw KV, pooling logits, raw indexer
                keys and their logits, queries, indexer queries and weights
  csa_decode    B sequences, one new token each, compressed caches resident
  hca_decode    B sequences, heavily compressed cache, one new token each
  mixed_decode  B ragged sequences, 4 layers CSA/HCA/CSA/HCA, paged caches
"""
from __future__ import annotations

import dataclasses
import math

import torch

BF16 = torch.bfloat16


# ---------------------------------------------------------------------------
# workload descriptions
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class CsaPrefill:
    name: str
    L: int
    H: int
    d: int
    H_I: int
    c_I: int
    m: int
    k: int
    W: int
    q_scale: float      # queries drawn N(0,1) * q_scale
    lam: float          # softmax scale passed to the attention
    low_rank: int = 0   # rank of the shared key component (0 = none)
    seed: int = 0
    w_dist: str = "uniform"


@dataclasses.dataclass(frozen=True)
class CsaDecode:
    name: str
    B: int
    N: int
    H: int
    d: int
    H_I: int
    c_I: int
    m: int
    k: int
    W: int
    lam: float
    seed: int = 1
    w_dist: str = "uniform"


@dataclasses.dataclass(frozen=True)
class HcaDecode:
    name: str
    B: int
    N: int
    H: int
    d: int
    m: int
    W: int
    lam: float
    seed: int = 3


@dataclasses.dataclass(frozen=True)
class MixedDecode:
    name: str
    B: int
    N_lo: int
    N_hi: int
    H: int
    d: int
    H_I: int
    c_I: int
    m_csa: int
    m_hca: int
    k: int
    W: int
    lam: float
    page_size: int
    layers: tuple = ("csa", "hca", "csa", "hca")
    seed: int = 4


INV_SQRT_128 = 1.0 / math.sqrt(128.0)

# The five long-context workloads.
CFG_PREFILL_4K = CsaPrefill("csa_prefill_L4096", L=4096, H=8, d=128, H_I=4, c_I=64, m=4,
                            k=64, W=128, q_scale=INV_SQRT_128, lam=1.0, seed=0)
CFG_DECODE_128K = CsaDecode("csa_decode_B64_N131072", B=64, N=131072, H=64, d=128, H_I=8,
                            c_I=64, m=4, k=2048, W=128, lam=INV_SQRT_128, seed=1)
CFG_PREFILL_64K = CsaPrefill("csa_prefill_L65536", L=65536, H=64, d=128, H_I=8, c_I=64, m=4,
                             k=2048, W=128, q_scale=1.0, lam=INV_SQRT_128, low_rank=16, seed=2)
CFG_HCA_1M = HcaDecode("hca_decode_B8_N1048576", B=8, N=1 << 20, H=64, d=128, m=128, W=128,
                       lam=INV_SQRT_128, seed=3)
CFG_MIXED = MixedDecode("mixed_decode_B16_N256K_1M", B=16, N_lo=1 << 18, N_hi=1 << 20, H=64,
                        d=128, H_I=8, c_I=64, m_csa=4, m_hca=128, k=2048, W=128,
                        lam=INV_SQRT_128, page_size=64, seed=4)

# The 128K decode with the indexer keys and queries held in 4-bit storage
# (same seeded inputs; the keys are quantized when the cache is built).
CFG_DECODE_128K_MXFP4 = dataclasses.replace(CFG_DECODE_128K, name="csa_decode_B64_N131072_mxfp4_indexer")
# ... and the main entries in FP8 content + bf16 rotary storage as well.
CFG_DECODE_128K_LOWPREC = dataclasses.replace(CFG_DECODE_128K, name="csa_decode_B64_N131072_lowprec")

WORKLOADS = {c.name: c for c in (CFG_PREFILL_4K, CFG_DECODE_128K, CFG_PREFILL_64K, CFG_HCA_1M,
                                 CFG_MIXED, CFG_DECODE_128K_MXFP4, CFG_DECODE_128K_LOWPREC)}


# ---------------------------------------------------------------------------
# drawing helpers
# ---------------------------------------------------------------------------
def generator(seed):
    return torch.Generator().manual_seed(int(seed))


def normal(g, shape, scale=1.0, dtype=BF16):
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def uniform(g, shape, dtype=torch.float32):
    return torch.rand(shape, generator=g, dtype=torch.float32).to(dtype)


def head_weights(g, shape, dist):
    return uniform(g, shape) if dist == "uniform" else normal(g, shape, dtype=torch.float32)


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------
def csa_prefill_inputs(cfg: CsaPrefill, L=None):
    """Raw inputs of one CSA prefill.  With ``low_rank`` r > 0 both the raw KV
    and the raw indexer keys get a shared rank-r component A_t @ U (A_t ~
    N(0,1)^r per token, U ~ N(0,1)^(r x dim) / 4, its own U per tensor)."""
    L = cfg.L if L is None else L
    g = generator(cfg.seed)
    q = normal(g, (L, cfg.H, cfg.d), cfg.q_scale)
    kv = torch.randn((L, cfg.d), generator=g)
    kI = torch.randn((L, cfg.c_I), generator=g)
    if cfg.low_rank:
        A = torch.randn((L, cfg.low_rank), generator=g)
        U = torch.randn((cfg.low_rank, cfg.d), generator=g) / 4
        UI = torch.randn((cfg.low_rank, cfg.c_I), generator=g) / 4
        kv += A @ U
        kI += A @ UI
    return dict(
        q=q,
        kv_raw=kv.to(BF16),
        Z=normal(g, (L, cfg.d)),
        kI_raw=kI.to(BF16),
        ZI=normal(g, (L, cfg.c_I)),
        qI=normal(g, (L, cfg.H_I, cfg.c_I)),
        w=head_weights(g, (L, cfg.H_I), cfg.w_dist),
    )


def csa_decode_inputs(cfg: CsaDecode, B=None):
    """Resident compressed caches (contiguous, [B, S, dim]) plus one new token
    per sequence at position N: its query, indexer query, head weights and
    the window buffer of its last W raw tokens (oldest first, itself last)."""
    B = cfg.B if B is None else B
    S = cfg.N // cfg.m
    g = generator(cfg.seed)
    return dict(
        q=normal(g, (B, cfg.H, cfg.d)),
        qI=normal(g, (B, cfg.H_I, cfg.c_I)),
        w=head_weights(g, (B, cfg.H_I), cfg.w_dist),
        kv_comp=normal(g, (B, S, cfg.d)),
        kI_comp=normal(g, (B, S, cfg.c_I)),
        win=normal(g, (B, cfg.W, cfg.d)),
        win_len=torch.full((B,), min(cfg.W, cfg.N + 1), dtype=torch.int32),
        pos=torch.full((B,), cfg.N, dtype=torch.int64),
    )


def hca_decode_inputs(cfg: HcaDecode, B=None):
    B = cfg.B if B is None else B
    S = cfg.N // cfg.m
    g = generator(cfg.seed)
    return dict(
        q=normal(g, (B, cfg.H, cfg.d)),
        kv_comp=normal(g, (B, S, cfg.d)),
        win=normal(g, (B, cfg.W, cfg.d)),
        win_len=torch.full((B,), min(cfg.W, cfg.N + 1), dtype=torch.int32),
        pos=torch.full((B,), cfg.N, dtype=torch.int64),
    )


def paged_pool(g, n_entries, dim, page_size):
    """A shuffled page pool holding len(n_entries) logical caches.

    Returns (pool [P*page_size, dim] bf16, page_table [B, max_pages] int32,
    padded with -1).  Sequence b's logical entry s lives at physical row
    page_table[b, s // page_size] * page_size + s % page_size."""
    pages = [-(-int(n) // page_size) for n in n_entries]
    total = sum(pages)
    perm = torch.randperm(total, generator=g).to(torch.int32)
    table = torch.full((len(pages), max(pages)), -1, dtype=torch.int32)
    off = 0
    for b, p in enumerate(pages):
        table[b, :p] = perm[off:off + p]
        off += p
    pool = normal(g, (total * page_size, dim))
    return pool, table


def mixed_decode_inputs(cfg: MixedDecode, B=None):
    """Ragged lengths N_b ~ U[N_lo, N_hi]; per layer its own paged caches
    (one page table shared by the main and indexer caches of a CSA layer),
    queries and window buffers."""
    B = cfg.B if B is None else B
    g = generator(cfg.seed)
    N = torch.randint(cfg.N_lo, cfg.N_hi + 1, (B,), generator=g, dtype=torch.int64)
    layers = []
    for kind in cfg.layers:
        m = cfg.m_csa if kind == "csa" else cfg.m_hca
        S = [int(n) // m for n in N]
        lay = dict(kind=kind, m=m, S=torch.tensor(S, dtype=torch.int64),
                   q=normal(g, (B, cfg.H, cfg.d)),
                   win=normal(g, (B, cfg.W, cfg.d)),
                   win_len=torch.clamp(N + 1, max=cfg.W).to(torch.int32))
        lay["kv_pool"], lay["page_table"] = paged_pool(g, S, cfg.d, cfg.page_size)
        if kind == "csa":
            lay["qI"] = normal(g, (B, cfg.H_I, cfg.c_I))
            lay["w"] = uniform(g, (B, cfg.H_I))
            # indexer keys share the layer's page table
            lay["kI_pool"] = normal(g, (lay["kv_pool"].shape[0], cfg.c_I))
        layers.append(lay)
    return dict(pos=N, layers=layers)


def random_topk_lists(g, T, k, n_eligible):
    """Valid entry lists for attention-only cases: per query a random subset
    of min(k, n_eligible[t]) distinct eligible entries, ascending, padded with
    -1.  Returns (idx [T, k] int32, count [T] int32)."""
    idx = torch.full((T, k), -1, dtype=torch.int32)
    cnt = torch.zeros(T, dtype=torch.int32)
    for t in range(T):
        n = int(n_eligible[t])
        c = min(k, n)
        if c:
            sel = torch.randperm(n, generator=g)[:c].sort().values
            idx[t, :c] = sel.to(torch.int32)
        cnt[t] = c
    return idx, cnt


def fp4_codes(g, rows_shape, dim, scale_lo=124, scale_hi=129):
    """Random 4-bit storage of vectors of `dim` elements: uniform code bytes
    (every E2M1 code equally likely in each nibble) [*rows_shape, dim/2] and
    uniform scale bytes in [scale_lo, scale_hi) [*rows_shape, dim/32]
    (uint8).  Raw bytes only: both sides decode them."""
    shape = tuple(rows_shape)
    codes = torch.randint(0, 256, shape + (dim // 2,), generator=g, dtype=torch.int32).to(torch.uint8)
    scales = torch.randint(scale_lo, scale_hi, shape + (dim // 32,), generator=g,
                           dtype=torch.int32).to(torch.uint8)
    return codes, scales
