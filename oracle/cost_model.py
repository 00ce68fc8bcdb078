"""Cost model of the DeepSeek-V4 book, Ch.8 "A Cost Model for Long Context"
(and Ch.6 "Grouped output projections", Ch.7 "HCA's 128:1 non-overlapping
compressor").

TEST INFRASTRUCTURE ONLY.  Exact integer / rational arithmetic from the model
dimensions the pages state; the tests compare the results with the figures
the pages print.
"""
from __future__ import annotations

from fractions import Fraction


def gqa8_bytes_per_token_layer(kv_heads=8, head_dim=128, elem_bytes=2):
    """Separate K and V vectors per token per layer ("Baseline: conventional
    GQA8 cache payload")."""
    return 2 * kv_heads * head_dim * elem_bytes


def gqa8_cache_bytes(n_tokens, n_layers, **kw):
    return gqa8_bytes_per_token_layer(**kw) * n_tokens * n_layers


def v4_entry_bytes(c=512, rope_dims=64, content_bytes=1, rope_bytes=2):
    """One shared KV entry: non-rotary channels in FP8, the last rope_dims
    channels in BF16 ("V4 compressed-entry payload")."""
    return (c - rope_dims) * content_bytes + rope_dims * rope_bytes


def main_cache_bytes_per_token(m, **kw):
    """Amortised growth of one layer's compressed main cache per raw token."""
    return Fraction(v4_entry_bytes(**kw), m)


def indexer_key_bytes(c_idx=128, bits=4):
    return Fraction(c_idx * bits, 8)


def csa_bytes_per_token(m=4, c_idx=128):
    """Main entry plus indexer key, per raw token, in one CSA layer."""
    return main_cache_bytes_per_token(m) + indexer_key_bytes(c_idx) / m


def model_cache_bytes(n_tokens, n_csa, n_hca, m_csa=4, m_hca=128):
    """Whole-model growing cache ("Whole-model KV cache footprint")."""
    per_tok = n_csa * csa_bytes_per_token(m_csa) + n_hca * main_cache_bytes_per_token(m_hca)
    return per_tok * n_tokens


def fp4_scale_overhead(c_idx=128, group=32, scale_bytes=1):
    """Scale bytes over payload bytes for an FP4 key with one scale per group
    ("Quantization scales and bounded tail buffers")."""
    return Fraction(c_idx // group * scale_bytes, indexer_key_bytes(c_idx))


def hca_entries(n_tokens, m=128):
    """Completed HCA entries and the trailing tokens left to the window."""
    return n_tokens // m, n_tokens % m


def attention_flops(n_heads, c, n_entries):
    """2cE for QK plus 2cE for PV per head ("Main-attention versus indexer
    arithmetic")."""
    return 4 * n_heads * c * n_entries


def indexer_ops(n_tokens, m, idx_heads, c_idx):
    """Multiply-add count x2 of one decode indexer scan over N/m keys."""
    return 2 * (n_tokens // m) * idx_heads * c_idx


def grouped_out_proj_params(n_heads, c, d, groups, d_g):
    """(direct, grouped) parameter counts of the output projection
    (Ch.6 "Grouped output projections")."""
    direct = n_heads * c * d
    grouped = n_heads * c * d_g + groups * d_g * d
    return direct, grouped
