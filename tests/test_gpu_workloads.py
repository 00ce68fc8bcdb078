"""The five long-context workloads at full size, run through the C ABI in the
launch configuration the bench times, checked against the oracle on sampled
outputs (the oracle computes each sampled query from the raw inputs)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_attn, assert_mostly_exact, check_topk, dev, f64, score_eps

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_kv_03_b200 as csa
    csa.load()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _csa():
    import compressed_sparse_kv_03_b200 as csa
    return csa


def e2e_eps(qI, w, KI):
    """Score tolerance when both sides compress the keys themselves: the
    fp32 accumulation bound plus one bf16 rounding step (2^-8 relative) of
    each stored key coordinate."""
    if KI.shape[0] == 0:
        return 0.0
    kmax = np.abs(KI).max(axis=0)
    return score_eps(qI, w, KI) + 2.0 ** -8 * float(np.abs(w) @ (np.abs(qI) @ kmax))


def _prefill_pipeline(cfg, x):
    csa = _csa()
    kv_raw, kI_raw = dev(x["kv_raw"]), dev(x["kI_raw"])
    kv_comp = csa.compress_kv(kv_raw, dev(x["Z"]), cfg.m)
    kI_comp = csa.compress_kv(kI_raw, dev(x["ZI"]), cfg.m)
    idx, cnt = csa.indexer_topk(dev(x["qI"]), dev(x["w"]), csa.Cache(kI_comp), cfg.m, cfg.k)
    out = csa.sparse_attn_prefill(dev(x["q"]), kv_comp, kv_raw, idx, cnt, cfg.W, cfg.lam)
    torch.cuda.synchronize()
    return kv_comp, kI_comp, idx, cnt, out


def _check_prefill(cfg, x, rows):
    kv_comp, kI_comp, idx, cnt, out = _prefill_pipeline(cfg, x)
    kvc_ref = oracle.bf16_round(oracle.pool_block(f64(x["kv_raw"]), f64(x["Z"]), cfg.m))
    kIc_ref = oracle.bf16_round(oracle.pool_block(f64(x["kI_raw"]), f64(x["ZI"]), cfg.m))
    assert_close_attn(kv_comp, kvc_ref, "compressed main KV")
    assert_close_attn(kI_comp, kIc_ref, "compressed indexer keys")
    qI, w = x["qI"], x["w"]
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    stats = {"exact": 0, "near-tie": 0}
    ref_idx = np.full((len(rows), cfg.k), -1, dtype=np.int64)
    ref_cnt = np.zeros(len(rows), dtype=np.int64)
    for r, t in enumerate(rows):
        n = t // cfg.m
        s = oracle.indexer_scores(f64(qI[t]), f64(w[t]), kIc_ref[:n])
        stats[check_topk(idx_h[t], cnt_h[t], s, cfg.k, e2e_eps(f64(qI[t]), f64(w[t]), kIc_ref[:n]))] += 1
        sel = oracle.topk_select(s, cfg.k)
        ref_idx[r, :sel.shape[0]] = sel
        ref_cnt[r] = sel.shape[0]
    q_rows = np.zeros((max(rows) + 1, cfg.H, cfg.d))
    q_rows[rows] = f64(x["q"][rows])
    ref_out, _ = oracle.csa_prefill_attention(q_rows, kvc_ref, f64(x["kv_raw"]), ref_idx, ref_cnt,
                                              cfg.W, cfg.lam, rows=rows)
    assert_close_attn(out[rows], ref_out, "prefill output")
    return stats


def test_csa_prefill_L4096_full():
    cfg = synth.CFG_PREFILL_4K
    x = synth.csa_prefill_inputs(cfg)
    stats = _check_prefill(cfg, x, list(range(cfg.L)))
    assert stats["exact"] >= 0.99 * cfg.L, stats


def test_csa_prefill_L65536_sampled():
    cfg = synth.CFG_PREFILL_64K
    x = synth.csa_prefill_inputs(cfg)
    g = np.random.default_rng(3)
    rows = sorted(set([0, 1, 3, 4, 5, 8191, 8192, 8195, 8196, cfg.L - 1, cfg.L - 2]
                      + g.integers(0, cfg.L, 21).tolist()))
    stats = _check_prefill(cfg, x, rows)
    assert stats["exact"] >= len(rows) - 2, stats


def _decode_check(cfg, x, seqs):
    csa = _csa()
    B, S = cfg.B, cfg.N // cfg.m
    d = {k: dev(v) for k, v in x.items()}
    idx, cnt = csa.indexer_topk(d["qI"], d["w"], csa.Cache.contiguous(d["kI_comp"]), cfg.m, cfg.k,
                                seq_id=torch.arange(B, dtype=torch.int32, device="cuda"),
                                q_pos=d["pos"], max_entries=S)
    out = csa.sparse_attn_decode(d["q"], csa.Cache.contiguous(d["kv_comp"]), d["win"], d["win_len"],
                                 idx, cnt, cfg.lam)
    torch.cuda.synchronize()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    kvc = lambda b: f64(x["kv_comp"][b])
    kIc = lambda b: f64(x["kI_comp"][b])

    class Lazy:
        def __init__(self, fn):
            self.fn = fn

        def __getitem__(self, b):
            return self.fn(b)

    ref_out, _, ref_idx, ref_cnt = oracle.csa_decode(
        f64(x["q"][: max(seqs) + 1]), Lazy(kvc), Lazy(kIc), f64(x["qI"]), f64(x["w"]), f64(x["win"]),
        x["win_len"].numpy(), x["pos"].numpy(), cfg.m, cfg.k, cfg.lam, seqs=seqs)
    stats = {"exact": 0, "near-tie": 0}
    for r, b in enumerate(seqs):
        KI = kIc(b)
        s = oracle.indexer_scores(f64(x["qI"][b]), f64(x["w"][b]), KI)
        stats[check_topk(idx_h[b], cnt_h[b], s, cfg.k, score_eps(f64(x["qI"][b]), f64(x["w"][b]), KI))] += 1
        assert_close_attn(out[b], ref_out[r], f"decode seq {b}")
    assert_mostly_exact(stats, len(seqs))
    return stats


def test_csa_decode_B64_N131072_sampled():
    cfg = synth.CFG_DECODE_128K
    x = synth.csa_decode_inputs(cfg)
    stats = _decode_check(cfg, x, [0, 17, 42, 63])
    assert stats["exact"] >= 3, stats


def test_hca_decode_B8_N1M_full():
    csa = _csa()
    cfg = synth.CFG_HCA_1M
    x = synth.hca_decode_inputs(cfg)
    d = {k: dev(v) for k, v in x.items()}
    S = cfg.N // cfg.m
    out = csa.hca_attn(d["q"], csa.Cache.contiguous(d["kv_comp"]), d["win"], cfg.m, cfg.W, cfg.lam,
                       win_len=d["win_len"], q_pos=d["pos"], max_entries=S)
    ref, _ = oracle.hca_decode(f64(x["q"]), f64(x["kv_comp"]), f64(x["win"]), x["win_len"].numpy(),
                               x["pos"].numpy(), cfg.m, cfg.lam)
    assert_close_attn(out, ref, "hca decode 1M")


def test_mixed_decode_paged_sampled():
    csa = _csa()
    cfg = synth.CFG_MIXED
    x = synth.mixed_decode_inputs(cfg)
    B, P = cfg.B, cfg.page_size
    pos = x["pos"]
    seqs = [0, 7, 15]
    seq_id = torch.arange(B, dtype=torch.int32, device="cuda")
    near = 0
    for li, lay in enumerate(x["layers"]):
        S = [int(s) for s in lay["S"]]
        table = dev(lay["page_table"])
        kv = csa.Cache(dev(lay["kv_pool"]), page_table=table, page_size=P)
        if lay["kind"] == "csa":
            kI = csa.Cache(dev(lay["kI_pool"]), page_table=table, page_size=P)
            idx, cnt = csa.indexer_topk(dev(lay["qI"]), dev(lay["w"]), kI, lay["m"], cfg.k,
                                        seq_id=seq_id, q_pos=dev(pos), max_entries=max(S))
            out = csa.sparse_attn_decode(dev(lay["q"]), kv, dev(lay["win"]), dev(lay["win_len"]),
                                         idx, cnt, cfg.lam)
            idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        else:
            out = csa.hca_attn(dev(lay["q"]), kv, dev(lay["win"]), lay["m"], cfg.W, cfg.lam,
                               win_len=dev(lay["win_len"]), q_pos=dev(pos), max_entries=max(S))
        torch.cuda.synchronize()
        for b in seqs:
            kv_b = f64(oracle.unpage(lay["kv_pool"], lay["page_table"][b], S[b], P))
            win_b = f64(lay["win"][b, : int(lay["win_len"][b])])
            if lay["kind"] == "csa":
                kI_b = f64(oracle.unpage(lay["kI_pool"], lay["page_table"][b], S[b], P))
                qI_b, w_b = f64(lay["qI"][b]), f64(lay["w"][b])
                s = oracle.indexer_scores(qI_b, w_b, kI_b[: int(pos[b]) // lay["m"]])
                near += check_topk(idx_h[b], cnt_h[b], s, cfg.k, score_eps(qI_b, w_b, kI_b)) != "exact"
                sel = oracle.topk_select(s, cfg.k)
                rows = np.concatenate([kv_b[sel], win_b])
            else:
                rows = np.concatenate([kv_b[: int(pos[b]) // lay["m"]], win_b])
            ref, _ = oracle.attend_shared_kv(f64(lay["q"][b]), rows, cfg.lam)
            assert_close_attn(out[b], ref, f"layer {li} ({lay['kind']}) seq {b}")
    assert near <= 1, f"{near} near-tie queries among the checked CSA layers"
