"""Pins of the fp64 oracle to things other than itself: the pages' worked
numbers (tests/golden, each with its citation), closed forms, special cases
that reduce to a library routine, and brute force on tiny inputs."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from conftest import read_golden

rng = np.random.default_rng(1234)


# ---------------------------------------------------------------------------
# step 1: pooling
# ---------------------------------------------------------------------------
def _worked_example_inputs(weight_on):
    """m = 2, entry i = 1: a branch = tokens 2, 3, b branch = tokens 0, 1."""
    g = read_golden("pooling_worked_example.txt")
    a = [float(x) for x in g["a_content"][0]]
    b = [float(x) for x in g["b_content"][0]]
    ex = [float(x) for x in g["exp_logits"][0]]
    Ca = np.zeros((4, 1)); Cb = np.zeros((4, 1)); Za = np.zeros((4, 1)); Zb = np.zeros((4, 1))
    Ca[2, 0], Ca[3, 0] = a
    Cb[0, 0], Cb[1, 0] = b
    # logits whose exponentials are the printed (2, 1, 1, 1), in the given order
    slots = {"a1": (Za, 2), "a2": (Za, 3), "b1": (Zb, 0), "b2": (Zb, 1)}
    for name, e in zip(weight_on, ex):
        arr, row = slots[name]
        arr[row, 0] = math.log(e)
    return Ca, Za, Cb, Zb, g


def test_pooling_worked_example_listed_order():
    Ca, Za, Cb, Zb, g = _worked_example_inputs(["a1", "a2", "b1", "b2"])
    out = oracle.pool_overlap(Ca, Za, Cb, Zb, m=2)
    assert out.shape == (2, 1)
    assert out[1, 0] == pytest.approx(float(g["result_listed_order"][0][0]), abs=1e-12)


def test_pooling_worked_example_chronological_order():
    Ca, Za, Cb, Zb, g = _worked_example_inputs(["b1", "b2", "a1", "a2"])
    out = oracle.pool_overlap(Ca, Za, Cb, Zb, m=2)
    assert out[1, 0] == pytest.approx(float(g["result_chronological_order"][0][0]), abs=1e-12)


def test_pooling_weights_printed():
    g = read_golden("pooling_worked_example.txt")
    ex = np.array([float(x) for x in g["exp_logits"][0]])
    w = np.array([float(x) for x in g["weights"][0]])
    # the oracle's pooling with content = one-hot picks out each weight
    for j in range(4):
        C = np.zeros((4, 1)); C[j, 0] = 1.0
        Z = np.log(ex)[:, None]
        assert oracle.pool_block(C, Z, m=4)[0, 0] == pytest.approx(w[j], abs=1e-12)


def test_overlap_first_entry_closed_form():
    """Entry 0 has no previous block: b branch masked, all weight on tokens
    0..m-1 (Ch.5 'Receptive field versus compression stride').  Closed form:
    logits (0, ln 3) on contents (4, 8) -> 0.25*4 + 0.75*8 = 7."""
    Ca = np.array([[4.0], [8.0], [100.0], [100.0]])
    Za = np.array([[0.0], [math.log(3.0)], [0.0], [0.0]])
    Cb = np.full((4, 1), 1e6)   # must not leak into entry 0
    Zb = np.full((4, 1), 50.0)
    out = oracle.pool_overlap(Ca, Za, Cb, Zb, m=2)
    assert out[0, 0] == pytest.approx(7.0, abs=1e-12)


def test_overlap_m1_is_two_way_sigmoid():
    """m = 1: entry i mixes token i (a) and token i-1 (b) with weight
    sigmoid(za - zb) on the a side."""
    N = 6
    Ca, Za, Cb, Zb = (rng.standard_normal((N, 3)) for _ in range(4))
    out = oracle.pool_overlap(Ca, Za, Cb, Zb, m=1)
    for i in range(1, N):
        wa = 1.0 / (1.0 + np.exp(Zb[i - 1] - Za[i]))
        np.testing.assert_allclose(out[i], wa * Ca[i] + (1 - wa) * Cb[i - 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[0], Ca[0], atol=1e-12)


def test_overlap_b_branch_uses_previous_block_and_bias_positions():
    """m = 2 with all logits equal except biases: Ba = (ln 3, 0), Bb = (0, ln 2)
    give weights 3:1 on the a tokens and 1:2 on the b tokens."""
    m = 2
    Ca = np.array([[1.0], [2.0], [3.0], [4.0]])
    Cb = np.array([[10.0], [20.0], [30.0], [40.0]])
    Z = np.zeros((4, 1))
    Ba = np.array([[math.log(3.0)], [0.0]])
    Bb = np.array([[0.0], [math.log(2.0)]])
    out = oracle.pool_overlap(Ca, Z, Cb, Z, m, Ba, Bb)
    # entry 1: a = tokens 2,3 (weights 3,1), b = tokens 0,1 (weights 1,2); total 7
    want = (3 * 3.0 + 1 * 4.0 + 1 * 10.0 + 2 * 20.0) / 7.0
    assert out[1, 0] == pytest.approx(want, abs=1e-12)


def test_block_bias_is_indexed_by_position_in_block():
    m = 2
    C = np.array([[1.0], [5.0], [7.0], [11.0], [13.0]])   # 5 tokens -> 2 entries
    Z = np.zeros((5, 1))
    B = np.array([[math.log(3.0)], [0.0]])
    out = oracle.pool_block(C, Z, m, B)
    assert out.shape == (2, 1)     # the trailing token makes no entry
    np.testing.assert_allclose(out[:, 0], [(3 * 1 + 5) / 4, (3 * 7 + 11) / 4], atol=1e-12)


def test_block_special_cases():
    C = rng.standard_normal((12, 5))
    Z = rng.standard_normal((12, 5))
    np.testing.assert_allclose(oracle.pool_block(C, Z, m=1), C, atol=1e-15)          # identity
    np.testing.assert_allclose(oracle.pool_block(C, np.zeros_like(Z), m=4),
                               C.reshape(3, 4, 5).mean(axis=1), atol=1e-12)           # mean
    np.testing.assert_allclose(oracle.pool_block(np.full_like(C, 2.5), Z, m=3),
                               np.full((4, 5), 2.5), atol=1e-12)                      # sums to 1
    Zbig = np.zeros_like(Z); Zbig[5] = 1000.0                                          # stability
    out = oracle.pool_block(C, Zbig, m=4)
    np.testing.assert_allclose(out[1], C[5], atol=1e-12)


def test_coordinatewise_independence():
    """Weights are computed per coordinate: coordinate 0 may favour token 0
    while coordinate 1 favours token 3 (Ch.5 'Coordinate-wise softmax
    pooling')."""
    C = np.arange(8.0).reshape(4, 2)
    Z = np.array([[50.0, 0.0], [0.0, 0.0], [0.0, 0.0], [0.0, 50.0]])
    out = oracle.pool_block(C, Z, m=4)
    np.testing.assert_allclose(out[0], [C[0, 0], C[3, 1]], atol=1e-12)


# ---------------------------------------------------------------------------
# steps 2-3: indexer and top-k
# ---------------------------------------------------------------------------
def _toy_indexer():
    g = read_golden("indexer_toy_example.txt")
    table = {row[0]: [float(x) for x in row[1:]] for row in g["table"]}
    names = ["A", "B", "C"]
    # keys / queries with q_h . K_s = table[s][h]; q is not the identity so a
    # transposed operand would change the numbers: q1 = (1, 1), q2 = (0, 1)
    qI = np.array([[1.0, 1.0], [0.0, 1.0]])
    KI = np.array([[table[n][0] - table[n][1], table[n][1]] for n in names])
    np.testing.assert_allclose(KI @ qI.T, [table[n] for n in names])
    return g, names, qI, KI


@pytest.mark.parametrize("overlap", [True, False])
def test_decode_cache_state_equals_bulk_pooling(overlap):
    """Appending a sequence token by token (Ch.5 "Decode-time cache state")
    yields, entry for entry, the bulk pooling of the whole sequence; one entry
    appears every m tokens; the window holds the last W raw rows in order."""
    rng = np.random.default_rng(31)
    N, d, m, W = 27, 6, 4, 5
    Ca, Za, Cb, Zb = (rng.standard_normal((N, d)) for _ in range(4))
    Ba, Bb = rng.standard_normal((m, d)), rng.standard_normal((m, d))
    st = oracle.DecodeCacheState(m, W, overlap, Ba, Bb if overlap else None)
    for t in range(N):
        st.append(Ca[t], Za[t], Cb[t], Zb[t])
        assert len(st.entries) == (t + 1) // m
        assert np.array_equal(np.array(st.window), Ca[max(0, t + 1 - W):t + 1])
    ref = oracle.pool_overlap(Ca, Za, Cb, Zb, m, Ba, Bb) if overlap else oracle.pool_block(Ca, Za, m, Ba)
    np.testing.assert_allclose(np.array(st.entries), ref, rtol=0, atol=1e-12)


def test_decode_cache_state_entry_reads_only_its_blocks():
    """Overlap entry i depends on tokens m(i-1) .. m(i+1)-1 only: changing any
    other token leaves it unchanged (and changing one inside changes it)."""
    rng = np.random.default_rng(32)
    N, d, m = 24, 4, 4
    X = [rng.standard_normal((N, d)) for _ in range(4)]

    def entries(X):
        st = oracle.DecodeCacheState(m, 0, True)
        for t in range(N):
            st.append(*(x[t] for x in X))
        return np.array(st.entries)

    base = entries(X)
    i = 3
    for t, same in ((m * (i - 1) - 1, True), (m * (i + 1), True), (m * (i - 1), False), (m * i + 1, False)):
        Y = [x.copy() for x in X]
        Y[0][t] += 1.0          # content of token t (a branch of its block, b branch of the next)
        Y[1][t] += 1.0
        Y[2][t] += 1.0
        Y[3][t] += 1.0
        changed = not np.allclose(entries(Y)[i], base[i])
        assert changed != same, (t, same)


def test_rmsnorm_closed_forms():
    """Ch.2 "Normalization and rotary position embeddings": unit RMS without a
    gain, invariant to a positive scale, gain per coordinate, zeros stay zero."""
    rng = np.random.default_rng(41)
    x = rng.standard_normal((5, 128)) * 3.0
    y = oracle.rmsnorm(x, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-12)
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * x, eps=0.0), y, rtol=1e-12)
    g = rng.standard_normal(128)
    np.testing.assert_allclose(oracle.rmsnorm(x, g, eps=0.0), y * g, rtol=1e-12)
    assert np.all(oracle.rmsnorm(np.zeros((2, 64))) == 0.0)


def test_rope_closed_forms():
    """Ch.7 "Partial RoPE and output de-rotation": only the last 64
    coordinates move; pair j of the slice turns by t * 10000^(-2j/64); R_t is
    orthogonal with inverse R_{-t}; q.k after rotation depends only on s - t."""
    rng = np.random.default_rng(42)
    d, r0 = 128, 64
    t = 1234567
    for j in (0, 5, 31):
        e = np.zeros(d)
        e[r0 + 2 * j] = 1.0
        y = oracle.rope_rotate(e, t)
        ang = t * 10000.0 ** (-2.0 * j / 64)
        np.testing.assert_allclose(y[r0 + 2 * j:r0 + 2 * j + 2], [np.cos(ang), np.sin(ang)], atol=1e-9)
        assert np.count_nonzero(np.abs(y) > 1e-12) <= 2
    x = rng.standard_normal((4, d))
    y = oracle.rope_rotate(x, [3, 70, 9000, 2 ** 20])
    np.testing.assert_array_equal(y[:, :r0], x[:, :r0])
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    np.testing.assert_allclose(oracle.rope_rotate(y, [3, 70, 9000, 2 ** 20], inverse=True), x, atol=1e-9)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    dot = lambda tq, ts: oracle.rope_rotate(q, tq) @ oracle.rope_rotate(k, ts)
    np.testing.assert_allclose(dot(500, 120), dot(500 + 4099, 120 + 4099), rtol=1e-9)


def test_output_derotation_gives_relative_positions():
    """Applying R_{-t} to an attention output over values rotated by R_s gives
    the sum of values rotated by R_{s-t} (the pages' de-rotation identity)."""
    rng = np.random.default_rng(43)
    d, n, t = 128, 6, 777
    v = rng.standard_normal((n, d))
    s = np.array([3, 100, 640, 701, 760, 777])
    p = rng.dirichlet(np.ones(n))
    o = (p[:, None] * oracle.rope_rotate(v, s)).sum(0)
    lhs = oracle.rope_rotate(o, t, inverse=True)
    rhs = (p[:, None] * oracle.rope_rotate(v, s - t)).sum(0)
    np.testing.assert_allclose(lhs, rhs, atol=1e-9)


def test_indexer_toy_scores():
    g, names, qI, KI = _toy_indexer()
    w = np.array([float(x) for x in g["w_second"][0]])
    want = [float(x) for x in g["scores_second"][0]]
    np.testing.assert_allclose(oracle.indexer_scores(qI, w, KI), want, atol=1e-12)
    assert names[int(np.argmax(oracle.indexer_scores(qI, w, KI)))] == "B"


def test_indexer_toy_ranking():
    g, names, qI, KI = _toy_indexer()
    w = np.array([float(x) for x in g["w_first"][0]])
    sel = oracle.topk_select(oracle.indexer_scores(qI, w, KI), 2)
    assert [names[i] for i in sel] == g["top2_first"][0]


def test_indexer_relu_clips_each_head():
    qI = np.array([[1.0, 0.0], [0.0, 1.0]])
    KI = np.array([[-2.0, 3.0], [-1.0, -1.0]])
    w = np.array([0.2, 0.8])
    # head 1 negative -> 0; block 2 all heads negative -> exactly 0
    np.testing.assert_allclose(oracle.indexer_scores(qI, w, KI), [0.8 * 3.0, 0.0], atol=0)


def _brute_topk(scores, k):
    """Element i is selected iff fewer than k elements beat it, where j beats
    i when s_j > s_i or (s_j == s_i and j < i)."""
    s = np.asarray(scores, dtype=np.float32)
    n = s.shape[0]
    sel = [i for i in range(n) if sum(1 for j in range(n) if s[j] > s[i] or (s[j] == s[i] and j < i)) < k]
    return np.array(sel, dtype=np.int64)


@pytest.mark.parametrize("n,k", [(1, 1), (5, 2), (17, 4), (40, 7), (64, 63), (9, 20)])
def test_topk_matches_brute_force_with_ties(n, k):
    for trial in range(5):
        s = rng.integers(-3, 4, size=n).astype(np.float64)        # many exact ties
        s[rng.random(n) < 0.2] = -0.0                               # signed zeros tie with +0
        got = oracle.topk_select(s, k)
        np.testing.assert_array_equal(got, _brute_topk(s, k))
        assert np.all(np.diff(got) > 0)                             # ascending
        assert got.shape[0] == min(n, k)


def test_topk_decides_in_fp32():
    """Scores equal after fp32 rounding are ties (lower index wins)."""
    s = np.array([1.0, 1.0 + 1e-12, 0.5])
    np.testing.assert_array_equal(oracle.topk_select(s, 1), [0])


def test_causal_eligibility():
    assert [oracle.eligible_entries(t, 4) for t in range(10)] == [0, 0, 0, 0, 1, 1, 1, 1, 2, 2]
    L, m, k = 40, 4, 3
    qI = rng.standard_normal((L, 2, 8)); w = rng.random((L, 2)); KI = rng.standard_normal((L // m, 8))
    idx, cnt = oracle.csa_prefill_topk(qI, w, KI, m, k)
    for t in range(L):
        n = t // m
        assert cnt[t] == min(k, n)
        assert np.all(idx[t, :cnt[t]] < n) and np.all(idx[t, cnt[t]:] == -1)


# ---------------------------------------------------------------------------
# step 4: attention
# ---------------------------------------------------------------------------
def _sdpa_causal(q, kv, lam, bias=None):
    """torch's scaled_dot_product_attention in float64, one shared KV head
    serving as both K and V, causal."""
    L, H, d = q.shape
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                       # [1, H, L, d]
    kt = torch.from_numpy(kv)[None, None].expand(1, H, L, d)
    if bias is None:
        o = F.scaled_dot_product_attention(qt, kt, kt, is_causal=True, scale=lam)
    else:
        o = F.scaled_dot_product_attention(qt, kt, kt, attn_mask=torch.from_numpy(bias), scale=lam)
    return o[0].permute(1, 0, 2).numpy()


def _csa_m1_inputs(L=24, H=3, d=16):
    q = rng.standard_normal((L, H, d))
    kv = rng.standard_normal((L, d))
    Z = rng.standard_normal((L, d))
    kI = rng.standard_normal((L, 8)); ZI = rng.standard_normal((L, 8))
    qI = rng.standard_normal((L, 2, 8)); w = rng.random((L, 2))
    return q, kv, Z, kI, ZI, qI, w


def test_csa_m1_full_topk_window1_is_dense_causal():
    """m = 1 pooling is the identity, k >= L selects every earlier token and a
    window of 1 adds the current one: exactly dense causal MQA."""
    q, kv, Z, kI, ZI, qI, w = _csa_m1_inputs()
    L = q.shape[0]
    lam = 0.37
    # no bf16 storage rounding here: compare the definitions exactly
    kv_comp = oracle.pool_block(kv, Z, 1)
    idx, cnt = oracle.csa_prefill_topk(qI, w, oracle.pool_block(kI, ZI, 1), 1, L)
    out, _ = oracle.csa_prefill_attention(q, kv_comp, kv, idx, cnt, 1, lam)
    np.testing.assert_allclose(out, _sdpa_causal(q, kv, lam), atol=1e-12)


def test_csa_m1_window_duplicates_closed_form():
    """With W > 1 the tokens t-W+1 .. t-1 appear both as selected entries and
    in the window; each duplicate adds ln 2 to that position's logit."""
    q, kv, Z, kI, ZI, qI, w = _csa_m1_inputs()
    L, W, lam = q.shape[0], 5, 0.2
    idx, cnt = oracle.csa_prefill_topk(qI, w, kI, 1, L)
    out, _ = oracle.csa_prefill_attention(q, kv, kv, idx, cnt, W, lam)
    bias = np.full((L, L), -np.inf)
    for t in range(L):
        bias[t, : t + 1] = 0.0
        bias[t, max(0, t - W + 1): t] = math.log(2.0)
    np.testing.assert_allclose(out, _sdpa_causal(q, kv, lam, bias), atol=1e-12)


def test_hca_m1_window1_is_dense_causal():
    q, kv, *_ = _csa_m1_inputs()
    lam = 0.5
    out, _ = oracle.hca_prefill(q, kv, kv, 1, 1, lam)
    np.testing.assert_allclose(out, _sdpa_causal(q, kv, lam), atol=1e-12)


def test_decode_m1_is_last_row_of_dense_causal():
    """Decode of token N with m = 1, k >= N and a window of 1 (the new token)
    equals the last row of dense causal attention over N+1 tokens."""
    N, H, d = 30, 4, 8
    kv = rng.standard_normal((N + 1, d))
    q = rng.standard_normal((N + 1, H, d))
    qI = rng.standard_normal((1, 2, 8)); w = rng.random((1, 2)); kI = rng.standard_normal((N, 8))
    out, _, idx, cnt = oracle.csa_decode(q[N:N + 1], [kv[:N]], [kI], qI, w, kv[None, N:N + 1],
                                         [1], [N], 1, N, 0.3)
    assert cnt[0] == N
    np.testing.assert_allclose(out[0], _sdpa_causal(q, kv, 0.3)[N], atol=1e-12)
    out_h, _ = oracle.hca_decode(q[N:N + 1], [kv[:N]], kv[None, N:N + 1], [1], [N], 1, 0.3)
    np.testing.assert_allclose(out_h[0], out[0], atol=1e-12)


def test_attention_weights_sum_to_one():
    v = rng.standard_normal(6)
    rows = np.tile(v, (9, 1))
    o, _ = oracle.attend_shared_kv(rng.standard_normal((4, 6)), rows, 0.7)
    np.testing.assert_allclose(o, np.tile(v, (4, 1)), atol=1e-12)


def test_sink_worked_example():
    g = read_golden("sink_example.txt")
    real, sink, want = (float(g[k][0][0]) for k in ("real_mass", "sink_mass", "real_weight"))
    # one real entry whose logit is ln(real): q . kv = ln(real) with lam = 1
    kv = np.array([[math.log(real), 2.0]])
    q = np.array([[1.0, 0.0]])
    o, lse = oracle.attend_shared_kv(q, kv, 1.0, sink=np.array([math.log(sink)]))
    np.testing.assert_allclose(o[0], want * kv[0], atol=1e-12)
    assert lse[0] == pytest.approx(math.log(real + sink), abs=1e-12)


def test_lse_without_sink():
    q = rng.standard_normal((3, 5)); rows = rng.standard_normal((7, 5))
    _, lse = oracle.attend_shared_kv(q, rows, 0.4)
    np.testing.assert_allclose(lse, np.log(np.exp(0.4 * q @ rows.T).sum(1)), atol=1e-12)


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------
def test_bf16_round_matches_torch():
    x = rng.standard_normal(10000) * 10.0 ** rng.integers(-5, 5, 10000)
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(oracle.bf16_round(x), want)


# ---------------------------------------------------------------------------
# cost model (Ch.8)
# ---------------------------------------------------------------------------
def test_cost_model_matches_pages():
    cm = oracle.cost_model
    g = read_golden("cost_model.txt")
    gqa_pro = cm.gqa8_cache_bytes(10**6, 61)
    gqa_flash = cm.gqa8_cache_bytes(10**6, 43)
    pro = cm.model_cache_bytes(10**6, 30, 31)
    flash = cm.model_cache_bytes(10**6, 21, 20)
    d_f, g_f = cm.grouped_out_proj_params(64, 512, 4096, 8, 1024)
    d_p, g_p = cm.grouped_out_proj_params(128, 512, 7168, 16, 1024)
    csa_fl = cm.attention_flops(128, 512, 1024 + 128)
    got = {
        "gqa8_bytes_per_token_layer": cm.gqa8_bytes_per_token_layer(),
        "gqa8_layer_bytes_1M": cm.gqa8_cache_bytes(10**6, 1),
        "gqa8_61_layers_1M": gqa_pro,
        "gqa8_43_layers_1M": gqa_flash,
        "entry_bytes": cm.v4_entry_bytes(),
        "csa_main_bytes_per_token": cm.main_cache_bytes_per_token(4),
        "hca_main_bytes_per_token": cm.main_cache_bytes_per_token(128),
        "indexer_key_bytes": cm.indexer_key_bytes(),
        "indexer_bytes_per_token": cm.indexer_key_bytes() / 4,
        "csa_total_bytes_per_token": cm.csa_bytes_per_token(),
        "pro_cache_1M_bytes": pro,
        "flash_cache_1M_bytes": flash,
        "pro_over_gqa8": pro / gqa_pro,
        "flash_over_gqa8": flash / gqa_flash,
        "fp4_scale_overhead": cm.fp4_scale_overhead(),
        "csa_attention_flops": csa_fl,
        "hca_attention_flops": cm.attention_flops(128, 512, cm.hca_entries(10**6)[0] + 128),
        "indexer_ops": cm.indexer_ops(10**6, 4, 64, 128),
        "indexer_over_csa_main": cm.indexer_ops(10**6, 4, 64, 128) / csa_fl,
        "hca_entries_1M": cm.hca_entries(10**6)[0],
        "hca_trailing_1M": cm.hca_entries(10**6)[1],
        "flash_out_proj_ratio": g_f / d_f,
        "pro_out_proj_ratio": g_p / d_p,
        "pro_out_proj_saving": d_p - g_p,
    }
    assert set(got) == set(g)
    for name, rows in g.items():
        want, tol = float(rows[0][0]), float(rows[0][1])
        v = float(got[name])
        if tol == 0:
            assert v == want, name
        else:
            assert abs(v - want) <= tol * abs(want), (name, v, want)


# ---------------------------------------------------------------------------
# 4-bit indexer storage (Ch.8 "V4 compressed-entry payload" and "Quantization
# scales and bounded tail buffers")
# ---------------------------------------------------------------------------
from oracle import mxfp4 as ofp4   # noqa: E402


def test_e2m1_values_are_the_fp4_grid():
    # the eight E2M1 magnitudes as the OCP MX format tabulates them, +/- by bit 3
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    got = ofp4.e2m1_value(np.arange(16))
    assert got[:8].tolist() == mags
    assert (-got[8:]).tolist() == mags
    assert np.signbit(got[8])   # code 8 is -0


def test_e2m1_encode_matches_library_rounding():
    import ml_dtypes
    # every midpoint and every grid value, both signs, plus random values over
    # and beyond the range (saturation)
    mags = ofp4.e2m1_value(np.arange(8))
    mids = (mags[1:] + mags[:-1]) / 2
    y = np.concatenate([mags, mids, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20),
                        rng.uniform(-9, 9, 4000), [6.5, 7.99, 1e6, -1e6]])
    y = np.concatenate([y, -y]).astype(np.float32)
    lib = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ofp4.e2m1_encode(y.astype(np.float64)), lib)


def test_e2m1_ties_go_to_even_codes():
    # midpoints of adjacent magnitudes -> the neighbour with mantissa bit 0
    assert ofp4.e2m1_encode([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]).tolist() == [0, 2, 2, 4, 4, 6, 6]


def test_mxfp4_scale_puts_block_max_in_top_binade():
    # X = floor(log2 amax) - 2, so amax / 2^X lies in [4, 8)
    for _ in range(200):
        blk = rng.standard_normal(32) * 2.0 ** rng.integers(-30, 30)
        X = ofp4.mxfp4_scale_exponent(blk)
        r = np.abs(blk).max() / 2.0 ** X
        assert 4.0 <= r < 8.0
    assert ofp4.mxfp4_scale_exponent(np.zeros(32)) == -127
    assert ofp4.mxfp4_scale_exponent(np.full(32, 2.0 ** -200)) == -127   # clamped
    assert ofp4.mxfp4_scale_exponent(np.full(32, 6.0)) == 0
    assert ofp4.mxfp4_scale_exponent(np.full(32, 4.0)) == 0
    assert ofp4.mxfp4_scale_exponent(np.full(32, 3.99)) == -1


def test_mxfp4_roundtrip_and_error_bound():
    x = oracle.bf16_round(rng.standard_normal((64, 128)))
    packed, scales = ofp4.mxfp4_quantize(x)
    assert packed.shape == (64, 64) and scales.shape == (64, 4)
    y = ofp4.mxfp4_dequantize(packed, scales)
    # representable values survive unchanged
    p2, s2 = ofp4.mxfp4_quantize(y)
    assert np.array_equal(p2, packed) and np.array_equal(s2, scales)
    # the error of an element is at most half the grid step at its magnitude,
    # except above 6 (saturation), where it is below 2 * 2^X
    X = np.repeat(scales.astype(np.int64) - 127, 32, axis=1)
    u = np.abs(x) / 2.0 ** X
    half_step = np.where(u < 2, 0.25, np.where(u < 4, 0.5, 1.0))
    bound = np.where(u > 6, 2.0, half_step) * 2.0 ** X
    assert np.all(np.abs(y - x) <= bound)


def test_mxfp4_packing_order():
    # element 2i in the low nibble of byte i, element 2i+1 in the high nibble
    x = np.zeros(32)
    x[0], x[1], x[30], x[31] = 4.0, -1.0, 0.5, 6.0     # amax 6 -> X = 0
    packed, scales = ofp4.mxfp4_quantize(x)
    assert scales.tolist() == [127]
    assert packed[0] == (0x6 | (0xA << 4)) and packed[15] == (0x1 | (0x7 << 4))


def test_mxfp4_key_bytes_match_pages():
    # a 128-dim FP4 indexer key is 64 bytes; one scale byte per 32 elements adds
    # 4 bytes, +6.25 % (Ch.8 "Quantization scales and bounded tail buffers")
    packed, scales = ofp4.mxfp4_quantize(rng.standard_normal(128))
    assert packed.nbytes == 64 and scales.nbytes == 4
    assert scales.nbytes / packed.nbytes == 0.0625


def test_mxfp4_indexer_scores_brute_force():
    # scores from codes decoded by the printed grid, in plain loops
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    H, c, n = 3, 64, 5
    qp, qs = ofp4.mxfp4_quantize(rng.standard_normal((H, c)))
    kp, ks = ofp4.mxfp4_quantize(rng.standard_normal((n, c)))
    w = rng.uniform(0, 1, H)

    def val(packed, scales, r):
        b = int(packed[r // 2])
        code = (b & 0xF) if r % 2 == 0 else (b >> 4)
        v = grid[code & 7] * (-1.0 if code & 8 else 1.0)
        return v * 2.0 ** (int(scales[r // 32]) - 127)

    got = ofp4.indexer_scores_mxfp4(qp, qs, w, kp, ks)
    for s in range(n):
        want = 0.0
        for h in range(H):
            dot = sum(val(qp[h], qs[h], r) * val(kp[s], ks[s], r) for r in range(c))
            want += w[h] * max(dot, 0.0)
        assert got[s] == pytest.approx(want, rel=1e-12, abs=1e-12)


def test_mxfp4_quantize_is_blockwise_definition():
    # each 32-element block: scale byte from its own maximum, codes of x / 2^X
    x = oracle.bf16_round(rng.standard_normal((7, 96)) * 2.0 ** rng.integers(-60, 60, (7, 1)))
    x[0, :32] = 0.0
    packed, scales = ofp4.mxfp4_quantize(x)
    for r in range(7):
        for b in range(3):
            blk = x[r, 32 * b:32 * b + 32]
            X = ofp4.mxfp4_scale_exponent(blk)
            assert scales[r, b] == X + 127
            codes = ofp4.e2m1_encode(blk / 2.0 ** X)
            assert np.array_equal(packed[r, 16 * b:16 * b + 16], codes[0::2] | (codes[1::2] << 4))


# ---------------------------------------------------------------------------
# mixed-precision entries: FP8 content + bf16 rotary part (Ch.8 "V4
# compressed-entry payload")
# ---------------------------------------------------------------------------
from oracle import fp8_entry as ofp8   # noqa: E402


def test_e4m3_grid_closed_forms():
    v = ofp8.e4m3_value(np.arange(256))
    finite = v[np.isfinite(v)]
    assert np.nanmax(v) == 448.0 and np.nanmin(v) == -448.0          # largest normal
    assert v[1] == 2.0 ** -9 and v[8] == 2.0 ** -6                     # smallest subnormal / normal
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and finite.size == 254
    assert np.all(np.diff(v[:0x7F]) > 0)                               # codes ordered by value
    assert np.signbit(v[0x80]) and v[0x80] == 0.0


def test_e4m3_encode_matches_library_rounding():
    import ml_dtypes
    mags = ofp8.e4m3_value(np.arange(0x7F))
    mids = (mags[1:] + mags[:-1]) / 2
    y = np.concatenate([mags, mids, mids * (1 + 2.0 ** -30), mids * (1 - 2.0 ** -30),
                        rng.uniform(-448, 448, 6000), rng.standard_normal(3000) * 0.01])
    y = np.concatenate([y, -y]).astype(np.float32)
    lib = y.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ofp8.e4m3_encode(y.astype(np.float64)), lib)


def test_e4m3_saturates_and_keeps_sign():
    assert ofp8.e4m3_encode([449.0, 480.0, 1e9, -1e9]).tolist() == [0x7E, 0x7E, 0x7E, 0xFE]
    assert ofp8.e4m3_encode([-0.0, -2.0 ** -12]).tolist() == [0x80, 0x80]


def test_mxfp8_scale_binade_and_roundtrip():
    for _ in range(200):
        blk = rng.standard_normal(32) * 2.0 ** rng.integers(-40, 40)
        X = ofp8.mxfp8_scale_exponent(blk)
        assert 256.0 <= np.abs(blk).max() / 2.0 ** X < 512.0
    x = oracle.bf16_round(rng.standard_normal((20, 64)) * 2.0 ** rng.integers(-20, 20, (20, 1)))
    codes, scales = ofp8.mxfp8_quantize(x)
    y = ofp8.mxfp8_dequantize(codes, scales)
    c2, s2 = ofp8.mxfp8_quantize(y)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    # error at most half a quantum of the element's binade (quantum 2^(e-3),
    # subnormal quantum 2^-9), in units of 2^X; saturated elements below 64
    X = np.repeat(scales.astype(np.int64) - 127, 32, axis=1)
    u = np.abs(x) / 2.0 ** X
    e = np.floor(np.log2(np.maximum(u, 2.0 ** -6)))
    bound = np.where(u > 448, 64.0, 2.0 ** (e - 4)) * 2.0 ** X
    assert np.all(np.abs(y - x) <= bound)


def test_mxfp8_quantize_is_blockwise_definition():
    x = oracle.bf16_round(rng.standard_normal((5, 64)) * 2.0 ** rng.integers(-60, 60, (5, 1)))
    x[0, 32:] = 0.0
    codes, scales = ofp8.mxfp8_quantize(x)
    for r in range(5):
        for b in range(2):
            blk = x[r, 32 * b:32 * b + 32]
            X = ofp8.mxfp8_scale_exponent(blk)
            assert scales[r, b] == X + 127
            assert np.array_equal(codes[r, 32 * b:32 * b + 32], ofp8.e4m3_encode(blk / 2.0 ** X))


def test_fp8_entry_payload_matches_pages():
    # c = 512 with the last 64 coordinates rotary: 448 FP8 bytes + 64 bf16 values = 576 B
    # (Ch.8 "V4 compressed-entry payload"), plus 14 scale bytes of metadata
    x = oracle.bf16_round(rng.standard_normal(512))
    codes, scales, rope = ofp8.entry_quantize(x, 64)
    assert codes.nbytes + 2 * rope.size == 576
    assert scales.size == 14
    # the rotary part is kept as given
    y = ofp8.entry_dequantize(codes, scales, rope)
    assert np.array_equal(y[448:], x[448:])
    assert np.array_equal(y[:448], ofp8.mxfp8_dequantize(codes, scales))


def test_fp8_entry_values_are_bf16_numbers():
    # every dequantized content value is exactly representable in bf16 (3
    # mantissa bits, power-of-two scale), so the dequantized cache is a bf16 cache
    x = oracle.bf16_round(rng.standard_normal((50, 128)) * 3)
    codes, scales, rope = ofp8.entry_quantize(x, 64)
    y = ofp8.entry_dequantize(codes, scales, rope)
    assert np.array_equal(oracle.bf16_round(y), y)


# ---------------------------------------------------------------------------
# paged cache addressing (oracle.page_rows / oracle.unpage)
# ---------------------------------------------------------------------------
def test_page_rows_hand_mapping():
    """Three sequences, pages of two rows, page ids written out by hand:
    seq 0 holds pages (3, 0), seq 1 pages (1, 4), seq 2 page (2) and an unused
    slot (-1).  Logical entry s of a sequence sits at row page * 2 + s % 2 of
    the page table[s // 2]; the rows below are counted on paper."""
    table = np.array([[3, 0], [1, 4], [2, -1]], dtype=np.int32)
    assert list(oracle.page_rows(table[0], 4, 2)) == [6, 7, 0, 1]
    assert list(oracle.page_rows(table[1], 3, 2)) == [2, 3, 8]
    assert list(oracle.page_rows(table[2], 2, 2)) == [4, 5]
    assert list(oracle.page_rows(table[2], 0, 2)) == []
    # the sequences' rows never collide, and every used row of the pool is hit once
    rows = np.concatenate([oracle.page_rows(table[0], 4, 2), oracle.page_rows(table[1], 4, 2),
                           oracle.page_rows(table[2], 2, 2)])
    assert sorted(rows) == list(range(10))


def test_unpage_gathers_the_mapped_rows():
    """A pool whose row r holds (r, -r): the logical view of a sequence is the
    listed rows in logical order (a swapped page or a transposed offset fails).
    Pages of 4 rows, table (5, 2, 0): entries 0-3 are rows 20-23, entry 4 is
    row 8."""
    pool = np.stack([np.arange(24.0), -np.arange(24.0)], axis=1)
    table = np.array([5, 2, 0], dtype=np.int32)
    want = np.array([[20, -20], [21, -21], [22, -22], [23, -23], [8, -8]], dtype=np.float64)
    np.testing.assert_array_equal(oracle.unpage(pool, table, 5, 4), want)
