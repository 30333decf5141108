"""Pins for the fp64 CPU oracle, independent of the oracle's own code paths.

Each check comes from something other than the oracle: a closed form derived
by hand, an invariant of the mathematics, a brute-force search on tiny
inputs, or a separately written dense-attention reduction.  The last test
plants plausible mistakes in the oracle (on the CPU) and shows that the pins
catch them.

Sources: "Tencent released Simple-Attention-Sparsification ..." (aigc.news,
2026-09-14), release paragraph, and "Simple-Attention-Sparsification Text
Generation Model: 12GB+ VRAM" (localmodelwatch), "Specifications and
Configuration Table": 64-token blocks, Top-K 31, a 128-wide gate, the Qproj
query projection, keys pooled by maximum, minimum and average, normalised
queries and keys, RoPE in the gate, budgets of 1,024 / 2,048 / 4,096 tokens.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import sas_oracle as O

EPS = 1e-6
SCALE = 1.0 / math.sqrt(128.0)


# ---------------------------------------------------------------- pooling
def test_pool_closed_form():
    # K[j][d] = 0.5 j - 0.25 d : max at j=63, min at j=0, mean at j=31.5
    j = np.arange(64)[:, None]
    d = np.arange(128)[None, :]
    kb = 0.5 * j - 0.25 * d
    p = O.pool_block(kb)
    dd = np.arange(128)
    assert np.array_equal(p[:128], 0.5 * 63 - 0.25 * dd)
    assert np.array_equal(p[128:256], -0.25 * dd)
    assert np.allclose(p[256:], 0.5 * 31.5 - 0.25 * dd, rtol=0, atol=1e-12)


def test_pool_brute_force_random():
    rng = np.random.default_rng(5)
    kb = rng.standard_normal((64, 128)).astype(np.float32).astype(np.float64)
    p = O.pool_block(kb)
    for dim in (0, 17, 127):
        col = [kb[t][dim] for t in range(64)]
        m_hi = col[0]
        m_lo = col[0]
        tot = 0.0
        for x in col:
            m_hi = x if x > m_hi else m_hi
            m_lo = x if x < m_lo else m_lo
            tot += x
        assert p[dim] == m_hi and p[128 + dim] == m_lo  # order-free: bit-exact
        assert abs(p[256 + dim] - tot / 64) <= 1e-12


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_unit_rms_and_scale_free():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(128) * 3.0
    y = O.rms_norm(x, np.ones(128), EPS)
    ms = np.mean(x * x)
    assert abs(math.sqrt(np.mean(y * y)) - math.sqrt(ms / (ms + EPS))) < 1e-12
    y2 = O.rms_norm(7.0 * x, np.ones(128), EPS)
    assert np.allclose(y, y2, rtol=1e-6, atol=0)
    g = rng.standard_normal(128)
    assert np.allclose(O.rms_norm(x, g, EPS), y * g, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- RoPE
def test_rope_pos0_identity_and_norm():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(128)
    assert np.allclose(O.rope_rotate_half(x, 0), x, atol=0, rtol=0)
    y = O.rope_rotate_half(x, 1234)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-10


def test_rope_closed_form_basis_vectors():
    # pair (0, 64) turns at 1 rad per position; pair (1, 65) at 10000^(-1/64)
    e = np.eye(128)
    for pos in (0, 1, 5, 511, 2047):
        y0 = O.rope_rotate_half(e[0], pos)
        exp0 = math.cos(pos) * e[0] + math.sin(pos) * e[64]
        assert np.allclose(y0, exp0, atol=1e-12)
        y64 = O.rope_rotate_half(e[64], pos)
        assert np.allclose(y64, -math.sin(pos) * e[0] + math.cos(pos) * e[64], atol=1e-12)
        th1 = 10000.0 ** (-2.0 / 128.0)
        y1 = O.rope_rotate_half(e[1], pos)
        assert np.allclose(y1, math.cos(pos * th1) * e[1] + math.sin(pos * th1) * e[65], atol=1e-12)


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(3)
    x, y = rng.standard_normal(128), rng.standard_normal(128)
    a = np.dot(O.rope_rotate_half(x, 40), O.rope_rotate_half(y, 13))
    b = np.dot(O.rope_rotate_half(x, 40 + 300), O.rope_rotate_half(y, 13 + 300))
    assert abs(a - b) < 1e-9 * max(1.0, abs(a))


# ---------------------------------------------------------------- gate, hand-derived closed form
def _closed_form_inputs(c):
    """Blocks whose dim 64 alternates +1 / -3 (max 1, min -3, avg -1), all other
    dims 0; W_k sends max(dim64) -> u_64, min(dim64) -> u_0, avg(dim64) -> u_1;
    W_q = I; q = e_0; gains 1."""
    n = c
    k = np.zeros((64 * (c + 1), 128))
    k[0::2, 64] = 1.0
    k[1::2, 64] = -3.0
    w_k = np.zeros((384, 128))
    w_k[64, 64] = 1.0            # max part
    w_k[128 + 64, 0] = 1.0       # min part
    w_k[256 + 64, 1] = 1.0       # avg part
    w_q = np.eye(128)[None]
    q = np.zeros((1, 128))
    q[0, 0] = 1.0
    return n, k, w_k, w_q, q


def test_gate_scores_closed_form():
    # u = 1 e64 - 3 e0 - 1 e1 ; |u|^2/128 = 11/128 ; RoPE at b; q~ = a(cos c e0 + sin c e64)
    # s_b = a * kn * (-3 cos(c-b) + sin(c-b) + 0) * scale   (pair (1,65) meets q~ = 0)
    c = 9
    n, k, w_k, w_q, q = _closed_form_inputs(c)
    gk = O.gate_keys_for_sequence(k, n, w_k, np.ones(128), EPS)
    s, S = O.gate_scores(q, w_q, np.ones((1, 128)), gk, n, c, SCALE, EPS)
    a = 1.0 / math.sqrt(1.0 / 128 + EPS)
    kn = 1.0 / math.sqrt(11.0 / 128 + EPS)
    for b in range(n):
        want = a * kn * (-3.0 * math.cos(c - b) + math.sin(c - b)) * SCALE
        assert abs(s[0, b] - want) < 1e-12, (b, s[0, b], want)
        assert S[b] == s[0, b]


# Asymmetric projection, non-unit gains.  q = e3; head 0's W_q has a single 1
# at row 3, column 0, so q @ W_q = e0, while W_q @ q (the transposed
# reading) would give e64 from the 1 at row 64, column 3.  Head 1's W_q sends
# q to e64.  Gains: gamma_q[0] = 2, gamma_q[64] = 0.5, gamma_k[0] = 1.5,
# gamma_k[1] = 0.25, gamma_k[64] = 3, every other entry 1 + (i mod 5)/10 (so
# a gain read at the wrong index, dropped, or taken from the other vector
# changes the value).
def _gains():
    i = np.arange(128)
    g_q = 1.0 + (i % 5) / 10.0
    g_k = 1.0 + ((i + 2) % 5) / 10.0
    g_q[0], g_q[64] = 2.0, 0.5
    g_k[0], g_k[1], g_k[64] = 1.5, 0.25, 3.0
    return g_q, g_k


def _asym_w_q():
    w0 = np.zeros((128, 128))
    w0[3, 0] = 1.0      # q @ W_q = e0
    w0[64, 3] = 1.0     # W_q @ q = e64 (must not be used)
    w1 = np.zeros((128, 128))
    w1[3, 64] = 1.0     # q @ W_q = e64
    w1[0, 3] = 1.0      # W_q @ q = e0 (must not be used)
    return np.stack([w0, w1])


def _asym_closed_form(c):
    """Hand-derived scores of the two heads for the blocks of
    _closed_form_inputs(c) (u = e64 - 3 e0 - e1 before the gain):
      k^ = kn (3 e64 - 4.5 e0 - 0.25 e1),  kn = 1/sqrt(11/128 + eps);
      q~_0 = 2a (cos c e0 + sin c e64),  q~_1 = 0.5a (-sin c e0 + cos c e64),
      a = 1/sqrt(1/128 + eps);  RoPE turns pair (0, 64) by the position, so
      s_0b = 2a kn (-4.5 cos(c-b) + 3 sin(c-b)) scale
      s_1b = 0.5a kn (4.5 sin(c-b) + 3 cos(c-b)) scale
    (pair (1, 65) meets zeros in both queries)."""
    a = 1.0 / math.sqrt(1.0 / 128 + EPS)
    kn = 1.0 / math.sqrt(11.0 / 128 + EPS)
    s0 = [2 * a * kn * (-4.5 * math.cos(c - b) + 3 * math.sin(c - b)) * SCALE for b in range(c)]
    s1 = [0.5 * a * kn * (4.5 * math.sin(c - b) + 3 * math.cos(c - b)) * SCALE for b in range(c)]
    return np.array(s0), np.array(s1)


def test_gate_scores_closed_form_asymmetric_projection_and_gains():
    c = 11
    n, k, w_k, _, _ = _closed_form_inputs(c)
    g_q, g_k = _gains()
    q = np.zeros((2, 128))
    q[:, 3] = 1.0
    gk = O.gate_keys_for_sequence(k, n, w_k, g_k, EPS)
    s, S = O.gate_scores(q, _asym_w_q(), np.stack([g_q, g_q]), gk, n, c, SCALE, EPS)
    s0, s1 = _asym_closed_form(c)
    assert np.allclose(s[0], s0, rtol=0, atol=1e-12)
    assert np.allclose(s[1], s1, rtol=0, atol=1e-12)
    # group score: the mean of the two heads' closed forms (not their max)
    assert np.allclose(S, 0.5 * (s0 + s1), rtol=0, atol=1e-12)
    assert not np.allclose(S, np.maximum(s0, s1))


def test_decode_step_driver_closed_form_gains():
    """The batched driver gives gamma_q to the queries and gamma_k to the keys:
    the same closed form through O.decode_step (one sequence, one KV head,
    G = 2)."""
    c = 11
    _, k, w_k, _, _ = _closed_form_inputs(c)
    g_q, g_k = _gains()
    L = 64 * c + 5
    kc = np.zeros((1, 1, L, 128))
    kc[0, 0] = k[:L]
    q = np.zeros((1, 2, 128))
    q[0, :, 3] = 1.0
    res = O.decode_step(q, kc, np.zeros_like(kc), [L], _asym_w_q(), g_q, w_k[None], g_k, 64 * 4)
    s0, s1 = _asym_closed_form(c)
    assert np.allclose(res[(0, 0)]["S"], 0.5 * (s0 + s1), rtol=0, atol=1e-12)


def test_rms_norm_closed_form_with_gain():
    # x = 3 e0 + 4 e1: mean(x^2) = 25/128; gain 2 at 0, -1 at 1
    x = np.zeros(128)
    x[0], x[1] = 3.0, 4.0
    g = np.full(128, 7.0)
    g[0], g[1] = 2.0, -1.0
    r = math.sqrt(25.0 / 128 + EPS)
    want = np.zeros(128)
    want[0], want[1] = 6.0 / r, -4.0 / r
    assert np.allclose(O.rms_norm(x, g, EPS), want, rtol=0, atol=1e-12)


def test_gate_group_score_is_mean_over_heads():
    rng = np.random.default_rng(4)
    G, c = 4, 12
    k = rng.standard_normal((64 * (c + 1), 128))
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    gk = O.gate_keys_for_sequence(k, c, w_k, np.ones(128), EPS)
    q = rng.standard_normal((G, 128))
    w_q = rng.standard_normal((G, 128, 128)) / math.sqrt(128)
    s, S = O.gate_scores(q, w_q, np.ones((G, 128)), gk, c, c, SCALE, EPS)
    # each head scored alone gives the same row (heads do not interact)
    for g in range(G):
        s1, S1 = O.gate_scores(q[g:g + 1], w_q[g:g + 1], np.ones((1, 128)), gk, c, c, SCALE, EPS)
        assert np.allclose(s1[0], s[g], atol=1e-14)
        assert np.allclose(S1, s1[0], atol=1e-14)   # one head: the group score is that head's


def test_gate_scores_invariant_to_positive_key_scale():
    rng = np.random.default_rng(6)
    c = 10
    k = rng.standard_normal((64 * (c + 1), 128))
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    q = rng.standard_normal((2, 128))
    w_q = rng.standard_normal((2, 128, 128)) / math.sqrt(128)
    g1 = O.gate_keys_for_sequence(k, c, w_k, np.ones(128), EPS)
    g2 = O.gate_keys_for_sequence(3.0 * k, c, w_k, np.ones(128), EPS)
    s1, _ = O.gate_scores(q, w_q, np.ones((2, 128)), g1, c, c, SCALE, EPS)
    s2, _ = O.gate_scores(q, w_q, np.ones((2, 128)), g2, c, c, SCALE, EPS)
    assert np.allclose(s1, s2, rtol=1e-5, atol=1e-7)


def test_gate_query_shift_invariance():
    # shifting query and key positions together leaves the score unchanged
    rng = np.random.default_rng(7)
    q = rng.standard_normal(128)
    w_q = rng.standard_normal((128, 128)) / math.sqrt(128)
    pooled = rng.standard_normal(384)
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    s1 = np.dot(O.gate_query(q, w_q, np.ones(128), 50), O.gate_key(pooled, w_k, np.ones(128), 20))
    s2 = np.dot(O.gate_query(q, w_q, np.ones(128), 950), O.gate_key(pooled, w_k, np.ones(128), 920))
    assert abs(s1 - s2) < 1e-9 * max(1.0, abs(s1))


# ---------------------------------------------------------------- Top-K selection
def _dominance_ok(S, sel_hist, n):
    rest = [b for b in range(n) if b not in sel_hist]
    return all((S[b] > S[r]) or (S[b] == S[r] and b < r) for b in sel_hist for r in rest)


@pytest.mark.parametrize("n,topk", [(0, 3), (1, 3), (5, 3), (6, 6), (8, 3), (8, 1), (7, 7), (9, 4)])
def test_select_brute_force_tiny(n, topk):
    rng = np.random.default_rng(100 + 10 * n + topk)
    for trial in range(20):
        S = rng.integers(-3, 4, size=n).astype(np.float64) * 0.5  # many ties
        if trial % 2:
            S = S + rng.standard_normal(n) * 1e-3
        sel = O.select_blocks(S, n, topk)
        assert sel[-1] == n and sel == sorted(sel) and len(set(sel)) == len(sel)
        want_k = min(topk, n)
        cands = [list(c) for c in itertools.combinations(range(n), want_k) if _dominance_ok(S, c, n)]
        assert len(cands) == 1
        assert sel[:-1] == cands[0]


@pytest.mark.parametrize("L", [1, 63, 64, 65, 128, 4096, 4097, 32768])
@pytest.mark.parametrize("budget", [64, 1024, 2048, 4096])
def test_selected_count(L, budget):
    c = (L - 1) // 64
    S = np.random.default_rng(L + budget).standard_normal(c)
    sel = O.select_blocks(S, c, O.topk_for_budget(budget))
    assert len(sel) == min(budget // 64, c + 1)


def test_topk_for_budget_matches_training_setting():
    # 31 historical + current = 2048/64 (release settings)
    assert O.topk_for_budget(2048) == 31
    assert O.topk_for_budget(1024) == 15 and O.topk_for_budget(4096) == 63


# ---------------------------------------------------------------- attention reductions
def _rand_group(rng, L, G=4):
    k = rng.standard_normal((L, 128))
    v = rng.standard_normal((L, 128))
    q = rng.standard_normal((G, 128))
    w_q = rng.standard_normal((G, 128, 128)) / math.sqrt(128)
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    return k, v, q, w_q, w_k


@pytest.mark.parametrize("L", [1, 64, 65, 300, 1000])
def test_budget_covering_context_is_dense_causal(L):
    rng = np.random.default_rng(L)
    k, v, q, w_q, w_k = _rand_group(rng, L)
    c = (L - 1) // 64
    gk = O.gate_keys_for_sequence(k, c, w_k, np.ones(128), EPS)
    budget = 64 * (c + 1)
    r = O.decode_one_group(q, k, v, L, gk, w_q, np.ones((4, 128)), budget)
    assert r["sel"] == list(range(c + 1))
    dense = O.dense_causal_decode(q, k, v, L)
    assert np.max(np.abs(r["out"] - dense)) < 1e-12


def test_equal_values_and_zero_query():
    rng = np.random.default_rng(11)
    L = 700
    k, v, q, w_q, w_k = _rand_group(rng, L)
    c = (L - 1) // 64
    gk = O.gate_keys_for_sequence(k, c, w_k, np.ones(128), EPS)
    vconst = np.tile(rng.standard_normal(128), (L, 1))
    r = O.decode_one_group(q, k, vconst, L, gk, w_q, np.ones((4, 128)), 256)
    assert np.allclose(r["out"], vconst[0][None, :], atol=1e-12)
    # q = 0 for attention -> plain mean of the selected tokens' values
    toks = O.selected_token_ids(r["sel"], L)
    z = O.attention_over_tokens(np.zeros(128), k, v, toks, SCALE)
    assert np.allclose(z, v[toks].mean(axis=0), atol=1e-12)


def test_budget_64_attends_current_block_only():
    rng = np.random.default_rng(12)
    L = 1000
    k, v, q, w_q, w_k = _rand_group(rng, L)
    c = (L - 1) // 64
    gk = O.gate_keys_for_sequence(k, c, w_k, np.ones(128), EPS)
    r = O.decode_one_group(q, k, v, L, gk, w_q, np.ones((4, 128)), 64)
    assert r["sel"] == [c]
    lo = 64 * c
    for g in range(4):
        logits = (k[lo:L] @ q[g]) * SCALE
        w = np.exp(logits - logits.max())
        assert np.allclose(r["out"][g], (w @ v[lo:L]) / w.sum(), atol=1e-12)


def test_closed_form_selection_ranks_by_relative_position():
    # with the closed-form gate above, block b's score is f(c-b); Top-K must
    # follow the ranking of f over the offsets
    c = 20
    n, k, w_k, w_q, q = _closed_form_inputs(c)
    L = 64 * c + 1
    v = np.zeros_like(k)
    gk = O.gate_keys_for_sequence(k, n, w_k, np.ones(128), EPS)
    r = O.decode_one_group(q, k[:L], v[:L], L, gk, w_q, np.ones((1, 128)), 64 * 6)
    f = [(-3.0 * math.cos(c - b) + math.sin(c - b), b) for b in range(c)]
    want = sorted(b for _, b in sorted(f, key=lambda t: (-t[0], t[1]))[:5])
    assert r["sel"] == want + [c]


# ---------------------------------------------------------------- prefill
def test_prefill_full_budget_is_dense_causal():
    rng = np.random.default_rng(13)
    nb, G = 4, 2
    T = 64 * nb
    q = rng.standard_normal((G, T, 128))
    k = rng.standard_normal((T, 128))
    v = rng.standard_normal((T, 128))
    w_q = rng.standard_normal((G, 128, 128)) / math.sqrt(128)
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    gk = O.gate_keys_for_sequence(k, nb, w_k, np.ones(128), EPS)
    dense = [O.dense_causal_prefill(q[g], k, v) for g in range(G)]
    for i in range(nb):
        r = O.prefill_query_block(q[:, 64 * i:64 * (i + 1)], k, v, i, gk, w_q,
                                  np.ones((G, 128)), topk=nb)
        assert r["sel"] == list(range(i + 1))
        for g in range(G):
            assert np.max(np.abs(r["out"][g] - dense[g][64 * i:64 * (i + 1)])) < 1e-12


def test_prefill_gate_query_is_block_mean():
    rng = np.random.default_rng(14)
    nb, G, i = 6, 2, 5
    T = 64 * nb
    q = rng.standard_normal((G, T, 128))
    k = rng.standard_normal((T, 128))
    v = rng.standard_normal((T, 128))
    w_q = rng.standard_normal((G, 128, 128)) / math.sqrt(128)
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    gk = O.gate_keys_for_sequence(k, nb, w_k, np.ones(128), EPS)
    r = O.prefill_query_block(q[:, 64 * i:64 * (i + 1)], k, v, i, gk, w_q, np.ones((G, 128)), topk=2)
    qbar = q[:, 64 * i:64 * (i + 1)].mean(axis=1)
    _, S = O.gate_scores(qbar, w_q, np.ones((G, 128)), gk, i, i, SCALE, EPS)
    assert np.allclose(r["S"], S, atol=1e-14)
    assert len(r["sel"]) == 3 and r["sel"][-1] == i
    # token 0 of the query block sees the kept blocks plus itself only
    toks = O.selected_token_ids(r["sel"][:-1], 64 * i) + [64 * i]
    ref = O.attention_over_tokens(q[0, 64 * i], k, v, toks, SCALE)
    assert np.allclose(r["out"][0, 0], ref, atol=1e-12)


# ---------------------------------------------------------------- gated inference mode (R18)
def _gated_case(gate_scale=SCALE):
    """Two heads, one complete historical block and the query token (L = 65).
    Block 0's keys are a*e1, so the pooled block projects (W_k maps max, min
    and mean of dim 1 to output 0) onto k~_0 = sqrt(128) e0 after RMSNorm;
    W_q = I and q_g = +-b e0 give q~_g = +-sqrt(128) (cos 1 e0 + sin 1 e64) at
    query position 1, so s_g = +-sqrt(128) cos(1) * sqrt(128) * gate_scale.
    Every attention logit is 0 (q _|_ keys, current key 0)."""
    a, b, L = 1.5, 2.0, 65
    rng = np.random.default_rng(3)
    k = np.zeros((L, 128))
    k[:64, 1] = a
    v = np.zeros((L, 128))
    v0 = rng.standard_normal(128)
    v1 = rng.standard_normal(128)
    v[:64] = v0
    v[64] = v1
    w_k = np.zeros((384, 128))
    w_k[1, 0] = w_k[129, 0] = w_k[257, 0] = 1.0
    gk = O.gate_keys_for_sequence(k, 1, w_k, np.ones(128))
    q = np.zeros((2, 128))
    q[0, 0], q[1, 0] = b, -b
    w_q = np.stack([np.eye(128)] * 2)
    gam = np.ones((2, 128))
    res = {}
    for mode in (O.GATE_SELECT_ONLY, O.GATE_LOGSIGMOID_BIAS):
        res[mode] = O.decode_one_group(q, k, v, L, gk, w_q, gam, 2048, gate_scale=gate_scale,
                                       gate_mode=mode)
    eps = 1e-6  # RMSNorm epsilon (R5)
    kn = 3 * a / math.sqrt((3 * a) ** 2 / 128 + eps)   # |k~_0|
    qn = b / math.sqrt(b ** 2 / 128 + eps)             # |q~_g|
    s = np.array([1.0, -1.0]) * qn * math.cos(1.0) * kn * gate_scale
    return res, s, v0, v1


def test_gated_mode_closed_form():
    """out_g = (64 sigmoid(s_g) v0 + v1) / (64 sigmoid(s_g) + 1): the bias is
    log(sigmoid(s_g)) per head on the historical block only."""
    res, s, v0, v1 = _gated_case()
    r = res[O.GATE_LOGSIGMOID_BIAS]
    assert r["sel"] == [0, 1]
    assert np.allclose(r["s"][:, 0], s, rtol=1e-12, atol=1e-12)
    for g in range(2):
        w = 64.0 / (1.0 + math.exp(-s[g]))
        want = (w * v0 + v1) / (w + 1.0)
        assert np.allclose(r["out"][g], want, rtol=1e-12, atol=1e-12), g
    plain = res[O.GATE_SELECT_ONLY]["out"]
    assert np.allclose(plain, (64.0 * v0 + v1) / 65.0, rtol=1e-12, atol=1e-12)
    assert not np.allclose(r["out"][0], plain[0])


def test_gated_mode_saturated_gates():
    """Gates near 1 reduce the gated mode to select-only (R12); gates near 0
    leave the current block alone."""
    res, s, v0, v1 = _gated_case(gate_scale=1e3)
    assert s[0] > 700 and s[1] < -700
    assert np.allclose(res[O.GATE_LOGSIGMOID_BIAS]["out"][0], res[O.GATE_SELECT_ONLY]["out"][0],
                       rtol=1e-12, atol=1e-12)
    assert np.allclose(res[O.GATE_LOGSIGMOID_BIAS]["out"][1], v1, rtol=1e-12, atol=1e-12)


def test_gated_prefill_closed_form():
    """Query block 1 of a 128-token sequence: block 0's keys a*e1 (gate key
    sqrt(128)-ish e0 as in the decode case), block 1's keys 0, every query of
    head g equal to +-b e0 (so the block-mean gate query is the same vector,
    at position 1).  All attention logits are 0, so token t of block 1 gives
    (64 sigmoid(s_g) v0 + (t + 1) v1) / (64 sigmoid(s_g) + t + 1)."""
    a, b = 1.5, 2.0
    rng = np.random.default_rng(4)
    k = np.zeros((128, 128))
    k[:64, 1] = a
    v = np.zeros((128, 128))
    v0, v1 = rng.standard_normal(128), rng.standard_normal(128)
    v[:64], v[64:] = v0, v1
    w_k = np.zeros((384, 128))
    w_k[1, 0] = w_k[129, 0] = w_k[257, 0] = 1.0
    gk = O.gate_keys_for_sequence(k, 2, w_k, np.ones(128))
    q = np.zeros((2, 64, 128))
    q[0, :, 0], q[1, :, 0] = b, -b
    w_q = np.stack([np.eye(128)] * 2)
    r = O.prefill_query_block(q, k, v, 1, gk, w_q, np.ones((2, 128)), 31, gate_mode=O.GATE_LOGSIGMOID_BIAS)
    eps = 1e-6
    kn = 3 * a / math.sqrt((3 * a) ** 2 / 128 + eps)
    qn = b / math.sqrt(b ** 2 / 128 + eps)
    s = np.array([1.0, -1.0]) * qn * math.cos(1.0) * kn * SCALE
    assert r["sel"] == [0, 1]
    for g in range(2):
        w = 64.0 / (1.0 + math.exp(-s[g]))
        for t in (0, 17, 63):
            want = (w * v0 + (t + 1) * v1) / (w + t + 1)
            assert np.allclose(r["out"][g, t], want, rtol=1e-12, atol=1e-12), (g, t)


def test_log_sigmoid_values():
    assert O.log_sigmoid(0.0) == pytest.approx(-math.log(2.0), abs=1e-15)
    for x in (-50.0, -3.0, -0.5, 0.25, 4.0):
        assert O.log_sigmoid(x) == pytest.approx(math.log(1.0 / (1.0 + math.exp(-x))), rel=1e-12, abs=1e-300)
    assert O.log_sigmoid(60.0) == pytest.approx(-math.exp(-60.0), rel=1e-12)
    assert O.log_sigmoid(-800.0) == pytest.approx(-800.0)
    assert -1e-300 < O.log_sigmoid(800.0) <= 0.0


# ---------------------------------------------------------------- bf16 gate-key storage (R19)
def test_round_to_bf16_worked_values():
    """Hand-worked bfloat16 roundings: 8 significant bits (1 implicit + 7)."""
    cases = [
        (1.0, 1.0),
        (1.0 + 2 ** -8, 1.0),                  # exactly half an ulp above 1: tie, 1.0 is even
        (1.0 + 3 * 2 ** -8, 1.0 + 2 ** -6),    # tie between 1+2^-7 (odd) and 1+2^-6 (even)
        (1.0 + 2 ** -8 + 2 ** -20, 1.0 + 2 ** -7),   # just above the tie: up
        (1.0 + 2 ** -7, 1.0 + 2 ** -7),        # representable
        (-2.5, -2.5),
        (3.0e38, 1.765625 * 2.0 ** 127),       # 1.11000011..b * 2^127 rounds up to 1.1100010b
        (1.0e-40, 9.99e-41),                   # binary32 subnormal, kept to 7 fraction bits
        (0.1, 0.10009765625),                  # 0x3DCD
        (65504.0, 65536.0),
    ]
    for x, want in cases:
        got = float(O.round_to_bf16(x))
        assert got == pytest.approx(want, rel=2 ** -9), (x, got, want)
    assert float(O.round_to_bf16(0.1)) == 0.10009765625
    assert float(O.round_to_bf16(1.0 + 2 ** -8)) == 1.0
    assert float(O.round_to_bf16(1.0 + 3 * 2 ** -8)) == 1.0 + 2 ** -6
    assert np.isinf(O.round_to_bf16(np.inf)) and np.isnan(O.round_to_bf16(np.nan))


def test_round_to_bf16_is_idempotent_and_within_half_ulp():
    x = np.random.default_rng(9).standard_normal(10000) * 10.0 ** np.random.default_rng(10).integers(-6, 6, 10000)
    r = O.round_to_bf16(x)
    assert np.array_equal(O.round_to_bf16(r), r)
    # |x - r| <= 2^-8 |x|: unit roundoff of an 8-bit significand (float32 step aside)
    assert np.all(np.abs(x - r) <= 2.0 ** -8 * np.abs(x) * (1 + 2 ** -14) + 1e-300)
    # an independent implementation: torch's float32 -> bfloat16 conversion
    import torch
    assert np.array_equal(torch.tensor(x).float().bfloat16().double().numpy(), r)
    # the bf16 pattern has a zero low half
    assert np.all((r.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)


# ---------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle (CPU) and show a pin fails."""
    good_rope = O.rope_rotate_half

    def rope_wrong_sign(x, pos, base=10000.0):
        return good_rope(x, -pos, base)

    monkeypatch.setattr(O, "rope_rotate_half", rope_wrong_sign)
    with pytest.raises(AssertionError):
        test_gate_scores_closed_form()
    monkeypatch.setattr(O, "rope_rotate_half", good_rope)

    good_pool = O.pool_block

    def pool_swapped(kb):
        p = good_pool(kb)
        return np.concatenate([p[128:256], p[:128], p[256:]])

    monkeypatch.setattr(O, "pool_block", pool_swapped)
    with pytest.raises(AssertionError):
        test_gate_scores_closed_form()
    monkeypatch.setattr(O, "pool_block", good_pool)

    good_select = O.select_blocks

    def select_high_index_ties(S, n, topk):
        order = sorted(range(n), key=lambda b: (-float(S[b]), -b))
        return sorted(order[:min(topk, n)]) + [n]

    monkeypatch.setattr(O, "select_blocks", select_high_index_ties)
    with pytest.raises(AssertionError):
        test_select_brute_force_tiny(8, 3)
    monkeypatch.setattr(O, "select_blocks", good_select)

    good_attn = O.attention_over_tokens

    def attn_no_scale(q, k, v, toks, scale, bias=None):
        return good_attn(q, k, v, toks, 1.0, bias)

    monkeypatch.setattr(O, "attention_over_tokens", attn_no_scale)
    with pytest.raises(AssertionError):
        test_budget_covering_context_is_dense_causal(300)
    monkeypatch.setattr(O, "attention_over_tokens", good_attn)

    # gated mode: log(1 - sigmoid) instead of log(sigmoid); the gate itself
    # instead of its log; a bias on the current block too
    good_ls = O.log_sigmoid
    monkeypatch.setattr(O, "log_sigmoid", lambda x: good_ls(-x))
    with pytest.raises(AssertionError):
        test_gated_mode_closed_form()
    monkeypatch.setattr(O, "log_sigmoid", lambda x: math.exp(good_ls(x)))
    with pytest.raises(AssertionError):
        test_gated_mode_closed_form()
    monkeypatch.setattr(O, "log_sigmoid", good_ls)

    good_bias = O.gated_token_bias

    def bias_on_current_too(s_g, blocks, seq_len, cur):
        b = good_bias(s_g, blocks, seq_len, cur)
        return [x if x != 0.0 else good_ls(0.0) for x in b]

    monkeypatch.setattr(O, "gated_token_bias", bias_on_current_too)
    with pytest.raises(AssertionError):
        test_gated_mode_closed_form()
    monkeypatch.setattr(O, "log_sigmoid", lambda x: good_ls(-x))
    with pytest.raises(AssertionError):
        test_gated_prefill_closed_form()
    monkeypatch.setattr(O, "log_sigmoid", good_ls)
    monkeypatch.setattr(O, "gated_token_bias", good_bias)

    # projection read transposed (W_q @ q instead of q @ W_q)
    good_gq = O.gate_query

    def gate_query_transposed(q, w_q, gamma_q, pos, eps=1e-6, base=10000.0):
        return good_gq(q, np.asarray(w_q).T, gamma_q, pos, eps, base)

    monkeypatch.setattr(O, "gate_query", gate_query_transposed)
    with pytest.raises(AssertionError):
        test_gate_scores_closed_form_asymmetric_projection_and_gains()
    monkeypatch.setattr(O, "gate_query", good_gq)

    # gain read at the wrong index (rotate-half partner), or dropped
    good_rms = O.rms_norm
    monkeypatch.setattr(O, "rms_norm", lambda x, g, eps=1e-6: good_rms(x, np.roll(g, 64), eps))
    with pytest.raises(AssertionError):
        test_gate_scores_closed_form_asymmetric_projection_and_gains()
    monkeypatch.setattr(O, "rms_norm", lambda x, g, eps=1e-6: good_rms(x, np.ones(128), eps))
    with pytest.raises(AssertionError):
        test_gate_scores_closed_form_asymmetric_projection_and_gains()
    with pytest.raises(AssertionError):
        test_rms_norm_closed_form_with_gain()
    monkeypatch.setattr(O, "rms_norm", good_rms)

    # the key gain given to the queries (driver level)
    good_step = O.decode_step

    def step_gains_swapped(q, kc, vc, lens, w_q, gamma_q, w_k, gamma_k, budget, **kw):
        return good_step(q, kc, vc, lens, w_q, gamma_k, w_k, gamma_k, budget, **kw)

    monkeypatch.setattr(O, "decode_step", step_gains_swapped)
    with pytest.raises(AssertionError):
        test_decode_step_driver_closed_form_gains()
    monkeypatch.setattr(O, "decode_step", good_step)

    # group score as the max over heads instead of the mean
    good_gs = O.gate_scores

    def gate_scores_max(*a, **kw):
        s, S = good_gs(*a, **kw)
        return s, (s.max(axis=0) if s.shape[1] else S)

    monkeypatch.setattr(O, "gate_scores", gate_scores_max)
    with pytest.raises(AssertionError):
        test_gate_scores_closed_form_asymmetric_projection_and_gains()
    monkeypatch.setattr(O, "gate_scores", good_gs)
