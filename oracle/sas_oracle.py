"""Plain fp64 CPU oracle for SAS (Simple-Attention-Sparsification) gated
block-sparse attention: decode step and block-sparse chunked prefill.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  The CUDA library never calls it, links it or reads its output;
it shares no code, tables or helpers with ``gated_block_sparse_token_b200``.

Everything here is computed in float64 with numpy, one (sequence, KV head)
or (sequence, KV head, query block) at a time, in the order the method
states its steps.  Inputs are the exact values the GPU receives (bf16 or
fp32 numbers widened to float64).

Sources (web pages describing the release; they print no formula, so every
formula below is a reading, flagged ``ASSUMPTION``):

* [aigc-0914] "Tencent released Simple-Attention-Sparsification, a method for
  efficient sparse attention in Qwen3 models" (aigc.news, 2026-09-14), release
  paragraph: 64-token KV blocks; 31 historical blocks kept in training; a
  128-wide gate; the query goes through a projection called Qproj; each key
  block is summarised by its maximum, minimum and average; queries and keys
  are normalised and the gate applies RoPE; training sequences of 32,768
  tokens; a 2,048-token decode budget by default, 1,024 and 4,096 also
  usable; continuous gates weight the blocks that were selected.
* [lmw-en] "Simple-Attention-Sparsification Text Generation Model: 12GB+
  VRAM" (localmodelwatch, English), "Specifications and Configuration Table":
  the same settings, and gate parameter counts 33.0M / 33.0M / 42.0M.
* [lmw-ja] "Tencent、Qwen3向けSASスパースアテンションチェックポイント公開"
  (localmodelwatch, Japanese), "スペック・構成表": the same tables.
* [nedoborov] ai-news.nedoborov.com post of 2026-09-14 on the SAS release
  (Russian), list of sparse-attention settings: block 64, Top-K 31, length
  32,768, budget 2,048 with 1,024 / 4,096 usable without retraining.

Readings fixed where the pages are silent (each also marked in code):

R1  W_q is [128][128] per query head, W_k is [384][128] per KV head, no bias,
    applied as row vector times matrix (x @ W).  The gate parameter counts
    ([lmw-en] table) equal layers*(Hq*128*128 + Hkv*384*128) for the Qwen3
    head layouts.
R2  The query fed to Qproj is the per-head attention query (head_dim 128).
R3  The pooled keys are the K cache values attention reads.
R4  Pooled vector order is [max; min; avg] (the order in which the release
    paragraph lists the three poolings).
R5  Q/K normalization is RMSNorm x / sqrt(mean(x^2) + eps) * gamma, eps 1e-6,
    applied after the projection and before RoPE.  The gain is one
    128-vector per layer for q and one for k, shared by all heads: with
    per-head gains the printed counts would read 33.2M, not 33.0M.
R6  Gate RoPE is rotate-half (pairs i, i+64), theta_i = base^(-2i/128),
    base 10000; key position = block index b, query position = current block
    index c (decode) or query block index i (prefill).
R7  Gate score s_{g,b} = (q~_g . k~_b) * gate_scale, gate_scale = 1/sqrt(128).
R8  One block set per KV head, ranked by the mean over the G query heads of
    the group of their gate scores.
R9  Equal group scores: the lower block index wins.
R10 The current block c = floor((L-1)/64) is always attended and never
    scored; the query is token L-1, which is already in the cache.
R11 With fewer historical blocks than Top-K, all of them are kept.
R12 Inference weights every selected block 1 (the continuous gate is the
    training path); a budget covering the context gives dense causal
    attention.
R13 Prefill gate query for query block i is the mean over the block's 64
    token queries, per query head.
R14 Attention logits use scale 1/sqrt(128); softmax in float64.
R18 Gated inference mode (a variant of R12; the release paragraph of
    [aigc-0914] has continuous gates on the chosen blocks): the logits of every
    token of a selected historical block b, for query head g, get the
    additive bias log(sigmoid(s_{g,b})) with s_{g,b} the head's gate score
    (R7); the current block gets 0.  Gates equal to 1 reduce it to R12.
R19 bf16 gate-key cache (a storage option, not a change of the method): the
    gate key k~_b is computed as before and stored rounded to the nearest
    bf16 value (ties to even); scores use the stored value.  The release
    ships its gate weights in bf16 ([lmw-en] table: the printed checkpoint
    sizes fit bf16 weights).

R20 Gradient through the gates (the release paragraph of [aigc-0914] says the
    continuous gates on the selected blocks let a gradient reach the gate
    through the discrete Top-K; second paragraph of [nedoborov] likewise):
    in the gated mode (R18), for an upstream gradient dL/dout, the gradients
    of the gate parameters W_q, W_k, gamma_q and gamma_k flow through
    log(sigmoid(s_gb)) of every selected historical block; the selected set
    is held fixed (the Top-K itself has no gradient).  In the select-only
    mode (R12) the gate parameters get no gradient.

Parity status: the gate formula as a whole (R1-R8) is pinned only by the
invariants and hand-derived closed forms in tests/test_oracle.py, not by any
value the pages print ("parity unpinned" against the pages for the exact gate
arithmetic; the pages print no worked example).
"""
from __future__ import annotations

import math
import numpy as np

BLOCK = 64          # KV block size in tokens  [aigc-0914], [lmw-en] table
HEAD_DIM = 128      # Qwen3 head_dim (attention query/key width)
GATE_HIDDEN = 128   # gate hidden size  [aigc-0914], [lmw-en] table
POOL_DIM = 3 * HEAD_DIM   # max, min, avg stacked  (R4)


# --------------------------------------------------------------------------
# Step 1: key-block pooling (release paragraph of [aigc-0914]: every key
# block is summarised by its maximum, minimum and average; R3, R4).
# --------------------------------------------------------------------------
def pool_block(k_block: np.ndarray) -> np.ndarray:
    """Pooled key of one complete 64-token block.

    k_block: [64][128] keys of the block.  Returns [384] =
    [per-dim max ; per-dim min ; per-dim mean].  ASSUMPTION R4 (order).
    """
    k_block = np.asarray(k_block, dtype=np.float64)
    assert k_block.shape == (BLOCK, HEAD_DIM)
    mx = k_block.max(axis=0)
    mn = k_block.min(axis=0)
    avg = k_block.sum(axis=0) / BLOCK
    return np.concatenate([mx, mn, avg])


# --------------------------------------------------------------------------
# Step 2 pieces: Q/K normalisation and gate RoPE (release paragraph of
# [aigc-0914]: queries and keys are normalised, the gate applies RoPE; R5, R6).
# --------------------------------------------------------------------------
def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gamma.  ASSUMPTION R5."""
    x = np.asarray(x, dtype=np.float64)
    return x / math.sqrt(float(np.mean(x * x)) + eps) * np.asarray(gamma, np.float64)


def rope_rotate_half(x: np.ndarray, pos: int, base: float = 10000.0) -> np.ndarray:
    """Rotary embedding of a 128-vector at integer position ``pos``.

    Pairs (i, i+64), angle pos * base^(-2i/128):
      y_i      = x_i cos - x_{i+64} sin
      y_{i+64} = x_{i+64} cos + x_i sin
    ASSUMPTION R6 (rotate-half convention, base 10000).
    """
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    i = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * i / x.shape[-1])
    ang = float(pos) * theta
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[:half], x[half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s])


def gate_key(pooled: np.ndarray, w_k: np.ndarray, gamma_k: np.ndarray, pos: int,
             eps: float = 1e-6, base: float = 10000.0) -> np.ndarray:
    """k~_b = RoPE(RMSNorm(pooled @ W_k) , b).  W_k: [384][128].  R1, R5, R6."""
    u = np.asarray(pooled, np.float64) @ np.asarray(w_k, np.float64)
    return rope_rotate_half(rms_norm(u, gamma_k, eps), pos, base)


def gate_query(q: np.ndarray, w_q: np.ndarray, gamma_q: np.ndarray, pos: int,
               eps: float = 1e-6, base: float = 10000.0) -> np.ndarray:
    """q~ = RoPE(RMSNorm(q @ W_q), pos): the gate's query projection, which the
    pages name Qproj.  W_q: [128][128].
    R1, R2, R5, R6."""
    v = np.asarray(q, np.float64) @ np.asarray(w_q, np.float64)
    return rope_rotate_half(rms_norm(v, gamma_q, eps), pos, base)


def gate_keys_for_sequence(k_seq: np.ndarray, num_blocks: int, w_k: np.ndarray,
                           gamma_k: np.ndarray, eps: float = 1e-6,
                           base: float = 10000.0) -> np.ndarray:
    """Gate keys of blocks 0..num_blocks-1 of one (sequence, KV head).

    k_seq: [>= 64*num_blocks][128].  Returns [num_blocks][128]."""
    out = np.zeros((num_blocks, GATE_HIDDEN))
    for b in range(num_blocks):
        pooled = pool_block(k_seq[b * BLOCK:(b + 1) * BLOCK])
        out[b] = gate_key(pooled, w_k, gamma_k, b, eps, base)
    return out


# --------------------------------------------------------------------------
# Steps 2-3: gate scores and Top-K selection ([aigc-0914]: the gate ranks
# the KV blocks and the best are kept, training Top-K 31, budget 2,048;
# [nedoborov] list).
# --------------------------------------------------------------------------
def gate_scores(q_group: np.ndarray, w_q_group: np.ndarray, gamma_q_group: np.ndarray,
                gate_keys: np.ndarray, n_hist: int, q_pos: int,
                gate_scale: float = 1.0 / math.sqrt(128.0), eps: float = 1e-6,
                base: float = 10000.0):
    """Per-head and group gate scores of the historical blocks 0..n_hist-1.

    q_group:       [G][128] queries of the G query heads sharing a KV head.
    w_q_group:     [G][128][128].   gamma_q_group: [G][128].
    gate_keys:     [>= n_hist][128] k~ of the KV head.
    Returns (s [G][n_hist], S [n_hist]) with s_{g,b} = q~_g . k~_b * scale
    (R7) and S_b = mean_g s_{g,b} (R8).
    """
    G = q_group.shape[0]
    s = np.zeros((G, n_hist))
    for g in range(G):
        qt = gate_query(q_group[g], w_q_group[g], gamma_q_group[g], q_pos, eps, base)
        for b in range(n_hist):
            s[g, b] = float(np.dot(qt, gate_keys[b])) * gate_scale
    S = s.sum(axis=0) / G if n_hist else np.zeros(0)
    return s, S


def select_blocks(S: np.ndarray, n_hist: int, topk: int) -> list[int]:
    """Ascending block list: the min(topk, n_hist) historical blocks with the
    largest group score (ties -> lower index, R9), then the current block
    ``n_hist`` (R10, R11).  Selection by a full sort of (-S_b, b)."""
    order = sorted(range(n_hist), key=lambda b: (-float(S[b]), b))
    kept = sorted(order[:min(topk, n_hist)])
    return kept + [n_hist]


def topk_for_budget(token_budget: int) -> int:
    """Historical blocks kept for a token budget: budget/64 - 1 (the current
    block takes the remaining 64 tokens: 31 + 1 = 2048/64)."""
    assert token_budget % BLOCK == 0 and token_budget >= BLOCK
    return token_budget // BLOCK - 1


# --------------------------------------------------------------------------
# Step 4: attention over the selected blocks (R12, R14).
# --------------------------------------------------------------------------
def round_to_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 value, ties to even (R19).  bfloat16 is
    the upper half of an IEEE binary32: 1 sign, 8 exponent, 7 fraction bits.
    The value is first rounded to binary32 (float64 -> float32 is itself
    round-to-nearest-even), then the low 16 bits of the binary32 pattern are
    rounded away: add 0x7FFF plus the lowest kept bit, clear the low half.
    Infinities stay, NaN stays NaN."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + keep_lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).astype(np.float64)
    nan = np.isnan(f)
    if np.any(nan):
        out = np.where(nan, np.nan, out)
    return out


GATE_SELECT_ONLY = 0       # R12: selected blocks weighted 1
GATE_LOGSIGMOID_BIAS = 1   # R18: + log(sigmoid(s_{g,b})) on block b's logits


def log_sigmoid(x: float) -> float:
    """log(1 / (1 + exp(-x))), evaluated without overflow for either sign."""
    x = float(x)
    if x >= 0.0:
        return -math.log1p(math.exp(-x))
    return x - math.log1p(math.exp(x))


def attention_over_tokens(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                          token_ids, scale: float, bias=None) -> np.ndarray:
    """softmax(q . k_j * scale + bias_j) weighted sum of v_j over the listed
    tokens, two-pass (max, then exp-sum) in float64.  bias: None, or one
    additive logit term per listed token (the gated mode, R18)."""
    idx = np.asarray(list(token_ids), dtype=np.int64)
    logits = (k[idx].astype(np.float64) @ np.asarray(q, np.float64)) * scale
    if bias is not None:
        logits = logits + np.asarray(bias, np.float64)
    m = logits.max()
    p = np.exp(logits - m)
    return (p @ v[idx].astype(np.float64)) / p.sum()


def selected_token_ids(blocks, seq_len: int):
    """Token positions covered by the listed blocks, clipped to the context
    (only the current block can be partial)."""
    out = []
    for b in blocks:
        out.extend(range(b * BLOCK, min((b + 1) * BLOCK, seq_len)))
    return out


def gated_token_bias(s_g, blocks, seq_len: int, cur: int):
    """The gated mode's logit bias for one query head (R18), one entry per
    token of selected_token_ids(blocks, seq_len): log(sigmoid(s_g[b])) for a
    historical block b, 0 for the current block."""
    out = []
    for b in blocks:
        n = min((b + 1) * BLOCK, seq_len) - b * BLOCK
        out.extend([0.0 if b == cur else log_sigmoid(s_g[b])] * n)
    return out


def decode_one_group(q_group, k_seq, v_seq, seq_len, gate_keys, w_q_group,
                     gamma_q_group, token_budget, attn_scale=1.0 / math.sqrt(128.0),
                     gate_scale=1.0 / math.sqrt(128.0), eps=1e-6, base=10000.0,
                     gate_mode=GATE_SELECT_ONLY):
    """Decode step of one (sequence, KV head): gate, select, attend.

    q_group [G][128]: queries of token L-1 for the G heads of the group.
    k_seq, v_seq [>= L][128]: the head's cache.  gate_keys [>= c][128].
    gate_mode: GATE_SELECT_ONLY (R12) or GATE_LOGSIGMOID_BIAS (R18).
    Returns dict(out [G][128], sel (ascending list), s [G][c], S [c]).
    """
    c = (seq_len - 1) // BLOCK            # current block (R10)
    s, S = gate_scores(q_group, w_q_group, gamma_q_group, gate_keys, c, c,
                       gate_scale, eps, base)
    sel = select_blocks(S, c, topk_for_budget(token_budget))
    toks = selected_token_ids(sel, seq_len)
    outs = []
    for g in range(q_group.shape[0]):
        bias = None
        if gate_mode == GATE_LOGSIGMOID_BIAS:
            bias = gated_token_bias(s[g], sel, seq_len, c)
        outs.append(attention_over_tokens(q_group[g], k_seq, v_seq, toks, attn_scale, bias))
    return {"out": np.stack(outs), "sel": sel, "s": s, "S": S}


def dense_causal_decode(q_group, k_seq, v_seq, seq_len,
                        attn_scale=1.0 / math.sqrt(128.0)):
    """Plain dense attention of token L-1 over tokens 0..L-1 (no gate, no
    blocks); what a budget covering the whole context must reduce to."""
    out = np.zeros((q_group.shape[0], HEAD_DIM))
    for g in range(q_group.shape[0]):
        logits = np.array([float(np.dot(q_group[g], k_seq[j])) for j in range(seq_len)]) * attn_scale
        w = np.exp(logits - logits.max())
        w /= w.sum()
        acc = np.zeros(HEAD_DIM)
        for j in range(seq_len):
            acc += w[j] * np.asarray(v_seq[j], np.float64)
        out[g] = acc
    return out


# --------------------------------------------------------------------------
# Block-sparse chunked prefill (training setting: Top-K 31 over 32,768-token
# sequences, [aigc-0914]; R13).
# --------------------------------------------------------------------------
def prefill_query_block(q_blk_group, k_seq, v_seq, i, gate_keys, w_q_group,
                        gamma_q_group, topk, attn_scale=1.0 / math.sqrt(128.0),
                        gate_scale=1.0 / math.sqrt(128.0), eps=1e-6, base=10000.0,
                        gate_mode=GATE_SELECT_ONLY):
    """One (sequence, KV head, query block i) of block-sparse causal prefill.

    q_blk_group [G][64][128]: queries of block i for the G heads.
    Gate query of head g = mean over the block's 64 queries (R13), placed at
    position i; historical blocks 0..i-1 scored; top-min(topk, i) kept plus
    the diagonal block i; token t of block i attends to all tokens of the
    kept historical blocks and to tokens 64i..t of block i.  Gated mode
    (R18): the tokens of a kept historical block b get + log(sigmoid(s_gb))
    on head g's logits, the diagonal block 0.
    Returns dict(out [G][64][128], sel, S, s).
    """
    G = q_blk_group.shape[0]
    qbar = q_blk_group.astype(np.float64).mean(axis=1)
    s, S = gate_scores(qbar, w_q_group, gamma_q_group, gate_keys, i, i,
                       gate_scale, eps, base)
    sel = select_blocks(S, i, topk)
    hist_toks = selected_token_ids(sel[:-1], (i + 1) * BLOCK)
    out = np.zeros((G, BLOCK, HEAD_DIM))
    for g in range(G):
        hist_bias = None
        if gate_mode == GATE_LOGSIGMOID_BIAS:
            hist_bias = gated_token_bias(s[g], sel[:-1], (i + 1) * BLOCK, i)
        for t in range(BLOCK):
            toks = hist_toks + list(range(i * BLOCK, i * BLOCK + t + 1))
            bias = None if hist_bias is None else hist_bias + [0.0] * (t + 1)
            out[g, t] = attention_over_tokens(q_blk_group[g, t], k_seq, v_seq, toks, attn_scale, bias)
    return {"out": out, "sel": sel, "S": S, "s": s}


def dense_causal_prefill(q_seq, k_seq, v_seq, attn_scale=1.0 / math.sqrt(128.0)):
    """Dense causal attention of every token of one head: [T][128] -> [T][128]."""
    T = q_seq.shape[0]
    logits = (q_seq.astype(np.float64) @ k_seq.astype(np.float64).T) * attn_scale
    out = np.zeros((T, HEAD_DIM))
    for t in range(T):
        row = logits[t, :t + 1]
        w = np.exp(row - row.max())
        out[t] = (w @ v_seq[:t + 1].astype(np.float64)) / w.sum()
    return out


# --------------------------------------------------------------------------
# Batched drivers (loops over sequences and KV heads) used by tests/bench.
# Layouts: q [B][Hq][128]; contiguous cache [B][Hkv][cap][128]; gate weights
# w_q [Hq][128][128], w_k [Hkv][384][128]; gains gamma_q [128] and gamma_k
# [128], one each per layer (reading R5b: the printed parameter counts fit
# one shared gain per layer, not one per head).  Query head g belongs to KV
# head g // G (G = Hq / Hkv).
# --------------------------------------------------------------------------
def decode_step(q, k_cache, v_cache, seq_lens, w_q, gamma_q, w_k, gamma_k,
                token_budget, gate_keys=None, pairs=None, eps=1e-6, base=10000.0,
                gate_mode=GATE_SELECT_ONLY):
    """Full decode step for the listed (sequence, KV head) pairs (all if None).

    gate_keys: optional precomputed [B][Hkv][>=c][128]; computed from the
    cache when None.  Returns {(s, h): decode_one_group(...)}.
    """
    B, Hq = q.shape[0], q.shape[1]
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    if pairs is None:
        pairs = [(s, h) for s in range(B) for h in range(Hkv)]
    res = {}
    for (s, h) in pairs:
        L = int(seq_lens[s])
        c = (L - 1) // BLOCK
        ks, vs = k_cache[s, h], v_cache[s, h]
        if gate_keys is None:
            gk = gate_keys_for_sequence(ks, c, w_k[h], gamma_k, eps, base)
        else:
            gk = np.asarray(gate_keys[s, h, :c], np.float64)
        heads = slice(h * G, (h + 1) * G)
        res[(s, h)] = decode_one_group(np.asarray(q[s, heads], np.float64), ks, vs, L, gk,
                                       w_q[heads], np.tile(gamma_q, (G, 1)), token_budget,
                                       eps=eps, base=base, gate_mode=gate_mode)
    return res


# --------------------------------------------------------------------------
# Gradient of the gated decode step with respect to the gate parameters
# (R20): the continuous gates on the selected blocks make the gate
# differentiable; the Top-K set is held fixed.
# --------------------------------------------------------------------------
def rms_norm_backward(x, gamma, dy, eps: float = 1e-6):
    """Backward of y = x / r * gamma, r = sqrt(mean(x^2) + eps): returns
    (dL/dx, dL/dgamma) for dL/dy = dy.  From dy_i/dx_k = gamma_i (delta_ik / r
    - x_i x_k / (n r^3))."""
    x = np.asarray(x, np.float64)
    gamma = np.asarray(gamma, np.float64)
    dy = np.asarray(dy, np.float64)
    n = x.shape[-1]
    r = math.sqrt(float(np.mean(x * x)) + eps)
    gdy = gamma * dy
    dx = gdy / r - x * float(np.dot(gdy, x)) / (n * r ** 3)
    dgamma = dy * x / r
    return dx, dgamma


def log_sigmoid_grad(x: float) -> float:
    """d log(sigmoid(x)) / dx = 1 - sigmoid(x) = sigmoid(-x)."""
    return math.exp(log_sigmoid(-x))


def matmul_weight_grad(x, dy):
    """Gradient of W in y = x @ W (row vector x): dL/dW[i][j] = x_i dL/dy_j."""
    return np.outer(np.asarray(x, np.float64), np.asarray(dy, np.float64))


def rope_backward(dy, pos: int, base: float = 10000.0):
    """Backward of the gate RoPE at `pos`: each (i, i+64) pair is a plane
    rotation, so its transpose is the rotation by -pos."""
    return rope_rotate_half(dy, -pos, base)


def decode_gate_grads(q_group, k_seq, v_seq, seq_len, w_q_group, gamma_q, w_k, gamma_k,
                      token_budget, d_out, attn_scale=1.0 / math.sqrt(128.0),
                      gate_scale=1.0 / math.sqrt(128.0), eps=1e-6, base=10000.0, sel=None):
    """Gated-mode decode step of one (sequence, KV head) and the gradients of
    L = sum_g d_out[g] . out[g] with respect to the gate parameters (R20).

    q_group [G][128]; k_seq, v_seq [>= L][128]; w_q_group [G][128][128];
    gamma_q [128]; w_k [384][128]; gamma_k [128]; d_out [G][128].
    sel: the block list to hold fixed (None: the gate's own Top-K).
    Returns dict(out, sel, s, dw_q [G][128][128], dw_k [384][128],
    dgamma_q [128], dgamma_k [128]).

    Forward, in the method's order: pooled keys P_b, u_b = P_b @ W_k,
    k^_b = RMSNorm(u_b) * gamma_k, k~_b = RoPE(k^_b, b); v_g = q_g @ W_q[g],
    q^_g = RMSNorm(v_g) * gamma_q, q~_g = RoPE(q^_g, c); s_gb = q~_g . k~_b *
    gate_scale; logits q_g . k_j * attn_scale + log(sigmoid(s_gb)) on the
    tokens j of a selected historical block b (0 on the current block);
    softmax; out_g = sum_j p_gj v_j.  Backward in reverse order."""
    q_group = np.asarray(q_group, np.float64)
    d_out = np.asarray(d_out, np.float64)
    G = q_group.shape[0]
    c = (seq_len - 1) // BLOCK
    # forward
    P = [pool_block(k_seq[b * BLOCK:(b + 1) * BLOCK]) for b in range(c)]
    u = [P[b] @ np.asarray(w_k, np.float64) for b in range(c)]
    kt = np.array([rope_rotate_half(rms_norm(u[b], gamma_k, eps), b, base) for b in range(c)]).reshape(c, HEAD_DIM)
    v = [q_group[g] @ np.asarray(w_q_group[g], np.float64) for g in range(G)]
    qt = np.array([rope_rotate_half(rms_norm(v[g], gamma_q, eps), c, base) for g in range(G)])
    s = (qt @ kt.T) * gate_scale if c else np.zeros((G, 0))
    if sel is None:
        sel = select_blocks(s.mean(axis=0) if c else np.zeros(0), c, topk_for_budget(token_budget))
    toks = selected_token_ids(sel, seq_len)
    blk = [t // BLOCK for t in toks]
    out = np.zeros((G, HEAD_DIM))
    dw_q = np.zeros((G, HEAD_DIM, HEAD_DIM))
    dgamma_q = np.zeros(HEAD_DIM)
    dkt = np.zeros((c, HEAD_DIM))
    ds_all = np.zeros((G, c))
    for g in range(G):
        bias = np.array([0.0 if b == c else log_sigmoid(s[g, b]) for b in blk])
        logits = (k_seq[toks].astype(np.float64) @ q_group[g]) * attn_scale + bias
        w = np.exp(logits - logits.max())
        p = w / w.sum()
        out[g] = p @ v_seq[toks].astype(np.float64)
        # softmax backward: dL/dlogit_j = p_j (d_out . v_j - d_out . out)
        dv_dot = v_seq[toks].astype(np.float64) @ d_out[g]
        dlogit = p * (dv_dot - float(np.dot(d_out[g], out[g])))
        # the bias of block b is shared by its tokens; d log(sigmoid(s))/ds = 1 - sigmoid(s)
        dq_t = np.zeros(HEAD_DIM)
        for b in sel[:-1]:
            dbias = sum(dl for dl, bj in zip(dlogit, blk) if bj == b)
            ds = dbias * log_sigmoid_grad(s[g, b])
            ds_all[g, b] = ds
            dq_t += ds * gate_scale * kt[b]
            dkt[b] += ds * gate_scale * qt[g]
        dq_hat = rope_backward(dq_t, c, base)
        dvg, dgq = rms_norm_backward(v[g], gamma_q, dq_hat, eps)
        dgamma_q += dgq
        dw_q[g] = matmul_weight_grad(q_group[g], dvg)
    dw_k = np.zeros((POOL_DIM, HEAD_DIM))
    dgamma_k = np.zeros(HEAD_DIM)
    for b in sel[:-1]:
        dk_hat = rope_backward(dkt[b], b, base)
        dub, dgk = rms_norm_backward(u[b], gamma_k, dk_hat, eps)
        dgamma_k += dgk
        dw_k += matmul_weight_grad(P[b], dub)
    return {"out": out, "sel": sel, "s": s, "ds": ds_all, "dw_q": dw_q, "dw_k": dw_k,
            "dgamma_q": dgamma_q, "dgamma_k": dgamma_k}


def gated_decode_loss(q_group, k_seq, v_seq, seq_len, w_q_group, gamma_q, w_k, gamma_k,
                      d_out, sel, attn_scale=1.0 / math.sqrt(128.0),
                      gate_scale=1.0 / math.sqrt(128.0), eps=1e-6, base=10000.0):
    """L = sum_g d_out[g] . out[g] of the gated decode step over the fixed
    block list `sel` (the scalar whose gradient decode_gate_grads returns),
    through the forward functions above (gate_keys_for_sequence,
    gate_scores, attention_over_tokens)."""
    G = len(q_group)
    c = (seq_len - 1) // BLOCK
    keys = gate_keys_for_sequence(k_seq, c, w_k, gamma_k, eps, base)
    s, _ = gate_scores(q_group, w_q_group, np.tile(gamma_q, (G, 1)), keys, c, c, gate_scale, eps, base)
    toks = selected_token_ids(sel, seq_len)
    tot = 0.0
    for g in range(G):
        o = attention_over_tokens(q_group[g], k_seq, v_seq, toks, attn_scale,
                                  gated_token_bias(s[g], sel, seq_len, c))
        tot += float(np.dot(d_out[g], o))
    return tot


# --------------------------------------------------------------------------
# Gradient of the gated prefill with respect to the gate parameters (R20 for
# the chunked prefill: every query block i has its own gate query, its own
# block list and its own gates log(sigmoid(s_{g,i,b}))).
# --------------------------------------------------------------------------
def prefill_gate_grads(q_seq_group, k_seq, v_seq, w_q_group, gamma_q, w_k, gamma_k, sels, d_out,
                       attn_scale=1.0 / math.sqrt(128.0), gate_scale=1.0 / math.sqrt(128.0),
                       eps=1e-6, base=10000.0):
    """Gated-mode prefill of one (sequence, KV head) over the fixed block lists
    `sels` (sels[i]: ascending historical blocks of query block i, then i) and
    the gradients of L = sum_{g,t} d_out[g][t] . out[g][t] with respect to the
    gate parameters (R20).

    q_seq_group, d_out [G][T][128]; k_seq, v_seq [T][128]; T a multiple of 64;
    w_q_group [G][128][128]; gamma_q, gamma_k [128]; w_k [384][128].
    Returns dict(out [G][T][128], s (dict (g, i) -> scores over blocks < i),
    dw_q [G][128][128], dw_k [384][128], dgamma_q, dgamma_k).

    Forward as prefill_query_block (R13, R18): gate query of head g for block
    i = RoPE(RMSNorm(mean_t q[g][t] @ W_q[g]) * gamma_q, i); gate key of block
    b as decode; token t of block i attends to the kept historical blocks'
    tokens (+ log(sigmoid(s_{g,i,b}))) and causally to block i (+ 0).
    Backward: dL/dlogit_j = p_j (d_out_t . v_j - d_out_t . out_t); a block's
    bias is shared by all (t, j) of query block i and key block b."""
    q_seq_group = np.asarray(q_seq_group, np.float64)
    d_out = np.asarray(d_out, np.float64)
    k_seq = np.asarray(k_seq, np.float64)
    v_seq = np.asarray(v_seq, np.float64)
    G, T = q_seq_group.shape[0], q_seq_group.shape[1]
    nblk = T // BLOCK
    P = [pool_block(k_seq[b * BLOCK:(b + 1) * BLOCK]) for b in range(nblk)]
    u = [P[b] @ np.asarray(w_k, np.float64) for b in range(nblk)]
    kt = np.array([rope_rotate_half(rms_norm(u[b], gamma_k, eps), b, base) for b in range(nblk)])
    out = np.zeros((G, T, HEAD_DIM))
    dw_q = np.zeros((G, HEAD_DIM, HEAD_DIM))
    dgamma_q = np.zeros(HEAD_DIM)
    dkt = np.zeros((nblk, HEAD_DIM))
    s_all = {}
    for i in range(nblk):
        sel = list(sels[i])
        hist = sel[:-1]
        toks_hist = selected_token_ids(hist, (i + 1) * BLOCK)  # 64 tokens per kept block, in list order
        k_hist, v_hist = k_seq[toks_hist], v_seq[toks_hist]
        for g in range(G):
            qbar = q_seq_group[g, i * BLOCK:(i + 1) * BLOCK].mean(axis=0)
            v = qbar @ np.asarray(w_q_group[g], np.float64)
            qt = rope_rotate_half(rms_norm(v, gamma_q, eps), i, base)
            s = np.array([float(qt @ kt[b]) * gate_scale for b in range(i)])
            s_all[(g, i)] = s
            bias_hist = np.repeat([log_sigmoid(s[b]) for b in hist], BLOCK)
            dbias = np.zeros(len(hist))
            for t in range(BLOCK):
                tok = i * BLOCK + t
                k_diag, v_diag = k_seq[i * BLOCK:tok + 1], v_seq[i * BLOCK:tok + 1]
                logits = np.concatenate([k_hist @ q_seq_group[g, tok] * attn_scale + bias_hist,
                                         k_diag @ q_seq_group[g, tok] * attn_scale])
                w = np.exp(logits - logits.max())
                p = w / w.sum()
                vv = np.concatenate([v_hist, v_diag])
                out[g, tok] = p @ vv
                dlogit = p * (vv @ d_out[g, tok] - float(np.dot(d_out[g, tok], out[g, tok])))
                # a kept block's bias is shared by its 64 tokens
                dbias += dlogit[:len(toks_hist)].reshape(len(hist), BLOCK).sum(axis=1)
            dq_t = np.zeros(HEAD_DIM)
            for n, b in enumerate(hist):
                ds = dbias[n] * log_sigmoid_grad(s[b])
                dq_t += ds * gate_scale * kt[b]
                dkt[b] += ds * gate_scale * qt
            dq_hat = rope_backward(dq_t, i, base)
            dvg, dgq = rms_norm_backward(v, gamma_q, dq_hat, eps)
            dgamma_q += dgq
            dw_q[g] += matmul_weight_grad(qbar, dvg)
    dw_k = np.zeros((POOL_DIM, HEAD_DIM))
    dgamma_k = np.zeros(HEAD_DIM)
    for b in range(nblk):
        if not np.any(dkt[b]):
            continue
        dk_hat = rope_backward(dkt[b], b, base)
        dub, dgk = rms_norm_backward(u[b], gamma_k, dk_hat, eps)
        dgamma_k += dgk
        dw_k += matmul_weight_grad(P[b], dub)
    return {"out": out, "s": s_all, "dw_q": dw_q, "dw_k": dw_k, "dgamma_q": dgamma_q, "dgamma_k": dgamma_k}


def gated_prefill_loss(q_seq_group, k_seq, v_seq, w_q_group, gamma_q, w_k, gamma_k, sels, d_out,
                       attn_scale=1.0 / math.sqrt(128.0), gate_scale=1.0 / math.sqrt(128.0),
                       eps=1e-6, base=10000.0):
    """L = sum_{g,t} d_out[g][t] . out[g][t] of the gated prefill over the
    fixed block lists `sels` (the scalar whose gradient prefill_gate_grads
    returns), through the forward functions above (gate_keys_for_sequence,
    gate_scores, gated_token_bias, attention_over_tokens)."""
    q_seq_group = np.asarray(q_seq_group, np.float64)
    G, T = q_seq_group.shape[0], q_seq_group.shape[1]
    nblk = T // BLOCK
    keys = gate_keys_for_sequence(k_seq, nblk, w_k, gamma_k, eps, base)
    tot = 0.0
    for i in range(nblk):
        qbar = q_seq_group[:, i * BLOCK:(i + 1) * BLOCK].mean(axis=1)
        s, _ = gate_scores(qbar, w_q_group, np.tile(gamma_q, (G, 1)), keys, i, i, gate_scale, eps, base)
        hist = list(sels[i])[:-1]
        toks_hist = selected_token_ids(hist, (i + 1) * BLOCK)
        for g in range(G):
            hb = gated_token_bias(s[g], hist, (i + 1) * BLOCK, i)
            for t in range(BLOCK):
                tok = i * BLOCK + t
                toks = toks_hist + list(range(i * BLOCK, tok + 1))
                o = attention_over_tokens(q_seq_group[g, tok], k_seq, v_seq, toks, attn_scale,
                                          hb + [0.0] * (t + 1))
                tot += float(np.dot(d_out[g, tok], o))
    return tot
