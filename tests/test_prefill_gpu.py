"""GPU parity of the block-sparse chunked prefill (tcgen05 attention) against
the CPU oracle, through the C ABI: gate keys of every block, the block list of
every query block (exact up to the tie window), and the attention output of
every token (bf16 storage, 1e-2 max-abs)."""
import math

import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import PrefillSpec, make_prefill_inputs, qwen3_8b_prefill_32k
from oracle import sas_oracle as O

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(spec, gk16=0, gate_mode=sas.GATE_SELECT_ONLY, budgets=None, want_status=sas.SAS_OK):
    inp = make_prefill_inputs(spec, DEV)
    B, Tn = spec.batch, spec.seq_len
    nblk = Tn // 64
    cfg = sas.Config(spec.hq, spec.hkv, token_budget=spec.token_budget, gate_keys_bf16=gk16,
                     gate_mode=gate_mode)
    ws = sas.make_workspace(cfg, DEV, batch=B, max_seq_len=Tn)
    gk = torch.zeros(B, spec.hkv, nblk, 128, dtype=sas.gate_key_dtype(cfg), device=DEV)
    out = torch.full((B, spec.hq, Tn, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    sel = torch.full((B, spec.hkv, nblk, cfg.max_sel), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, spec.hkv, nblk), -1, dtype=torch.int32, device=DEV)
    tb = None if budgets is None else torch.tensor(budgets, dtype=torch.int32, device=DEV)
    sas.prefill_block_sparse(cfg, inp["q"], inp["k"], inp["v"], inp["w_q"], inp["gamma_q"], inp["w_k"],
                             inp["gamma_k"], gk, out, ws, sel_idx=sel, sel_count=cnt, token_budgets=tb)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == want_status
    return inp, cfg, gk, out, sel, cnt


def _check(spec, inp, cfg, gk, out, sel, cnt, triples, budgets=None, sets_only=()):
    """Compare the listed (sequence, KV head, query block) triples with the
    oracle: gate keys of the pair, the block list, and the 64 x G outputs
    (only the block list for the triples also listed in sets_only)."""
    G = spec.hq // spec.hkv
    wq = inp["w_q"].double().cpu().numpy()
    wk = inp["w_k"].double().cpu().numpy()
    gq = np.tile(inp["gamma_q"].double().cpu().numpy(), (G, 1))
    gkn = inp["gamma_k"].double().cpu().numpy()
    gk_h = gk.double().cpu().numpy()
    out_h, sel_h, cnt_h = out.float().cpu().numpy(), sel.cpu().numpy(), cnt.cpu().numpy()
    sets_only = set(sets_only)
    cache = {}
    for (s, h, i) in triples:
        if (s, h) not in cache:
            ks = inp["k"][s, h].double().cpu().numpy()
            vs = inp["v"][s, h].double().cpu().numpy()
            keys = O.gate_keys_for_sequence(ks, spec.seq_len // 64, wk[h], gkn)
            stored, flipped = None, set()
            if cfg.gate_keys_bf16:
                # the oracle scores from its own rounded keys; stored keys lie within
                # one bf16 ulp of them (> 99 % equal), and a row one ulp off is
                # consulted only to trace a set difference to it
                keys = O.round_to_bf16(keys)
                T.assert_close_rel(gk_h[s, h], keys, f"prefill bf16 gate keys s={s} h={h}", rtol=T.BF16_ULP)
                assert float(np.mean(gk_h[s, h] == keys)) > 0.99
                stored = gk_h[s, h]
                flipped = {b for b in range(keys.shape[0]) if not np.array_equal(stored[b], keys[b])}
            else:
                T.assert_close_rel(gk_h[s, h], keys, f"prefill gate keys s={s} h={h}")
            cache[(s, h)] = (ks, vs, keys, stored, flipped)
        ks, vs, keys, stored, flipped = cache[(s, h)]
        qb = inp["q"][s, h * G:(h + 1) * G, 64 * i:64 * (i + 1)].double().cpu().numpy()
        topk = (cfg.max_sel if budgets is None else budgets[s] // 64) - 1
        m = int(cnt_h[s, h, i])
        got_sel = list(sel_h[s, h, i, :m])
        tag = f"{spec.name} s={s} h={h} i={i}"
        if (s, h, i) in sets_only:
            qbar = qb.mean(axis=1)
            sg, S = O.gate_scores(qbar, wq[h * G:(h + 1) * G], gq, keys, i, i)
            r = {"sel": O.select_blocks(S, i, topk), "S": S, "s": sg}
        else:
            r = O.prefill_query_block(qb, ks, vs, i, keys, wq[h * G:(h + 1) * G], gq, topk,
                                      gate_mode=cfg.gate_mode)
        try:
            swapped = T.assert_selection(got_sel, r["sel"], r["S"], topk, tag)
        except AssertionError:
            if not flipped:
                raise
            assert (set(int(b) for b in got_sel) ^ set(r["sel"])) & flipped, \
                f"{tag}: set mismatch not traceable to a one-ulp key flip"
            sg, S = O.gate_scores(qb.mean(axis=1), wq[h * G:(h + 1) * G], gq, stored, i, i)
            T.assert_selection(got_sel, O.select_blocks(S, i, topk), S, topk, tag + " (stored keys)")
            swapped, r = True, dict(r, s=sg)
        if (s, h, i) in sets_only:
            continue
        want = r["out"]
        if swapped:
            # the kernel kept a tie-window swap: attend over its list, gates from the oracle's scores
            hist = O.selected_token_ids(got_sel[:-1], 64 * (i + 1))
            want = np.zeros((G, 64, 128))
            for g in range(G):
                hb = O.gated_token_bias(r["s"][g], got_sel[:-1], 64 * (i + 1), i) if cfg.gate_mode else None
                for t in range(64):
                    bias = None if hb is None else hb + [0.0] * (t + 1)
                    want[g, t] = O.attention_over_tokens(qb[g, t], ks, vs, hist + list(range(64 * i, 64 * i + t + 1)),
                                                         cfg.attn_scale, bias)
        got = out_h[s, h * G:(h + 1) * G, 64 * i:64 * (i + 1)]
        err = float(np.max(np.abs(got - want)))
        assert np.all(np.isfinite(got)) and err <= T.OUT_ATOL, f"{tag}: out max-abs err {err}"


def test_prefill_small_all_blocks():
    spec = PrefillSpec("pf_small", 1, 4, 2, 1024, token_budget=256, seed=41)
    res = _run(spec)
    triples = [(0, h, i) for h in range(2) for i in range(16)]
    _check(spec, *res, triples)


def test_prefill_small_bf16_gate_keys():
    spec = PrefillSpec("pf_small_bf16", 1, 4, 2, 1024, token_budget=256, seed=41)
    res = _run(spec, gk16=1)
    triples = [(0, h, i) for h in range(2) for i in range(16)]
    _check(spec, *res, triples)


def test_prefill_gated_mode():
    spec = PrefillSpec("pf_gated", 1, 4, 2, 1024, token_budget=256, seed=44)
    res = _run(spec, gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    _check(spec, *res, [(0, h, i) for h in range(2) for i in range(16)])


def test_prefill_gated_mode_bf16_keys_eight_heads_per_group():
    spec = PrefillSpec("pf_gated_g8", 1, 8, 1, 768, token_budget=320, seed=45)
    res = _run(spec, gk16=1, gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    _check(spec, *res, [(0, 0, i) for i in range(12)])


def test_prefill_gated_mode_full_size_sampled():
    spec = qwen3_8b_prefill_32k()
    res = _run(spec, gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    _check(spec, *res, [(0, 1, 1), (1, 6, 100), (3, 4, 511)])


def test_prefill_per_sequence_budgets():
    spec = PrefillSpec("pf_budgets", 3, 4, 2, 1024, token_budget=512, seed=46)
    res = _run(spec, budgets=[128, 512, 256])
    _check(spec, *res, [(s, h, i) for s in range(3) for h in range(2) for i in (1, 2, 5, 9, 15)],
           budgets=[128, 512, 256])
    cnt = res[-1].cpu().numpy()
    for s, kmax in enumerate((1, 7, 3)):
        assert list(cnt[s, 0]) == [min(i, kmax) + 1 for i in range(16)]


def test_prefill_per_sequence_budgets_gated():
    spec = PrefillSpec("pf_budgets_gated", 2, 4, 1, 768, token_budget=384, seed=47)
    res = _run(spec, gate_mode=sas.GATE_LOGSIGMOID_BIAS, budgets=[384, 192])
    _check(spec, *res, [(s, 0, i) for s in range(2) for i in range(12)], budgets=[384, 192])


def test_prefill_bad_budget_skips_that_sequence():
    spec = PrefillSpec("pf_bad_budget", 2, 4, 1, 512, token_budget=256, seed=48)
    inp, cfg, gk, out, sel, cnt = _run(spec, budgets=[256, 100], want_status=sas.SAS_ERR_DEVICE_BOUNDS)
    assert torch.all(cnt[1] == 0)
    assert torch.all(out[1] == 0)  # skipped: rows zeroed
    assert not torch.isnan(out[0].float()).any()
    _check(spec, inp, cfg, gk, out, sel, cnt, [(0, 0, i) for i in range(8)])


def test_prefill_budget_covering_context_is_dense_causal():
    spec = PrefillSpec("pf_dense", 2, 4, 1, 512, token_budget=1024, seed=42)
    inp, cfg, gk, out, sel, cnt = _run(spec)
    q = inp["q"].double().cpu().numpy()
    outh = out.float().cpu().numpy()
    for s in range(2):
        ks = inp["k"][s, 0].double().cpu().numpy()
        vs = inp["v"][s, 0].double().cpu().numpy()
        for g in range(4):
            dense = O.dense_causal_prefill(q[s, g], ks, vs)
            err = float(np.max(np.abs(outh[s, g] - dense)))
            assert err <= T.OUT_ATOL, (s, g, err)
    assert torch.equal(cnt.cpu(), torch.arange(1, 9, dtype=torch.int32).repeat(2, 1, 1))


def test_prefill_eight_query_heads_per_kv_head():
    spec = PrefillSpec("pf_g8", 1, 8, 1, 768, token_budget=320, seed=43)
    res = _run(spec)
    _check(spec, *res, [(0, 0, i) for i in range(12)])


def test_prefill_beyond_512_blocks():
    """33,920 tokens: query blocks past 512 historical blocks take the
    16-keys-per-thread selection."""
    spec = PrefillSpec("pf_530_blocks", 1, 2, 1, 64 * 530, token_budget=1024, seed=49)
    res = _run(spec)
    _check(spec, *res, [(0, 0, i) for i in (5, 512, 513, 520, 529)])


def test_prefill_qwen3_8b_32k_full_size():
    """Block lists of every query block of two (sequence, KV head) pairs and of
    a spread of query blocks over all pairs; outputs on a sample."""
    spec = qwen3_8b_prefill_32k()
    res = _run(spec)
    nblk = spec.seq_len // 64
    every = [(0, 0, i) for i in range(nblk)] + [(3, 7, i) for i in range(nblk)]
    spread = [(s, h, (37 * (8 * s + h) + 11) % nblk) for s in range(spec.batch) for h in range(spec.hkv)]
    outs = [(0, 0, 0), (0, 0, 30), (1, 3, 31), (2, 5, 200), (3, 7, 511), (3, 2, 64)]
    sets = [t for t in every + spread if t not in outs]
    _check(spec, *res, sets + outs, sets_only=sets)


def test_prefill_odd_group_small():
    """Five query heads per KV head (the Qwen3-14B grouping): the last tile of
    each group holds one head."""
    spec = PrefillSpec("pf_g5", 1, 10, 2, 768, token_budget=320, seed=51)
    res = _run(spec)
    _check(spec, *res, [(0, h, i) for h in range(2) for i in range(12)])


def test_prefill_odd_group_gated():
    spec = PrefillSpec("pf_g5_gated", 2, 5, 1, 640, token_budget=256, seed=52)
    res = _run(spec, gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    _check(spec, *res, [(s, 0, i) for s in range(2) for i in range(10)])


def test_prefill_qwen3_14b_heads_8k():
    """Qwen3-14B head layout (40 query / 8 KV heads), 8,192 tokens, budget
    2,048: block lists of every query block of two pairs, outputs sampled."""
    spec = PrefillSpec("pf_qwen3_14b_8k", 1, 40, 8, 8192, token_budget=2048, seed=53)
    res = _run(spec)
    nblk = spec.seq_len // 64
    outs = [(0, 0, 5), (0, 7, 127), (0, 3, 64)]
    sets = [t for t in [(0, 0, i) for i in range(nblk)] + [(0, 7, i) for i in range(nblk)] if t not in outs]
    _check(spec, *res, sets + outs, sets_only=sets)


def test_prefill_qwen3_14b_32k_full_size_sampled():
    """The Qwen3-14B head layout (40 query / 8 KV heads, five heads per group)
    at the full 32,768-token training length, budget 2,048: block lists of
    every query block of one pair and of a spread over the other pairs,
    outputs on a sample."""
    spec = PrefillSpec("pf_qwen3_14b_32k", 1, 40, 8, 32768, token_budget=2048, seed=55)
    res = _run(spec)
    nblk = spec.seq_len // 64
    every = [(0, 5, i) for i in range(nblk)]
    spread = [(0, h, (97 * h + 13) % nblk) for h in range(spec.hkv) if h != 5]
    outs = [(0, 5, 0), (0, 5, 31), (0, 0, 300), (0, 7, 511)]
    sets = [t for t in every + spread if t not in outs]
    _check(spec, *res, sets + outs, sets_only=sets)


@pytest.mark.parametrize("budget", [8192, 16384])
def test_prefill_budgets_beyond_4096(budget):
    """Budgets above 4,096 tokens (lists of up to 256 blocks; one attention
    CTA per SM)."""
    spec = PrefillSpec(f"pf_budget{budget}", 1, 4, 1, 64 * 300, token_budget=budget, seed=54)
    res = _run(spec)
    nblk = spec.seq_len // 64
    outs = [(0, 0, 3), (0, 0, 200), (0, 0, nblk - 1)]
    sets = [(0, 0, i) for i in range(nblk) if (0, 0, i) not in outs]
    _check(spec, *res, sets + outs, sets_only=sets)
