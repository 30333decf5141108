"""GPU parity of the decode path against the CPU oracle, through the C ABI.

Small shapes span several gate-key chunks, several selected blocks per CTA
and ragged current blocks; the full-size workloads (Qwen3-4B 32k batch 8,
Qwen3-8B ragged batch 32 at three budgets, Qwen3-14B paged 128k) are checked
on every (sequence, KV head) pair, which the oracle computes one by one.  The
workloads carry non-unit RMSNorm gains, so every kernel's use of gamma_q and
gamma_k is compared too."""
import math

import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import (DecodeSpec, make_decode_inputs, qwen3_4b_32k,
                                                     qwen3_8b_ragged, qwen3_14b_paged_128k,
                                                     tiny_decode, logical_kv)
from oracle import sas_oracle as O

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _all_pairs(spec):
    return [(s, h) for s in range(spec.batch) for h in range(spec.hkv)]


def _run_and_check(spec, budget, out_dtype="bf16", pairs=None, out_atol=T.OUT_ATOL):
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, budget, out_dtype)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    pairs = pairs or _all_pairs(spec)
    orc = T.oracle_pairs(inp, budget, pairs)
    T.check_pairs(inp, cfg, gpu, orc, gate_keys=gk, out_atol=out_atol)
    return inp, cfg, gpu, orc


SMALL = [
    # name, B, hq, hkv, lens, budget, dtype
    ("g4_multi_tile", 2, 8, 2, [4096, 2500], 1024, "bf16"),
    ("g4_ragged_tail", 3, 4, 1, [65, 1000, 2049], 256, "bf16"),
    ("g5_qwen14b_heads", 2, 10, 2, [3000, 4097], 512, "bf16"),
    ("g8", 1, 8, 1, [1800], 320, "bf16"),
    ("g1", 2, 2, 2, [777, 64], 128, "bf16"),
    ("budget64_current_only", 2, 8, 2, [1000, 3], 64, "bf16"),
    ("single_token", 1, 4, 1, [1], 2048, "bf16"),
    ("full_first_block", 1, 4, 1, [64], 2048, "bf16"),
    ("budget_covers_context", 2, 8, 2, [1500, 640], 2048, "bf16"),
    ("long_slices", 1, 4, 1, [20000], 1024, "bf16"),
    ("f32_small", 2, 8, 2, [1500, 333], 512, "f32"),
]


@pytest.mark.parametrize("name,B,hq,hkv,lens,budget,dt", SMALL, ids=[s[0] for s in SMALL])
def test_decode_step_small(name, B, hq, hkv, lens, budget, dt):
    spec = DecodeSpec(name, B, hq, hkv, lens, (budget,), kv_dtype=dt, block_offset_std=0.5, seed=11)
    _run_and_check(spec, budget, out_atol=(2e-4 if dt == "f32" else T.OUT_ATOL),
                   out_dtype=("f32" if dt == "f32" else "bf16"))


def test_decode_step_f32_out_from_bf16_cache():
    spec = DecodeSpec("bf16_to_f32", 2, 8, 2, [3000, 1234], (512,), seed=12)
    _run_and_check(spec, 512, out_dtype="f32")


def test_paged_small():
    spec = DecodeSpec("paged_small", 2, 8, 2, [2000, 4096], (512,), paged=True, capacity=4096, seed=13)
    _run_and_check(spec, 512)


def test_tiny_config_full():
    """One sequence, one KV head, G 4, 4,096 tokens, budget 1,024, fp32 Q/K/V."""
    spec = tiny_decode()
    _run_and_check(spec, 1024, out_dtype="f32", out_atol=2e-4)


def test_budget_covering_context_equals_dense():
    spec = DecodeSpec("dense", 2, 8, 2, [1200, 2048], (2048,), seed=14)
    inp, cfg, gpu, _ = _run_and_check(spec, 2048)
    out = gpu["out"].float().cpu().numpy()
    q = inp["q"].double().cpu().numpy()
    for s in range(2):
        for h in range(2):
            ks, vs = logical_kv(inp, s, h, spec.seq_lens[s])
            dense = O.dense_causal_decode(q[s, 4 * h:4 * h + 4], ks, vs, spec.seq_lens[s])
            assert np.max(np.abs(out[s, 4 * h:4 * h + 4] - dense)) <= T.OUT_ATOL


def test_values_past_context_are_ignored():
    """NaN in cache rows past L (the unwritten tail of the current block) must
    not reach the output."""
    spec = DecodeSpec("nan_tail", 2, 8, 2, [1000, 2050], (512,), capacity=4096, seed=15)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    for s, L in enumerate(spec.seq_lens):
        inp["k"][s, :, L:] = float("nan")
        inp["v"][s, :, L:] = float("nan")
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    orc = T.oracle_pairs(inp, 512, _all_pairs(spec))
    T.check_pairs(inp, cfg, gpu, orc, gate_keys=gk)


def test_pool_keys_vs_oracle_and_raw_pooling():
    spec = DecodeSpec("pool", 2, 8, 2, [3000, 700], (512,), capacity=4096, block_offset_std=0.5, seed=16)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    mg = T.gate_key_rows(spec)
    raw = torch.zeros(2, 2, mg, 384, dtype=torch.float32, device=DEV)
    gk = T.run_pool(inp, cfg, ws, pooled_raw=raw)
    torch.cuda.synchronize()
    gk, raw = gk.cpu().numpy(), raw.cpu().numpy()
    wk = inp["w_k"].double().cpu().numpy()
    gam_k = inp["gamma_k"].double().cpu().numpy()
    assert not np.allclose(gam_k, 1.0)   # the gain is exercised
    for s in range(2):
        for h in range(2):
            L = spec.seq_lens[s]
            ks, _ = logical_kv(inp, s, h, L)
            nfull = L // 64
            want = O.gate_keys_for_sequence(ks, nfull, wk[h], gam_k)
            T.assert_close_rel(gk[s, h, :nfull], want, f"gate keys s={s} h={h}")
            assert np.all(gk[s, h, nfull:] == 0), "incomplete blocks must not be pooled"
            for b in range(nfull):
                p = O.pool_block(ks[64 * b:64 * b + 64])
                assert np.array_equal(raw[s, h, b, :256], p[:256])  # max, min exact
                assert np.allclose(raw[s, h, b, 256:], p[256:], rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("gk16", [0, 1])
def test_pool_keys_tiles_offsets_and_ragged_ends(gk16):
    """Pooling calls that start mid-cache and cross the 128-block tiles of the
    tensor-core projection: blocks blk_begin[s] .. blk_begin[s] + 199 that are
    complete, every other row left alone."""
    spec = DecodeSpec("pool_tiles", 2, 8, 2, [64 * 300, 64 * 250 + 17], (512,), capacity=64 * 300,
                      block_offset_std=0.5, seed=19)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    cfg.gate_keys_bf16 = gk16
    ws = sas.make_workspace(cfg, DEV)
    mg = T.gate_key_rows(spec)
    gk = torch.full((2, 2, mg, 128), 7.0, dtype=sas.gate_key_dtype(cfg), device=DEV)
    begin = torch.tensor([5, 130], dtype=torch.int32, device=DEV)
    sas.pool_keys(cfg, T.kv_of(inp), inp["w_k"], inp["gamma_k"], gk, ws, blk_begin=begin, num_blocks=200)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    got = gk.double().cpu().numpy()
    wk = inp["w_k"].double().cpu().numpy()
    gam_k = inp["gamma_k"].double().cpu().numpy()
    for s, L in enumerate(spec.seq_lens):
        lo, hi = int(begin[s]), min(int(begin[s]) + 200, L // 64)
        for h in range(2):
            ks, _ = logical_kv(inp, s, h, L)
            want = np.stack([O.gate_key(O.pool_block(ks[64 * b:64 * b + 64]), wk[h], gam_k, b) for b in range(lo, hi)])
            if gk16:
                want = O.round_to_bf16(want)
                T.assert_close_rel(got[s, h, lo:hi], want, f"pooled s={s} h={h}", rtol=T.BF16_ULP)
            else:
                T.assert_close_rel(got[s, h, lo:hi], want, f"pooled s={s} h={h}")
            keep = [b for b in range(mg) if not lo <= b < hi]
            assert np.all(got[s, h, keep] == 7.0), "rows outside the range must be left alone"


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_decode_step_pools_the_completed_block(dt):
    """With W_k / gamma_k the fused step writes the gate key of the block the
    decoded token completes (L % 64 == 0) and leaves other rows alone."""
    spec = DecodeSpec("fused_pool_" + dt, 4, 8, 2, [4096, 2048, 2049, 64], (512,), kv_dtype=dt,
                      capacity=4096, block_offset_std=0.5, seed=22)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512, "f32" if dt == "f32" else "bf16")
    ws = sas.make_workspace(cfg, DEV)
    ref = T.run_pool(inp, cfg, ws)           # every complete block, by the pooling kernel
    gk = ref.clone()
    for s, L in enumerate(spec.seq_lens):
        gk[s, :, (L - 1) // 64] = 0.0          # forget the current block's row
    gpu = T.run_decode_step(inp, cfg, ws, gk, pool=True)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    wk = inp["w_k"].double().cpu().numpy()
    gam_k = inp["gamma_k"].double().cpu().numpy()
    for s, L in enumerate(spec.seq_lens):
        c = (L - 1) // 64
        for h in range(2):
            row = gk[s, h, c].cpu().numpy()
            if L % 64 == 0:
                ks, _ = logical_kv(inp, s, h, L)
                want = O.gate_key(O.pool_block(ks[64 * c:64 * c + 64]), wk[h], gam_k, c)
                T.assert_close_rel(row, want, f"fused pooled key s={s} h={h}")
                # same fp32 arithmetic in another accumulation order (384-term dot products)
                T.assert_close_rel(row, ref[s, h, c].cpu().numpy(), "fused vs pooling kernel",
                                   rtol=2e-4)
            else:
                assert np.all(row == 0), "an incomplete block must not be pooled"
    for s, L in enumerate(spec.seq_lens):  # every other row untouched
        c = (L - 1) // 64
        keep = [b for b in range(gk.shape[2]) if b != c]
        assert torch.equal(gk[s, :, keep], ref[s, :, keep])
    orc = T.oracle_pairs(inp, 512, _all_pairs(spec))
    T.check_pairs(inp, cfg, gpu, orc, out_atol=(2e-4 if dt == "f32" else T.OUT_ATOL))


def test_incremental_pooling_matches_full_pooling():
    spec = DecodeSpec("incr", 2, 8, 2, [4096, 3000], (512,), capacity=4096, seed=17)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    full = T.run_pool(inp, cfg, ws)
    # pool the first part, then the rest block by block from per-sequence starts
    part = torch.zeros_like(full)
    T.run_pool(inp, cfg, ws, gate_keys=part, num_blocks=20)
    begin = torch.full((2,), 20, dtype=torch.int32, device=DEV)
    for _ in range(50):
        T.run_pool(inp, cfg, ws, gate_keys=part, blk_begin=begin, num_blocks=1)
        begin += 1
    torch.cuda.synchronize()
    assert torch.equal(part, full)


def test_gate_scores_entry_point():
    spec = DecodeSpec("gate", 3, 10, 2, [4000, 129, 2500], (1024,), capacity=4096, seed=18)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 1024)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    mg = gk.shape[2]
    head = torch.full((3, 10, mg), float("nan"), device=DEV)
    group = torch.full((3, 2, mg), float("nan"), device=DEV)
    sas.gate_scores(cfg, inp["q"], inp["seq_lens"], inp["w_q"], inp["gamma_q"], gk, group, ws,
                    head_scores=head)
    torch.cuda.synchronize()
    orc = T.oracle_pairs(inp, 1024, _all_pairs(spec))
    head, group = head.cpu().numpy(), group.cpu().numpy()
    for (s, h), r in orc.items():
        c = len(r["S"])
        T.assert_close_rel(group[s, h, :c], r["S"], f"group s={s} h={h}")
        T.assert_close_rel(head[s, 5 * h:5 * h + 5, :c], r["s"], f"head s={s} h={h}")


@pytest.mark.parametrize("budget", [64, 256, 1024, 4096])
def test_topk_exact_with_ties(budget):
    """Selection on given scores must equal the full-sort rule exactly, ties
    included (scores drawn from a handful of values)."""
    g = torch.Generator().manual_seed(budget)
    B, hkv, mg = 3, 4, 2048
    lens = torch.tensor([1, 2000, 64 * 2047 + 5], dtype=torch.int32)
    scores = (torch.randint(-4, 5, (B, hkv, mg), generator=g).float() * 0.25)
    scores[1, 1] += torch.randn(mg, generator=g) * 1e-3
    scores[2, 3] = torch.randn(mg, generator=g)
    scores[2, 0] = 0.5                      # all equal: index order decides
    scores[2, 1, 100:300] = float("-inf")   # extreme values next to ordinary ones
    scores[2, 2, 7] = 3.0e38
    cfg = sas.Config(4 * hkv, hkv, token_budget=budget)
    ws = sas.make_workspace(cfg, DEV)
    sel = torch.full((B, hkv, budget // 64), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, hkv), -1, dtype=torch.int32, device=DEV)
    sas.topk_blocks(cfg, scores.to(DEV), lens.to(DEV), sel, cnt, ws)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for s in range(B):
        c = (int(lens[s]) - 1) // 64
        for h in range(hkv):
            want = O.select_blocks(scores[s, h, :c].double().numpy(), c, budget // 64 - 1)
            assert int(cnt[s, h]) == len(want)
            assert list(sel[s, h, :len(want)]) == want, (s, h)


@pytest.mark.parametrize("budget", [1024, 2048, 4096, 16384])
def test_topk_exact_up_to_512_blocks(budget):
    """Up to 512 historical blocks (contexts to 32k) take the short selection
    path: value-linear buckets, a bit mask, a crowded-bucket fallback.  Ties,
    equal scores, infinities and a span that overflows fp32 must still give
    the full-sort rule exactly."""
    g = torch.Generator().manual_seed(budget + 7)
    B, hkv, mg = 2, 4, 512
    lens = torch.tensor([64 * 257 + 1, 64 * 512], dtype=torch.int32)   # 257 and 511 blocks
    scores = torch.randn(B, hkv, mg, generator=g)
    scores[:, 0] = torch.randint(-4, 5, (B, mg), generator=g).float() * 0.25   # 9 values, many ties
    scores[:, 1] = -1.25                                                     # all equal
    scores[0, 2, 3] = float("inf")
    scores[0, 2, 50:60] = float("-inf")
    scores[1, 2, 10] = 3.0e38
    scores[1, 2, 11] = -3.0e38                                               # max - min overflows
    scores[1, 3, 200:220] = 2.0                                              # a tied plateau at the top
    cfg = sas.Config(4 * hkv, hkv, token_budget=budget)
    ws = sas.make_workspace(cfg, DEV)
    sel = torch.full((B, hkv, budget // 64), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, hkv), -1, dtype=torch.int32, device=DEV)
    sas.topk_blocks(cfg, scores.to(DEV), lens.to(DEV), sel, cnt, ws)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for s in range(B):
        c = (int(lens[s]) - 1) // 64
        for h in range(hkv):
            want = O.select_blocks(scores[s, h, :c].double().numpy(), c, budget // 64 - 1)
            assert int(cnt[s, h]) == len(want)
            assert list(sel[s, h, :len(want)]) == want, (s, h)


@pytest.mark.parametrize("budget", [1024, 4096, 16384])
def test_topk_exact_513_to_2048_blocks(budget):
    """513 .. 2,048 historical blocks (contexts to 128k) take the 16-keys-per-
    thread path, 2,049 and more the general one; ties, equal scores,
    infinities and a span that overflows fp32 must give the full-sort rule
    exactly on both sides of each boundary."""
    g = torch.Generator().manual_seed(budget + 11)
    B, hkv, mg = 5, 4, 2100
    nblocks = [513, 1024, 1999, 2048, 2049]
    lens = torch.tensor([64 * n + 1 for n in nblocks], dtype=torch.int32)
    scores = torch.randn(B, hkv, mg, generator=g)
    scores[:, 0] = torch.randint(-4, 5, (B, mg), generator=g).float() * 0.25   # 9 values, many ties
    scores[:, 1] = -1.25                                                     # all equal
    scores[0, 2, 3] = float("inf")
    scores[2, 2, 50:60] = float("-inf")
    scores[3, 2, 10] = 3.0e38
    scores[3, 2, 11] = -3.0e38                                               # max - min overflows
    scores[1, 3, 700:720] = 2.0                                              # a tied plateau at the top
    cfg = sas.Config(4 * hkv, hkv, token_budget=budget)
    ws = sas.make_workspace(cfg, DEV)
    sel = torch.full((B, hkv, budget // 64), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, hkv), -1, dtype=torch.int32, device=DEV)
    sas.topk_blocks(cfg, scores.to(DEV), lens.to(DEV), sel, cnt, ws)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for s in range(B):
        c = (int(lens[s]) - 1) // 64
        assert c == nblocks[s]
        for h in range(hkv):
            want = O.select_blocks(scores[s, h, :c].double().numpy(), c, budget // 64 - 1)
            assert int(cnt[s, h]) == len(want)
            assert list(sel[s, h, :len(want)]) == want, (s, h)


def test_sparse_decode_given_blocks():
    spec = DecodeSpec("given", 2, 8, 2, [3000, 2100], (512,), capacity=4096, seed=19)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    orc = T.oracle_pairs(inp, 512, _all_pairs(spec))
    sel = torch.full((2, 2, 8), -1, dtype=torch.int32)
    cnt = torch.zeros((2, 2), dtype=torch.int32)
    for (s, h), r in orc.items():
        sel[s, h, :len(r["sel"])] = torch.tensor(r["sel"], dtype=torch.int32)
        cnt[s, h] = len(r["sel"])
    out = torch.full((2, 8, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    sas.sparse_decode(cfg, inp["q"], T.kv_of(inp), sel.to(DEV), cnt.to(DEV), out, ws)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    out = out.float().cpu().numpy()
    for (s, h), r in orc.items():
        assert np.max(np.abs(out[s, 4 * h:4 * h + 4] - r["out"])) <= T.OUT_ATOL


def test_device_bounds_are_reported_not_faulted():
    """A sequence longer than its cache, and a block table entry outside the
    page pool, are caught by the kernels' own checks (no access is issued):
    status bit set, that (seq, head) zeroed, the others still correct."""
    spec = DecodeSpec("bounds", 2, 8, 2, [1000, 2000], (512,), capacity=2048, seed=20)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    torch.cuda.synchronize()
    inp["seq_lens"][1] = 5000  # beyond capacity 2048
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_ERR_DEVICE_BOUNDS
    assert torch.all(gpu["out"][1] == 0)
    assert int(gpu["sel_count"][1, 0]) == 0
    inp["seq_lens"][1] = 2000
    orc = T.oracle_pairs(inp, 512, [(0, 0), (0, 1)])
    T.check_pairs(inp, cfg, gpu, orc)
    # paged: a page id past the pool
    spec = DecodeSpec("bounds_paged", 2, 8, 2, [1000, 2000], (512,), paged=True, capacity=2048, seed=21)
    inp = make_decode_inputs(spec, DEV)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    torch.cuda.synchronize()
    inp["block_table"][0, 3] = 10 ** 6
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_ERR_DEVICE_BOUNDS
    assert torch.all(gpu["out"][0] == 0)
    sas.reset_device_status(ws)
    assert sas.get_device_status(ws) == sas.SAS_OK


# ------------------------------------------------------------ full-size workloads
# Gate keys, group scores, block sets and outputs are compared with the
# oracle on EVERY (sequence, KV head) pair of the workload.


def test_qwen3_4b_32k_full_size():
    spec = qwen3_4b_32k()
    inp, *_ = _run_and_check(spec, 2048)
    assert not torch.allclose(inp["gamma_q"], torch.ones_like(inp["gamma_q"]))


def test_qwen3_8b_ragged_full_size():
    """Batch 32, contexts uniform in [8,192, 65,536]: every pair at each of the
    budgets 1,024 / 2,048 / 4,096 (one set of gate keys, as in serving)."""
    spec = qwen3_8b_ragged()
    inp = make_decode_inputs(spec, DEV)
    keys = {}
    for budget in (1024, 2048, 4096):
        cfg = T.config_for(spec, budget)
        ws = sas.make_workspace(cfg, DEV)
        gk = T.run_pool(inp, cfg, ws)
        gpu = T.run_decode_step(inp, cfg, ws, gk)
        torch.cuda.synchronize()
        assert sas.get_device_status(ws) == sas.SAS_OK
        orc = T.oracle_pairs(inp, budget, _all_pairs(spec), keys_cache=keys)
        T.check_pairs(inp, cfg, gpu, orc, gate_keys=gk)


def test_qwen3_14b_paged_128k_incremental():
    """Pool all but the last 256 tokens, then append them 64 at a time (one
    pooling call per completed block) and decode at 131,072."""
    spec = qwen3_14b_paged_128k()
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 4096)
    ws = sas.make_workspace(cfg, DEV)
    full_len = spec.seq_lens[0]
    start = full_len - spec.appended
    lens = inp["seq_lens"].clone()
    inp["seq_lens"].fill_(start)
    gk = T.run_pool(inp, cfg, ws)
    begin = torch.full((spec.batch,), start // 64, dtype=torch.int32, device=DEV)
    for t in range(64, spec.appended + 1, 64):
        inp["seq_lens"].fill_(start + t)
        T.run_pool(inp, cfg, ws, gate_keys=gk, blk_begin=begin, num_blocks=1)
        begin += 1
    inp["seq_lens"].copy_(lens)
    ref = T.run_pool(inp, cfg, ws)
    torch.cuda.synchronize()
    assert torch.equal(gk, ref)
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    orc = T.oracle_pairs(inp, 4096, _all_pairs(spec))
    T.check_pairs(inp, cfg, gpu, orc, gate_keys=gk)
