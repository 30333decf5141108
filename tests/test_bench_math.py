"""The algorithmic byte and FLOP counts behind bench.py's roofline fractions,
checked against hand-derived totals for the benchmark workloads (CPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_decode_bytes_qwen3_4b_32k():
    """Batch 8, 32/8 heads, 32,768 tokens, budget 2,048, pooling the completed
    block: per (sequence, KV head) 32 blocks of K and V (bf16) = 32*64*128*2*2
    bytes, 511 fp32 gate keys, q and out of 4 heads, the new gate key; per
    launch W_q of 32 heads and W_k of 8 heads (bf16)."""
    per_pair = 32 * 64 * 128 * 2 * 2 + 511 * 128 * 4 + 2 * 4 * 128 * 2 + 128 * 4
    want = 8 * 8 * per_pair + 32 * 128 * 128 * 2 + 8 * 384 * 128 * 2
    assert want == 85_852_160
    assert bench.decode_bytes([32768] * 8, 32, 8, 2048) == want


def test_decode_bytes_qwen3_14b_paged_128k():
    """Batch 16, 40/8 heads, 131,072 tokens, budget 4,096: per (sequence, KV
    head) 63 historical blocks plus the full current block (64 tokens) of K
    and V, 2,047 fp32 gate keys, q and out of 5 heads, the new gate key (the
    token completes block 2,047); per launch W_q of 40 heads and W_k of 8."""
    per_pair = 64 * 64 * 128 * 2 * 2 + 2047 * 128 * 4 + 2 * 5 * 128 * 2 + 128 * 4
    want = 16 * 8 * per_pair + 40 * 128 * 128 * 2 + 8 * 384 * 128 * 2
    assert want == 405_078_016
    assert bench.decode_bytes([131072] * 16, 40, 8, 4096) == want


def test_decode_bytes_bf16_keys_and_mixed_budgets():
    per_pair16 = 32 * 64 * 128 * 4 + 511 * 128 * 2 + 2 * 4 * 128 * 2 + 128 * 2
    assert bench.decode_bytes([32768] * 8, 32, 8, 2048, gk_elem=2) == \
        8 * 8 * per_pair16 + 32 * 128 * 128 * 2 + 8 * 384 * 128 * 2
    budgets = [1024, 4096]
    per = [(b // 64) * 64 * 128 * 4 + 511 * 512 + 2 * 4 * 128 * 2 + 512 for b in budgets]
    assert bench.decode_bytes([32768] * 2, 32, 8, budgets) == 8 * sum(per) + 32 * 128 * 128 * 2 + 8 * 384 * 128 * 2


def test_decode_bytes_partial_current_block_and_short_context():
    # L = 100: current block 1 holds 36 tokens, one historical block; no block
    # completes, so neither W_k nor a new gate key is read or written
    per_pair = (1 * 64 + 36) * 128 * 2 * 2 + 1 * 512 + 2 * 4 * 128 * 2
    assert bench.decode_bytes([100], 32, 8, 2048) == 8 * per_pair + 32 * 128 * 128 * 2


def test_prefill_flops_qwen3_8b_32k():
    """512 query blocks, Top-K 31: block i attends min(31, i) + 1 blocks, so
    sum_i = 496 + 481 * 32 = 15,888 tile pairs per (sequence, query head), each
    2 * 64 * 64 * 128 FLOPs for Q K^T and as many for P V."""
    pairs = sum(min(31, i) + 1 for i in range(512))
    assert pairs == 15_888
    assert bench.prefill_flops(512, 32, 8, 2048, 4) == 4 * 32 * 15_888 * 4 * 64 * 64 * 128


def test_traffic_digest_ignores_comments_but_not_code():
    src = "int f(int x) {  // doubles\n  /* the\n     rule */\n  return 2 * x;\n}\n"
    base = bench.code_only(src)
    assert base == "int f(int x) {\n  return 2 * x;\n}"
    assert bench.code_only(src.replace("doubles", "twice")) == base
    assert bench.code_only("\n\n" + src.replace("/* the", "/* a")) == base
    assert bench.code_only(src.replace("2 * x", "3 * x")) != base


def test_all_cores_oracle_baseline_runs_in_spawned_processes():
    r = bench.cpu_baseline_all_cores(0.3, workers=2)
    assert r["cores"] == 2 and r["kind"] == "oracle" and r["value"] > 0
    assert "2 processes" in r["sample"]
