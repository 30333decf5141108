"""Checks the oracle's constants and the gate layout against the settings the
release pages print (tests/golden/sas_settings.txt, sources cited there)."""
import os

from oracle import sas_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def _settings():
    out = {}
    with open(os.path.join(HERE, "golden", "sas_settings.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(None, 1)
            out.setdefault(k, []).append(v)
    return out


def test_oracle_constants_match_pages():
    s = _settings()
    assert O.BLOCK == int(s["kv_block_size_tokens"][0])
    assert O.GATE_HIDDEN == int(s["gate_hidden_size"][0])
    assert s["key_block_pooling"][0] == "max+min+average"
    assert O.POOL_DIM == 3 * O.HEAD_DIM
    budgets = [int(s["default_decode_budget_tokens"][0])] + [int(x) for x in s["alt_decode_budget_tokens"]]
    # training Top-K 31 historical blocks + current = default budget / 64
    assert O.topk_for_budget(budgets[0]) == int(s["training_topk_historical_blocks"][0])
    for b in budgets:
        assert b % O.BLOCK == 0


def test_gate_layout_reproduces_printed_parameter_counts():
    # Reading R1: W_q [128x128] per query head, W_k [384x128] per KV head, no
    # bias, one 128-gain per layer for q and for k.  Qwen3 head layouts
    # (layers, query heads, KV heads): 4B/8B (36, 32, 8), 14B (40, 40, 8).
    s = _settings()

    def count(layers, hq, hkv):
        per_layer = hq * O.GATE_HIDDEN * O.HEAD_DIM + hkv * O.POOL_DIM * O.GATE_HIDDEN + 2 * O.GATE_HIDDEN
        return layers * per_layer

    assert round(count(36, 32, 8) / 1e6, 1) == float(s["gate_params_M_qwen3_4b"][0])
    assert round(count(36, 32, 8) / 1e6, 1) == float(s["gate_params_M_qwen3_8b"][0])
    assert round(count(40, 40, 8) / 1e6, 1) == float(s["gate_params_M_qwen3_14b"][0])
    # a per-head gain would give 33.2M, not the printed 33.0M
    per_head_gain = 36 * (32 * 128 * 128 + 8 * 384 * 128 + (32 + 8) * 128)
    assert round(per_head_gain / 1e6, 1) != float(s["gate_params_M_qwen3_4b"][0])
