"""GPU parity of the gated inference mode (SAS_GATE_LOGSIGMOID_BIAS) of the
fused decode step against the CPU oracle, through the C ABI.

The mode adds log(sigmoid(s_gb)) -- s_gb the query head's gate score -- to
the attention logits of every token of a selected historical block, and 0 to
the current block.  Small shapes span several selected blocks per CTA, GQA
groups of 1 to 8 and ragged current blocks (with and without pooling of a
completed block); the Qwen3-4B 32k workload is checked on sampled pairs."""
import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import DecodeSpec, make_decode_inputs, qwen3_4b_32k
from oracle import sas_oracle as O

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"
GATED = sas.GATE_LOGSIGMOID_BIAS


def _run(spec, budget, pairs=None, pool=False, out_dtype="bf16", out_atol=T.OUT_ATOL):
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, budget, out_dtype, gate_mode=GATED)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    if pool:  # the step itself pools blocks its token completes
        for s, L in enumerate(spec.seq_lens):
            if L % 64 == 0:
                gk[s, :, (L - 1) // 64] = 0.0
    gpu = T.run_decode_step(inp, cfg, ws, gk, pool=pool)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    pairs = pairs or [(s, h) for s in range(spec.batch) for h in range(spec.hkv)]
    orc = T.oracle_pairs(inp, budget, pairs, gate_mode=O.GATE_LOGSIGMOID_BIAS)
    T.check_pairs(inp, cfg, gpu, orc, gate_keys=gk, out_atol=out_atol)
    return inp, gpu, orc


CASES = [
    ("g4", 2, 8, 2, [4096, 2500], 1024, "bf16", False),
    ("g4_pool", 2, 8, 2, [4096, 1984], 512, "bf16", True),
    ("g8", 1, 8, 1, [1800], 320, "bf16", False),
    ("g1_ragged", 3, 2, 2, [777, 64, 65], 192, "bf16", False),
    ("g5", 2, 10, 2, [3000, 4097], 512, "bf16", False),
    ("f32", 2, 8, 2, [1500, 333], 512, "f32", False),
]


@pytest.mark.parametrize("name,B,hq,hkv,lens,budget,dt,pool", CASES, ids=[c[0] for c in CASES])
def test_gated_decode_step_small(name, B, hq, hkv, lens, budget, dt, pool):
    spec = DecodeSpec(name, B, hq, hkv, lens, (budget,), kv_dtype=dt, block_offset_std=0.5, seed=23)
    _run(spec, budget, pool=pool, out_dtype=("f32" if dt == "f32" else "bf16"),
         out_atol=(2e-4 if dt == "f32" else T.OUT_ATOL))


def test_gated_differs_from_select_only():
    """The gate must change the output (the two modes share the block set)."""
    spec = DecodeSpec("gated_vs_plain", 2, 8, 2, [4096, 3000], (1024,), block_offset_std=0.5, seed=29)
    inp = make_decode_inputs(spec, DEV)
    outs = {}
    for mode in (sas.GATE_SELECT_ONLY, GATED):
        cfg = T.config_for(spec, 1024, gate_mode=mode)
        ws = sas.make_workspace(cfg, DEV)
        gk = T.run_pool(inp, cfg, ws)
        outs[mode] = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert torch.equal(outs[GATED]["sel_idx"], outs[sas.GATE_SELECT_ONLY]["sel_idx"])
    d = (outs[GATED]["out"].float() - outs[sas.GATE_SELECT_ONLY]["out"].float()).abs().max().item()
    assert d > 1e-2


def test_gated_qwen3_4b_32k_full_size():
    spec = qwen3_4b_32k()
    _run(spec, 2048, pairs=[(0, 0), (3, 5), (7, 7)], pool=True)
