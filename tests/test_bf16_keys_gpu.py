"""The bf16 gate-key cache (gate_keys_bf16 = 1): keys are computed as before
and stored rounded to nearest-even bf16; every reader scores from the stored
value.  Parity: stored keys within one bf16 ulp of the oracle's keys rounded
the same way (the two sides differ below fp32 precision, so a value on a
rounding boundary may land one ulp apart), then scores, block sets and
outputs against the oracle run on its own rounded keys; a set difference is
accepted only where a block involved has a stored key one ulp off and the
oracle run on the stored keys agrees with the GPU."""
import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import (DecodeSpec, make_decode_inputs, qwen3_4b_32k,
                                                     logical_kv)
from oracle import sas_oracle as O

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _pool(inp, cfg, ws):
    spec = inp["spec"]
    gk = torch.zeros(spec.batch, spec.hkv, spec.cap // 64, 128, dtype=torch.bfloat16, device=DEV)
    sas.pool_keys(cfg, T.kv_of(inp), inp["w_k"], inp["gamma_k"], gk, ws)
    return gk


def _oracle_on_stored_keys(inp, cfg, gk, pairs):
    return T.oracle_on_rounded_keys(inp, cfg, gk, pairs)


@pytest.mark.parametrize("gate_mode", [sas.GATE_SELECT_ONLY, sas.GATE_LOGSIGMOID_BIAS])
def test_bf16_keys_decode_small(gate_mode):
    spec = DecodeSpec("bf16_keys", 3, 8, 2, [4096, 2500, 1000], (1024,), block_offset_std=0.5, seed=53)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 1024, gate_mode=gate_mode)
    cfg.gate_keys_bf16 = 1
    ws = sas.make_workspace(cfg, DEV)
    gk = _pool(inp, cfg, ws)
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    pairs = [(s, h) for s in range(spec.batch) for h in range(spec.hkv)]
    T.check_pairs(inp, cfg, gpu, _oracle_on_stored_keys(inp, cfg, gk, pairs))


def test_bf16_keys_fused_pooling_writes_bf16_row():
    """A step whose token completes its block writes the new key as bf16, equal
    (within one ulp) to what the pooling call stores."""
    spec = DecodeSpec("bf16_pool", 2, 8, 2, [4096, 1984], (512,), block_offset_std=0.5, seed=59)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    cfg.gate_keys_bf16 = 1
    ws = sas.make_workspace(cfg, DEV)
    ref = _pool(inp, cfg, ws)
    gk = ref.clone()
    for s, L in enumerate(spec.seq_lens):
        gk[s, :, (L - 1) // 64] = 0
    T.run_decode_step(inp, cfg, ws, gk, pool=True)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    for s, L in enumerate(spec.seq_lens):
        c = (L - 1) // 64
        T.assert_close_rel(gk[s, :, c].double().cpu().numpy(), ref[s, :, c].double().cpu().numpy(),
                           f"pooled row s={s}", rtol=T.BF16_ULP)


def test_bf16_keys_qwen3_4b_32k_full_size():
    spec = qwen3_4b_32k()
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 2048)
    cfg.gate_keys_bf16 = 1
    ws = sas.make_workspace(cfg, DEV)
    gk = _pool(inp, cfg, ws)
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    pairs = [(s, h) for s in range(spec.batch) for h in range(spec.hkv)]
    T.check_pairs(inp, cfg, gpu, _oracle_on_stored_keys(inp, cfg, gk, pairs))


def test_bf16_keys_dtype_is_checked_by_the_binding():
    cfg = sas.Config(8, 2, gate_keys_bf16=1)
    with pytest.raises(ValueError):
        sas._check_gk(cfg, torch.zeros(1, 1, 1, 128, dtype=torch.float32))
