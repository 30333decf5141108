"""Mixed token budgets in one batch (pages: 1,024-, 2,048- or 4,096-token
budgets usable without retraining): per-sequence budgets through sas_kv and
sas_topk_blocks, against the CPU oracle at each sequence's own budget."""
import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import DecodeSpec, make_decode_inputs
from oracle import sas_oracle as O

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _kv(inp, budgets):
    return sas.KvCache(inp["k"], inp["v"], inp["seq_lens"], inp["block_table"],
                       token_budgets=torch.tensor(budgets, dtype=torch.int32, device=DEV))


def _step(inp, cfg, ws, gk, kv):
    spec = inp["spec"]
    B = spec.batch
    out = torch.full((B, spec.hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    sel = torch.full((B, spec.hkv, cfg.max_sel), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, spec.hkv), -1, dtype=torch.int32, device=DEV)
    gs = torch.full((B, spec.hkv, gk.shape[2]), float("nan"), device=DEV)
    sas.decode_step(cfg, inp["q"], kv, inp["w_q"], inp["gamma_q"], gk, out, ws, sel_idx=sel,
                    sel_count=cnt, group_scores=gs)
    return {"out": out, "sel_idx": sel, "sel_count": cnt, "group_scores": gs}


@pytest.mark.parametrize("gate_mode", [sas.GATE_SELECT_ONLY, sas.GATE_LOGSIGMOID_BIAS])
def test_mixed_budgets_decode_step(gate_mode):
    budgets = [64, 1024, 2048, 4096, 1536]
    spec = DecodeSpec("mixed_budgets", 5, 8, 2, [8192, 8192, 8000, 8192, 5000], (4096,),
                      block_offset_std=0.5, seed=41)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 4096, gate_mode=gate_mode)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    gpu = _step(inp, cfg, ws, gk, _kv(inp, budgets))
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    orc = {}
    for s in range(spec.batch):
        orc.update(T.oracle_pairs(inp, budgets[s], [(s, h) for h in range(spec.hkv)],
                                  gate_mode=gate_mode))
    T.check_pairs(inp, cfg, gpu, orc, gate_keys=gk, budgets=budgets)
    cnt = gpu["sel_count"].cpu().numpy()
    for s, L in enumerate(spec.seq_lens):
        assert (cnt[s] == min(budgets[s] // 64, (L - 1) // 64 + 1)).all()


def test_mixed_budgets_topk_blocks():
    g = torch.Generator().manual_seed(43)
    B, hkv, mg = 4, 2, 256
    lens = torch.tensor([64 * 200 + 7, 64 * 255 + 1, 3000, 640], dtype=torch.int32)
    budgets = [4096, 64, 2048, 1024]
    scores = torch.randn(B, hkv, mg, generator=g)
    cfg = sas.Config(8, hkv, token_budget=4096)
    ws = sas.make_workspace(cfg, DEV)
    sel = torch.full((B, hkv, 64), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, hkv), -1, dtype=torch.int32, device=DEV)
    sas.topk_blocks(cfg, scores.to(DEV), lens.to(DEV), sel, cnt, ws,
                    token_budgets=torch.tensor(budgets, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for s in range(B):
        c = (int(lens[s]) - 1) // 64
        for h in range(hkv):
            want = O.select_blocks(scores[s, h, :c].double().numpy(), c, budgets[s] // 64 - 1)
            assert int(cnt[s, h]) == len(want)
            assert list(sel[s, h, :len(want)]) == want, (s, h)


def test_bad_budget_is_reported_and_skipped():
    """A budget that is not a multiple of 64, or above the configured one,
    skips that sequence (zero output) and sets the bounds bit."""
    spec = DecodeSpec("bad_budget", 3, 8, 2, [4096, 4096, 4096], (2048,), seed=47)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 2048)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    gpu = _step(inp, cfg, ws, gk, _kv(inp, [2048, 100, 4096]))
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_ERR_DEVICE_BOUNDS
    out = gpu["out"].float()
    assert torch.isfinite(out[0]).all() and out[0].abs().max() > 0
    assert torch.all(out[1] == 0) and torch.all(out[2] == 0)
    assert torch.all(gpu["sel_count"][1:] == 0)
