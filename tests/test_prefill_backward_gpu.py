"""GPU parity of the gradient through the gates of the gated prefill
(sas_prefill_gate_backward) against the oracle's fp64 gradient (reading R20
for the chunked prefill: every query block has its own block-mean gate
query, block list and gates; the lists are held fixed and a gate key's
gradient sums over the query blocks that kept it).  Source: "Tencent
released Simple-Attention-Sparsification ..." (aigc.news, 2026-09-14),
release paragraph.

Tolerance: every gradient tensor within 1e-3 of its largest magnitude
(max-abs error / max |oracle|): the kernels accumulate in fp32 (dot products
of 128 on the tensor cores with dL/dout as two bf16 terms, exact to about
2^-16; softmax statistics over up to 4,096 tokens; 384-term projections;
fixed-order sums over tokens, query blocks and sequences), whose rounding
stays far below that."""
import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import PrefillSpec, make_prefill_inputs
from oracle import sas_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRAD_RTOL = 1e-3


def _forward(spec, gate_mode=sas.GATE_LOGSIGMOID_BIAS):
    inp = make_prefill_inputs(spec, DEV)
    B, Tn = spec.batch, spec.seq_len
    nblk = Tn // 64
    cfg = sas.Config(spec.hq, spec.hkv, token_budget=spec.token_budget, gate_mode=gate_mode)
    ws = sas.make_workspace(cfg, DEV, batch=B, max_seq_len=Tn)
    gk = torch.zeros(B, spec.hkv, nblk, 128, dtype=torch.float32, device=DEV)
    out = torch.empty(B, spec.hq, Tn, 128, dtype=torch.bfloat16, device=DEV)
    sel = torch.full((B, spec.hkv, nblk, cfg.max_sel), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, spec.hkv, nblk), -1, dtype=torch.int32, device=DEV)
    sas.prefill_block_sparse(cfg, inp["q"], inp["k"], inp["v"], inp["w_q"], inp["gamma_q"], inp["w_k"],
                             inp["gamma_k"], gk, out, ws, sel_idx=sel, sel_count=cnt)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    return inp, cfg, ws, gk, sel, cnt


def _backward(spec, inp, cfg, ws, gk, sel, cnt, d_out):
    dw_q = torch.zeros(spec.hq, 128, 128, device=DEV)
    dw_k = torch.zeros(spec.hkv, 384, 128, device=DEV)
    dgq = torch.zeros(128, device=DEV)
    dgk = torch.zeros(128, device=DEV)
    sas.prefill_gate_backward(cfg, inp["q"], inp["k"], inp["v"], inp["w_q"], inp["gamma_q"], inp["w_k"],
                              inp["gamma_k"], gk, sel, cnt, d_out, dw_q, dw_k, dgq, dgk, ws)
    torch.cuda.synchronize()
    return dw_q, dw_k, dgq, dgk


def _oracle(spec, inp, sel, cnt, d_out):
    G = spec.hq // spec.hkv
    nblk = spec.seq_len // 64
    wq = inp["w_q"].double().cpu().numpy()
    wk = inp["w_k"].double().cpu().numpy()
    gq = inp["gamma_q"].double().cpu().numpy()
    gkn = inp["gamma_k"].double().cpu().numpy()
    sel_h, cnt_h = sel.cpu().numpy(), cnt.cpu().numpy()
    dw_q = np.zeros((spec.hq, 128, 128))
    dw_k = np.zeros((spec.hkv, 384, 128))
    dgq, dgk = np.zeros(128), np.zeros(128)
    for s in range(spec.batch):
        for h in range(spec.hkv):
            heads = slice(h * G, (h + 1) * G)
            sels = [[int(b) for b in sel_h[s, h, i, :int(cnt_h[s, h, i])]] for i in range(nblk)]
            r = O.prefill_gate_grads(inp["q"][s, heads].double().cpu().numpy(),
                                     inp["k"][s, h].double().cpu().numpy(), inp["v"][s, h].double().cpu().numpy(),
                                     wq[heads], gq, wk[h], gkn, sels, d_out[s, heads].double().cpu().numpy())
            dw_q[heads] += r["dw_q"]
            dw_k[h] += r["dw_k"]
            dgq += r["dgamma_q"]
            dgk += r["dgamma_k"]
    return dw_q, dw_k, dgq, dgk


def _compare(got, want, what):
    got = got.double().cpu().numpy()
    scale = float(np.max(np.abs(want)))
    assert scale > 0, f"{what}: the oracle gradient is zero"
    err = float(np.max(np.abs(got - want)))
    assert np.all(np.isfinite(got)) and err <= GRAD_RTOL * scale, f"{what}: max-abs err {err:.3g} vs scale {scale:.3g}"


SMALL = [
    # name, B, hq, hkv, T, budget
    ("g4", 1, 4, 1, 640, 192),
    ("g2_two_seqs", 2, 4, 2, 512, 256),
    ("g5_qwen14b_grouping", 1, 10, 2, 768, 320),
    ("g8_budget_covers_context", 1, 8, 1, 512, 1024),
    ("g4_budget_4096", 1, 4, 1, 64 * 70, 4096),
]


@pytest.mark.parametrize("name,B,hq,hkv,T,budget", SMALL, ids=[s[0] for s in SMALL])
def test_prefill_gate_backward_small(name, B, hq, hkv, T, budget):
    spec = PrefillSpec("pfbwd_" + name, B, hq, hkv, T, token_budget=budget, seed=81)
    inp, cfg, ws, gk, sel, cnt = _forward(spec)
    d_out = torch.randn(B, hq, T, 128, generator=torch.Generator(device=DEV).manual_seed(9), device=DEV)
    got = _backward(spec, inp, cfg, ws, gk, sel, cnt, d_out)
    assert sas.get_device_status(ws) == sas.SAS_OK
    want = _oracle(spec, inp, sel, cnt, d_out)
    for g, w, what in zip(got, want, ("dW_q", "dW_k", "dgamma_q", "dgamma_k")):
        _compare(g, w, f"{name} {what}")


def test_prefill_gate_backward_is_reproducible_bit_for_bit():
    spec = PrefillSpec("pfbwd_repro", 2, 8, 2, 1024, token_budget=512, seed=82)
    inp, cfg, ws, gk, sel, cnt = _forward(spec)
    d_out = torch.randn(2, 8, 1024, 128, generator=torch.Generator(device=DEV).manual_seed(10), device=DEV)
    a = _backward(spec, inp, cfg, ws, gk, sel, cnt, d_out)
    b = _backward(spec, inp, cfg, ws, gk, sel, cnt, d_out)
    assert sas.get_device_status(ws) == sas.SAS_OK
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_prefill_gate_backward_select_only_adds_nothing():
    spec = PrefillSpec("pfbwd_select_only", 1, 4, 1, 512, token_budget=192, seed=83)
    inp, cfg, ws, gk, sel, cnt = _forward(spec, gate_mode=sas.GATE_SELECT_ONLY)
    d_out = torch.ones(1, 4, 512, 128, device=DEV)
    for t in _backward(spec, inp, cfg, ws, gk, sel, cnt, d_out):
        assert torch.count_nonzero(t) == 0


def test_prefill_gate_backward_bad_list_is_reported_and_skipped():
    spec = PrefillSpec("pfbwd_bad", 1, 4, 1, 512, token_budget=192, seed=84)
    inp, cfg, ws, gk, sel, cnt = _forward(spec)
    sel[0, 0, 5, 0] = 7          # a block after query block 5
    d_out = torch.randn(1, 4, 512, 128, generator=torch.Generator(device=DEV).manual_seed(11), device=DEV)
    _backward(spec, inp, cfg, ws, gk, sel, cnt, d_out)
    assert sas.get_device_status(ws) == sas.SAS_ERR_DEVICE_BOUNDS
