"""GPU parity of the gradient through the gates (sas_gate_backward) against the
oracle's fp64 gradient (reading R20: in the gated mode the continuous gates on
the selected blocks give W_q, W_k, gamma_q and gamma_k a gradient; the block
lists are held fixed).  Source: "Tencent released
Simple-Attention-Sparsification ..." (aigc.news, 2026-09-14), release
paragraph.

Tolerance: every gradient tensor within 1e-3 of its largest magnitude (max-abs
error / max |oracle|): the kernels accumulate in fp32 (dot products of 128 --
dL/dout entering the tensor cores as two bf16 terms, exact to about 2^-16 --,
softmax sums over up to 4,096 tokens, 384-term projections, fixed-order sums
over sequences and entries), whose rounding stays orders of magnitude below
that."""
import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import DecodeSpec, make_decode_inputs, qwen3_4b_32k, logical_kv
from oracle import sas_oracle as O

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRAD_RTOL = 1e-3


def _forward(inp, budget, gate_mode=sas.GATE_LOGSIGMOID_BIAS):
    spec = inp["spec"]
    cfg = T.config_for(spec, budget, gate_mode=gate_mode)
    ws = sas.make_workspace(cfg, DEV, batch=spec.batch)  # the backward's per-pair terms
    gk = T.run_pool(inp, cfg, ws)
    gpu = T.run_decode_step(inp, cfg, ws, gk)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    return cfg, ws, gk, gpu


def _backward(inp, cfg, ws, gpu, d_out):
    spec = inp["spec"]
    dw_q = torch.zeros(spec.hq, 128, 128, device=DEV)
    dw_k = torch.zeros(spec.hkv, 384, 128, device=DEV)
    dgq = torch.zeros(128, device=DEV)
    dgk = torch.zeros(128, device=DEV)
    sas.gate_backward(cfg, inp["q"], T.kv_of(inp), inp["w_q"], inp["gamma_q"], inp["w_k"], inp["gamma_k"],
                      gpu["sel_idx"], gpu["sel_count"], d_out, dw_q, dw_k, dgq, dgk, ws)
    torch.cuda.synchronize()
    return dw_q, dw_k, dgq, dgk


def _oracle(inp, budget, gpu, d_out):
    spec = inp["spec"]
    G = spec.hq // spec.hkv
    q = inp["q"].double().cpu().numpy()
    wq = inp["w_q"].double().cpu().numpy()
    wk = inp["w_k"].double().cpu().numpy()
    gq = inp["gamma_q"].double().cpu().numpy()
    gkn = inp["gamma_k"].double().cpu().numpy()
    dout = d_out.double().cpu().numpy()
    sel_idx, sel_count = gpu["sel_idx"].cpu().numpy(), gpu["sel_count"].cpu().numpy()
    dw_q = np.zeros((spec.hq, 128, 128))
    dw_k = np.zeros((spec.hkv, 384, 128))
    dgq, dgk = np.zeros(128), np.zeros(128)
    for s in range(spec.batch):
        L = int(spec.seq_lens[s])
        for h in range(spec.hkv):
            ks, vs = logical_kv(inp, s, h, L)
            heads = slice(h * G, (h + 1) * G)
            gpu_sel = [int(b) for b in sel_idx[s, h, :int(sel_count[s, h])]]
            # the gate's own list first (forward parity), then the gradient over
            # the list the step used, held fixed
            own = O.decode_gate_grads(q[s, heads], ks, vs, L, wq[heads], gq, wk[h], gkn, budget, dout[s, heads])
            if own["sel"] != gpu_sel:
                T.assert_selection(gpu_sel, own["sel"], own["s"].mean(axis=0), budget // 64 - 1,
                                   f"backward s={s} h={h}")
                own = O.decode_gate_grads(q[s, heads], ks, vs, L, wq[heads], gq, wk[h], gkn, budget,
                                          dout[s, heads], sel=gpu_sel)
            dw_q[heads] += own["dw_q"]
            dw_k[h] += own["dw_k"]
            dgq += own["dgamma_q"]
            dgk += own["dgamma_k"]
    return dw_q, dw_k, dgq, dgk


def _compare(got, want, what):
    got = got.double().cpu().numpy()
    scale = float(np.max(np.abs(want)))
    assert scale > 0, f"{what}: the oracle gradient is zero"
    err = float(np.max(np.abs(got - want)))
    assert np.all(np.isfinite(got)) and err <= GRAD_RTOL * scale, f"{what}: max-abs err {err:.3g} vs scale {scale:.3g}"


SMALL = [
    ("g4_ragged", 3, 8, 2, [4096, 2500, 1000], 512),
    ("g5_qwen14b_heads", 2, 10, 2, [3000, 4097], 1024),
    ("budget_covers_context", 2, 8, 2, [700, 640], 2048),
    ("budget_4096", 1, 8, 1, [9000], 4096),
]


@pytest.mark.parametrize("name,B,hq,hkv,lens,budget", SMALL, ids=[s[0] for s in SMALL])
def test_gate_backward_small(name, B, hq, hkv, lens, budget):
    spec = DecodeSpec("bwd_" + name, B, hq, hkv, lens, (budget,), block_offset_std=0.5, seed=71)
    inp = make_decode_inputs(spec, DEV)
    cfg, ws, gk, gpu = _forward(inp, budget)
    d_out = torch.randn(B, hq, 128, generator=torch.Generator(device=DEV).manual_seed(5), device=DEV)
    got = _backward(inp, cfg, ws, gpu, d_out)
    assert sas.get_device_status(ws) == sas.SAS_OK
    want = _oracle(inp, budget, gpu, d_out)
    for g, w, what in zip(got, want, ("dW_q", "dW_k", "dgamma_q", "dgamma_k")):
        _compare(g, w, f"{name} {what}")


def test_gate_backward_qwen3_4b_32k_full_size():
    """Every (sequence, KV head) pair of the Qwen3-4B 32k workload (batch 8,
    budget 2,048), gated mode."""
    spec = qwen3_4b_32k()
    inp = make_decode_inputs(spec, DEV)
    cfg, ws, gk, gpu = _forward(inp, 2048)
    d_out = torch.randn(spec.batch, spec.hq, 128, generator=torch.Generator(device=DEV).manual_seed(6), device=DEV)
    got = _backward(inp, cfg, ws, gpu, d_out)
    assert sas.get_device_status(ws) == sas.SAS_OK
    want = _oracle(inp, 2048, gpu, d_out)
    for g, w, what in zip(got, want, ("dW_q", "dW_k", "dgamma_q", "dgamma_k")):
        _compare(g, w, f"qwen3_4b_32k {what}")


def test_gate_backward_select_only_adds_nothing():
    spec = DecodeSpec("bwd_select_only", 2, 8, 2, [3000, 1000], (512,), seed=72)
    inp = make_decode_inputs(spec, DEV)
    cfg, ws, gk, gpu = _forward(inp, 512, gate_mode=sas.GATE_SELECT_ONLY)
    d_out = torch.ones(2, 8, 128, device=DEV)
    for t in _backward(inp, cfg, ws, gpu, d_out):
        assert torch.count_nonzero(t) == 0


def test_gate_backward_bad_list_is_reported_and_skipped():
    spec = DecodeSpec("bwd_bad", 2, 8, 2, [3000, 1000], (512,), seed=73)
    inp = make_decode_inputs(spec, DEV)
    cfg, ws, gk, gpu = _forward(inp, 512)
    gpu["sel_idx"][1, 0, 0] = 10 ** 6        # a block past the current one
    d_out = torch.randn(2, 8, 128, generator=torch.Generator(device=DEV).manual_seed(7), device=DEV)
    _backward(inp, cfg, ws, gpu, d_out)
    assert sas.get_device_status(ws) == sas.SAS_ERR_DEVICE_BOUNDS


def test_gate_backward_is_reproducible_bit_for_bit():
    """The sums over sequences and entries run in a fixed order: two calls on
    the same inputs add exactly the same values."""
    spec = DecodeSpec("bwd_repro", 4, 16, 4, [3000, 1000, 2500, 4096], (1024,), block_offset_std=0.5, seed=74)
    inp = make_decode_inputs(spec, DEV)
    cfg, ws, gk, gpu = _forward(inp, 1024)
    d_out = torch.randn(4, 16, 128, generator=torch.Generator(device=DEV).manual_seed(8), device=DEV)
    a = _backward(inp, cfg, ws, gpu, d_out)
    b = _backward(inp, cfg, ws, gpu, d_out)
    assert sas.get_device_status(ws) == sas.SAS_OK
    for x, y in zip(a, b):
        assert torch.equal(x, y)
