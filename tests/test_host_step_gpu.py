"""The decode step with host-memory query and output (sas_decode_step_host):
a chain of steps enqueued back to back -- each one a copy in, the fused step
and a copy out on one stream, with a fresh query every step and blocks
pooled as their tokens complete them -- gives outputs, block lists and gate
keys bit-identical to sas_decode_step run on the same queries already on the
device, and one of its steps matches the oracle.  Pinned and pageable host
buffers are both accepted."""
import dataclasses

import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import DecodeSpec, make_decode_inputs

from oracle import sas_oracle as O
import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"
STEPS = 40


def _setup(gate_mode):
    spec = DecodeSpec("host_chain", 2, 8, 2, [4000, 2020], (512,), capacity=4096, seed=61)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512, gate_mode=gate_mode)
    ws = sas.make_workspace(cfg, DEV)
    gk0 = T.run_pool(inp, cfg, ws)
    base = inp["seq_lens"].clone()       # 4,001 .. 4,040 and 2,021 .. 2,060: blocks 62 and 31 complete
    g = torch.Generator().manual_seed(62)
    q_host = [torch.randn(spec.batch, spec.hq, 128, generator=g).to(torch.bfloat16).pin_memory()
              for _ in range(STEPS)]
    kvs = [sas.KvCache(inp["k"], inp["v"], base + 1 + t) for t in range(STEPS)]
    return spec, inp, cfg, ws, gk0, q_host, kvs


def _lists(spec, cfg):
    return (torch.full((STEPS, spec.batch, spec.hkv, cfg.max_sel), -1, dtype=torch.int32, device=DEV),
            torch.full((STEPS, spec.batch, spec.hkv), -1, dtype=torch.int32, device=DEV))


@pytest.mark.parametrize("gate_mode", [sas.GATE_SELECT_ONLY, sas.GATE_LOGSIGMOID_BIAS])
def test_host_buffer_chain_matches_device_steps(gate_mode):
    spec, inp, cfg, ws, gk0, q_host, kvs = _setup(gate_mode)
    stream = torch.cuda.Stream()
    shape = (spec.batch, spec.hq, 128)

    # device entry, the queries copied up beforehand, one step at a time
    gk_want = gk0.clone()
    out_want = torch.empty((STEPS,) + shape, dtype=torch.bfloat16, device=DEV)
    sel_want, cnt_want = _lists(spec, cfg)
    q_all = torch.stack(q_host).to(DEV)
    for t in range(STEPS):
        sas.decode_step(cfg, q_all[t], kvs[t], inp["w_q"], inp["gamma_q"], gk_want, out_want[t], ws,
                        sel_idx=sel_want[t], sel_count=cnt_want[t], w_k=inp["w_k"], gamma_k=inp["gamma_k"],
                        stream=stream)
        torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    assert not torch.equal(gk_want, gk0)   # the chain pooled blocks

    # host entry, every step enqueued back to back through one staging pair
    gk = gk0.clone()
    q_dev = torch.empty(shape, dtype=torch.bfloat16, device=DEV)
    out_dev = torch.empty(shape, dtype=torch.bfloat16, device=DEV)
    out_host = [torch.full(shape, float("nan"), dtype=torch.bfloat16).pin_memory() for _ in range(STEPS)]
    sel, cnt = _lists(spec, cfg)
    torch.cuda.synchronize()
    for t in range(STEPS):
        sas.decode_step_host(cfg, q_host[t], q_dev, kvs[t], inp["w_q"], inp["gamma_q"], gk, out_dev, out_host[t],
                             ws, sel_idx=sel[t], sel_count=cnt[t], w_k=inp["w_k"], gamma_k=inp["gamma_k"],
                             stream=stream)
    stream.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    assert torch.equal(gk, gk_want)
    for t in range(STEPS):
        assert torch.equal(cnt[t], cnt_want[t]), t
        assert torch.equal(sel[t], sel_want[t]), t
        assert torch.equal(out_host[t], out_want[t].cpu()), t

    # the first step against the oracle
    first = dict(inp, q=q_all[0], seq_lens=kvs[0].seq_lens,
                 spec=dataclasses.replace(spec, seq_lens=[int(x) for x in kvs[0].seq_lens.cpu()]))
    gpu = {"out": out_host[0], "sel_idx": sel[0], "sel_count": cnt[0],
           "group_scores": _scores(cfg, first, gk0, ws, stream)}
    pairs = [(s, h) for s in range(spec.batch) for h in range(spec.hkv)]
    orc = T.oracle_pairs(first, 512, pairs,
                         gate_mode=O.GATE_LOGSIGMOID_BIAS if gate_mode else O.GATE_SELECT_ONLY)
    T.check_pairs(first, cfg, gpu, orc, gate_keys=gk0)


def _scores(cfg, inputs, gk, ws, stream):
    """Group scores of the step, from the device entry (the host entry's
    outputs equal that entry's bit for bit, checked above)."""
    r = T.run_decode_step(inputs, cfg, ws, gk.clone())
    torch.cuda.synchronize()
    return r["group_scores"]


def test_pageable_host_buffers_give_the_same_step():
    spec, inp, cfg, ws, gk0, q_host, kvs = _setup(sas.GATE_SELECT_ONLY)
    shape = (spec.batch, spec.hq, 128)
    q_dev = torch.empty(shape, dtype=torch.bfloat16, device=DEV)
    out_dev = torch.empty(shape, dtype=torch.bfloat16, device=DEV)
    pinned = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    pageable = torch.empty(shape, dtype=torch.bfloat16)
    for q, out in ((q_host[3], pinned), (q_host[3].clone(), pageable)):
        sas.decode_step_host(cfg, q, q_dev, kvs[3], inp["w_q"], inp["gamma_q"], gk0.clone(), out_dev, out, ws)
        torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    assert torch.equal(pinned, pageable)
    assert torch.isfinite(pinned.float()).all()


def _host_vs_device(spec, out_dtype, q_pinned=True, out_pinned=True):
    """One step through sas_decode_step_host against sas_decode_step on the
    same inputs: outputs and block lists bit-identical."""
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512, out_dtype=out_dtype)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    want = T.run_decode_step(inp, cfg, ws, gk.clone())
    torch.cuda.synchronize()
    q_host = inp["q"].cpu()
    out_host = torch.full(tuple(want["out"].shape), float("nan"), dtype=want["out"].dtype)
    if q_pinned:
        q_host = q_host.pin_memory()
    if out_pinned:
        out_host = out_host.pin_memory()
    q_dev = torch.empty_like(inp["q"])
    out_dev = torch.empty_like(want["out"])
    sel = torch.full_like(want["sel_idx"], -1)
    cnt = torch.full_like(want["sel_count"], -1)
    sas.decode_step_host(cfg, q_host, q_dev, T.kv_of(inp), inp["w_q"], inp["gamma_q"], gk.clone(), out_dev,
                         out_host, ws, sel_idx=sel, sel_count=cnt)
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK
    assert torch.equal(cnt, want["sel_count"]) and torch.equal(sel, want["sel_idx"])
    assert torch.equal(out_host, want["out"].cpu())


@pytest.mark.parametrize("name,kv_dtype,out_dtype,hq,hkv", [
    ("f32_in_f32_out_g4", "f32", "f32", 8, 2),     # four 16-byte words of q per head and CTA
    ("f32_in_bf16_out_g4", "f32", "bf16", 8, 2),
    ("bf16_g5", "bf16", "bf16", 10, 2),            # an odd group: ten words per CTA
])
def test_host_step_query_types_and_groups(name, kv_dtype, out_dtype, hq, hkv):
    spec = DecodeSpec("host_" + name, 2, hq, hkv, [3001, 1500], (512,), kv_dtype=kv_dtype, capacity=4096, seed=64)
    _host_vs_device(spec, out_dtype)


@pytest.mark.parametrize("q_pinned,out_pinned", [(True, False), (False, True)])
def test_host_step_mixed_pinned_and_pageable(q_pinned, out_pinned):
    spec = DecodeSpec("host_mixed", 2, 8, 2, [3001, 1500], (512,), capacity=4096, seed=65)
    _host_vs_device(spec, "bf16", q_pinned, out_pinned)
