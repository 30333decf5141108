"""Decode steps enqueued back to back, where each launch may start while the
one ahead of it drains (programmatic dependent launch), give bit-identical
results to the same steps run one at a time with a device synchronisation
in between -- with the weights declared static and without, eagerly and
replayed from a CUDA graph.  The chains pool blocks as their tokens
complete them, so a step reads the gate key the step before it wrote (one
layer), or runs between two steps of another layer (two layers
interleaved, as in a model)."""
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import DecodeSpec, make_decode_inputs

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"
STEPS = 100


def _layer(seed):
    # lengths 3,991 .. 4,090 and 2,001 .. 2,100 over the chain: blocks 62
    # and 31 complete inside it
    spec = DecodeSpec("chain", 2, 8, 2, [3990, 2000], (512,), capacity=4096, seed=seed)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    gk0 = T.run_pool(inp, cfg, ws)
    base = inp["seq_lens"].clone()
    B, hq, hkv = spec.batch, spec.hq, spec.hkv
    return dict(inp=inp, cfg=cfg, ws=ws, gk0=gk0, gk=torch.empty_like(gk0),
                kvs=[sas.KvCache(inp["k"], inp["v"], base + 1 + t) for t in range(STEPS)],
                out=torch.empty(STEPS, B, hq, 128, dtype=torch.bfloat16, device=DEV),
                sel=torch.empty(STEPS, B, hkv, cfg.max_sel, dtype=torch.int32, device=DEV),
                cnt=torch.empty(STEPS, B, hkv, dtype=torch.int32, device=DEV))


def _enqueue(layers, static_weights, sync_each, stream):
    for t in range(STEPS):
        for L in layers:
            inp, c0 = L["inp"], L["cfg"]
            cfg = sas.Config(c0.num_q_heads, c0.num_kv_heads, token_budget=c0.token_budget,
                             static_weights=static_weights)
            sas.decode_step(cfg, inp["q"], L["kvs"][t], inp["w_q"], inp["gamma_q"], L["gk"], L["out"][t],
                            L["ws"], sel_idx=L["sel"][t], sel_count=L["cnt"][t], w_k=inp["w_k"],
                            gamma_k=inp["gamma_k"], stream=stream)
            if sync_each:
                torch.cuda.synchronize()


def _reset(layers):
    for L in layers:
        L["gk"].copy_(L["gk0"])
        L["out"].fill_(float("nan"))
        L["sel"].fill_(-1)
        L["cnt"].fill_(-1)
    torch.cuda.synchronize()


def _snapshot(layers):
    torch.cuda.synchronize()
    for L in layers:
        assert sas.get_device_status(L["ws"]) == sas.SAS_OK
    return [{k: L[k].clone() for k in ("gk", "out", "sel", "cnt")} for L in layers]


def _check(got, want, layers):
    for R, W, L in zip(got, want, layers):
        assert not torch.equal(W["gk"], L["gk0"])  # the chain pooled blocks
        assert torch.equal(R["gk"], W["gk"])
        for t in range(STEPS):
            assert torch.equal(R["cnt"][t], W["cnt"][t]), t
            assert torch.equal(R["sel"][t], W["sel"][t]), t
            assert torch.equal(R["out"][t], W["out"][t]), t


@pytest.mark.parametrize("nlayers", [1, 2])
@pytest.mark.parametrize("static_weights", [0, 1])
def test_back_to_back_steps_match_synchronised_steps(nlayers, static_weights):
    layers = [_layer(40 + i) for i in range(nlayers)]
    stream = torch.cuda.Stream()
    _reset(layers)
    _enqueue(layers, 0, True, stream)
    want = _snapshot(layers)
    # eager, no synchronisation between the steps
    _reset(layers)
    _enqueue(layers, static_weights, False, stream)
    _check(_snapshot(layers), want, layers)
    # the same chain captured once and replayed
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        _enqueue(layers, static_weights, False, stream)
    _reset(layers)
    with torch.cuda.stream(stream):
        g.replay()
    _check(_snapshot(layers), want, layers)
