"""The allocation-free decode step against the ordinary one, through the C ABI.

Callers that cannot allocate device memory -- a serving loop that must not
allocate once warmed up, a plugin whose host framework owns the GPU memory, a
plain C caller with no allocator -- cannot pass sas_decode_step its workspace.
sas_decode_step_static keeps that scratch (the device status word) in a
device array inside the library instead.  These tests call it twice in a row
and compare every output with sas_decode_step on the same inputs, and check
that the shared status word is cleared between calls.

The file name makes pytest collect it last, so a failure here leaves every
other test already run; it also passes on its own in a fresh process (the
first call looks up the array's device address).
"""
import numpy as np
import pytest
import torch

from gated_block_sparse_token_b200 import sas
from gated_block_sparse_token_b200.workloads import DecodeSpec, make_decode_inputs

import sas_testlib as T

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(spec, cfg, mg):
    B = spec.batch
    return (torch.full((B, spec.hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV),
            torch.full((B, spec.hkv, cfg.max_sel), -1, dtype=torch.int32, device=DEV),
            torch.full((B, spec.hkv), -1, dtype=torch.int32, device=DEV),
            torch.full((B, spec.hkv, mg), float("nan"), dtype=torch.float32, device=DEV))


def test_static_step_matches_workspace_step_on_two_calls():
    spec = DecodeSpec("no_alloc", 3, 8, 2, [4096, 2500, 1024], (512,), capacity=4096,
                      block_offset_std=0.5, seed=31)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    gk0 = T.run_pool(inp, cfg, ws)
    for s, L in enumerate(spec.seq_lens):      # the step itself pools the completed blocks
        gk0[s, :, (L - 1) // 64] = 0.0
    mg = gk0.shape[2]
    kv = T.kv_of(inp)

    gk_ref = gk0.clone()
    out_ref, sel_ref, cnt_ref, gs_ref = _outputs(spec, cfg, mg)
    sas.decode_step(cfg, inp["q"], kv, inp["w_q"], inp["gamma_q"], gk_ref, out_ref, ws,
                    sel_idx=sel_ref, sel_count=cnt_ref, group_scores=gs_ref,
                    w_k=inp["w_k"], gamma_k=inp["gamma_k"])
    torch.cuda.synchronize()
    assert sas.get_device_status(ws) == sas.SAS_OK

    for call in range(2):
        gk = gk0.clone()
        out, sel, cnt, gs = _outputs(spec, cfg, mg)
        status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        sas.decode_step_static(cfg, inp["q"], kv, inp["w_q"], inp["gamma_q"], gk, out,
                               sel_idx=sel, sel_count=cnt, group_scores=gs,
                               w_k=inp["w_k"], gamma_k=inp["gamma_k"], status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: status bits {int(status.item())}"
        err = float((out.float() - out_ref.float()).abs().max())
        assert np.isfinite(err) and err <= T.OUT_ATOL, f"call {call}: out differs by {err}"
        assert torch.equal(cnt, cnt_ref) and torch.equal(sel, sel_ref), f"call {call}: block lists"
        for s, L in enumerate(spec.seq_lens):
            c = (L - 1) // 64
            T.assert_close_rel(gs[s, :, :c].cpu().numpy(), gs_ref[s, :, :c].cpu().numpy(),
                               f"call {call} group scores s={s}")
        T.assert_close_rel(gk.cpu().numpy(), gk_ref.cpu().numpy(), f"call {call} gate keys")


def test_static_step_clears_the_shared_status_word():
    """A call that trips a device range check reports it; the next clean call
    starts from a cleared status word and reports 0."""
    spec = DecodeSpec("no_alloc_status", 2, 8, 2, [1000, 2000], (512,), capacity=2048, seed=32)
    inp = make_decode_inputs(spec, DEV)
    cfg = T.config_for(spec, 512)
    ws = sas.make_workspace(cfg, DEV)
    gk = T.run_pool(inp, cfg, ws)
    kv = T.kv_of(inp)
    out, sel, cnt, gs = _outputs(spec, cfg, gk.shape[2])
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    inp["seq_lens"][1] = 5000  # longer than the 2,048-token cache: caught before any access
    sas.decode_step_static(cfg, inp["q"], kv, inp["w_q"], inp["gamma_q"], gk, out,
                           sel_idx=sel, sel_count=cnt, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 1 == 1
    inp["seq_lens"][1] = 2000
    sas.decode_step_static(cfg, inp["q"], kv, inp["w_q"], inp["gamma_q"], gk, out,
                           sel_idx=sel, sel_count=cnt, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
