"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, the ctypes mirrors match the C struct layouts (checked
against a gcc build of the header), and host-side validation rejects bad
arguments before touching CUDA."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

from gated_block_sparse_token_b200 import build as B
from gated_block_sparse_token_b200 import sas

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sas.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return sas.lib()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"^SAS_API\s+[\w\s\*]+?\b(sas_\w+)\(", src, flags=re.M)


def test_header_declares_all_entry_points():
    names = set(declared_functions())
    want = {"sas_pool_keys", "sas_gate_scores", "sas_topk_blocks", "sas_sparse_decode",
            "sas_decode_step", "sas_workspace_bytes", "sas_get_device_status",
            "sas_reset_device_status", "sas_status_string", "sas_abi_version", "sas_gate_backward",
            "sas_prefill_gate_backward", "sas_decode_step_host"}
    assert want <= names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", sas.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (sas_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)


def test_library_needs_no_driver_at_load():
    out = subprocess.run(["ldd", sas.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libtorch" not in out


def test_struct_layout_matches_header():
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "sas.h"
#define O(T, f) printf("%s.%s %zu\n", #T, #f, offsetof(T, f))
int main(void) {
  printf("sizeof.sas_config %zu\nsizeof.sas_kv %zu\n", sizeof(sas_config), sizeof(sas_kv));
  O(sas_config, token_budget); O(sas_config, rope_base); O(sas_config, gate_scale);
  O(sas_config, kv_dtype); O(sas_config, out_dtype); O(sas_config, gate_mode); O(sas_config, gate_keys_bf16);
  O(sas_config, static_weights);
  O(sas_kv, block_table); O(sas_kv, seq_lens); O(sas_kv, batch); O(sas_kv, capacity);
  O(sas_kv, num_pages); O(sas_kv, max_blocks_per_seq); O(sas_kv, token_budgets);
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(l.split() for l in lines if l.strip())
    assert int(got["sizeof.sas_config"]) == ctypes.sizeof(sas._Config)
    assert int(got["sizeof.sas_kv"]) == ctypes.sizeof(sas._Kv)
    for key, val in got.items():
        if key.startswith("sizeof"):
            continue
        struct, fieldname = key.split(".")
        cls = sas._Config if struct == "sas_config" else sas._Kv
        assert getattr(cls, fieldname).offset == int(val), key


def test_abi_version_and_status_strings(L):
    assert sas.abi_version() == sas.ABI_VERSION == 10
    for st in range(7):
        assert len(sas.status_string(st)) > 0
    assert sas.status_string(sas.SAS_OK) == "ok"


# Host validation.  Every call below must fail in the host checks, which come
# before any CUDA call; pointers are dummies that are never dereferenced.
# Skipped where a GPU is present so that a validation bug can never launch a
# kernel on dummy pointers.
nogpu = pytest.mark.skipif(torch.cuda.is_available(), reason="host validation runs on CPU-only hosts")
FAKE = 0x100000  # 16-byte aligned dummy address


def _cfg(**kw):
    base = dict(num_q_heads=32, num_kv_heads=8, token_budget=2048)
    base.update(kw)
    return sas.Config(**base)


def _kv(batch=2, cap=4096, **kw):
    k = sas._Kv(FAKE, FAKE, None, FAKE, batch, cap, 0, 0)
    for key, val in kw.items():
        setattr(k, key, val)
    return k


def _decode(L, cfg, kv=None, ws_bytes=256, ws=FAKE, q=FAKE, out=FAKE, mg=64):
    c = cfg.c()
    kv = kv or _kv()
    return L.sas_decode_step(ctypes.byref(c), q, ctypes.byref(kv), FAKE, FAKE, None, None, FAKE, mg,
                             out, None, None, None, ws, ws_bytes, None)


@nogpu
@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), sas.SAS_ERR_UNSUPPORTED),
    (dict(block_size=32), sas.SAS_ERR_INVALID_ARG),
    (dict(gate_hidden=64), sas.SAS_ERR_INVALID_ARG),
    (dict(token_budget=100), sas.SAS_ERR_INVALID_ARG),
    (dict(token_budget=0), sas.SAS_ERR_INVALID_ARG),
    (dict(token_budget=32768), sas.SAS_ERR_UNSUPPORTED),
    (dict(num_q_heads=30), sas.SAS_ERR_INVALID_ARG),
    (dict(num_q_heads=72, num_kv_heads=8), sas.SAS_ERR_UNSUPPORTED),
    (dict(attn_scale=0.0), sas.SAS_ERR_INVALID_ARG),
    (dict(gate_scale=float("nan")), sas.SAS_ERR_INVALID_ARG),
    (dict(norm_eps=-1.0), sas.SAS_ERR_INVALID_ARG),
    (dict(rope_base=-5.0), sas.SAS_ERR_INVALID_ARG),
    (dict(gate_mode=2), sas.SAS_ERR_INVALID_ARG),
    (dict(gate_mode=-1), sas.SAS_ERR_INVALID_ARG),
    (dict(gate_keys_bf16=2), sas.SAS_ERR_INVALID_ARG),
    (dict(static_weights=2), sas.SAS_ERR_INVALID_ARG),
])
def test_config_validation(L, kw, status):
    assert _decode(L, _cfg(**kw)) == status


@nogpu
def test_workspace_and_pointer_validation(L):
    cfg = _cfg()
    assert _decode(L, cfg, ws_bytes=8) == sas.SAS_ERR_WORKSPACE
    assert _decode(L, cfg, ws=0) == sas.SAS_ERR_WORKSPACE
    assert _decode(L, cfg, ws=FAKE + 4) == sas.SAS_ERR_WORKSPACE
    assert _decode(L, cfg, kv=_kv(cap=1000)) == sas.SAS_ERR_INVALID_ARG
    assert _decode(L, cfg, kv=_kv(k=FAKE + 2)) == sas.SAS_ERR_INVALID_ARG
    assert _decode(L, cfg, kv=_kv(seq_lens=None)) == sas.SAS_ERR_INVALID_ARG
    assert _decode(L, cfg, kv=_kv(batch=-1)) == sas.SAS_ERR_INVALID_ARG
    # a paged cache needs pages and a block-table width
    assert _decode(L, cfg, kv=_kv(block_table=FAKE, num_pages=0, max_blocks_per_seq=4)) == sas.SAS_ERR_INVALID_ARG
    # TMA row coordinates are 32-bit
    assert _decode(L, cfg, kv=_kv(batch=4096, cap=1 << 20)) == sas.SAS_ERR_UNSUPPORTED
    assert _decode(L, cfg, q=0) == sas.SAS_ERR_INVALID_ARG
    assert _decode(L, cfg, q=FAKE + 4) == sas.SAS_ERR_INVALID_ARG   # q is bulk-copied: 16 bytes
    assert _decode(L, cfg, mg=0) == sas.SAS_ERR_INVALID_ARG
    c = cfg.c()
    kv = _kv()
    # fused pooling needs both W_k and gamma_k
    assert L.sas_decode_step(ctypes.byref(c), FAKE, ctypes.byref(kv), FAKE, FAKE, FAKE, None, FAKE, 64,
                             FAKE, None, None, None, FAKE, 256, None) == sas.SAS_ERR_INVALID_ARG


@nogpu
def test_empty_batch_is_a_no_op(L):
    assert _decode(L, _cfg(), kv=_kv(batch=0)) == sas.SAS_OK


def _decode_host(L, cfg, kv=None, q_host=FAKE, q_dev=FAKE, out_dev=FAKE, out_host=FAKE, ws_bytes=256):
    c = cfg.c()
    kv = kv or _kv()
    return L.sas_decode_step_host(ctypes.byref(c), q_host, q_dev, ctypes.byref(kv), FAKE, FAKE, None, None,
                                  FAKE, 64, out_dev, out_host, None, None, None, FAKE, ws_bytes, None)


@nogpu
def test_host_buffer_step_validates_before_any_copy(L):
    """sas_decode_step_host checks every argument, the host buffers included,
    before it enqueues its first copy; an empty batch enqueues nothing."""
    cfg = _cfg()
    assert _decode_host(L, cfg, q_host=None) == sas.SAS_ERR_INVALID_ARG
    assert _decode_host(L, cfg, out_host=None) == sas.SAS_ERR_INVALID_ARG
    assert _decode_host(L, cfg, q_dev=None) == sas.SAS_ERR_INVALID_ARG
    assert _decode_host(L, cfg, q_dev=FAKE + 4) == sas.SAS_ERR_INVALID_ARG    # bulk-copied: 16 bytes
    assert _decode_host(L, cfg, out_dev=None) == sas.SAS_ERR_INVALID_ARG
    assert _decode_host(L, cfg, ws_bytes=8) == sas.SAS_ERR_WORKSPACE
    assert _decode_host(L, _cfg(gate_mode=3)) == sas.SAS_ERR_INVALID_ARG
    assert _decode_host(L, cfg, kv=_kv(batch=0), q_host=None, out_host=None) == sas.SAS_OK


def test_host_step_binding_refuses_mismatched_host_buffers(monkeypatch):
    """The library sizes the host transfers from the config: the binding
    refuses a host tensor whose shape, dtype or placement disagrees with its
    staging buffer before any library call."""
    def no_library():
        raise AssertionError("the library was called before the buffer check")

    monkeypatch.setattr(sas, "lib", no_library)
    cfg = sas.Config(8, 2)
    kv = sas.KvCache(torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16),
                     torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16), torch.ones(1, dtype=torch.int32))
    gk = torch.zeros(1, 2, 4, 128)
    ws = torch.zeros(256, dtype=torch.uint8)
    dev = torch.zeros(1, 8, 128, dtype=torch.bfloat16)   # stands for a device buffer
    good = torch.zeros(1, 8, 128, dtype=torch.bfloat16)
    for q_host, out_host in ((torch.zeros(1, 4, 128, dtype=torch.bfloat16), good),
                             (good, torch.zeros(1, 8, 128, dtype=torch.float32)),
                             (torch.zeros(1, 8, 256, dtype=torch.bfloat16)[..., :128], good)):
        with pytest.raises(ValueError):
            sas.decode_step_host(cfg, q_host, dev, kv, None, None, gk, dev, out_host, ws)


@nogpu
def test_other_entry_points_validate(L):
    c = _cfg(token_budget=96).c()
    kv = _kv()
    assert L.sas_pool_keys(ctypes.byref(c), ctypes.byref(kv), None, 4, FAKE, FAKE, FAKE, 64, None,
                           FAKE, 256, None) == sas.SAS_ERR_INVALID_ARG
    c = _cfg().c()
    assert L.sas_pool_keys(ctypes.byref(c), ctypes.byref(kv), None, -1, FAKE, FAKE, FAKE, 64, None,
                           FAKE, 256, None) == sas.SAS_ERR_INVALID_ARG
    assert L.sas_gate_scores(ctypes.byref(c), FAKE, FAKE, 2, FAKE, FAKE, FAKE, 64, None, None,
                             FAKE, 256, None) == sas.SAS_ERR_INVALID_ARG
    assert L.sas_topk_blocks(ctypes.byref(c), FAKE, FAKE, None, 2, 64, FAKE, None, FAKE, 256,
                             None) == sas.SAS_ERR_INVALID_ARG
    assert L.sas_topk_blocks(ctypes.byref(c), FAKE, FAKE, FAKE + 2, 2, 64, FAKE, FAKE, FAKE, 256,
                             None) == sas.SAS_ERR_INVALID_ARG  # misaligned budgets
    assert L.sas_sparse_decode(ctypes.byref(c), FAKE, ctypes.byref(kv), None, FAKE, FAKE, FAKE,
                               256, None) == sas.SAS_ERR_INVALID_ARG
    st = ctypes.c_int(0)
    assert L.sas_get_device_status(None, None, ctypes.byref(st)) == sas.SAS_ERR_INVALID_ARG
    assert L.sas_reset_device_status(None, None) == sas.SAS_ERR_WORKSPACE


@nogpu
def test_gated_mode_not_in_sparse_decode(L):
    """The gated mode needs the gate query and keys: sas_sparse_decode, which
    has neither, refuses it on the host, before any CUDA call."""
    c = _cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS).c()
    kv = _kv()
    assert L.sas_sparse_decode(ctypes.byref(c), FAKE, ctypes.byref(kv), FAKE, FAKE, FAKE, FAKE,
                               256, None) == sas.SAS_ERR_UNSUPPORTED


def test_gated_mode_needs_no_more_workspace(L):
    # the gates live in shared memory (decode and prefill alike)
    for b, t in ((8, 32768), (2, 4096)):
        assert sas.workspace_bytes(_cfg(), b, t) == sas.workspace_bytes(_cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS), b, t)


def _prefill(L, c, budgets=None, batch=2, seq_len=4096, mg=64, ws=FAKE, ws_bytes=1 << 30, sel_count=None):
    return L.sas_prefill_block_sparse(ctypes.byref(c), FAKE, FAKE, FAKE, batch, seq_len, budgets, FAKE, FAKE,
                                      FAKE, FAKE, FAKE, mg, FAKE, None, sel_count, ws, ws_bytes, None)


@nogpu
def test_prefill_validates_on_the_host(L):
    c = _cfg().c()
    assert _prefill(L, c, budgets=FAKE + 2) == sas.SAS_ERR_INVALID_ARG     # misaligned budgets
    assert _prefill(L, c, seq_len=4000) == sas.SAS_ERR_UNSUPPORTED        # not a multiple of 64
    assert _prefill(L, c, mg=63) == sas.SAS_ERR_INVALID_ARG                # gate-key rows < T/64
    assert _prefill(L, c, ws=FAKE + 16) == sas.SAS_ERR_WORKSPACE           # not 256-byte aligned
    assert _prefill(L, c, ws_bytes=1024) == sas.SAS_ERR_WORKSPACE
    assert _prefill(L, c, sel_count=FAKE + 1) == sas.SAS_ERR_INVALID_ARG
    assert _prefill(L, _cfg(kv_dtype="f32").c()) == sas.SAS_ERR_UNSUPPORTED  # bf16 only
    assert _prefill(L, c, batch=0) == sas.SAS_OK


@nogpu
def test_gate_backward_validates_on_the_host(L):
    def bwd(c, **kw):
        a = dict(q=FAKE, w_q=FAKE, g_q=FAKE, w_k=FAKE, g_k=FAKE, sel=FAKE, cnt=FAKE, dout=FAKE, dwq=FAKE,
                 dwk=FAKE, dgq=FAKE, dgk=FAKE, ws=FAKE, ws_bytes=256)
        a.update(kw)
        kv = sas._Kv(FAKE, FAKE, None, FAKE, 2, 4096, 0, 0, None)
        return L.sas_gate_backward(ctypes.byref(c), a["q"], ctypes.byref(kv), a["w_q"], a["g_q"], a["w_k"],
                                   a["g_k"], a["sel"], a["cnt"], a["dout"], a["dwq"], a["dwk"], a["dgq"],
                                   a["dgk"], a["ws"], a["ws_bytes"], None)
    gated = _cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    assert bwd(gated.c(), dout=None) == sas.SAS_ERR_INVALID_ARG
    assert bwd(gated.c(), dwq=FAKE + 2) == sas.SAS_ERR_INVALID_ARG
    assert bwd(gated.c(), ws=None) == sas.SAS_ERR_WORKSPACE
    # the per-pair terms of the reduction need sas_workspace_bytes(cfg, B, 0)
    need = L.sas_workspace_bytes(ctypes.byref(gated.c()), 2, 0)
    assert need > L.sas_workspace_bytes(ctypes.byref(gated.c()), 0, 0)
    assert bwd(gated.c(), ws_bytes=need - 1) == sas.SAS_ERR_WORKSPACE
    assert bwd(_cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS, token_budget=8192).c()) == sas.SAS_ERR_UNSUPPORTED
    assert bwd(_cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS, kv_dtype="f32").c()) == sas.SAS_ERR_UNSUPPORTED
    # the select-only mode gives the gate parameters no gradient: nothing to do
    assert bwd(_cfg().c()) == sas.SAS_OK


@nogpu
def test_static_step_needs_no_batch_workspace(L):
    """The allocation-free step's 256-byte scratch covers a decode step of any
    batch (the workspace a decode step needs is sas_workspace_bytes(cfg, 0, 0));
    its host checks then refuse a missing q before anything is enqueued."""
    c = _cfg().c()
    for batch in (1, 8, 64):
        kv = _kv(batch=batch)
        st = L.sas_decode_step_static(ctypes.byref(c), None, ctypes.byref(kv), FAKE, FAKE, None, None, FAKE, 64,
                                      FAKE, None, None, None, None, None)
        assert st == sas.SAS_ERR_INVALID_ARG, (batch, st)


@nogpu
def test_prefill_gate_backward_validates_on_the_host(L):
    def bwd(c, seq_len=4096, mg=64, ws_bytes=1 << 34, dout=FAKE, batch=2):
        return L.sas_prefill_gate_backward(ctypes.byref(c), FAKE, FAKE, FAKE, batch, seq_len, FAKE, FAKE, FAKE,
                                           FAKE, FAKE, mg, FAKE, FAKE, dout, FAKE, FAKE, FAKE, FAKE, FAKE,
                                           ws_bytes, None)
    gated = _cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    assert bwd(gated.c(), dout=None) == sas.SAS_ERR_INVALID_ARG
    assert bwd(gated.c(), dout=FAKE + 4) == sas.SAS_ERR_INVALID_ARG               # d_out not 16-byte aligned
    assert bwd(gated.c(), mg=63) == sas.SAS_ERR_INVALID_ARG                       # gate-key rows < T/64
    assert bwd(gated.c(), seq_len=4000) == sas.SAS_ERR_UNSUPPORTED                # not a multiple of 64
    assert bwd(_cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS, gate_keys_bf16=1).c()) == sas.SAS_ERR_UNSUPPORTED
    assert bwd(_cfg(gate_mode=sas.GATE_LOGSIGMOID_BIAS, token_budget=8192).c()) == sas.SAS_ERR_UNSUPPORTED
    need = L.sas_workspace_bytes(ctypes.byref(gated.c()), 2, 4096)
    assert bwd(gated.c(), ws_bytes=need - 1) == sas.SAS_ERR_WORKSPACE
    assert bwd(gated.c(), batch=0) == sas.SAS_OK
    assert bwd(_cfg().c(), ws_bytes=256) == sas.SAS_OK  # select-only: no gradient, nothing enqueued


@pytest.mark.parametrize("gk16", [0, 1])
def test_every_gate_key_entry_point_checks_the_dtype_first(monkeypatch, gk16):
    """A gate-key tensor whose dtype disagrees with cfg.gate_keys_bf16 is refused
    by the binding before any library call (a bf16 array read as fp32 would be
    over-run by the kernels)."""
    def no_library():
        raise AssertionError("the library was called before the dtype check")

    monkeypatch.setattr(sas, "lib", no_library)
    cfg = sas.Config(8, 2, gate_keys_bf16=gk16)
    wrong = torch.zeros(1, 2, 4, 128, dtype=torch.float32 if gk16 else torch.bfloat16)
    kv = sas.KvCache(torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16),
                     torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16), torch.ones(1, dtype=torch.int32))
    q = torch.zeros(1, 8, 128, dtype=torch.bfloat16)
    ws = torch.zeros(256, dtype=torch.uint8)
    calls = [
        lambda: sas.decode_step_static(cfg, q, kv, None, None, wrong, q),
        lambda: sas.decode_step(cfg, q, kv, None, None, wrong, q, ws),
        lambda: sas.decode_step_host(cfg, q, q, kv, None, None, wrong, q, q, ws),
        lambda: sas.pool_keys(cfg, kv, None, None, wrong, ws),
        lambda: sas.gate_scores(cfg, q, kv.seq_lens, None, None, wrong, None, ws),
        lambda: sas.prefill_block_sparse(cfg, q, q, q, None, None, None, None, wrong, q, ws),
    ]
    for call in calls:
        with pytest.raises(ValueError):
            call()
