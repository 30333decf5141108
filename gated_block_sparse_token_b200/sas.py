"""Thin ctypes binding of libsas (include/sas.h): argument marshalling only.

Every function here forwards torch tensors' device pointers and sizes to the
C ABI of the same name and raises ``SasError`` on a non-OK status.  All
arithmetic runs in the library's CUDA kernels; there is no fallback.  The
library must have been built (``python -m gated_block_sparse_token_b200.build``).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SAS_LIBRARY selects another build of the same ABI (e.g. the phase-trace build).
LIB_PATH = os.environ.get("SAS_LIBRARY", os.path.join(_HERE, "libsas.so"))
ABI_VERSION = 10            # the include/sas.h this binding marshals for

SAS_OK = 0
SAS_ERR_INVALID_ARG = 1
SAS_ERR_UNSUPPORTED = 2
SAS_ERR_WORKSPACE = 3
SAS_ERR_CUDA = 4
SAS_ERR_DEVICE_BOUNDS = 5
SAS_ERR_TIMEOUT = 6

GATE_SELECT_ONLY = 0       # selected blocks weighted 1
GATE_LOGSIGMOID_BIAS = 1   # + log(sigmoid(gate score)) on a selected historical block's logits

DTYPE_BF16 = 0
DTYPE_F32 = 1
_DT = {"bf16": DTYPE_BF16, "f32": DTYPE_F32}
_TORCH_DT = {DTYPE_BF16: torch.bfloat16, DTYPE_F32: torch.float32}


class SasError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class _Config(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("gate_hidden", ctypes.c_int32), ("token_budget", ctypes.c_int32),
                ("rope_base", ctypes.c_float), ("norm_eps", ctypes.c_float),
                ("attn_scale", ctypes.c_float), ("gate_scale", ctypes.c_float),
                ("kv_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("gate_mode", ctypes.c_int32), ("gate_keys_bf16", ctypes.c_int32),
                ("static_weights", ctypes.c_int32)]


class _Kv(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
                ("token_budgets", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsas.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m gated_block_sparse_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        cfgp, kvp = ctypes.POINTER(_Config), ctypes.POINTER(_Kv)
        sigs = {
            "sas_abi_version": (i32, []),
            "sas_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "sas_workspace_bytes": (sz, [cfgp, i32, i32]),
            "sas_reset_device_status": (ctypes.c_int, [vp, vp]),
            "sas_get_device_status": (ctypes.c_int, [vp, vp, ctypes.POINTER(ctypes.c_int)]),
            "sas_pool_keys": (ctypes.c_int, [cfgp, kvp, vp, i32, vp, vp, vp, i32, vp, vp, sz, vp]),
            "sas_gate_scores": (ctypes.c_int, [cfgp, vp, vp, i32, vp, vp, vp, i32, vp, vp, vp, sz, vp]),
            "sas_topk_blocks": (ctypes.c_int, [cfgp, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]),
            "sas_sparse_decode": (ctypes.c_int, [cfgp, vp, kvp, vp, vp, vp, vp, sz, vp]),
            "sas_decode_step": (ctypes.c_int, [cfgp, vp, kvp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]),
            "sas_decode_step_static": (ctypes.c_int, [cfgp, vp, kvp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]),
            "sas_decode_step_host": (ctypes.c_int, [cfgp, vp, vp, kvp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp,
                                                    sz, vp]),
            "sas_gate_backward": (ctypes.c_int, [cfgp, vp, kvp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "sas_prefill_block_sparse": (ctypes.c_int, [cfgp, vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]),
            "sas_prefill_gate_backward": (ctypes.c_int, [cfgp, vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp, vp,
                                                         vp, vp, vp, vp, vp, sz, vp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        if L.sas_abi_version() != ABI_VERSION:
            raise RuntimeError(f"{LIB_PATH} has ABI {L.sas_abi_version()}, this binding wants {ABI_VERSION}: "
                               "rebuild it")
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sas_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != SAS_OK:
        raise SasError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


@dataclass
class Config:
    """Mirror of sas_config.  Defaults are the released setting (budget 2,048)."""
    num_q_heads: int
    num_kv_heads: int
    token_budget: int = 2048
    kv_dtype: str = "bf16"
    out_dtype: str = "bf16"
    rope_base: float = 10000.0
    norm_eps: float = 1e-6
    attn_scale: float = 1.0 / math.sqrt(128.0)
    gate_scale: float = 1.0 / math.sqrt(128.0)
    head_dim: int = 128
    block_size: int = 64
    gate_hidden: int = 128
    gate_mode: int = 0        # GATE_SELECT_ONLY or GATE_LOGSIGMOID_BIAS
    gate_keys_bf16: int = 0   # 1: the gate-key cache is bf16 (else fp32)
    # 1: w_q, gamma_q, w_k and gamma_k are never written while decode kernels
    # may run, so the kernels read them before the kernels ahead of them on
    # the stream have finished; 0: every input after those have finished
    static_weights: int = 0

    def c(self) -> _Config:
        return _Config(self.num_q_heads, self.num_kv_heads, self.head_dim, self.block_size,
                       self.gate_hidden, self.token_budget, self.rope_base, self.norm_eps,
                       self.attn_scale, self.gate_scale, _DT[self.kv_dtype], _DT[self.out_dtype],
                       self.gate_mode, self.gate_keys_bf16, self.static_weights)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_sel(self) -> int:
        return self.token_budget // 64


@dataclass
class KvCache:
    """Mirror of sas_kv holding the tensors alive.  block_table None: contiguous
    [B][Hkv][capacity][128]; else paged [num_pages][Hkv][64][128]."""
    k: torch.Tensor
    v: torch.Tensor
    seq_lens: torch.Tensor
    block_table: Optional[torch.Tensor] = None
    token_budgets: Optional[torch.Tensor] = None   # int32 [B]; None: the config's budget
    _c: Optional[_Kv] = field(default=None, repr=False)

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    def c(self) -> _Kv:
        if self.block_table is None:
            return _Kv(_ptr(self.k), _ptr(self.v), None, _ptr(self.seq_lens), self.batch,
                       int(self.k.shape[2]), 0, 0, _ptr(self.token_budgets))
        return _Kv(_ptr(self.k), _ptr(self.v), _ptr(self.block_table), _ptr(self.seq_lens),
                   self.batch, 0, int(self.k.shape[0]), int(self.block_table.shape[1]),
                   _ptr(self.token_budgets))


def abi_version() -> int:
    return int(lib().sas_abi_version())


def workspace_bytes(cfg: Config, batch: int = 0, max_seq_len: int = 0) -> int:
    c = cfg.c()
    return int(lib().sas_workspace_bytes(ctypes.byref(c), batch, max_seq_len))


def make_workspace(cfg: Config, device, batch: int = 0, max_seq_len: int = 0) -> torch.Tensor:
    """Caller-side workspace allocation (torch), zeroed."""
    return torch.zeros(workspace_bytes(cfg, batch, max_seq_len), dtype=torch.uint8, device=device)


def reset_device_status(ws: torch.Tensor, stream=None) -> None:
    _check(lib().sas_reset_device_status(_ptr(ws), _stream(stream)), "sas_reset_device_status")


def get_device_status(ws: torch.Tensor, stream=None) -> int:
    out = ctypes.c_int(-1)
    _check(lib().sas_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(out)),
           "sas_get_device_status")
    return int(out.value)


def pool_keys(cfg: Config, kv: KvCache, w_k, gamma_k, gate_keys, ws, blk_begin=None,
              num_blocks: Optional[int] = None, pooled_raw=None, stream=None) -> None:
    """sas_pool_keys.  num_blocks defaults to gate_keys.shape[2] (all rows)."""
    _check_gk(cfg, gate_keys)
    mg = int(gate_keys.shape[2])
    nb = mg if num_blocks is None else int(num_blocks)
    c, k = cfg.c(), kv.c()
    _check(lib().sas_pool_keys(ctypes.byref(c), ctypes.byref(k), _ptr(blk_begin), nb, _ptr(w_k),
                               _ptr(gamma_k), _ptr(gate_keys), mg, _ptr(pooled_raw), _ptr(ws),
                               ws.numel(), _stream(stream)), "sas_pool_keys")


def gate_scores(cfg: Config, q, seq_lens, w_q, gamma_q, gate_keys, group_scores, ws,
                head_scores=None, stream=None) -> None:
    _check_gk(cfg, gate_keys)
    c = cfg.c()
    _check(lib().sas_gate_scores(ctypes.byref(c), _ptr(q), _ptr(seq_lens), int(seq_lens.shape[0]),
                                 _ptr(w_q), _ptr(gamma_q), _ptr(gate_keys), int(gate_keys.shape[2]),
                                 _ptr(head_scores), _ptr(group_scores), _ptr(ws), ws.numel(),
                                 _stream(stream)), "sas_gate_scores")


def topk_blocks(cfg: Config, group_scores, seq_lens, sel_idx, sel_count, ws, stream=None,
                token_budgets=None) -> None:
    c = cfg.c()
    _check(lib().sas_topk_blocks(ctypes.byref(c), _ptr(group_scores), _ptr(seq_lens), _ptr(token_budgets),
                                 int(seq_lens.shape[0]), int(group_scores.shape[2]), _ptr(sel_idx),
                                 _ptr(sel_count), _ptr(ws), ws.numel(), _stream(stream)),
           "sas_topk_blocks")


def sparse_decode(cfg: Config, q, kv: KvCache, sel_idx, sel_count, out, ws, stream=None) -> None:
    c, k = cfg.c(), kv.c()
    _check(lib().sas_sparse_decode(ctypes.byref(c), _ptr(q), ctypes.byref(k), _ptr(sel_idx),
                                   _ptr(sel_count), _ptr(out), _ptr(ws), ws.numel(),
                                   _stream(stream)), "sas_sparse_decode")


def decode_step(cfg: Config, q, kv: KvCache, w_q, gamma_q, gate_keys, out, ws, sel_idx=None,
                sel_count=None, group_scores=None, w_k=None, gamma_k=None, stream=None) -> None:
    """sas_decode_step.  With w_k / gamma_k the step also pools the block the
    decoded token completes into gate_keys (see include/sas.h)."""
    _check_gk(cfg, gate_keys)
    c, k = cfg.c(), kv.c()
    _check(lib().sas_decode_step(ctypes.byref(c), _ptr(q), ctypes.byref(k), _ptr(w_q),
                                 _ptr(gamma_q), _ptr(w_k), _ptr(gamma_k), _ptr(gate_keys),
                                 int(gate_keys.shape[2]), _ptr(out), _ptr(sel_idx), _ptr(sel_count),
                                 _ptr(group_scores), _ptr(ws), ws.numel(), _stream(stream)),
           "sas_decode_step")


def decode_step_host(cfg: Config, q_host, q_dev, kv: KvCache, w_q, gamma_q, gate_keys, out_dev, out_host, ws,
                     sel_idx=None, sel_count=None, group_scores=None, w_k=None, gamma_k=None,
                     stream=None) -> None:
    """sas_decode_step_host: the step with q and out in host memory (pinned
    CPU tensors keep the copies asynchronous); q_dev / out_dev are device
    staging buffers of the same shapes.  out_host holds the output once the
    stream has passed the call.  The library sizes both transfers from the
    config, so each host tensor must be a contiguous CPU tensor of its
    staging buffer's shape and dtype (checked here)."""
    _check_gk(cfg, gate_keys)
    for name, h, d in (("q_host", q_host, q_dev), ("out_host", out_host, out_dev)):
        if h.device.type != "cpu" or not h.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor")
        if h.shape != d.shape or h.dtype != d.dtype:
            raise ValueError(f"{name} is {tuple(h.shape)} {h.dtype}, its device buffer {tuple(d.shape)} {d.dtype}")
    c, k = cfg.c(), kv.c()
    _check(lib().sas_decode_step_host(ctypes.byref(c), _ptr(q_host), _ptr(q_dev), ctypes.byref(k), _ptr(w_q),
                                      _ptr(gamma_q), _ptr(w_k), _ptr(gamma_k), _ptr(gate_keys),
                                      int(gate_keys.shape[2]), _ptr(out_dev), _ptr(out_host), _ptr(sel_idx),
                                      _ptr(sel_count), _ptr(group_scores), _ptr(ws), ws.numel(),
                                      _stream(stream)), "sas_decode_step_host")


def decode_step_static(cfg: Config, q, kv: KvCache, w_q, gamma_q, gate_keys, out, sel_idx=None,
                       sel_count=None, group_scores=None, w_k=None, gamma_k=None, status_out=None,
                       stream=None) -> None:
    """sas_decode_step_static: the same step with no workspace argument, for
    callers that cannot allocate; status_out (optional device uint32/int32
    tensor) receives the call's status bits."""
    _check_gk(cfg, gate_keys)
    c, k = cfg.c(), kv.c()
    _check(lib().sas_decode_step_static(ctypes.byref(c), _ptr(q), ctypes.byref(k), _ptr(w_q),
                                        _ptr(gamma_q), _ptr(w_k), _ptr(gamma_k), _ptr(gate_keys),
                                        int(gate_keys.shape[2]), _ptr(out), _ptr(sel_idx),
                                        _ptr(sel_count), _ptr(group_scores), _ptr(status_out),
                                        _stream(stream)), "sas_decode_step_static")


def gate_backward(cfg: Config, q, kv: KvCache, w_q, gamma_q, w_k, gamma_k, sel_idx, sel_count, d_out,
                  dw_q, dw_k, dgamma_q, dgamma_k, ws, stream=None) -> None:
    """sas_gate_backward: adds dL/dW_q, dL/dW_k, dL/dgamma_q, dL/dgamma_k (fp32)
    of the gated decode step, block lists held fixed, for d_out = dL/dout."""
    c, k = cfg.c(), kv.c()
    _check(lib().sas_gate_backward(ctypes.byref(c), _ptr(q), ctypes.byref(k), _ptr(w_q), _ptr(gamma_q),
                                   _ptr(w_k), _ptr(gamma_k), _ptr(sel_idx), _ptr(sel_count), _ptr(d_out),
                                   _ptr(dw_q), _ptr(dw_k), _ptr(dgamma_q), _ptr(dgamma_k), _ptr(ws),
                                   ws.numel(), _stream(stream)), "sas_gate_backward")


def prefill_block_sparse(cfg: Config, q, k, v, w_q, gamma_q, w_k, gamma_k, gate_keys, out, ws,
                         sel_idx=None, sel_count=None, stream=None, token_budgets=None) -> None:
    """sas_prefill_block_sparse: q [B][Hq][T][128], k / v [B][Hkv][T][128] (bf16),
    out like q; writes gate_keys [B][Hkv][MG][128]; ws from
    make_workspace(cfg, device, batch=B, max_seq_len=T); token_budgets: None or
    int32 [B] on the device (each a multiple of 64, at most cfg.token_budget)."""
    _check_gk(cfg, gate_keys)
    c = cfg.c()
    B, T = int(q.shape[0]), int(q.shape[2])
    _check(lib().sas_prefill_block_sparse(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), B, T,
                                          _ptr(token_budgets), _ptr(w_q),
                                          _ptr(gamma_q), _ptr(w_k), _ptr(gamma_k), _ptr(gate_keys),
                                          int(gate_keys.shape[2]), _ptr(out), _ptr(sel_idx),
                                          _ptr(sel_count), _ptr(ws), ws.numel(), _stream(stream)),
           "sas_prefill_block_sparse")


def prefill_gate_backward(cfg: Config, q, k, v, w_q, gamma_q, w_k, gamma_k, gate_keys, sel_idx, sel_count,
                          d_out, dw_q, dw_k, dgamma_q, dgamma_k, ws, stream=None) -> None:
    """sas_prefill_gate_backward: adds dL/dW_q, dL/dW_k, dL/dgamma_q, dL/dgamma_k
    (fp32) of the gated prefill, its block lists held fixed, for d_out =
    dL/dout [B][Hq][T][128] fp32; ws from make_workspace(cfg, device, batch=B,
    max_seq_len=T)."""
    _check_gk(cfg, gate_keys)
    c = cfg.c()
    B, T = int(q.shape[0]), int(q.shape[2])
    _check(lib().sas_prefill_gate_backward(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), B, T, _ptr(w_q),
                                           _ptr(gamma_q), _ptr(w_k), _ptr(gamma_k), _ptr(gate_keys),
                                           int(gate_keys.shape[2]), _ptr(sel_idx), _ptr(sel_count), _ptr(d_out),
                                           _ptr(dw_q), _ptr(dw_k), _ptr(dgamma_q), _ptr(dgamma_k), _ptr(ws),
                                           ws.numel(), _stream(stream)), "sas_prefill_gate_backward")


def out_dtype(cfg: Config) -> torch.dtype:
    return _TORCH_DT[_DT[cfg.out_dtype]]


def gate_key_dtype(cfg: Config) -> torch.dtype:
    """Element type of the gate-key cache under cfg (bf16 or fp32)."""
    return torch.bfloat16 if cfg.gate_keys_bf16 else torch.float32


def _check_gk(cfg: Config, gate_keys) -> None:
    if gate_keys is not None and gate_keys.dtype != gate_key_dtype(cfg):
        raise ValueError(f"gate_keys is {gate_keys.dtype}, the config wants {gate_key_dtype(cfg)}")


def kv_dtype(cfg: Config) -> torch.dtype:
    return _TORCH_DT[_DT[cfg.kv_dtype]]
