"""Seeded synthetic workloads (Qwen3-shaped decode layers and prefill).

Random inputs only: this module holds none of the method's arithmetic.  The
same tensors feed the CUDA library and the CPU oracle in the tests, and the
benchmark.  Shapes follow the Qwen3 4B / 8B / 14B attention layouts the SAS
checkpoints target (32 or 40 query heads, 8 KV heads, head_dim 128); the
pages' evaluation data (OpenR1-Math, LongBench-E, ...) is not used, these
i.i.d. normal inputs stand in for it.

Recipe (every draw from one torch.Generator seeded with ``seed``, in this
order): q ~ N(0,1) [B][Hq][128]; K ~ N(0,1) then V ~ N(0,1) in the cache
layout, plus, when ``block_offset_std`` > 0, a per-(seq, head, block) offset
vector N(0, std^2) added to all 64 tokens of the block (K's offsets drawn
right after K, V's after V); paged caches take a random permutation of the
page ids as block table; W_q ~ N(0, 1/128) [Hq][128][128] and W_k ~
N(0, 1/384) [Hkv][384][128], rounded to bf16; then the RMSNorm gains
gamma_q = 1 + gain_std * N(0,1) and gamma_k = 1 + gain_std * N(0,1), [128]
fp32 each (gain_std 0.25; the tiny fp32 workload keeps gain 1, as its
description states, but still draws them so the draw order is the same).
Values are rounded to the storage dtype (bf16 or fp32) once.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

BLOCK = 64
DIM = 128


@dataclass
class DecodeSpec:
    name: str
    batch: int
    hq: int
    hkv: int
    seq_lens: list
    token_budgets: tuple
    kv_dtype: str = "bf16"
    capacity: Optional[int] = None          # contiguous tokens per (seq, head)
    paged: bool = False
    block_offset_std: float = 0.0
    appended: int = 0                       # tokens appended incrementally
    seed: int = 0
    gain_std: float = 0.25                  # RMSNorm gains 1 + gain_std * N(0,1)

    @property
    def cap(self) -> int:
        if self.capacity is not None:
            return self.capacity
        return ((max(self.seq_lens) + BLOCK - 1) // BLOCK) * BLOCK


def tiny_decode(seed: int = 0) -> DecodeSpec:
    """One sequence, one KV head, G = 4, context 4,096, budget 1,024, fp32."""
    return DecodeSpec("tiny_1x4q1kv_4k_f32", 1, 4, 1, [4096], (1024,), kv_dtype="f32", seed=seed,
                      gain_std=0.0)


def qwen3_4b_32k(batch: int = 8, seq_len: int = 32768, seed: int = 1) -> DecodeSpec:
    """Qwen3-4B layer: 32/8 heads, batch 8, context 32,768, budget 2,048, bf16 K/V
    with per-block mean offsets of std 0.5."""
    return DecodeSpec(f"qwen3_4b_b{batch}_{seq_len // 1024}k", batch, 32, 8, [seq_len] * batch,
                      (2048,), block_offset_std=0.5, seed=seed)


def qwen3_8b_ragged(batch: int = 32, lo: int = 8192, hi: int = 65536, seed: int = 2) -> DecodeSpec:
    """Qwen3-8B layer: 32/8 heads, batch 32, contexts uniform in [lo, hi] in
    steps of 64, budgets 1,024 / 2,048 / 4,096."""
    g = torch.Generator().manual_seed(seed)
    lens = (torch.randint(lo // BLOCK, hi // BLOCK + 1, (batch,), generator=g) * BLOCK).tolist()
    return DecodeSpec(f"qwen3_8b_ragged_b{batch}", batch, 32, 8, lens, (1024, 2048, 4096),
                      capacity=hi, seed=seed)


def qwen3_14b_paged_128k(batch: int = 16, seq_len: int = 131072, appended: int = 256,
                         seed: int = 3) -> DecodeSpec:
    """Qwen3-14B layer: 40/8 heads, batch 16, context 131,072 in 64-token pages
    behind a random block table, budget 4,096; the last `appended` tokens are
    added (and their blocks pooled) incrementally."""
    return DecodeSpec(f"qwen3_14b_paged_b{batch}_{seq_len // 1024}k", batch, 40, 8,
                      [seq_len] * batch, (4096,), paged=True, appended=appended, seed=seed)


def _gains(g, device, std):
    """RMSNorm gains of the gate query and key: 1 + std * N(0,1), [128] fp32
    each (drawn even when std is 0, so later draws do not move)."""
    gq = _randn((DIM,), g, device)
    gk = _randn((DIM,), g, device)
    return 1.0 + std * gq, 1.0 + std * gk


def _randn(shape, g, device, std=1.0):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x if std == 1.0 else x * std


def make_decode_inputs(spec: DecodeSpec, device="cpu") -> dict:
    """Materialise a decode workload on `device` (bf16/fp32 storage dtypes)."""
    dt = torch.bfloat16 if spec.kv_dtype == "bf16" else torch.float32
    g = torch.Generator(device=device).manual_seed(spec.seed)
    B, hq, hkv = spec.batch, spec.hq, spec.hkv
    q = _randn((B, hq, DIM), g, device).to(dt)
    cap = spec.cap
    nblk = cap // BLOCK
    out = {"spec": spec, "q": q}
    if spec.paged:
        num_pages = B * nblk
        shape = (num_pages, hkv, BLOCK, DIM)
    else:
        shape = (B, hkv, cap, DIM)

    def cache():
        x = _randn(shape, g, device)
        if spec.block_offset_std > 0:
            if spec.paged:
                off = _randn((shape[0], hkv, 1, DIM), g, device, spec.block_offset_std)
                x += off
            else:
                off = _randn((B, hkv, nblk, 1, DIM), g, device, spec.block_offset_std)
                x = (x.view(B, hkv, nblk, BLOCK, DIM) + off).view(shape)
        return x.to(dt)

    out["k"] = cache()
    out["v"] = cache()
    if spec.paged:
        perm = torch.randperm(B * nblk, generator=g, device=device)
        out["block_table"] = perm.view(B, nblk).to(torch.int32)
    else:
        out["block_table"] = None
    out["w_q"] = _randn((hq, DIM, DIM), g, device, 1.0 / math.sqrt(DIM)).to(torch.bfloat16)
    out["w_k"] = _randn((hkv, 3 * DIM, DIM), g, device, 1.0 / math.sqrt(3 * DIM)).to(torch.bfloat16)
    out["gamma_q"], out["gamma_k"] = _gains(g, device, spec.gain_std)
    out["seq_lens"] = torch.tensor(spec.seq_lens, dtype=torch.int32, device=device)
    return out


def logical_kv(inputs: dict, s: int, h: int, length: int):
    """K, V of (sequence s, KV head h) as [length][128] float64 numpy arrays,
    read through the block table when the cache is paged (host copy)."""
    k, v, bt = inputs["k"], inputs["v"], inputs["block_table"]
    nb = (length + BLOCK - 1) // BLOCK
    if bt is None:
        ks = k[s, h, :nb * BLOCK]
        vs = v[s, h, :nb * BLOCK]
    else:
        pages = bt[s, :nb].long()
        ks = k[pages, h].reshape(nb * BLOCK, DIM)
        vs = v[pages, h].reshape(nb * BLOCK, DIM)
    return (ks[:length].double().cpu().numpy(), vs[:length].double().cpu().numpy())


@dataclass
class PrefillSpec:
    name: str
    batch: int
    hq: int
    hkv: int
    seq_len: int
    token_budget: int = 2048
    seed: int = 4
    gain_std: float = 0.25   # RMSNorm gains 1 + gain_std * N(0,1)


def qwen3_8b_prefill_32k(batch: int = 4, seq_len: int = 32768, seed: int = 4) -> PrefillSpec:
    """Qwen3-8B head layout (32 query / 8 KV heads), batch 4, causal 32,768-token
    prefill, Top-K 31 + the diagonal block (2,048-token budget)."""
    return PrefillSpec(f"qwen3_8b_prefill_b{batch}_{seq_len // 1024}k", batch, 32, 8, seq_len, 2048, seed)


def make_prefill_inputs(spec: PrefillSpec, device="cpu") -> dict:
    """q [B][Hq][T][128], k / v [B][Hkv][T][128] ~ N(0,1) in bf16; gate weights and
    gains as for decode.  Draw order: q, K, V, W_q, W_k, gamma_q, gamma_k."""
    g = torch.Generator(device=device).manual_seed(spec.seed)
    B, hq, hkv, T = spec.batch, spec.hq, spec.hkv, spec.seq_len
    out = {"spec": spec}
    out["q"] = _randn((B, hq, T, DIM), g, device).to(torch.bfloat16)
    out["k"] = _randn((B, hkv, T, DIM), g, device).to(torch.bfloat16)
    out["v"] = _randn((B, hkv, T, DIM), g, device).to(torch.bfloat16)
    out["w_q"] = _randn((hq, DIM, DIM), g, device, 1.0 / math.sqrt(DIM)).to(torch.bfloat16)
    out["w_k"] = _randn((hkv, 3 * DIM, DIM), g, device, 1.0 / math.sqrt(3 * DIM)).to(torch.bfloat16)
    out["gamma_q"], out["gamma_k"] = _gains(g, device, spec.gain_std)
    return out
