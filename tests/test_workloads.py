"""The seeded input generators shared by the oracle tests and the CUDA path
(gated_block_sparse_token_b200/workloads.py): the same seed gives the same
tensors, the benchmark workloads have the shapes and structure the pages'
Qwen3 settings fix (64-token blocks, 32/8 and 40/8 heads, budgets 1,024 /
2,048 / 4,096, training length 32,768), the paged cache maps every block of
every sequence to its own page, and the draws have the stated distributions.
CPU only, at sizes that allocate a few MB."""
import math

import numpy as np
import torch

from gated_block_sparse_token_b200 import workloads as W


def _small(**kw):
    base = dict(name="w", batch=2, hq=8, hkv=2, seq_lens=[300, 640], token_budgets=(512,), capacity=1024, seed=5)
    base.update(kw)
    return W.DecodeSpec(**base)


def test_same_seed_same_tensors_and_another_seed_differs():
    a, b = W.make_decode_inputs(_small()), W.make_decode_inputs(_small())
    c = W.make_decode_inputs(_small(seed=6))
    for key in ("q", "k", "v", "w_q", "w_k", "gamma_q", "gamma_k", "seq_lens"):
        assert torch.equal(a[key], b[key]), key
    for key in ("q", "k", "v", "w_q", "w_k"):
        assert not torch.equal(a[key], c[key]), key


def test_decode_shapes_and_dtypes():
    x = W.make_decode_inputs(_small())
    assert x["q"].shape == (2, 8, 128) and x["q"].dtype == torch.bfloat16
    assert x["k"].shape == x["v"].shape == (2, 2, 1024, 128)
    assert x["w_q"].shape == (8, 128, 128) and x["w_k"].shape == (2, 384, 128)
    assert x["w_q"].dtype == x["w_k"].dtype == torch.bfloat16
    assert x["gamma_q"].shape == x["gamma_k"].shape == (128,) and x["gamma_q"].dtype == torch.float32
    assert x["block_table"] is None and x["seq_lens"].tolist() == [300, 640]
    f = W.make_decode_inputs(W.tiny_decode())
    assert f["q"].dtype == f["k"].dtype == torch.float32 and f["k"].shape == (1, 1, 4096, 128)


def test_paged_cache_gives_every_block_its_own_page():
    x = W.make_decode_inputs(_small(paged=True, capacity=None, seq_lens=[640, 640]))
    bt = x["block_table"]
    assert bt.shape == (2, 10) and bt.dtype == torch.int32
    assert sorted(bt.flatten().tolist()) == list(range(20))      # a permutation of the pool
    assert x["k"].shape == (20, 2, 64, 128)
    # logical_kv reads a sequence's tokens through its pages
    ks, _ = W.logical_kv(x, 1, 0, 130)
    page = int(bt[1, 2])
    assert np.array_equal(ks[128:130], x["k"][page, 0, :2].double().numpy())


def test_block_offsets_shift_each_block_by_one_vector():
    x = W.make_decode_inputs(_small(block_offset_std=0.5, seq_lens=[1024, 1024]))
    k = x["k"].float().view(2, 2, 16, 64, 128)
    # per-block means spread by the offset std (0.5), token noise by 1 / sqrt(64)
    block_means = k.mean(dim=3)
    assert 0.4 < float(block_means.std()) < 0.6
    assert abs(float((k - k.mean(dim=3, keepdim=True)).std()) - 1.0) < 0.05


def test_gains_and_weight_scales():
    x = W.make_decode_inputs(_small(batch=1, seq_lens=[64], capacity=64, hq=32, hkv=8))
    for gam in (x["gamma_q"], x["gamma_k"]):
        assert abs(float(gam.mean()) - 1.0) < 0.1 and 0.15 < float(gam.std()) < 0.35
    assert not torch.equal(x["gamma_q"], x["gamma_k"])
    assert abs(float(x["w_q"].float().std()) - 1 / math.sqrt(128)) < 0.01
    assert abs(float(x["w_k"].float().std()) - 1 / math.sqrt(384)) < 0.01
    unit = W.make_decode_inputs(W.tiny_decode())
    assert torch.equal(unit["gamma_q"], torch.ones(128)) and torch.equal(unit["gamma_k"], torch.ones(128))


def test_benchmark_workloads_follow_the_qwen3_settings():
    main = W.qwen3_4b_32k()
    assert (main.batch, main.hq, main.hkv, main.token_budgets) == (8, 32, 8, (2048,))
    assert main.seq_lens == [32768] * 8
    rag = W.qwen3_8b_ragged()
    assert (rag.batch, rag.hq, rag.hkv, rag.token_budgets) == (32, 32, 8, (1024, 2048, 4096))
    assert all(8192 <= n <= 65536 and n % 64 == 0 for n in rag.seq_lens)
    assert len(set(rag.seq_lens)) > 16 and rag.cap == 65536
    assert rag.seq_lens == W.qwen3_8b_ragged().seq_lens            # seeded
    long = W.qwen3_14b_paged_128k()
    assert (long.batch, long.hq, long.hkv, long.token_budgets, long.paged) == (16, 40, 8, (4096,), True)
    assert long.seq_lens == [131072] * 16 and long.appended == 256
    pf = W.qwen3_8b_prefill_32k()
    assert (pf.batch, pf.hq, pf.hkv, pf.seq_len, pf.token_budget) == (4, 32, 8, 32768, 2048)


def test_prefill_inputs_are_seeded_and_shaped():
    spec = W.PrefillSpec("p", 1, 4, 1, 256, token_budget=192, seed=9)
    a, b = W.make_prefill_inputs(spec), W.make_prefill_inputs(spec)
    for key in ("q", "k", "v", "w_q", "w_k", "gamma_q", "gamma_k"):
        assert torch.equal(a[key], b[key]), key
    assert a["q"].shape == (1, 4, 256, 128) and a["k"].shape == a["v"].shape == (1, 1, 256, 128)
    assert a["q"].dtype == torch.bfloat16
