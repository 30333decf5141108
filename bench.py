"""Benchmark of the SAS decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: Qwen3-4B-shaped decode layer, batch 8, 32 query / 8 KV heads,
head_dim 128, context 32,768 for every sequence, token budget 2,048
(31 historical blocks + the current block), bf16 K/V with per-block mean
offsets (seeded, synthetic).  A step is one pass of the whole decode path
over the batch in one launch of sas_decode_step: gate query, scores of all
511 historical blocks, Top-K, block-sparse attention, and pooling + gate key
of the block the decoded token completes (token 32,768 completes block 511).  Steps rotate over R layers with their own caches, so the
selected working set (R x ~85 MB) is far larger than the 126 MB L2.

Metric: decode steps/s per layer (whole job: summed over ranks), achieved
HBM GB/s of the dominant kernel against the measured B200 copy bandwidth.

The layers share one sequence-length vector (a model's decode step reads
the same lengths in every layer); K/V caches, gate keys, queries and gate
weights are per layer.

Multi-GPU: one process per GPU (torchrun); every rank decodes its own
independent batch (weak scaling, no collective on the data path); the only
collectives are the barrier and the max-reduce of the timings.

Timing: each timed region replays exactly K steps (CUDA graphs), bracketed
by a barrier and a device synchronisation; the region is repeated
(--repeats, default 21) and the line reports the median, with min and max
beside it.  Variants: the gated mode, mixed budgets, bf16 gate keys, the
Qwen3-8B ragged layer at budgets 1,024 / 2,048 / 4,096, and the Qwen3-14B
128k paged layer decoded incrementally (256 appended tokens, pooling at block
completion).

--impl reference times the CPU oracle (the plain fp64 restatement of the
method) on whole decode steps of the same workload (64 (sequence, KV head)
pairs each), reported as steps/s.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse decode steps/s per layer at 32k ctx; achieved HBM GB/s vs B200 peak"
UNIT = "steps/s"
WORKLOAD = "qwen3_4b_decode_b8_ctx32768_budget2048"
BATCH, HQ, HKV, CTX, BUDGET = 8, 32, 8, 32768, 2048
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=400)
    ap.add_argument("--repeats", type=int, default=21,
                    help="timed replays of the K-step graphs; the median is reported")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-batch", type=int, default=4)
    ap.add_argument("--prefill-steps", type=int, default=5)
    ap.add_argument("--skip-prefill", action="store_true")
    ap.add_argument("--prefill-only", action="store_true")
    ap.add_argument("--variant-steps", type=int, default=1000)
    ap.add_argument("--skip-variants", action="store_true")
    return ap.parse_args()


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus, backend=None):
    """One process per GPU from the torchrun environment (RANK, LOCAL_RANK,
    WORLD_SIZE, MASTER_ADDR/PORT).  NCCL on GPUs; gloo when asked (the CPU
    tests of this plumbing).  The group carries only the barrier and the
    max-reduce of timings."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    backend = backend or "nccl"
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest of the ranks' values (timings are max over ranks)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, seconds_max):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time."""
    return world * units_per_rank / seconds_max


# ---------------------------------------------------------------- measured peaks, clocks
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                smax = float(f[3])
            except ValueError:
                continue
            for nm, val in zip(names, f[6:10]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- algorithmic bytes
def decode_bytes(seq_lens, hq, hkv, budget, kv_elem=2, pool=True, gk_elem=4):
    """Bytes one fused decode step must move: the selected K/V tokens, the fp32
    gate key of every historical block, q and out of every head and W_q once;
    with pooling of the completed current block also W_k once and the new
    gate keys (the block's K is already among the selected tokens).  budget:
    one for the batch, or one per sequence."""
    G = hq // hkv
    tot = 0
    budgets = budget if isinstance(budget, (list, tuple)) else [budget] * len(seq_lens)
    for L, budget in zip(seq_lens, budgets):
        c = (L - 1) // 64
        m = min(budget // 64 - 1, c)
        cur_tokens = L - 64 * c
        per_pair = (m * 64 + cur_tokens) * 128 * kv_elem * 2 + c * 128 * gk_elem + 2 * G * 128 * 2
        if pool and L % 64 == 0:
            per_pair += 128 * gk_elem
        tot += hkv * per_pair
    tot += hq * 128 * 128 * 2
    if pool and any(L % 64 == 0 for L in seq_lens):  # W_k is read only when a block completes
        tot += hkv * 384 * 128 * 2
    return tot


def prefill_flops(nblk, hq, hkv, budget, batch):
    """Tensor FLOPs of the block-sparse prefill attention, counted as full
    64x64 tiles: per (sequence, query head, query block i) min(topk, i) + 1
    blocks, each 2*64*64*128 for Q K^T and as much for P V."""
    topk = budget // 64 - 1
    pairs = sum(min(topk, i) + 1 for i in range(nblk))
    return batch * hq * pairs * 4 * 64 * 64 * 128


def measured_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured sustained bf16"
    return 1400.0, "fallback sustained bf16"


def run_prefill(args, device, world):
    """Block-sparse chunked prefill, Qwen3-8B heads, 32,768 tokens per sequence,
    Top-K 31 + diagonal: one sas_prefill_block_sparse call per step (pooling,
    gate queries, selection, tcgen05 attention), in both gate modes and with
    per-sequence budgets."""
    import torch
    from gated_block_sparse_token_b200 import sas
    from gated_block_sparse_token_b200.workloads import make_prefill_inputs, qwen3_8b_prefill_32k

    spec = qwen3_8b_prefill_32k(batch=args.prefill_batch)
    inp = make_prefill_inputs(spec, device)
    B, T = spec.batch, spec.seq_len
    nblk = T // 64
    out = torch.empty(B, spec.hq, T, 128, dtype=torch.bfloat16, device=device)
    gk = torch.zeros(B, spec.hkv, nblk, 128, dtype=torch.float32, device=device)
    stream = torch.cuda.Stream(device)

    def make_call(gate_mode, budgets=None):
        cfg = sas.Config(spec.hq, spec.hkv, token_budget=spec.token_budget if budgets is None else max(budgets),
                         gate_mode=gate_mode)
        ws = sas.make_workspace(cfg, device, batch=B, max_seq_len=T)
        tb = None if budgets is None else torch.tensor(budgets, dtype=torch.int32, device=device)

        def call():
            sas.prefill_block_sparse(cfg, inp["q"], inp["k"], inp["v"], inp["w_q"], inp["gamma_q"], inp["w_k"],
                                     inp["gamma_k"], gk, out, ws, stream=stream, token_budgets=tb)
        return call, ws

    mixed = [1024, 2048, 4096, 2048][:B] if B <= 4 else None
    modes = [make_call(sas.GATE_SELECT_ONLY), make_call(sas.GATE_LOGSIGMOID_BIAS)]
    if mixed:
        modes.append(make_call(sas.GATE_SELECT_ONLY, mixed))
    # the modes take turns, call by call, so that all of them see the same
    # clocks (a long tensor-core run settles under the power cap)
    with torch.cuda.stream(stream):
        for _ in range(2):
            for call, _ws in modes:
                call()
    torch.cuda.synchronize()
    barrier(world)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.prefill_steps)] for _ in modes]
    clk = ClockSampler(torch.device(device).index or 0)
    clk.start()
    time.sleep(0.3)  # nvidia-smi's first sample
    with torch.cuda.stream(stream):
        for k in range(args.prefill_steps):
            for (call, _ws), evm in zip(modes, ev):
                evm[k][0].record(stream)
                call()
                evm[k][1].record(stream)
    torch.cuda.synchronize()
    clocks = clk.stop()
    barrier(world)
    times = [max_over_ranks(sum(a.elapsed_time(b) for a, b in evm) / 1e3 / args.prefill_steps, world) for evm in ev]
    for _call, ws in modes:
        if sas.get_device_status(ws, stream) != sas.SAS_OK:
            raise RuntimeError("device status not OK after the prefill run")
    t, t_gated = times[0], times[1]
    t_mixed = times[2] if mixed else None
    flops = prefill_flops(nblk, spec.hq, spec.hkv, spec.token_budget, B)
    peak, kind = measured_tensor_peak()
    achieved = flops / t / 1e12
    return {"workload": spec.name, "batch_per_gpu": B, "seq_len": T, "q_heads": spec.hq,
            "kv_heads": spec.hkv, "token_budget": spec.token_budget, "steps": args.prefill_steps,
            "ms_per_step": round(t * 1e3, 4), "tokens_per_s": round(job_throughput(B * T, world, t), 1),
            "launches_per_step": 4,
            "clocks": clocks,
            "gated_mode_ms_per_step": round(t_gated * 1e3, 4),
            "mixed_budgets": None if t_mixed is None else {"token_budgets": mixed,
                                                          "ms_per_step": round(t_mixed * 1e3, 4)},
            "roofline": {"kernel": "prefill_attn_kernel (tcgen05)", "bound": "tensor",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "peak_kind": kind,
                         "flops_per_step": flops,
                         "note": "FLOPs over the whole prefill call (pooling, gate, selection and "
                                 "attention launches): a lower bound on the attention kernel's rate"}}


def run_backward(args, rank, world, device):
    """Gradient through the gates on the main workload (Qwen3-4B layer, batch 8,
    32k context, budget 2,048, gated mode): one sas_gate_backward call per
    step with the block lists of the forward step held fixed and a seeded
    upstream gradient.  Algorithmic bytes: the selected K and V blocks, W_q
    and W_k once, q and dL/dout, and the fp32 gradients of W_q and W_k
    written once."""
    import torch
    from gated_block_sparse_token_b200 import sas
    cfg, layers = build_layers(2, rank, device, gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    stream = torch.cuda.Stream(device)
    for L in layers:
        L["ws"] = sas.make_workspace(cfg, device, batch=BATCH)   # the per-pair terms of the reduction
        L["sel"] = torch.zeros(BATCH, HKV, cfg.max_sel, dtype=torch.int32, device=device)
        L["cnt"] = torch.zeros(BATCH, HKV, dtype=torch.int32, device=device)
        L["dout"] = torch.randn(BATCH, HQ, 128, generator=torch.Generator(device=device).manual_seed(9),
                                device=device)
    grads = [torch.zeros(HQ, 128, 128, device=device), torch.zeros(HKV, 384, 128, device=device),
             torch.zeros(128, device=device), torch.zeros(128, device=device)]
    torch.cuda.synchronize()   # the tensors above come from torch's stream
    for L in layers:          # the forward step that fixes the block lists
        inp = L["inp"]
        sas.decode_step(cfg, inp["q"], L["kv"], inp["w_q"], inp["gamma_q"], L["gk"], L["out"], L["ws"],
                        sel_idx=L["sel"], sel_count=L["cnt"], stream=stream)
    torch.cuda.synchronize()

    def bwd(L, st):
        inp = L["inp"]
        sas.gate_backward(cfg, inp["q"], L["kv"], inp["w_q"], inp["gamma_q"], inp["w_k"], inp["gamma_k"],
                          L["sel"], L["cnt"], L["dout"], *grads, L["ws"], stream=st)

    with torch.cuda.stream(stream):
        for L in layers:
            bwd(L, stream)
    torch.cuda.synchronize()
    steps = 200
    main = plan(bwd, steps, layers, stream)
    with torch.cuda.stream(stream):
        run_graphs(main)
    torch.cuda.synchronize()
    med, lo, hi, ts = timed_repeats(main, world, stream, args.repeats)
    for L in layers:
        if sas.get_device_status(L["ws"], stream) != sas.SAS_OK:
            raise RuntimeError("device status not OK after the backward run")
    del layers, main
    torch.cuda.empty_cache()
    G = HQ // HKV
    kv_bytes = BATCH * HKV * (BUDGET // 64) * 64 * 128 * 2 * 2
    dbytes = (kv_bytes + HQ * 128 * 128 * 2 + HKV * 384 * 128 * 2 + 2 * BATCH * HQ * 128 * 2
              + HQ * 128 * 128 * 4 + HKV * 384 * 128 * 4)
    call_s = med / steps
    peak, peak_kind = measured_peaks()
    return {"workload": f"{WORKLOAD} gated-mode gradient (W_q, W_k, gains)", "steps": steps,
            "value": round(job_throughput(steps, world, med), 2), "unit": "backward steps/s",
            "ms_per_step": round(call_s * 1e3, 5), "timing": spread(ts, steps),
            "roofline": dict(roofline_of(dbytes, call_s, peak, peak_kind),
                             kernel="gate_backward_kernel + gate_grad_reduce_kernel (sas_gate_backward)")}


def run_prefill_backward(args, device, world):
    """Gradient through the gates of the gated prefill (Qwen3-8B heads, batch
    --prefill-batch x 32,768 tokens, Top-K 31 + diagonal): one
    sas_prefill_gate_backward call per step over the block lists of a gated
    forward call, with a seeded upstream gradient.  Tensor FLOPs counted like
    the forward's: per tile pair 2*64*64*128 for q K^T and as much for
    dout V^T."""
    import torch
    from gated_block_sparse_token_b200 import sas
    from gated_block_sparse_token_b200.workloads import make_prefill_inputs, qwen3_8b_prefill_32k

    spec = qwen3_8b_prefill_32k(batch=args.prefill_batch)
    inp = make_prefill_inputs(spec, device)
    B, T = spec.batch, spec.seq_len
    nblk = T // 64
    cfg = sas.Config(spec.hq, spec.hkv, token_budget=spec.token_budget, gate_mode=sas.GATE_LOGSIGMOID_BIAS)
    ws = sas.make_workspace(cfg, device, batch=B, max_seq_len=T)
    gk = torch.zeros(B, spec.hkv, nblk, 128, dtype=torch.float32, device=device)
    out = torch.empty(B, spec.hq, T, 128, dtype=torch.bfloat16, device=device)
    sel = torch.zeros(B, spec.hkv, nblk, cfg.max_sel, dtype=torch.int32, device=device)
    cnt = torch.zeros(B, spec.hkv, nblk, dtype=torch.int32, device=device)
    d_out = torch.randn(B, spec.hq, T, 128, generator=torch.Generator(device=device).manual_seed(12), device=device)
    grads = [torch.zeros(spec.hq, 128, 128, device=device), torch.zeros(spec.hkv, 384, 128, device=device),
             torch.zeros(128, device=device), torch.zeros(128, device=device)]
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        sas.prefill_block_sparse(cfg, inp["q"], inp["k"], inp["v"], inp["w_q"], inp["gamma_q"], inp["w_k"],
                                 inp["gamma_k"], gk, out, ws, sel_idx=sel, sel_count=cnt, stream=stream)

    def call():
        sas.prefill_gate_backward(cfg, inp["q"], inp["k"], inp["v"], inp["w_q"], inp["gamma_q"], inp["w_k"],
                                  inp["gamma_k"], gk, sel, cnt, d_out, *grads, ws, stream=stream)

    with torch.cuda.stream(stream):
        call()
    torch.cuda.synchronize()
    steps = max(1, args.prefill_steps)
    ts = []
    for _ in range(max(3, min(args.repeats, 7))):
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps):
                call()
            e1.record(stream)
        torch.cuda.synchronize()
        ts.append(max_over_ranks(e0.elapsed_time(e1) / 1e3 / steps, world))
    if sas.get_device_status(ws, stream) != sas.SAS_OK:
        raise RuntimeError("device status not OK after the prefill backward run")
    del inp, out, d_out, grads, ws
    torch.cuda.empty_cache()
    t = statistics.median(ts)
    flops = prefill_flops(nblk, spec.hq, spec.hkv, spec.token_budget, B)
    peak, kind = measured_tensor_peak()
    return {"workload": f"{spec.name} gated-mode gradient (W_q, W_k, gains)", "batch_per_gpu": B,
            "calls_per_repeat": steps, "ms_per_step": round(t * 1e3, 4),
            "timing": {"repeats": len(ts), "median_ms": round(t * 1e3, 4), "min_ms": round(min(ts) * 1e3, 4),
                       "max_ms": round(max(ts) * 1e3, 4)},
            "roofline": {"kernel": "prefill_bwd_attn_kernel (mma.sync) + key, reduction kernels",
                         "bound": "tensor", "achieved": round(flops / t / 1e12, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(flops / t / 1e12 / peak, 4), "peak_kind": kind,
                         "flops_per_step": flops}}


def run_pooling(args, device, world):
    """Pooled keys and gate keys of a whole prefill-shaped cache (the Qwen3-8B
    head layout, batch 4 x 32,768 tokens, 8 KV heads: 16,384 blocks) in one
    sas_pool_keys call: each block's K is read once, [max; min; mean] pooled,
    projected by W_k on the tensor cores, normalised, rotated and stored.
    Algorithmic bytes: K once, the gate keys written, W_k once per KV head."""
    import torch
    from gated_block_sparse_token_b200 import sas
    from gated_block_sparse_token_b200.workloads import make_prefill_inputs, qwen3_8b_prefill_32k

    spec = qwen3_8b_prefill_32k(batch=args.prefill_batch)
    inp = make_prefill_inputs(spec, device)
    B, T = spec.batch, spec.seq_len
    nblk = T // 64
    cfg = sas.Config(spec.hq, spec.hkv, token_budget=spec.token_budget)
    lens = torch.full((B,), T, dtype=torch.int32, device=device)
    # two copies of the cache alternate, so the timed calls read K from HBM
    caches = [inp["k"], inp["k"].clone()]
    kvs = [sas.KvCache(k, inp["v"], lens) for k in caches]
    gk = torch.zeros(B, spec.hkv, nblk, 128, dtype=torch.float32, device=device)
    ws = sas.make_workspace(cfg, device)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for kv in kvs:
            sas.pool_keys(cfg, kv, inp["w_k"], inp["gamma_k"], gk, ws, stream=stream)
    torch.cuda.synchronize()
    n = 20
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            sas.pool_keys(cfg, kvs[i % 2], inp["w_k"], inp["gamma_k"], gk, ws, stream=stream)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    med, lo, hi, ts = timed_repeats([(g, 1)], world, stream, args.repeats)
    if sas.get_device_status(ws, stream) != sas.SAS_OK:
        raise RuntimeError("device status not OK after the pooling run")
    del g, kvs, caches
    torch.cuda.empty_cache()
    dbytes = B * spec.hkv * T * 128 * 2 + B * spec.hkv * nblk * 128 * 4 + spec.hkv * 384 * 128 * 2
    call_s = med / n
    peak, peak_kind = measured_peaks()
    return {"workload": f"{spec.name} (all {B * spec.hkv * nblk} blocks)", "calls": n,
            "ms_per_call": round(call_s * 1e3, 4), "timing": spread(ts, n),
            "roofline": dict(roofline_of(dbytes, call_s, peak, peak_kind),
                             kernel="pool_project_kernel (tcgen05 projection)")}


# the sources the fused decode kernel is built and launched from (its ncu
# counters stay valid while the code in these does not change)
DECODE_SOURCES = ("sas_api.cu", "sas_decode.cu", "sas_device.cuh", "sas_internal.h", "sas_select.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def code_only(text):
    """C++ source without its comments, trailing blanks and empty lines, so
    that a comment edit leaves the digest alone."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def source_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_block_sparse_token_b200", "csrc")
    for f in DECODE_SOURCES:
        with open(os.path.join(csrc, f)) as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the
    fused decode kernel on `workload`, from the ncu capture recorded in the
    traffic data file, if that capture was taken on the current kernel
    sources; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f).get(workload)
    if not rec or rec.get("source_digest") != source_digest():
        return None
    return float(rec["dram_bytes_per_launch"])


# ---------------------------------------------------------------- our arm
def build_layers(R, rank, device, gate_mode=0, budgets=None, gk16=0):
    import torch
    from gated_block_sparse_token_b200 import sas
    from gated_block_sparse_token_b200.workloads import make_decode_inputs, qwen3_4b_32k

    cfg = sas.Config(HQ, HKV, token_budget=BUDGET if budgets is None else max(budgets), gate_mode=gate_mode,
                     gate_keys_bf16=gk16, static_weights=1)
    tb = None if budgets is None else torch.tensor(budgets, dtype=torch.int32, device=device)
    layers = []
    lens = None  # one length vector for every layer, as in a model's decode step
    for li in range(R):
        spec = qwen3_4b_32k(batch=BATCH, seq_len=CTX, seed=1000 * (rank + 1) + li)
        inp = make_decode_inputs(spec, device)
        if lens is None:
            lens = inp["seq_lens"]
        inp["seq_lens"] = lens
        kv = sas.KvCache(inp["k"], inp["v"], inp["seq_lens"], token_budgets=tb)
        mg = spec.cap // 64
        gk = torch.zeros(BATCH, HKV, mg, 128, dtype=sas.gate_key_dtype(cfg), device=device)
        ws = sas.make_workspace(cfg, device)
        sas.pool_keys(cfg, kv, inp["w_k"], inp["gamma_k"], gk, ws)  # prefill-time keys (untimed)
        cur = torch.full((BATCH,), (CTX - 1) // 64, dtype=torch.int32, device=device)
        out = torch.empty(BATCH, HQ, 128, dtype=torch.bfloat16, device=device)
        layers.append(dict(inp=inp, kv=kv, gk=gk, ws=ws, cur=cur, out=out))
    return cfg, layers


def step(cfg, L, stream=None, q=None):
    """One decode step of one layer: a single fused launch that gates, selects,
    attends and pools the block the decoded token completes."""
    from gated_block_sparse_token_b200 import sas
    inp = L["inp"]
    sas.decode_step(cfg, inp["q"] if q is None else q, L["kv"], inp["w_q"], inp["gamma_q"], L["gk"],
                    L["out"], L["ws"], w_k=inp["w_k"], gamma_k=inp["gamma_k"], stream=stream)


def capture(fn, n, layers, stream, offset=0):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fn(layers[(offset + i) % len(layers)], stream)
    return g


def run_graphs(graphs_plan):
    for g, reps in graphs_plan:
        for _ in range(reps):
            g.replay()


def plan(fn, K, layers, stream, chunk=512):
    """Graphs that replay exactly K steps (rotating over the layers)."""
    R = len(layers)
    chunk = max(R, (min(chunk, K) // R) * R) if K >= R else K
    out = []
    if K // chunk:
        out.append((capture(fn, chunk, layers, stream), K // chunk))
    rem = K - (K // chunk) * chunk
    if rem:
        out.append((capture(fn, rem, layers, stream), 1))
    return out


def timed(graphs, world, stream):
    """Device time of replaying `graphs` once (CUDAGraph.replay launches on the
    current stream, so replays and events both go to `stream`), bracketed by a
    barrier and a device synchronisation on both sides; max over ranks."""
    import torch
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        run_graphs(graphs)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1) / 1e3, world)


def timed_repeats(graphs, world, stream, repeats):
    """`repeats` timed replays of the same K-step graphs: (median, min, max)
    seconds of one replay, and the list."""
    ts = [timed(graphs, world, stream) for _ in range(repeats)]
    return statistics.median(ts), min(ts), max(ts), ts


def spread(ts, steps):
    """Per-step microseconds of the repeats: median, min and max."""
    return {"repeats": len(ts), "median_us": round(statistics.median(ts) / steps * 1e6, 3),
            "min_us": round(min(ts) / steps * 1e6, 3), "max_us": round(max(ts) / steps * 1e6, 3)}


MIXED_BUDGETS = [1024, 2048, 4096, 2048, 1024, 4096, 2048, 2048]


def roofline_of(dbytes, dec_s, peak, peak_kind):
    achieved = dbytes / dec_s / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
            "bytes_per_launch": int(round(dbytes)), "avg_launch_us": round(dec_s * 1e6, 3)}


def run_long_context(args, rank, world, device, layers=2):
    """Long-context decode as an incremental run: the Qwen3-14B layer (40 query
    / 8 KV heads), batch 16, 64-token pages behind a random block table,
    budget 4,096.  The gate keys are pooled for the first 131,072 - 256
    tokens; then 256 decode steps each add one token to every sequence
    (step t decodes at length 130,816 + t + 1, the token's K/V already in its
    page) and the fused step pools a block exactly when its token completes
    it (4 of the 256 steps).  Every layer decodes every token, as in a model;
    two layers of 8.6 GB caches alternate (far above L2)."""
    import torch
    from gated_block_sparse_token_b200 import sas
    from gated_block_sparse_token_b200.workloads import make_decode_inputs, qwen3_14b_paged_128k
    spec0 = qwen3_14b_paged_128k()
    n_app = spec0.appended
    full = spec0.seq_lens[0]
    start = full - n_app
    cfg = sas.Config(spec0.hq, spec0.hkv, token_budget=4096, static_weights=1)
    Ls = []
    # one length vector per appended token, shared by the layers
    lens = [torch.full((spec0.batch,), start + t + 1, dtype=torch.int32, device=device) for t in range(n_app)]
    for li in range(layers):
        spec = qwen3_14b_paged_128k(seed=2000 * (rank + 1) + li)
        inp = make_decode_inputs(spec, device)
        inp["seq_lens"] = torch.full((spec.batch,), start, dtype=torch.int32, device=device)
        kv = sas.KvCache(inp["k"], inp["v"], inp["seq_lens"], inp["block_table"])
        gk = torch.zeros(spec.batch, spec.hkv, spec.cap // 64, 128, dtype=torch.float32, device=device)
        ws = sas.make_workspace(cfg, device)
        sas.pool_keys(cfg, kv, inp["w_k"], inp["gamma_k"], gk, ws)    # the prompt's blocks (untimed)
        out = torch.empty(spec.batch, spec.hq, 128, dtype=torch.bfloat16, device=device)
        kvs = [sas.KvCache(inp["k"], inp["v"], ln, inp["block_table"]) for ln in lens]
        Ls.append(dict(inp=inp, kvs=kvs, gk=gk, ws=ws, out=out))
    stream = torch.cuda.Stream(device)

    def one_pass():
        for t in range(n_app):
            for L in Ls:
                inp = L["inp"]
                sas.decode_step(cfg, inp["q"], L["kvs"][t], inp["w_q"], inp["gamma_q"], L["gk"], L["out"],
                                L["ws"], w_k=inp["w_k"], gamma_k=inp["gamma_k"], stream=stream)

    with torch.cuda.stream(stream):
        one_pass()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_pass()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    med, lo, hi, ts = timed_repeats([(g, 1)], world, stream, args.repeats)
    for L in Ls:
        if sas.get_device_status(L["ws"], stream) != sas.SAS_OK:
            raise RuntimeError("device status not OK after the long-context run")
    del Ls, g
    torch.cuda.empty_cache()
    peak, peak_kind = measured_peaks()
    steps = n_app * layers
    dbytes = sum(decode_bytes([start + t + 1] * spec0.batch, spec0.hq, spec0.hkv, 4096) for t in range(n_app)) / n_app
    dec_s = med / steps
    return {"mode": "long context, incremental", "workload": "qwen3_14b_paged_b16_128k_budget4096",
            "protocol": f"{n_app} appended tokens x {layers} layers per timed pass, pooling at block completion",
            "steps": steps, "value": round(job_throughput(steps, world, med), 2), "unit": UNIT,
            "ms_per_step": round(dec_s * 1e3, 5), "timing": spread(ts, steps),
            "roofline": roofline_of(dbytes, dec_s, peak, peak_kind)}


def run_ragged(args, rank, world, device, layers=2):
    """The Qwen3-8B ragged layer: batch 32, contexts uniform in [8,192,
    65,536] (step 64), 32 query / 8 KV heads, at budgets 1,024, 2,048 and
    4,096 with the same caches and gate keys.  Two layers of 8.6 GB caches
    alternate."""
    import torch
    from gated_block_sparse_token_b200 import sas
    from gated_block_sparse_token_b200.workloads import make_decode_inputs, qwen3_8b_ragged
    Ls = []
    spec0 = qwen3_8b_ragged()
    lens = None
    for li in range(layers):
        spec = qwen3_8b_ragged(seed=3000 * (rank + 1) + li)
        spec.seq_lens = spec0.seq_lens          # one length vector for every layer
        inp = make_decode_inputs(spec, device)
        if lens is None:
            lens = inp["seq_lens"]
        inp["seq_lens"] = lens
        kv = sas.KvCache(inp["k"], inp["v"], inp["seq_lens"])
        gk = torch.zeros(spec.batch, spec.hkv, spec.cap // 64, 128, dtype=torch.float32, device=device)
        cfg0 = sas.Config(spec.hq, spec.hkv, token_budget=4096)
        ws = sas.make_workspace(cfg0, device)
        sas.pool_keys(cfg0, kv, inp["w_k"], inp["gamma_k"], gk, ws)
        out = torch.empty(spec.batch, spec.hq, 128, dtype=torch.bfloat16, device=device)
        Ls.append(dict(inp=inp, kv=kv, gk=gk, ws=ws, out=out))
    stream = torch.cuda.Stream(device)
    peak, peak_kind = measured_peaks()
    res = []
    for budget in (1024, 2048, 4096):
        cfg = sas.Config(spec0.hq, spec0.hkv, token_budget=budget, static_weights=1)
        fn = lambda L, st: step(cfg, L, st)  # noqa: E731
        with torch.cuda.stream(stream):
            for L in Ls:
                step(cfg, L, stream)
        torch.cuda.synchronize()
        warm = plan(fn, 8 * layers, Ls, stream)
        main = plan(fn, args.variant_steps, Ls, stream)
        with torch.cuda.stream(stream):
            run_graphs(warm)
        torch.cuda.synchronize()
        med, lo, hi, ts = timed_repeats(main, world, stream, args.repeats)
        for L in Ls:
            if sas.get_device_status(L["ws"], stream) != sas.SAS_OK:
                raise RuntimeError(f"device status not OK after the ragged run at budget {budget}")
        del main, warm
        dbytes = decode_bytes(spec0.seq_lens, spec0.hq, spec0.hkv, budget)
        dec_s = med / args.variant_steps
        res.append({"mode": f"ragged contexts, budget {budget}", "workload": f"qwen3_8b_ragged_b32_8k_64k_budget{budget}",
                    "token_budget": budget, "steps": args.variant_steps,
                    "value": round(job_throughput(args.variant_steps, world, med), 2), "unit": UNIT,
                    "ms_per_step": round(dec_s * 1e3, 5), "timing": spread(ts, args.variant_steps),
                    "roofline": roofline_of(dbytes, dec_s, peak, peak_kind)})
    del Ls
    torch.cuda.empty_cache()
    return res


def run_variant(args, rank, world, device, name, gate_mode=0, budgets=None, gk16=0):
    """The same decode workload in one of the widened modes (the gated
    inference mode, mixed per-sequence budgets, bf16 gate keys), timed like
    the main line on a shorter run; reports steps/s and the kernel's HBM
    roofline."""
    import torch
    from gated_block_sparse_token_b200 import sas
    cfg, layers = build_layers(args.layers, rank, device, gate_mode=gate_mode, budgets=budgets, gk16=gk16)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for L in layers:
            step(cfg, L, stream)
    torch.cuda.synchronize()
    fn = lambda L, st: step(cfg, L, st)  # noqa: E731
    warm = plan(fn, max(args.warmup, 3 * len(layers)), layers, stream)
    main = plan(fn, args.variant_steps, layers, stream)
    with torch.cuda.stream(stream):
        run_graphs(warm)
    torch.cuda.synchronize()
    med, lo, hi, ts = timed_repeats(main, world, stream, args.repeats)
    for L in layers:
        if sas.get_device_status(L["ws"], stream) != sas.SAS_OK:
            raise RuntimeError(f"device status not OK after the {name} run")
    del layers, main, warm
    torch.cuda.empty_cache()
    peak, peak_kind = measured_peaks()
    dbytes = decode_bytes([CTX] * BATCH, HQ, HKV, budgets if budgets is not None else BUDGET,
                          gk_elem=2 if gk16 else 4)
    dec_s = med / args.variant_steps
    return {"mode": name, "token_budgets": budgets if budgets is not None else [BUDGET] * BATCH,
            "gate_mode": gate_mode, "gate_keys": "bf16" if gk16 else "fp32", "steps": args.variant_steps,
            "value": round(job_throughput(args.variant_steps, world, med), 2), "unit": UNIT,
            "ms_per_step": round(dec_s * 1e3, 5), "timing": spread(ts, args.variant_steps),
            "roofline": roofline_of(dbytes, dec_s, peak, peak_kind)}


def cpu_baseline(seconds, all_cores_workers=None):
    """The oracle as it stands, single-threaded, on a bounded sample of the
    workload: whole decode steps (all 64 (sequence, KV head) pairs); plus the
    same over the host's cores (independent pairs in spawned processes)."""
    r = reference_sample(seconds_budget=seconds)
    out = {"value": r["value"], "unit": UNIT, "cores": 1, "kind": "oracle", "sample": r["sample"]}
    if all_cores_workers != 0:
        try:
            out["all_cores"] = cpu_baseline_all_cores(seconds, all_cores_workers)
        except Exception as e:  # an auxiliary figure: report why it is missing, keep the line
            out["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    return out


def _oracle_worker(job):
    seconds, h = job
    r = reference_sample(seconds_budget=seconds, heads=(h,), whole_steps=False)
    return r["pairs"], r["elapsed"]


def cpu_baseline_all_cores(seconds, workers=None, max_workers=32):
    """Oracle decode steps on every host core at once: one spawned process per
    core (at most max_workers, each ~0.3 GB), each timing its own KV head's
    pairs single-threaded; steps/s = pairs per second over all of them / 64.
    Runs before any CUDA use of the parent process."""
    import multiprocessing as mp
    n = workers or min(os.cpu_count() or 1, max_workers)
    with mp.get_context("spawn").Pool(n) as pool:  # leaving the block terminates the workers
        job = pool.map_async(_oracle_worker, [(seconds, i % HKV) for i in range(n)])
        res = job.get(timeout=3 * seconds + 180)  # a worker lost to the OOM killer would hang map()
    rate = sum(p / e for p, e in res)
    pairs = sum(p for p, _ in res)
    return {"value": rate / (BATCH * HKV), "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": f"{pairs} (sequence, KV head) decode steps in {n} processes of {seconds:.0f} s each, "
                      f"1 thread each; a full step is {BATCH * HKV} pairs"}


def run_ours(args):
    import torch
    from gated_block_sparse_token_b200 import sas

    rank, world, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    if args.prefill_only:
        pf = run_prefill(args, device, world)
        if rank == 0:
            print(json.dumps({"impl": "ours", "prefill": pf}), flush=True)
        return
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)   # before any pool could fork after CUDA use
    cfg, layers = build_layers(args.layers, rank, device)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for L in layers:       # first calls (one-time set-up) outside capture
            step(cfg, L, stream)
    torch.cuda.synchronize()

    fn = lambda L, st: step(cfg, L, st)  # noqa: E731
    warm = plan(fn, args.warmup, layers, stream)
    main = plan(fn, args.steps, layers, stream)
    with torch.cuda.stream(stream):
        run_graphs(warm)
    torch.cuda.synchronize()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    # every repeat times exactly K steps (barrier + synchronize on both sides);
    # the line reports the median repeat
    t, t_min, t_max, ts = timed_repeats(main, world, stream, args.repeats)
    clocks = clk.stop()
    for L in layers:
        if sas.get_device_status(L["ws"], stream) != sas.SAS_OK:
            raise RuntimeError("device status not OK after the timed run")

    # the step is one launch of the fused kernel: its average duration is the
    # step time measured above
    t_dec = t

    # end to end through the public API: each step is one call of the
    # host-buffer entry, which enqueues the copy of that step's q from pinned
    # host memory, the fused step and the copy of its output back to pinned
    # host memory
    from gated_block_sparse_token_b200 import sas
    R = len(layers)
    q_host = [L["inp"]["q"].cpu().pin_memory() for L in layers]
    out_host = [torch.empty(BATCH, HQ, 128, dtype=torch.bfloat16).pin_memory() for _ in range(R)]
    q_dev = torch.empty_like(layers[0]["inp"]["q"])
    out_dev = torch.empty_like(layers[0]["out"])
    ke = args.e2e_steps

    def e2e_loop(n):
        for i in range(n):
            L = layers[i % R]
            inp = L["inp"]
            sas.decode_step_host(cfg, q_host[i % R], q_dev, L["kv"], inp["w_q"], inp["gamma_q"], L["gk"], out_dev,
                                 out_host[i % R], L["ws"], w_k=inp["w_k"], gamma_k=inp["gamma_k"], stream=stream)

    with torch.cuda.stream(stream):
        e2e_loop(min(50, ke))
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_loop(ke)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)

    del layers, main, warm
    torch.cuda.empty_cache()
    variants = []
    if not args.skip_variants:
        variants.append(run_variant(args, rank, world, device, "gated (log-sigmoid bias)", gate_mode=1))
        variants.append(run_variant(args, rank, world, device, "mixed budgets", budgets=MIXED_BUDGETS))
        variants.append(run_variant(args, rank, world, device, "bf16 gate keys", gk16=1))
        variants.extend(run_ragged(args, rank, world, device))
        variants.append(run_long_context(args, rank, world, device))
    bwd = None if args.skip_variants else run_backward(args, rank, world, device)
    pf = None if args.skip_prefill else run_prefill(args, device, world)
    pool = None if args.skip_prefill else run_pooling(args, device, world)
    pf_bwd = None if (args.skip_prefill or args.skip_variants) else run_prefill_backward(args, device, world)

    if rank != 0:
        return
    peak, peak_kind = measured_peaks()
    dbytes = decode_bytes([CTX] * BATCH, HQ, HKV, BUDGET)
    dec_s = t_dec / args.steps
    achieved = dbytes / dec_s / 1e9
    step_s = t / args.steps
    value = job_throughput(args.steps, world, t)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal K/V with per-block offsets, random-init gate weights)",
        "config": {"workload": WORKLOAD, "batch_per_gpu": BATCH, "q_heads": HQ, "kv_heads": HKV,
                   "head_dim": 128, "context": CTX, "token_budget": BUDGET,
                   "layers_rotated": args.layers,
                   "l2": f"inputs larger than L2: {args.layers} layer caches rotated, "
                         f"{args.layers * dbytes / 1e6:.0f} MB touched per rotation",
                   "parallelism": f"replicas x{world} (independent batches)"},
        "hbm_gbs_step": round(dbytes / step_s / 1e9, 1),
        "timing": spread(ts, args.steps),
        "roofline": {"kernel": "decode_cluster_kernel (sas_decode_step)", "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
                     "bytes_per_launch": dbytes, "avg_launch_us": round(dec_s * 1e6, 3),
                     "traffic": profiled_traffic(WORKLOAD)},
        "e2e": {"value": round(job_throughput(ke, world, t_e2e), 2), "unit": UNIT,
                "h2d_bytes_per_step": BATCH * HQ * 128 * 2, "d2h_bytes_per_step": BATCH * HQ * 128 * 2,
                "call": "sas.decode_step_host (C-ABI sas_decode_step_host), pinned host q and out, one call per step"},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if variants:
        line["variants"] = variants
    if pf is not None:
        line["prefill"] = pf
    if pool is not None:
        line["pooling"] = pool
    if bwd is not None:
        line["gate_backward"] = bwd
    if pf_bwd is not None:
        line["prefill_gate_backward"] = pf_bwd
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- reference arm (CPU oracle)
def reference_sample(seconds_budget=None, steps=None, heads=None, whole_steps=True):
    """Time the oracle on the workload: one decode step of one (sequence, KV
    head) pair = pooling + gate key of the block the token completes, gate
    query, scores of the 511 historical blocks, Top-K and attention over the
    kept blocks.  The gate keys of the historical blocks are precomputed
    (untimed), as the GPU step also finds them in its cache.  The host holds
    one sequence's 8 KV heads (same shape and distributions as the batch's 8
    sequences) and a whole step runs its 64 pairs, each sequence slot reusing
    that data.  whole_steps: stop only at the end of a whole step (the
    all-cores workers count single pairs).  Only the oracle calls are timed."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from gated_block_sparse_token_b200.workloads import qwen3_4b_32k, make_decode_inputs, logical_kv
    from oracle import sas_oracle as O

    spec = qwen3_4b_32k(batch=1, seq_len=CTX, seed=1)
    inp = make_decode_inputs(spec, "cpu")
    G = HQ // HKV
    q = inp["q"].double().numpy()
    wq = inp["w_q"].double().numpy()
    wk = inp["w_k"].double().numpy()
    gq = np.tile(inp["gamma_q"].double().numpy(), (G, 1))
    gkn = inp["gamma_k"].double().numpy()
    c = (CTX - 1) // 64
    pairs = []
    for h in (range(HKV) if heads is None else heads):
        ks, vs = logical_kv(inp, 0, h, CTX)
        keys = O.gate_keys_for_sequence(ks, c, wk[h], gkn)
        pairs.append((h, ks, vs, keys))
    per_step = BATCH * HKV if whole_steps else 1
    done, step_times = 0, []
    el = 0.0
    with threadpool_limits(limits=1):
        while True:
            t0 = time.perf_counter()
            for _ in range(per_step):
                h, ks, vs, keys = pairs[done % len(pairs)]
                O.gate_key(O.pool_block(ks[64 * c:64 * c + 64]), wk[h], gkn, c)
                O.decode_one_group(q[0, h * G:(h + 1) * G], ks, vs, CTX, keys, wq[h * G:(h + 1) * G],
                                   gq, BUDGET)
                done += 1
            dt = time.perf_counter() - t0
            step_times.append(dt)
            el += dt
            n_steps = len(step_times)
            if (steps is not None and n_steps >= steps) or (seconds_budget is not None and el >= seconds_budget):
                break
    if whole_steps:
        med = statistics.median(step_times)
        value = 1.0 / med
        sample = (f"{len(step_times)} whole decode steps ({done} (sequence, KV head) pairs) of the "
                  f"workload in {el:.1f} s, 1 thread; per step median {med:.2f} s, min "
                  f"{min(step_times):.2f} s, max {max(step_times):.2f} s")
    else:
        value = done / el / (BATCH * HKV)
        sample = f"{done} (sequence, KV head) pairs in {el:.1f} s, 1 thread"
    return {"value": value, "elapsed": el, "pairs": done, "steps": len(step_times), "sample": sample}


def run_reference(args):
    """The reference arm: the CPU oracle on whole 64-pair decode steps of the
    workload (one warm-up step, then K steps or as many as fit in 150 s, so
    the run stays within a few minutes whatever K is; the count is stated)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    reference_sample(steps=1)
    r = reference_sample(steps=args.steps, seconds_budget=150.0)
    value = r["value"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": r["steps"],
        "warmup": 1, "ms_per_step": 1e3 / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": WORKLOAD, "batch_per_gpu": BATCH, "q_heads": HQ, "kv_heads": HKV,
                   "head_dim": 128, "context": CTX, "token_budget": BUDGET},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    run_ours(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
