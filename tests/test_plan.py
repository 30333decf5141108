"""Host-side checks of the decode kernel's shared-memory plan (no GPU): every
TMA destination is aligned as the copy requires, regions that are live at the
same time do not overlap, and the remote writes of other CTAs (scores during
their phase 1, merge partials after their attention phase) never land on a
region this CTA may still be reading."""
import os
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_block_sparse_token_b200", "csrc")


@pytest.fixture(scope="module")
def plans():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "plan_check")
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "native", "plan_check.cu"), "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    rows = []
    for line in out.splitlines():
        rows.append({k: int(v) for k, v in (f.split("=") for f in line.split())})
    return rows


def test_plan_alignment_and_overlap(plans):
    CS, dpc = 8, 16
    assert len(plans) == 8 * 8 * 5 * 2 * 2
    for p in plans:
        G, mg, ms = p["G"], max(p["mg"], 1), p["budget"] // 64
        tag = str(p)
        assert p["ok"] == 1, tag
        assert p["slots"] % 1024 == 0 and p["r_wq"] % 128 == 0, tag
        assert p["qraw"] % 16 == 0 and p["gam"] % 16 == 0 and p["bars"] % 8 == 0, tag
        # fixed regions, in order, disjoint
        fixed = [("slots", 2 * 16384), ("sel", 4 * ms), ("rows", 8 * ((ms + 7) // 8)),
                 ("gbias", 4 * ms * G * p["gated"]),
                 ("qraw", G * 128 * (4 if p["f32"] else 2)), ("qbar", 512), ("pml", 256), ("gam", 512),
                 ("bars", 8 * (2 + 9))]
        for (a, sa), (b, _) in zip(fixed, fixed[1:]):
            assert p[a] + sa <= p[b], (tag, a, b)
        r = p["r_qv"]
        assert p["bars"] + 8 * (2 + 9) <= r, tag
        # phase 0-1 layout: qv then the W_q slice
        qv_end = r + G * 128 * 4
        assert qv_end <= p["r_wq"], tag
        # phase 2-4 layout: inbox first; select-only: over qv, covering it
        # entirely; gated mode: after qv, which every CTA reads for its gates
        # once the list is in (other CTAs' partials may land before that)
        inbox_end = p["r_inbox"] + CS * G * (dpc + 2) * 4
        if p["gated"]:
            assert p["r_inbox"] >= qv_end, tag
        else:
            assert p["r_inbox"] == r and inbox_end >= qv_end, tag
        # scores pushed by other CTAs during their phase 1 must not touch qv
        assert p["r_keys"] >= inbox_end and p["r_keys"] >= qv_end, tag
        assert p["r_hist"] >= p["r_keys"] + 4 * mg, tag
        assert p["r_selbits"] >= p["r_hist"] + 4 * 1024, tag
        assert p["r_scan"] >= p["r_selbits"] + 4 * ((mg + 31) // 32), tag
        # distributed Top-K: local keys, then the candidates other CTAs push
        # after their phase 1 (past the inbox and qv, clear of the local keys)
        assert p["r_lkeys"] >= inbox_end and p["r_lkeys"] >= qv_end, tag
        assert p["r_gather"] >= p["r_lkeys"] + 8 * 256, tag
        assert p["r_gather"] % 16 == 0 and p["r_lkeys"] % 16 == 0, tag
        assert p["wq_heads"] in (G, (G + 1) // 2), tag
        end = max(p["r_wq"] + p["wq_heads"] * 128 * dpc * 2, p["r_scan"] + 64,
                  p["r_gather"] + 8 * CS * 64)
        assert p["total"] >= end + 1024, tag


def test_w_q_in_two_passes_only_where_it_buys_the_fourth_cta(plans):
    four = 228 * 1024 // 4 - 1024
    for p in plans:
        if p["wq_heads"] < p["G"]:
            assert p["total"] <= four, p
    # Qwen3-14B, 128k context: G = 5, 2,048 gate-key rows, budget 4,096, bf16
    p = next(q for q in plans if q["G"] == 5 and q["mg"] == 2048 and q["budget"] == 4096 and q["f32"] == 0
             and q["gated"] == 0)
    assert p["wq_heads"] == 3 and p["total"] <= four, p
    # Qwen3-4B, 32k: one pass
    p = next(q for q in plans if q["G"] == 4 and q["mg"] == 512 and q["budget"] == 2048 and q["f32"] == 0
             and q["gated"] == 0)
    assert p["wq_heads"] == 4, p


def test_plan_fits_four_ctas_per_sm_at_the_benchmark_shape(plans):
    # Qwen3-4B, 32k context: G = 4, 512 gate-key rows, budget 2,048, bf16
    for gated in (0, 1):
        p = next(q for q in plans if q["G"] == 4 and q["mg"] == 512 and q["budget"] == 2048 and q["f32"] == 0
                 and q["gated"] == gated)
        assert 4 * (p["total"] + 1024) <= 228 * 1024


def test_prefill_attention_keeps_two_ctas_per_sm():
    """The block list and its gates sit beside the Q tile and the K/V rings:
    for lists up to 64 blocks (budgets to 4,096 tokens) two CTAs of the
    tcgen05 attention kernel must still fit in an SM's 228 KiB (1 KiB of it
    reserved per CTA); every accepted list (to 16,384 tokens) fits one."""
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "prefill_plan_check")
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "native", "prefill_plan_check.cu"), "-o", exe],
                       check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    sizes = [int(line.split("bytes=")[1]) for line in out.splitlines()]
    assert len(sizes) == 256   # lists of 1 .. 256 blocks (budgets to 16,384 tokens)
    # two CTAs per SM up to the 4,096-token budget, one beyond
    assert all(2 * (b + 1024) <= 228 * 1024 for b in sizes[:64]), max(sizes[:64])
    assert all(b <= 227 * 1024 for b in sizes), max(sizes)


def test_gate_backward_ring_fits_every_accepted_shape():
    """The gate backward (a cluster of two CTAs per pair, one CTA per SM)
    takes as many K/V ring stages as fit: every group of 1 to 8 heads and
    every list of up to 64 blocks (budgets to 4,096 tokens) gets at least one
    within 227 KiB, the benchmark shape (4 heads, 32 blocks) the full four,
    and the second CTA's hand-over (a pooled row of 384 floats per
    historical entry, 3 statistics per head and entry, for half the list)
    stays far inside an mbarrier's transaction count."""
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "bwd_plan_check")
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "native", "bwd_plan_check.cu"), "-o", exe],
                       check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    rows = [{k: int(v) for k, v in (f.split("=") for f in line.split())} for line in out.splitlines()]
    assert len(rows) == 8 * 64
    for r in rows:
        assert 1 <= r["stages"] <= 4 and r["bytes"] <= 227 * 1024, r
        m = r["max_sel"]
        handover = (m // 2) * 3 * r["G"] * 4 + (m // 2) * 384 * 4
        assert handover < (1 << 20) - 1
    bench = next(r for r in rows if r["G"] == 4 and r["max_sel"] == 32)
    assert bench["stages"] == 4
