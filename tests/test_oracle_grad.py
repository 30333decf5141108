"""Pins for the oracle's gradient through the gates (reading R20: in the gated
mode the continuous gates on the selected blocks give the gate parameters a
gradient; the Top-K set is held fixed).  Source: "Tencent released
Simple-Attention-Sparsification ..." (aigc.news, 2026-09-14), release
paragraph, and the second paragraph of the ai-news.nedoborov.com post of the
same day: the gates on the chosen blocks make the discrete Top-K selection
differentiable.

The analytic gradient is checked against central finite differences of the
forward functions (gate_keys_for_sequence, gate_scores,
attention_over_tokens) on tiny shapes, against a hand-derived closed form,
and planted mistakes in the backward are shown to fail."""
import math

import numpy as np
import pytest

from oracle import sas_oracle as O

SCALE = 1.0 / math.sqrt(128.0)


def _tiny(seed=3, L=64 * 6 + 9, G=2):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((L, 128))
    v = rng.standard_normal((L, 128))
    q = rng.standard_normal((G, 128))
    w_q = rng.standard_normal((G, 128, 128)) / math.sqrt(128)
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    g_q = 1.0 + 0.25 * rng.standard_normal(128)
    g_k = 1.0 + 0.25 * rng.standard_normal(128)
    d_out = rng.standard_normal((G, 128))
    return dict(q=q, k=k, v=v, L=L, w_q=w_q, w_k=w_k, g_q=g_q, g_k=g_k, d_out=d_out)


def _grads(t, budget=64 * 3, sel=None):
    return O.decode_gate_grads(t["q"], t["k"], t["v"], t["L"], t["w_q"], t["g_q"], t["w_k"], t["g_k"],
                               budget, t["d_out"], sel=sel)


def _loss(t, sel):
    return O.gated_decode_loss(t["q"], t["k"], t["v"], t["L"], t["w_q"], t["g_q"], t["w_k"], t["g_k"],
                               t["d_out"], sel)


def _fd(t, name, idx, sel, h=1e-5):
    arr = t[name]
    old = arr[idx]
    arr[idx] = old + h
    lp = _loss(t, sel)
    arr[idx] = old - h
    lm = _loss(t, sel)
    arr[idx] = old
    return (lp - lm) / (2 * h)


def test_gate_grads_match_finite_differences():
    t = _tiny()
    r = _grads(t)
    sel = r["sel"]
    assert len(sel) == 3 and sel[-1] == (t["L"] - 1) // 64
    # the forward inside the backward equals the plain gated forward
    G = t["q"].shape[0]
    keys = O.gate_keys_for_sequence(t["k"], (t["L"] - 1) // 64, t["w_k"], t["g_k"])
    fw = O.decode_one_group(t["q"], t["k"], t["v"], t["L"], keys, t["w_q"], np.tile(t["g_q"], (G, 1)),
                            64 * 3, gate_mode=O.GATE_LOGSIGMOID_BIAS)
    assert fw["sel"] == sel and np.allclose(fw["out"], r["out"], atol=1e-12)
    rng = np.random.default_rng(7)
    checks = {"w_q": ("dw_q", [tuple(rng.integers(0, [G, 128, 128])) for _ in range(10)]),
              "w_k": ("dw_k", [(int(rng.integers(0, 128)) + 128 * part, int(rng.integers(0, 128)))
                               for part in (0, 1, 2) for _ in range(4)]),
              "g_q": ("dgamma_q", [(int(i),) for i in rng.integers(0, 128, 8)]),
              "g_k": ("dgamma_k", [(int(i),) for i in rng.integers(0, 128, 8)])}
    for name, (gname, idxs) in checks.items():
        ga = r[gname]
        scale = float(np.max(np.abs(ga)))
        assert scale > 1e-6, f"{gname} is zero"
        for idx in idxs:
            want = _fd(t, name, idx, sel)
            got = float(ga[idx])
            assert abs(got - want) <= 1e-6 * max(abs(want), 1e-3 * scale), (gname, idx, got, want)


def test_gate_grads_closed_form():
    """Two heads, one historical block (keys a*e1), W_q = I, q_g = +-b e0, every
    attention logit 0 (the case of the gated forward's closed form):
    out_g = (w v0 + v1) / (w + 1), w = 64 sigmoid(s_g), so
    dL/ds_g = d_out_g . (v0 - v1) * 64 sigmoid(s_g)(1 - sigmoid(s_g)) / (w + 1)^2.
    s_g is linear in gamma_q[0] and in gamma_k[0] (all other gain entries
    meet zeros), so dL/dgamma_q[0] = dL/dgamma_k[0] = sum_g dL/ds_g s_g and
    every other gain entry has gradient 0."""
    a, b, L = 1.5, 2.0, 65
    rng = np.random.default_rng(3)
    k = np.zeros((L, 128))
    k[:64, 1] = a
    v = np.zeros((L, 128))
    v0, v1 = rng.standard_normal(128), rng.standard_normal(128)
    v[:64], v[64] = v0, v1
    w_k = np.zeros((384, 128))
    w_k[1, 0] = w_k[129, 0] = w_k[257, 0] = 1.0
    q = np.zeros((2, 128))
    q[0, 0], q[1, 0] = b, -b
    d_out = rng.standard_normal((2, 128))
    r = O.decode_gate_grads(q, k, v, L, np.stack([np.eye(128)] * 2), np.ones(128), w_k, np.ones(128),
                            2048, d_out)
    assert r["sel"] == [0, 1]
    kn = 3 * a / math.sqrt((3 * a) ** 2 / 128 + 1e-6)
    qn = b / math.sqrt(b ** 2 / 128 + 1e-6)
    s = np.array([1.0, -1.0]) * qn * math.cos(1.0) * kn * SCALE
    assert np.allclose(r["s"][:, 0], s, rtol=1e-12)
    ds = []
    for g in range(2):
        sig = 1.0 / (1.0 + math.exp(-s[g]))
        w = 64.0 * sig
        ds.append(float(np.dot(d_out[g], v0 - v1)) * 64.0 * sig * (1.0 - sig) / (w + 1.0) ** 2)
    assert np.allclose(r["ds"][:, 0], ds, rtol=1e-10, atol=1e-14)
    want0 = sum(ds[g] * s[g] for g in range(2))
    assert r["dgamma_q"][0] == pytest.approx(want0, rel=1e-10)
    assert r["dgamma_k"][0] == pytest.approx(want0, rel=1e-10)
    assert np.max(np.abs(r["dgamma_q"][1:])) < 1e-12 and np.max(np.abs(r["dgamma_k"][1:])) < 1e-12


def test_gradient_planted_mistakes(monkeypatch):
    good = O.log_sigmoid_grad
    monkeypatch.setattr(O, "log_sigmoid_grad", lambda x: 1.0 - good(x))   # sigmoid, not 1 - sigmoid
    with pytest.raises(AssertionError):
        test_gate_grads_closed_form()
    monkeypatch.setattr(O, "log_sigmoid_grad", good)

    good_rope = O.rope_backward
    monkeypatch.setattr(O, "rope_backward", lambda dy, pos, base=10000.0: O.rope_rotate_half(dy, pos, base))
    with pytest.raises(AssertionError):
        test_gate_grads_match_finite_differences()
    monkeypatch.setattr(O, "rope_backward", good_rope)

    good_rms = O.rms_norm_backward

    def rms_first_term_only(x, gamma, dy, eps=1e-6):
        dx, dg = good_rms(x, gamma, dy, eps)
        r = math.sqrt(float(np.mean(np.asarray(x) ** 2)) + eps)
        return np.asarray(gamma) * np.asarray(dy) / r, dg

    monkeypatch.setattr(O, "rms_norm_backward", rms_first_term_only)
    with pytest.raises(AssertionError):
        test_gate_grads_match_finite_differences()
    monkeypatch.setattr(O, "rms_norm_backward", good_rms)

    good_mm = O.matmul_weight_grad
    monkeypatch.setattr(O, "matmul_weight_grad", lambda x, dy: good_mm(x, dy).T if len(x) == len(dy) else good_mm(x, dy))
    with pytest.raises(AssertionError):
        test_gate_grads_match_finite_differences()
    monkeypatch.setattr(O, "matmul_weight_grad", good_mm)


def test_rms_norm_backward_matches_finite_differences():
    rng = np.random.default_rng(11)
    x, g, dy = rng.standard_normal(128), 1 + 0.3 * rng.standard_normal(128), rng.standard_normal(128)
    dx, dg = O.rms_norm_backward(x, g, dy)
    for i in (0, 5, 77, 127):
        e = np.zeros(128)
        e[i] = 1e-6
        fd = (np.dot(dy, O.rms_norm(x + e, g)) - np.dot(dy, O.rms_norm(x - e, g))) / 2e-6
        assert dx[i] == pytest.approx(fd, rel=1e-6, abs=1e-9)
        fdg = (np.dot(dy, O.rms_norm(x, g + e)) - np.dot(dy, O.rms_norm(x, g - e))) / 2e-6
        assert dg[i] == pytest.approx(fdg, rel=1e-6, abs=1e-9)


# ---------------------------------------------------------------- prefill shape
def _tiny_prefill(seed=5, T=256, G=2):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((T, 128))
    k += np.repeat(0.5 * rng.standard_normal((T // 64, 128)), 64, axis=0)  # distinct blocks
    v = rng.standard_normal((T, 128))
    q = rng.standard_normal((G, T, 128))
    w_q = rng.standard_normal((G, 128, 128)) / math.sqrt(128)
    w_k = rng.standard_normal((384, 128)) / math.sqrt(384)
    g_q = 1.0 + 0.25 * rng.standard_normal(128)
    g_k = 1.0 + 0.25 * rng.standard_normal(128)
    d_out = rng.standard_normal((G, T, 128))
    # fixed block lists (any ascending lists ending with the query block are
    # valid: the Top-K is held fixed); block 1 is chosen by two query blocks
    sels = [[0], [0, 1], [1, 2], [0, 1, 3]]
    return dict(q=q, k=k, v=v, w_q=w_q, w_k=w_k, g_q=g_q, g_k=g_k, d_out=d_out, sels=sels)


def _pf_grads(t):
    return O.prefill_gate_grads(t["q"], t["k"], t["v"], t["w_q"], t["g_q"], t["w_k"], t["g_k"], t["sels"],
                                t["d_out"])


def _pf_fd(t, name, idx, h=1e-5):
    arr = t[name]
    old = arr[idx]
    loss = lambda: O.gated_prefill_loss(t["q"], t["k"], t["v"], t["w_q"], t["g_q"], t["w_k"], t["g_k"],  # noqa: E731
                                        t["sels"], t["d_out"])
    arr[idx] = old + h
    lp = loss()
    arr[idx] = old - h
    lm = loss()
    arr[idx] = old
    return (lp - lm) / (2 * h)


def test_prefill_gate_grads_match_finite_differences():
    """Every parameter tensor of the prefill-shaped gradient against central
    differences of the gated prefill's loss (built from the forward
    functions), on 4 query blocks of 2 heads with block 1 kept by two query
    blocks (its gate key's gradient sums over both)."""
    t = _tiny_prefill()
    r = _pf_grads(t)
    checks = [("w_q", "dw_q", (0, 3, 5)), ("w_q", "dw_q", (1, 100, 7)), ("w_q", "dw_q", (1, 64, 64)),
              ("w_k", "dw_k", (2, 9)), ("w_k", "dw_k", (130, 0)), ("w_k", "dw_k", (300, 77)),
              ("g_q", "dgamma_q", (4,)), ("g_q", "dgamma_q", (90,)),
              ("g_k", "dgamma_k", (11,)), ("g_k", "dgamma_k", (127,))]
    for name, key, idx in checks:
        want = _pf_fd(t, name, idx)
        got = r[key][idx]
        assert abs(got - want) <= 1e-6 * max(1.0, abs(want)), (key, idx, got, want)
    # the forward part is the prefill the GPU is compared with
    for i in range(4):
        fwd = O.prefill_query_block(t["q"][:, 64 * i:64 * (i + 1)], t["k"], t["v"], i,
                                    O.gate_keys_for_sequence(t["k"], 4, t["w_k"], t["g_k"]), t["w_q"],
                                    np.tile(t["g_q"], (2, 1)), topk=len(t["sels"][i]) - 1,
                                    gate_mode=O.GATE_LOGSIGMOID_BIAS)
        if list(fwd["sel"]) == t["sels"][i]:
            assert np.allclose(fwd["out"], r["out"][:, 64 * i:64 * (i + 1)], atol=1e-12)


def test_prefill_gradient_planted_mistakes(monkeypatch):
    t = _tiny_prefill(seed=6)
    idx = (1, 100, 7)

    def fd_ok():
        return abs(_pf_grads(t)["dw_q"][idx] - _pf_fd(t, "w_q", idx)) <= 1e-6 * max(1.0, abs(_pf_fd(t, "w_q", idx)))

    assert fd_ok()
    good = O.log_sigmoid_grad
    monkeypatch.setattr(O, "log_sigmoid_grad", lambda x: 1.0 - good(x))
    assert not fd_ok()
    monkeypatch.setattr(O, "log_sigmoid_grad", good)
    good_rope = O.rope_backward
    monkeypatch.setattr(O, "rope_backward", lambda dy, pos, base=10000.0: O.rope_rotate_half(dy, pos, base))
    assert not fd_ok()
    monkeypatch.setattr(O, "rope_backward", good_rope)
