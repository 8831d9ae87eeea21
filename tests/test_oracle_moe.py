"""Pins for the oracle's grouped MoE MLP (CPU only).

* the fp64 mode against torch autograd of an independent token-by-token
  formulation (forward value and every gradient);
* the MXFP8 mode against a token-by-token brute force (no permutation,
  no padding, no grouping);
* the quantisation axis of every GEMM operand, by directional exactness: an
  operand built to be exact under blocks along K but lossy across K must give
  the exact product, and the mirror construction must not;
* closeness of the MXFP8 and BF16 modes to the exact result, and exact zeros
  for the weight gradient of an expert with no tokens.
"""
import numpy as np
import pytest
import torch

from oracle import moe, mx
from mxfp8_quantize_b200 import workloads


def _tiny(T=24, d=64, f=64, E=4, k=2, seed=0, routing="uniform", empty=None, w_std=None):
    cfg = workloads.MoEConfig("tiny", T, d, f, E, k, "mxfp8", True, w_std, routing, seed, empty_expert=empty)
    inp = workloads.make_inputs(cfg)
    return cfg, {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in inp.items()}


def _torch_token_by_token(x, idx, prob, w1, w2, dy):
    x = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    w1 = torch.tensor(w1, dtype=torch.float64, requires_grad=True)
    w2 = torch.tensor(w2, dtype=torch.float64, requires_grad=True)
    p = torch.tensor(prob, dtype=torch.float64, requires_grad=True)
    f = w2.shape[2]
    rows = []
    for t in range(x.shape[0]):
        acc = 0
        for j in range(idx.shape[1]):
            e = int(idx[t, j])
            h = w1[e] @ x[t]
            a = torch.nn.functional.silu(h[:f]) * h[f:] * p[t, j]
            acc = acc + w2[e] @ a
        rows.append(acc)
    y = torch.stack(rows)
    (y * torch.tensor(dy, dtype=torch.float64)).sum().backward()
    return y.detach().numpy(), x.grad.numpy(), w1.grad.numpy(), w2.grad.numpy(), p.grad.numpy()


@pytest.mark.parametrize("seed,routing,empty", [(0, "uniform", None), (1, "zipf", 3), (2, "dirichlet", None)])
def test_fp64_matches_autograd(seed, routing, empty):
    cfg, inp = _tiny(seed=seed, routing=routing, empty=empty)
    y, st = moe.forward(inp["x"], inp["topk_idx"], inp["topk_prob"], inp["w_gate_up"], inp["w_down"], "fp64")
    g = moe.backward(inp["dy"], st, inp["w_gate_up"], inp["w_down"])
    ry, rdx, rdw1, rdw2, rdp = _torch_token_by_token(inp["x"], inp["topk_idx"], inp["topk_prob"],
                                                     inp["w_gate_up"], inp["w_down"], inp["dy"])
    for a, b in [(y, ry), (g["dx"], rdx), (g["dw_gate_up"], rdw1), (g["dw_down"], rdw2), (g["d_topk_prob"], rdp)]:
        assert np.max(np.abs(a - b)) <= 1e-10 * max(1.0, np.max(np.abs(b)))


def test_fp64_finite_difference_on_prob_and_weight():
    cfg, inp = _tiny(T=8, d=32, f=32, E=2, seed=3)
    dy = inp["dy"]

    def loss(x, prob, w1, w2):
        y, _ = moe.forward(x, inp["topk_idx"], prob, w1, w2, "fp64")
        return float(np.sum(y * dy))

    y, st = moe.forward(inp["x"], inp["topk_idx"], inp["topk_prob"], inp["w_gate_up"], inp["w_down"], "fp64")
    g = moe.backward(dy, st, inp["w_gate_up"], inp["w_down"])
    eps = 1e-6
    p = inp["topk_prob"].astype(np.float64)
    for (t, j) in [(0, 0), (5, 1)]:
        pp, pm = p.copy(), p.copy()
        pp[t, j] += eps
        pm[t, j] -= eps
        fd = (loss(inp["x"], pp, inp["w_gate_up"], inp["w_down"]) - loss(inp["x"], pm, inp["w_gate_up"], inp["w_down"])) / (2 * eps)
        assert fd == pytest.approx(g["d_topk_prob"][t, j], rel=1e-6, abs=1e-9)
    w2 = inp["w_down"].astype(np.float64)
    for (e, r_, c) in [(0, 3, 7), (1, 30, 0)]:
        wp, wm = w2.copy(), w2.copy()
        wp[e, r_, c] += eps
        wm[e, r_, c] -= eps
        fd = (loss(inp["x"], p, inp["w_gate_up"], wp) - loss(inp["x"], p, inp["w_gate_up"], wm)) / (2 * eps)
        assert fd == pytest.approx(g["dw_down"][e, r_, c], rel=1e-6, abs=1e-9)


def test_mxfp8_forward_matches_token_by_token_brute_force():
    cfg, inp = _tiny(T=40, d=64, f=96, E=4, seed=4, routing="zipf")
    x, idx, prob, w1, w2 = (inp[n] for n in ("x", "topk_idx", "topk_prob", "w_gate_up", "w_down"))
    y, _ = moe.forward(x, idx, prob, w1, w2, "mxfp8")
    f = w2.shape[2]
    w1q = [mx.fake_quant(w1[e], axis=1) for e in range(w1.shape[0])]   # blocks along d
    w2q = [mx.fake_quant(w2[e], axis=1) for e in range(w2.shape[0])]   # blocks along f
    ref = np.zeros_like(y)
    for t in range(x.shape[0]):
        xq = mx.fake_quant(x[t:t + 1], axis=1)
        acc = np.zeros((1, x.shape[1]), dtype=np.float32)
        for j in range(idx.shape[1]):
            e = idx[t, j]
            h = (xq @ w1q[e].T).astype(np.float32).astype(np.float64)
            a = (moe.silu(h[:, :f]) * h[:, f:] * float(prob[t, j])).astype(np.float32)
            aq = mx.fake_quant(a, axis=1)
            acc = acc + moe.bf16_round((aq @ w2q[e].T).astype(np.float32))
        ref[t] = moe.bf16_round(acc)[0]
    assert np.mean(y == ref) > 0.99
    assert np.max(np.abs(y - ref)) <= 2e-2 * np.max(np.abs(ref))


def _directional(rows, cols, exact_axis, seed):
    """A matrix whose MXFP8 quantisation is exact along ``exact_axis`` but lossy along the other.

    Each line along ``exact_axis`` is a fixed E4M3 pattern with a power-of-two
    scale of its own; lines differ by up to 2**24, so blocks taken across them
    flush the small lines to zero or round them.
    """
    rng = np.random.default_rng(seed)
    table = mx.e4m3_decode_table()
    codes = rng.integers(0, 0x7F, (rows, cols))
    if exact_axis == 0:
        codes[::32, :] = 0x7E
        scale = 2.0 ** rng.integers(-12, 12, (1, cols))
    else:
        codes[:, ::32] = 0x7E
        scale = 2.0 ** rng.integers(-12, 12, (rows, 1))
    sign = np.where(rng.integers(0, 2, (rows, cols)) == 1, -1.0, 1.0)
    return table[codes] * sign * scale


def test_gemm_quantises_each_operand_along_k():
    M, K, N = 64, 96, 64
    A = _directional(M, K, exact_axis=1, seed=1)       # exact in blocks along K (axis 1)
    B = _directional(K, N, exact_axis=0, seed=2)       # exact in blocks along K (axis 0)
    assert np.array_equal(moe.gemm(A, B, "mxfp8"), A @ B)
    A_bad = _directional(M, K, exact_axis=0, seed=3)   # exact only across K
    B_bad = _directional(K, N, exact_axis=1, seed=4)
    assert not np.allclose(moe.gemm(A_bad, B, "mxfp8"), A_bad @ B, rtol=1e-3, atol=0)
    assert not np.allclose(moe.gemm(A, B_bad, "mxfp8"), A @ B_bad, rtol=1e-3, atol=0)


@pytest.mark.parametrize("precision,tol", [("mxfp8", 0.1), ("bf16", 0.02)])
def test_quantised_modes_close_to_exact(precision, tol):
    cfg, inp = _tiny(T=64, d=128, f=128, E=4, seed=6)
    args = (inp["x"], inp["topk_idx"], inp["topk_prob"], inp["w_gate_up"], inp["w_down"])
    y0, s0 = moe.forward(*args, "fp64")
    g0 = moe.backward(inp["dy"], s0, inp["w_gate_up"], inp["w_down"])
    y1, s1 = moe.forward(*args, precision)
    g1 = moe.backward(inp["dy"], s1, inp["w_gate_up"], inp["w_down"])

    def rel(a, b):
        return np.linalg.norm(a - b) / np.linalg.norm(b)

    assert rel(y1, y0) < tol
    for n in ("dx", "dw_gate_up", "dw_down", "d_topk_prob"):
        assert rel(g1[n], g0[n]) < tol, n


def test_empty_expert_has_zero_weight_gradient():
    cfg, inp = _tiny(T=32, d=64, f=64, E=4, seed=7, routing="zipf", empty=2)
    assert not np.any(inp["topk_idx"] == 2)
    for precision in ("mxfp8", "bf16"):
        y, st = moe.forward(inp["x"], inp["topk_idx"], inp["topk_prob"], inp["w_gate_up"], inp["w_down"], precision)
        g = moe.backward(inp["dy"], st, inp["w_gate_up"], inp["w_down"])
        assert np.all(g["dw_gate_up"][2] == 0) and np.all(g["dw_down"][2] == 0)
        assert st["route"]["split_sizes"][2] == 0


def test_grouped_equals_loop_over_single_expert_calls():
    """Routing every token to one expert at a time reproduces the grouped result per expert."""
    cfg, inp = _tiny(T=32, d=64, f=64, E=3, k=1, seed=8)
    x, idx, prob, w1, w2 = (inp[n] for n in ("x", "topk_idx", "topk_prob", "w_gate_up", "w_down"))
    y, _ = moe.forward(x, idx, prob, w1, w2, "mxfp8")
    for e in range(3):
        tok = np.where(idx[:, 0] == e)[0]
        if tok.size == 0:
            continue
        ye, _ = moe.forward(x[tok], idx[tok] * 0, prob[tok], w1[e:e + 1], w2[e:e + 1], "mxfp8")
        assert np.array_equal(ye, y[tok])
