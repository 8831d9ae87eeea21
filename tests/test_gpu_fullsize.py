"""GPU parity at the full workload sizes (Mixtral-8x7B layer, and the 32768-token long sequence),
in the same fused calls the benchmark times, on outputs the oracle can compute one by one.

Why the sampled checks are exact restatements of the full oracle:
* every forward output row and every dgrad row depends only on its own token (row-wise
  quantisation, per-row epilogue), so the oracle run on a subset of one expert's slots gives
  exactly those rows of y_perm, h, dx_perm and the probability gradient;
* a 32-column slab of the ffn dimension depends only on the matching gate/up rows of W1 and
  columns of W2 (each slab is one whole MXFP8 block along f), so the oracle run on a one-expert,
  32-column sub-layer over all of that expert's tokens gives exactly those columns of dW2 and
  those rows of dW1;
* quantised operands and epilogue requantisations are checked bit-exactly on sampled rows and
  32-row blocks, the routing arrays in full.
"""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import mx, routing
from tests.gpu_util import has_b200, parity, unswizzle_scales
from mxfp8_quantize_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.slow, pytest.mark.skipif(not has_b200(), reason="needs a B200")]

import mxfp8_quantize_b200 as moe  # noqa: E402

TOL = {"mxfp8": 2e-2, "bf16": 1e-2}
N_ROWS = 128       # expert-0 slots whose rows are recomputed by the oracle
SLABS = (0, 5)     # 32-column ffn slabs whose weight gradients are recomputed


def _f(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


@pytest.fixture(scope="module", params=["mixtral_mxfp8", "mixtral_bf16", "longseq_mxfp8"])
def full(request):
    cfg = workloads.CONFIGS[request.param]
    prec = cfg.precision
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    cap = moe.capacity_rows(T, k, E)
    dims = (T, d, f, E, k, prec)
    sz = moe.sizes(T, d, f, E, k, prec, True)
    fws = torch.empty(sz["fwd_ws"], dtype=torch.uint8, device="cuda")
    bws = torch.empty(sz["bwd_ws"], dtype=torch.uint8, device="cuda")
    dump_a = torch.empty((cap, f), dtype=torch.float32, device="cuda")
    dump_dh = torch.empty((cap, 2 * f), dtype=torch.float32, device="cuda")
    moe.set_debug_dump(0, dump_a, dump_dh)
    try:
        y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                           dev["w_down"], precision=prec, training=True, workspace=fws)
        dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, dev["w_gate_up"], dev["w_down"], workspace=bws)
        moe.get_status(0)
    finally:
        moe.set_debug_dump(0, None, None)

    def view(buf, which, name, n, dtype=torch.uint8):
        return moe.buffer_view(buf, which, name, dims, True, n, dtype)

    route = routing.route(inp["topk_idx"].numpy(), E, 128, capacity=cap)
    poff = route["poffsets"]
    seg0 = slice(int(poff[0]), int(poff[0]) + N_ROWS)
    g = dict(cfg=cfg, prec=prec, route=route, cap=cap,
             y=_f(y), dx=_f(dx), dp=_f(dp), dw1_0=_f(dw1[0]), dw2_0=_f(dw2[0]),
             poffsets=_f(view(saved.buf, 0, "poffsets", E + 1, torch.int32)),
             sorted_to_src=_f(view(saved.buf, 0, "sorted_to_src", cap, torch.int32)),
             src_to_sorted=_f(view(saved.buf, 0, "src_to_sorted", T * k, torch.int32)),
             y_perm=_f(view(fws, 1, "y_perm", cap * d, torch.bfloat16).view(cap, d)),
             dx_perm=_f(view(bws, 2, "dx_perm", cap * d, torch.bfloat16).view(cap, d)),
             h0=_f(view(saved.buf, 0, "h", cap * 2 * f, torch.bfloat16).view(cap, 2 * f)[seg0]),
             a_dump=_f(dump_a[seg0]), dh_dump=_f(dump_dh[seg0]))
    if prec == "mxfp8":
        rows = seg0
        g["a_q"] = _f(view(fws, 1, "a_q", cap * f).view(cap, f)[rows])
        g["aT_q"] = _f(view(saved.buf, 0, "aT_q", f * cap).view(f, cap)[:, rows])
        g["dh_q"] = _f(view(bws, 2, "dh_q", cap * 2 * f).view(cap, 2 * f)[rows])
        g["dhT_q"] = _f(view(bws, 2, "dhT_q", 2 * f * cap).view(2 * f, cap)[:, rows])
        w1q = view(fws, 1, "w1_q", E * 2 * f * d).view(E * 2 * f, d)
        g["w1_q_rows"] = _f(w1q[:512])                       # 256 gate + 256 up rows of expert 0
        g["w1_s"] = _f(view(fws, 1, "w1_s", E * 2 * f * d // 32)[: 2 * (512 // 128) * (d // 128) * 512])
        g["w1c_q_rows"] = _f(view(saved.buf, 0, "w1c_q", E * d * 2 * f).view(E * d, 2 * f)[:64])
        g["x_q"] = _f(view(fws, 1, "x_q", cap * d).view(cap, d)[rows])
        g["xT_q"] = _f(view(saved.buf, 0, "xT_q", d * cap).view(d, cap)[:, rows])
        g["dy_q"] = _f(view(bws, 2, "dy_q", cap * d).view(cap, d)[rows])
    # host copies the oracle needs: activations, routing, and expert 0's weights
    g["np"] = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy())
               for n, t in inp.items() if n not in ("w_gate_up", "w_down")}
    g["np"]["w_gate_up"] = inp["w_gate_up"][0:1].float().numpy()
    g["np"]["w_down"] = inp["w_down"][0:1].float().numpy()
    del fws, bws, saved, dump_a, dump_dh, dev
    torch.cuda.empty_cache()
    return g


def _expert0_subset(g, n):
    """The first n slots of expert 0 as a one-expert, top-1 sub-problem (same slot order)."""
    r = g["route"]
    slots = r["sorted_to_src"][int(r["poffsets"][0]): int(r["poffsets"][0]) + n]
    assert np.all(slots >= 0)
    k = g["cfg"].k
    npi = g["np"]
    x = npi["x"][slots // k]
    dy = npi["dy"][slots // k]
    prob = npi["topk_prob"].reshape(-1)[slots][:, None]
    idx = np.zeros((n, 1), dtype=np.int32)
    return x, dy, prob, idx, slots


def test_full_routing_bit_exact(full):
    g, r = full, full["route"]
    assert np.array_equal(g["poffsets"], r["poffsets"])
    assert np.array_equal(g["sorted_to_src"], r["sorted_to_src"])
    assert np.array_equal(g["src_to_sorted"], r["src_to_sorted"])
    assert r["split_sizes"].sum() == g["cfg"].T * g["cfg"].k


def test_full_quantised_operands_bit_exact(full):
    g = full
    if g["prec"] != "mxfp8":
        pytest.skip("MXFP8 only")
    d, f = g["cfg"].d, g["cfg"].f
    w1 = g["np"]["w_gate_up"][0]
    # the row-wise copy of W1 interleaves 128 gate rows with the matching 128 up rows
    src = np.concatenate([w1[0:128], w1[f:f + 128], w1[128:256], w1[f + 128:f + 256]])
    rq, rs = mx.quantize_rowwise(src)
    assert np.array_equal(g["w1_q_rows"], rq)
    assert np.array_equal(unswizzle_scales(g["w1_s"], 512, d // 32), rs)
    # down the columns, transposed: row c of the copy is column c of W1 quantised along 2f
    assert np.array_equal(g["w1c_q_rows"], mx.quantize_colwise_t(w1[:, :64])[0])
    x, dy, prob, idx, slots = _expert0_subset(g, N_ROWS)
    assert np.array_equal(g["x_q"], mx.quantize_rowwise(x)[0])
    assert np.array_equal(g["xT_q"], mx.quantize_colwise_t(x)[0])
    assert np.array_equal(g["dy_q"], mx.quantize_rowwise(dy)[0])


def test_full_epilogue_requantisation_bit_exact(full):
    g = full
    if g["prec"] != "mxfp8":
        pytest.skip("MXFP8 only")
    assert np.array_equal(g["a_q"], mx.quantize_rowwise(g["a_dump"])[0])
    assert np.array_equal(g["aT_q"], mx.quantize_colwise_t(g["a_dump"])[0])
    assert np.array_equal(g["dh_q"], mx.quantize_rowwise(g["dh_dump"])[0])
    assert np.array_equal(g["dhT_q"], mx.quantize_colwise_t(g["dh_dump"])[0])


def test_full_expert0_rows_within_tolerance(full):
    g = full
    prec = g["prec"]
    name = g["cfg"].name
    x, dy, prob, idx, slots = _expert0_subset(g, N_ROWS)
    w1 = g["np"]["w_gate_up"][0:1]
    w2 = g["np"]["w_down"][0:1]
    y, st = omoe.forward(x, idx, prob, w1, w2, prec)
    gr = omoe.backward(dy, st, w1, w2)
    lo = int(g["route"]["poffsets"][0])
    rows = slice(lo, lo + N_ROWS)
    tol = TOL[prec]
    parity(f"{name}.y_perm", g["y_perm"][rows], y, tol)               # GEMM1 -> SwiGLU -> GEMM2 at K = d, f
    parity(f"{name}.h", g["h0"], st["h"][:N_ROWS], tol)
    parity(f"{name}.a", g["a_dump"], st["a"][:N_ROWS], tol)
    parity(f"{name}.dx_perm", g["dx_perm"][rows], gr["dx_perm"][:N_ROWS], tol)  # dgrad of down, dSwiGLU, dgrad of gate_up
    parity(f"{name}.dh", g["dh_dump"], gr["dh_perm"][:N_ROWS], tol)
    # probability gradient of those slots
    parity(f"{name}.d_topk_prob", g["dp"].reshape(-1)[slots], gr["d_topk_prob"][:, 0], tol)


@pytest.mark.parametrize("slab", SLABS)
def test_full_wgrad_slabs_within_tolerance(full, slab):
    g = full
    prec, f = g["prec"], g["cfg"].f
    r = g["route"]
    m0 = int(r["split_sizes"][0])
    x, dy, prob, idx, slots = _expert0_subset(g, m0)
    c0 = 32 * slab
    w1 = g["np"]["w_gate_up"][0]
    w1s = np.concatenate([w1[c0:c0 + 32], w1[f + c0:f + c0 + 32]])[None]   # [1, 64, d]
    w2s = g["np"]["w_down"][0][:, c0:c0 + 32][None]                          # [1, d, 32]
    _, st = omoe.forward(x, idx, prob, w1s, w2s, prec)
    gr = omoe.backward(dy, st, w1s, w2s)
    name, tol = g["cfg"].name, TOL[prec]
    parity(f"{name}.dw_down[slab {slab}]", g["dw2_0"][:, c0:c0 + 32], gr["dw_down"][0], tol)
    parity(f"{name}.dw_gate_up[gate slab {slab}]", g["dw1_0"][c0:c0 + 32], gr["dw_gate_up"][0][:32], tol)
    parity(f"{name}.dw_gate_up[up slab {slab}]", g["dw1_0"][f + c0:f + c0 + 32], gr["dw_gate_up"][0][32:], tol)


def test_full_combine_is_the_ordered_fp32_sum_of_expert_rows(full):
    """Property at any size: y[t] = bf16(sum_j fp32(y_perm[row(t, j)])), likewise dx."""
    g = full
    T, k = g["cfg"].T, g["cfg"].k
    s2 = g["src_to_sorted"]
    for out, rows in (("y", "y_perm"), ("dx", "dx_perm")):
        acc = np.zeros_like(g[out], dtype=np.float32)
        for j in range(k):
            acc = acc + g[rows][s2[j::k]].astype(np.float32)
        assert np.array_equal(g[out], omoe.bf16_round(acc))
