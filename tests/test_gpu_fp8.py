"""GPU parity of per-tensor FP8 (the standalone quantiser and the fused layer) against the oracle,
through the C ABI.

Per-tensor FP8 (ai4snews paragraph 2: FP8 and MXFP8 training; plain FP8 keeps one scale per tensor)
with current scaling, as oracle.fp8 states it.  Bit-exact: every tensor maximum, scale and code
the library computes (weights, the gathered rows of x and dy, and a and dh, the last two checked
against the oracle's quantiser applied to the bf16 rows the library wrote before quantising them);
the transposed copies hold the same codes.  Within tolerance (max|gpu - ref| / max|ref| <= 2e-2):
h, a, dh, y, dx, dW and the routing-probability gradient against the oracle's "fp8" layer.
"""
import numpy as np
import pytest
import torch

from oracle import fp8 as ofp8
from oracle import moe as omoe
from oracle import routing
from tests.gpu_util import bf16_np, has_b200, parity, rel_err
from mxfp8_quantize_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_b200(), reason="needs a B200")]

import mxfp8_quantize_b200 as moe  # noqa: E402

TOL = 2e-2
F32_MAX = float(np.finfo(np.float32).max)


# ------------------------------------------------------------------ standalone quantiser
@pytest.mark.parametrize("batch,rows,cols,fmt", [(1, 128, 128, "e4m3"), (3, 256, 384, "e4m3"),
                                                 (2, 384, 256, "e5m2"), (4, 128, 512, "e4m3")])
def test_fp8_quantize_bit_exact(batch, rows, cols, fmt):
    """Codes and scales of each [rows, cols] tensor of the batch; tensors of different magnitude,
    an all-zero one (scale 1) and one whose maximum is so small that vmax / amax overflows (the
    largest finite fp32)."""
    x = workloads.random_bf16((batch, rows, cols), seed=100 + batch).float()
    for b in range(batch):
        x[b] *= 2.0 ** (7 * b - 10)
    if batch >= 3:
        x[1] = 0.0
    if batch >= 4:
        x[3] = x[3] / x[3].abs().max() * 2.0 ** -120
    x = x.to(torch.bfloat16)
    out = moe.fp8_quantize(x.cuda(), colwise=True, fmt=fmt)
    torch.cuda.synchronize()
    q, qT, sc = out["q_row"].cpu().numpy(), out["q_colT"].cpu().numpy(), out["scale"].cpu().numpy()
    for b in range(batch):
        codes, s = ofp8.quantize(x[b].float().numpy(), fmt)
        assert np.array_equal(q[b], codes), b
        assert np.array_equal(qT[b], codes.T), b
        assert sc[b] == s, (b, sc[b], s)
    if batch >= 3:
        assert sc[1] == 1.0 and not q[1].any()
    if batch >= 4:
        assert sc[3] == np.float32(F32_MAX)


def test_fp8_quantize_refuses_bad_shapes():
    x = torch.zeros((100, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.fp8_quantize(x)


# ------------------------------------------------------------------ the fused layer
def _run(cfg, grad_format="e4m3", training=True, backward=True, w1=None, w2=None):
    inp = workloads.make_inputs(cfg, with_dy=backward)
    dev = {n: t.cuda() for n, t in inp.items()}
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    sz = moe.sizes(T, d, f, E, k, "fp8", training)
    ws = torch.zeros(sz["fwd_ws"], dtype=torch.uint8, device="cuda")
    w1 = dev["w_gate_up"] if w1 is None else w1(dev["w_gate_up"])
    w2 = dev["w_down"] if w2 is None else w2(dev["w_down"])
    moe.set_grad_format(0, grad_format)
    try:
        y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], w1, w2, precision="fp8",
                                           training=training, workspace=ws)
        out = dict(y=y, saved=saved, ws=ws, inp=inp, cap=moe.capacity_rows(T, k, E))
        if backward:
            bws = torch.zeros(sz["bwd_ws"], dtype=torch.uint8, device="cuda")
            dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, w1, w2, workspace=bws)
            out.update(dx=dx, dw1=dw1, dw2=dw2, dp=dp, bws=bws)
        moe.get_status(0)
    finally:
        moe.set_grad_format(0, "e4m3")
    return out


def _oracle(inp, grad_format="e4m3", backward=True):
    np_in = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in inp.items()}
    y, st = omoe.forward(np_in["x"], np_in["topk_idx"], np_in["topk_prob"], np_in["w_gate_up"], np_in["w_down"],
                         "fp8", grad_format=grad_format)
    res = dict(y=y, st=st, np=np_in)
    if backward:
        res.update(omoe.backward(np_in["dy"], st, np_in["w_gate_up"], np_in["w_down"]))
    return res


def _view(buf, which, name, cfg, training, n, dtype=torch.uint8):
    return moe.buffer_view(buf, which, name, (cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, "fp8"), training, n, dtype)


def _amax(v):
    v = np.asarray(v, dtype=np.float32)
    return np.float32(np.max(np.abs(v))) if v.size else np.float32(0)


@pytest.fixture(scope="module", params=["e4m3", "e5m2"])
def small(request):
    gf = request.param
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], precision="fp8", seed=51)
    g = _run(cfg, gf)
    ref = _oracle(g["inp"], gf)
    return cfg, gf, g, ref


def test_fp8_maxima_and_codes_bit_exact(small):
    cfg, gf, g, ref = small
    E, d, f, cap = cfg.E, cfg.d, cfg.f, g["cap"]
    st = ref["st"]
    poff = st["route"]["poffsets"]
    w1, w2 = ref["np"]["w_gate_up"], ref["np"]["w_down"]
    amax = _view(g["saved"].buf, 0, "pt_amax", cfg, True, 4 * E, torch.float32).cpu().numpy().reshape(4, E)
    a_gpu = _view(g["ws"], 1, "a", cfg, True, cap * f, torch.bfloat16).float().cpu().numpy().reshape(cap, f)
    dh_gpu = _view(g["bws"], 2, "dh", cfg, True, cap * 2 * f, torch.bfloat16).float().cpu().numpy().reshape(cap, 2 * f)
    amax2 = _view(g["bws"], 2, "pt_amax", cfg, True, 2 * E, torch.float32).cpu().numpy().reshape(2, E)
    dyp = routing.permute_rows(ref["np"]["dy"], st["route"]["sorted_to_src"], cfg.k)
    views = {
        "w1_q": _view(g["ws"], 1, "w1_q", cfg, True, E * 2 * f * d).cpu().numpy().reshape(E, 2 * f, d),
        "w1c_q": _view(g["saved"].buf, 0, "w1c_q", cfg, True, E * d * 2 * f).cpu().numpy().reshape(E, d, 2 * f),
        "w2_q": _view(g["ws"], 1, "w2_q", cfg, True, E * d * f).cpu().numpy().reshape(E, d, f),
        "w2c_q": _view(g["saved"].buf, 0, "w2c_q", cfg, True, E * f * d).cpu().numpy().reshape(E, f, d),
        "x_q": _view(g["ws"], 1, "x_q", cfg, True, cap * d).cpu().numpy().reshape(cap, d),
        "xT_q": _view(g["saved"].buf, 0, "xT_q", cfg, True, d * cap).cpu().numpy().reshape(d, cap),
        "a_q": _view(g["ws"], 1, "a_q", cfg, True, cap * f).cpu().numpy().reshape(cap, f),
        "aT_q": _view(g["saved"].buf, 0, "aT_q", cfg, True, f * cap).cpu().numpy().reshape(f, cap),
        "dy_q": _view(g["bws"], 2, "dy_q", cfg, True, cap * d).cpu().numpy().reshape(cap, d),
        "dyT_q": _view(g["bws"], 2, "dyT_q", cfg, True, d * cap).cpu().numpy().reshape(d, cap),
        "dh_q": _view(g["bws"], 2, "dh_q", cfg, True, cap * 2 * f).cpu().numpy().reshape(cap, 2 * f),
        "dhT_q": _view(g["bws"], 2, "dhT_q", cfg, True, 2 * f * cap).cpu().numpy().reshape(2 * f, cap),
    }
    for e in range(E):
        lo, hi = int(poff[e]), int(poff[e + 1])
        # maxima: x over the expert's rows, the weights, and a / dy / dh over the expert's rows
        assert amax[0, e] == _amax(st["x_perm"][lo:hi]), e
        assert amax[1, e] == _amax(w1[e]) and amax[2, e] == _amax(w2[e]), e
        assert amax[3, e] == _amax(a_gpu[lo:hi]), e
        assert amax2[0, e] == _amax(dyp[lo:hi]) and amax2[1, e] == _amax(dh_gpu[lo:hi]), e
        # codes
        c, _ = ofp8.quantize(w1[e])
        assert np.array_equal(views["w1_q"][e], c) and np.array_equal(views["w1c_q"][e], c.T), e
        c, _ = ofp8.quantize(w2[e])
        assert np.array_equal(views["w2_q"][e], c) and np.array_equal(views["w2c_q"][e], c.T), e
        if hi == lo:
            continue
        for name, rows, fmt in (("x", st["x_perm"][lo:hi], "e4m3"), ("a", a_gpu[lo:hi], "e4m3"),
                                ("dy", dyp[lo:hi], gf), ("dh", dh_gpu[lo:hi], gf)):
            c, _ = ofp8.quantize(rows, fmt)
            assert np.array_equal(views[name + "_q"][lo:hi], c), (name, e)
            assert np.array_equal(views[name + "T_q"][:, lo:hi], c.T), (name, e)


def test_fp8_intermediates_within_tolerance(small):
    cfg, gf, g, ref = small
    E, f, cap = cfg.E, cfg.f, g["cap"]
    Tp = int(ref["st"]["route"]["poffsets"][E])
    h = _view(g["saved"].buf, 0, "h", cfg, True, cap * 2 * f, torch.bfloat16).float().cpu().numpy()
    parity(f"small_fp8_{gf}.h", h.reshape(cap, 2 * f)[:Tp], ref["st"]["h"], TOL)
    a = _view(g["ws"], 1, "a", cfg, True, cap * f, torch.bfloat16).float().cpu().numpy().reshape(cap, f)
    parity(f"small_fp8_{gf}.a", a[:Tp], ref["st"]["a"], TOL)
    dh = _view(g["bws"], 2, "dh", cfg, True, cap * 2 * f, torch.bfloat16).float().cpu().numpy()
    parity(f"small_fp8_{gf}.dh", dh.reshape(cap, 2 * f)[:Tp], ref["dh_perm"], TOL)


@pytest.mark.parametrize("name", ["y", "dx", "dw1", "dw2", "dp"])
def test_fp8_outputs_within_tolerance(small, name):
    cfg, gf, g, ref = small
    refname = {"y": "y", "dx": "dx", "dw1": "dw_gate_up", "dw2": "dw_down", "dp": "d_topk_prob"}[name]
    got = g[name]
    got = got.float().cpu().numpy() if got.dtype == torch.bfloat16 else got.cpu().numpy()
    parity(f"small_fp8_{gf}.{name}", got, ref[refname], TOL)
    if name in ("dw1", "dw2"):
        assert np.all(got[7] == 0)   # expert 7 receives no tokens


def _scattered(w: torch.Tensor):
    """The experts of a stacked [E, r, c] weight at irregularly spaced places of one buffer."""
    E, r, c = w.shape
    buf = torch.zeros(E * r * c + 256 * E * E, dtype=w.dtype, device=w.device)
    out, off = [], 0
    for e in range(E):
        off += 256 * e
        v = buf[off:off + r * c].view(r, c)
        v.copy_(w[e])
        out.append(v)
        off += r * c
    return out


def test_fp8_scattered_experts_and_inference_match():
    """Experts given as separately placed tensors (one quantiser launch per expert) give the same
    results bit for bit; so do the inference forward and the allocation-free forward."""
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], precision="fp8", T=1024, seed=52)
    a = _run(cfg)
    b = _run(cfg, w1=_scattered, w2=_scattered)
    for name in ("y", "dx", "dw1", "dw2", "dp"):
        ga, gb = a[name], b[name]
        if isinstance(ga, list):
            assert all(torch.equal(u, v) for u, v in zip(ga, gb)), name
        else:
            assert torch.equal(ga, gb), name
    inf = _run(cfg, training=False, backward=False)
    assert torch.equal(inf["y"], a["y"])
    # the allocation-free forward (a shape whose workspace fits its static scratch)
    small = workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision="fp8", seed=53)
    ref = _run(small, training=False, backward=False)
    dev = {n: t.cuda() for n, t in ref["inp"].items()}
    y = moe.moe_grouped_mlp_fwd_noalloc(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                        dev["w_down"], precision="fp8")
    torch.cuda.synchronize()
    assert torch.equal(y, ref["y"])


@pytest.mark.parametrize("T", [1, 3])
def test_fp8_few_tokens(T):
    cfg = workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision="fp8", T=T, backward=True)
    g = _run(cfg)
    ref = _oracle(g["inp"])
    for name, rn in (("y", "y"), ("dx", "dx"), ("dw1", "dw_gate_up"), ("dw2", "dw_down"), ("dp", "d_topk_prob")):
        got = g[name]
        got = got.float().cpu().numpy() if got.dtype == torch.bfloat16 else got.cpu().numpy()
        assert rel_err(got, ref[rn]) <= TOL, name


def test_fp8_refuses_other_saved_h_modes():
    cfg = workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision="fp8", backward=False)
    inp = {n: t.cuda() for n, t in workloads.make_inputs(cfg).items()}
    assert moe.sizes(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, "fp8", True, "mxfp8")["saved"] == 0
    with pytest.raises(moe.MoeError):
        moe.moe_grouped_mlp_fwd(inp["x"], inp["topk_idx"], inp["topk_prob"], inp["w_gate_up"], inp["w_down"],
                                precision="fp8", training=True, saved_h="recompute")
