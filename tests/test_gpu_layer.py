"""GPU parity of the fused layer (forward + backward) against the oracle, through the C ABI.

Bit-exact: routing arrays and every MXFP8 operand the library quantises (weights, x, dy, and
the epilogue requantisations of a and dh, checked against the oracle's quantiser applied to
the fp32 values the epilogue dumps).  Within tolerance (max|gpu - ref| / max|ref|, 2e-2 for
MXFP8, 1e-2 for BF16, as the layer's accuracy target states): h, a, dh, y, dx, dW and the
routing-probability gradient, against the oracle run on the same seeded inputs.
"""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import mx, routing
from tests.gpu_util import bf16_np, has_b200, parity, rel_err, unswizzle_scales
from mxfp8_quantize_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_b200(), reason="needs a B200")]

import mxfp8_quantize_b200 as moe  # noqa: E402

TOL = {"mxfp8": 2e-2, "bf16": 1e-2}


def _run(cfg, precision, training=True, backward=True):
    inp = workloads.make_inputs(cfg, with_dy=backward)
    dev = {n: t.cuda() for n, t in inp.items()}
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    cap = moe.capacity_rows(T, k, E)
    dump_a = torch.full((cap, f), float("nan"), dtype=torch.float32, device="cuda")
    dump_dh = torch.full((cap, 2 * f), float("nan"), dtype=torch.float32, device="cuda")
    moe.set_debug_dump(0, dump_a, dump_dh)
    sz = moe.sizes(T, d, f, E, k, precision, training)
    ws = torch.zeros(sz["fwd_ws"], dtype=torch.uint8, device="cuda")
    try:
        y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                           dev["w_down"], precision=precision, training=training, workspace=ws)
        out = dict(y=y, saved=saved, ws=ws, dump_a=dump_a, inp=inp, cap=cap)
        if backward:
            bws = torch.zeros(sz["bwd_ws"], dtype=torch.uint8, device="cuda")
            dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, dev["w_gate_up"], dev["w_down"],
                                                      workspace=bws)
            out.update(dx=dx, dw1=dw1, dw2=dw2, dp=dp, bws=bws, dump_dh=dump_dh)
        moe.get_status(0)
    finally:
        moe.set_debug_dump(0, None, None)
    return out


def _oracle(inp, precision, backward=True):
    np_in = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in inp.items()}
    y, st = omoe.forward(np_in["x"], np_in["topk_idx"], np_in["topk_prob"], np_in["w_gate_up"], np_in["w_down"],
                         precision)
    res = dict(y=y, st=st, np=np_in)
    if backward:
        res.update(omoe.backward(np_in["dy"], st, np_in["w_gate_up"], np_in["w_down"]))
    return res


def _view(buf, which, name, cfg, precision, training, n, dtype=torch.uint8):
    dims = (cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, precision)
    return moe.buffer_view(buf, which, name, dims, training, n, dtype)


@pytest.fixture(scope="module")
def tiny():
    cfg = workloads.CONFIGS["tiny_bf16"]
    return cfg


@pytest.mark.parametrize("precision", ["bf16", "mxfp8"])
def test_tiny_forward(tiny, precision):
    cfg = tiny
    g = _run(cfg, precision, training=False, backward=False)
    ref = _oracle(g["inp"], precision, backward=False)
    assert rel_err(bf16_np(g["y"]), ref["y"]) <= TOL[precision]


@pytest.fixture(scope="module", params=["mxfp8", "bf16"])
def small(request):
    precision = request.param
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], precision=precision)
    g = _run(cfg, precision)
    ref = _oracle(g["inp"], precision)
    return cfg, precision, g, ref


def test_small_routing_bit_exact(small):
    cfg, precision, g, ref = small
    r = ref["st"]["route"]
    E, cap = cfg.E, g["cap"]
    poff = _view(g["saved"].buf, 0, "poffsets", cfg, precision, True, E + 1, torch.int32).cpu().numpy()
    assert np.array_equal(poff, r["poffsets"])
    s2 = _view(g["saved"].buf, 0, "sorted_to_src", cfg, precision, True, cap, torch.int32).cpu().numpy()
    assert np.array_equal(s2[:poff[E]], r["sorted_to_src"])
    assert np.all(s2[poff[E]:] == -1)
    sp = _view(g["saved"].buf, 0, "split_sizes", cfg, precision, True, E, torch.int32).cpu().numpy()
    assert np.array_equal(sp, r["split_sizes"])
    assert sp[7] == 0 and sp.sum() == cfg.T * cfg.k


def test_small_quantised_operands_bit_exact(small):
    cfg, precision, g, ref = small
    if precision != "mxfp8":
        pytest.skip("MXFP8 only")
    E, d, f, cap = cfg.E, cfg.d, cfg.f, g["cap"]
    Tp = int(ref["st"]["route"]["poffsets"][E])
    w1 = ref["np"]["w_gate_up"]
    w2 = ref["np"]["w_down"]
    # weights, row-wise (forward GEMMs) ...
    # (the row-wise copy of W1 is stored in 256-row groups of 128 gate rows + the matching 128 up rows)
    q = _view(g["ws"], 1, "w1_q", cfg, precision, True, E * 2 * f * d).cpu().numpy().reshape(E * 2 * f, d)
    s = _view(g["ws"], 1, "w1_s", cfg, precision, True, E * 2 * f * d // 32).cpu().numpy()
    rq, rs = mx.quantize_rowwise(w1.reshape(E * 2 * f, d))
    r = np.arange(2 * f)
    dst = np.where(r < f, (r // 128) * 256 + r % 128, ((r - f) // 128) * 256 + 128 + (r - f) % 128)
    dst = (np.arange(E)[:, None] * 2 * f + dst[None, :]).reshape(-1)
    assert np.array_equal(q[dst], rq)
    assert np.array_equal(unswizzle_scales(s, E * 2 * f, d // 32)[dst], rs)
    q = _view(g["ws"], 1, "w2_q", cfg, precision, True, E * d * f).cpu().numpy().reshape(E * d, f)
    assert np.array_equal(q, mx.quantize_rowwise(w2.reshape(E * d, f))[0])
    # ... and down the columns, transposed (dgrad GEMMs)
    q = _view(g["saved"].buf, 0, "w1c_q", cfg, precision, True, E * d * 2 * f).cpu().numpy().reshape(E, d, 2 * f)
    s = _view(g["saved"].buf, 0, "w1c_s", cfg, precision, True, E * d * 2 * f // 32).cpu().numpy()
    for e in (0, E - 1):
        rq, rs = mx.quantize_colwise_t(w1[e])
        assert np.array_equal(q[e], rq)
    assert np.array_equal(unswizzle_scales(s, E * d, 2 * f // 32)[:d], mx.quantize_colwise_t(w1[0])[1])
    # x gathered + quantised both ways
    xp = ref["st"]["x_perm"]
    q = _view(g["ws"], 1, "x_q", cfg, precision, True, cap * d).cpu().numpy().reshape(cap, d)
    assert np.array_equal(q[:Tp], mx.quantize_rowwise(xp)[0])
    q = _view(g["saved"].buf, 0, "xT_q", cfg, precision, True, d * cap).cpu().numpy().reshape(d, cap)
    assert np.array_equal(q[:, :Tp], mx.quantize_colwise_t(xp)[0])
    # epilogue requantisation of a: bit-exact from the fp32 values it quantised
    a32 = g["dump_a"].cpu().numpy()[:Tp]
    q = _view(g["ws"], 1, "a_q", cfg, precision, True, cap * f).cpu().numpy().reshape(cap, f)
    s = _view(g["ws"], 1, "a_s", cfg, precision, True, cap * f // 32).cpu().numpy()
    rq, rs = mx.quantize_rowwise(a32)
    assert np.array_equal(q[:Tp], rq)
    assert np.array_equal(unswizzle_scales(s, cap, f // 32)[:Tp], rs)
    q = _view(g["saved"].buf, 0, "aT_q", cfg, precision, True, f * cap).cpu().numpy().reshape(f, cap)
    s = _view(g["saved"].buf, 0, "aT_s", cfg, precision, True, f * cap // 32).cpu().numpy()
    rq, rs = mx.quantize_colwise_t(a32)
    assert np.array_equal(q[:, :Tp], rq)
    assert np.array_equal(unswizzle_scales(s, f, cap // 32)[:, :Tp // 32], rs)
    # dh requantisation
    dh32 = g["dump_dh"].cpu().numpy()[:Tp]
    q = _view(g["bws"], 2, "dh_q", cfg, precision, True, cap * 2 * f).cpu().numpy().reshape(cap, 2 * f)
    assert np.array_equal(q[:Tp], mx.quantize_rowwise(dh32)[0])
    q = _view(g["bws"], 2, "dhT_q", cfg, precision, True, 2 * f * cap).cpu().numpy().reshape(2 * f, cap)
    assert np.array_equal(q[:, :Tp], mx.quantize_colwise_t(dh32)[0])
    # dy gathered + quantised
    dyp = routing.permute_rows(ref["np"]["dy"], ref["st"]["route"]["sorted_to_src"], cfg.k)
    q = _view(g["bws"], 2, "dy_q", cfg, precision, True, cap * d).cpu().numpy().reshape(cap, d)
    assert np.array_equal(q[:Tp], mx.quantize_rowwise(dyp)[0])
    q = _view(g["bws"], 2, "dyT_q", cfg, precision, True, d * cap).cpu().numpy().reshape(d, cap)
    assert np.array_equal(q[:, :Tp], mx.quantize_colwise_t(dyp)[0])


def test_small_intermediates_within_tolerance(small):
    cfg, precision, g, ref = small
    E, f, cap = cfg.E, cfg.f, g["cap"]
    Tp = int(ref["st"]["route"]["poffsets"][E])
    h = _view(g["saved"].buf, 0, "h", cfg, precision, True, cap * 2 * f, torch.bfloat16).float().cpu().numpy()
    parity(f"small_{precision}.h", h.reshape(cap, 2 * f)[:Tp], ref["st"]["h"], TOL[precision])
    parity(f"small_{precision}.a", g["dump_a"].cpu().numpy()[:Tp], ref["st"]["a"], TOL[precision])


@pytest.mark.parametrize("name", ["y", "dx", "dw1", "dw2", "dp"])
def test_small_outputs_within_tolerance(small, name):
    cfg, precision, g, ref = small
    refname = {"y": "y", "dx": "dx", "dw1": "dw_gate_up", "dw2": "dw_down", "dp": "d_topk_prob"}[name]
    got = g[name]
    got = got.float().cpu().numpy() if got.dtype == torch.bfloat16 else got.cpu().numpy()
    parity(f"small_{precision}.{name}", got, ref[refname], TOL[precision])
    if name == "dw1":
        assert np.all(got[7] == 0)   # expert 7 receives no tokens
    if name == "dw2":
        assert np.all(got[7] == 0)


def _scattered(w: torch.Tensor):
    """The experts of a stacked [E, r, c] weight copied to irregularly spaced places of one buffer
    (gaps of 0, 256, 512, ... elements), so that no uniform stride covers them."""
    E, r, c = w.shape
    gaps = [256 * e for e in range(E)]
    buf = torch.zeros(E * r * c + sum(gaps), dtype=w.dtype, device=w.device)
    out, off = [], 0
    for e in range(E):
        off += gaps[e]
        v = buf[off:off + r * c].view(r, c)
        v.copy_(w[e])
        out.append(v)
        off += r * c
    return out


@pytest.mark.parametrize("precision", ["mxfp8", "bf16"])
def test_scattered_expert_weights_match_stacked(precision):
    """Experts given as separately placed tensors take the general paths (the tile quantiser, the
    bf16 weight gather) instead of the strided ones (TMA-fed quantiser, 3-D weight maps): every
    output must be identical."""
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], precision=precision, T=1024)
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    res = []
    for w1, w2 in [(dev["w_gate_up"], dev["w_down"]), (_scattered(dev["w_gate_up"]), _scattered(dev["w_down"]))]:
        y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], w1, w2,
                                           precision=precision, training=True)
        dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, w1, w2)
        moe.get_status(0)
        res.append([t.float().cpu() if t.dtype == torch.bfloat16 else t.cpu() for t in (y, dx, dw1, dw2, dp)])
    for name, a, b in zip(("y", "dx", "dw_gate_up", "dw_down", "d_topk_prob"), *res):
        assert torch.equal(a, b), name


@pytest.mark.parametrize("T", [1, 3])
@pytest.mark.parametrize("precision", ["mxfp8", "bf16"])
def test_few_tokens_forward_backward(T, precision):
    """A handful of tokens: every expert tile is almost all padding rows (gathered as zeros), and
    most experts receive nothing (zero weight gradients)."""
    cfg = workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision=precision, T=T, backward=True)
    g = _run(cfg, precision)
    ref = _oracle(g["inp"], precision)
    assert rel_err(bf16_np(g["y"]), ref["y"]) <= TOL[precision]
    assert rel_err(bf16_np(g["dx"]), ref["dx"]) <= TOL[precision]
    assert rel_err(bf16_np(g["dw1"]), ref["dw_gate_up"]) <= TOL[precision]
    assert rel_err(bf16_np(g["dw2"]), ref["dw_down"]) <= TOL[precision]
    assert rel_err(g["dp"].cpu().numpy(), ref["d_topk_prob"]) <= TOL[precision]
    used = set(np.asarray(g["inp"]["topk_idx"]).reshape(-1).tolist())
    for e in range(cfg.E):
        if e not in used:
            assert not bf16_np(g["dw1"][e]).any() and not bf16_np(g["dw2"][e]).any()


def test_floor_scale_rule_layer():
    """The fused layer with the OCP floor shared-exponent rule in every quantisation
    (moe_ctx_set_scale_rule): quantised operands and the epilogue requantisations bit-exact against
    the oracle's floor-rule codec, outputs within tolerance of the oracle's floor-rule layer."""
    precision = "mxfp8"
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], T=1024, seed=41)
    moe.set_scale_rule(0, "floor")
    try:
        g = _run(cfg, precision)
    finally:
        moe.set_scale_rule(0, "ceil")
    np_in = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in g["inp"].items()}
    y, st = omoe.forward(np_in["x"], np_in["topk_idx"], np_in["topk_prob"], np_in["w_gate_up"], np_in["w_down"],
                         precision, scale_rule="floor")
    gr = omoe.backward(np_in["dy"], st, np_in["w_gate_up"], np_in["w_down"])
    E, d, f, cap = cfg.E, cfg.d, cfg.f, g["cap"]
    Tp = int(st["route"]["poffsets"][E])
    w2 = np_in["w_down"]
    q = _view(g["ws"], 1, "w2_q", cfg, precision, True, E * d * f).cpu().numpy().reshape(E * d, f)
    assert np.array_equal(q, mx.quantize_rowwise(w2.reshape(E * d, f), rule="floor")[0])
    q = _view(g["ws"], 1, "x_q", cfg, precision, True, cap * d).cpu().numpy().reshape(cap, d)
    assert np.array_equal(q[:Tp], mx.quantize_rowwise(st["x_perm"], rule="floor")[0])
    a32 = g["dump_a"].cpu().numpy()[:Tp]
    q = _view(g["ws"], 1, "a_q", cfg, precision, True, cap * f).cpu().numpy().reshape(cap, f)
    assert np.array_equal(q[:Tp], mx.quantize_rowwise(a32, rule="floor")[0])
    dh32 = g["dump_dh"].cpu().numpy()[:Tp]
    q = _view(g["bws"], 2, "dhT_q", cfg, precision, True, 2 * f * cap).cpu().numpy().reshape(2 * f, cap)
    assert np.array_equal(q[:, :Tp], mx.quantize_colwise_t(dh32, rule="floor")[0])
    for name, ref in (("y", y), ("dx", gr["dx"]), ("dw1", gr["dw_gate_up"]), ("dw2", gr["dw_down"]),
                      ("dp", gr["d_topk_prob"])):
        got = g[name]
        got = got.float().cpu().numpy() if got.dtype == torch.bfloat16 else got.cpu().numpy()
        parity(f"small_floor_rule.{name}", got, ref, TOL[precision])


def test_e5m2_gradient_format_layer():
    """The backward with E5M2 gradient operands (moe_ctx_set_grad_format): dy quantised both ways
    and the dSwiGLU requantisation of dh bit-exact against the oracle's E5M2 codec, the backward
    GEMMs multiplying E5M2 A by E4M3 B, outputs within tolerance of the oracle's e5m2 layer."""
    precision = "mxfp8"
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], T=1024, seed=42)
    moe.set_grad_format(0, "e5m2")
    try:
        g = _run(cfg, precision)
    finally:
        moe.set_grad_format(0, "e4m3")
    np_in = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in g["inp"].items()}
    y, st = omoe.forward(np_in["x"], np_in["topk_idx"], np_in["topk_prob"], np_in["w_gate_up"], np_in["w_down"],
                         precision, grad_format="e5m2")
    gr = omoe.backward(np_in["dy"], st, np_in["w_gate_up"], np_in["w_down"])
    d, f, cap = cfg.d, cfg.f, g["cap"]
    Tp = int(st["route"]["poffsets"][cfg.E])
    dyp = routing.permute_rows(np_in["dy"], st["route"]["sorted_to_src"], cfg.k)
    q = _view(g["bws"], 2, "dy_q", cfg, precision, True, cap * d).cpu().numpy().reshape(cap, d)
    assert np.array_equal(q[:Tp], mx.quantize_rowwise(dyp, fmt="e5m2")[0])
    q = _view(g["bws"], 2, "dyT_q", cfg, precision, True, d * cap).cpu().numpy().reshape(d, cap)
    assert np.array_equal(q[:, :Tp], mx.quantize_colwise_t(dyp, fmt="e5m2")[0])
    dh32 = g["dump_dh"].cpu().numpy()[:Tp]
    q = _view(g["bws"], 2, "dh_q", cfg, precision, True, cap * 2 * f).cpu().numpy().reshape(cap, 2 * f)
    s = _view(g["bws"], 2, "dh_s", cfg, precision, True, cap * 2 * f // 32).cpu().numpy()
    rq, rs = mx.quantize_rowwise(dh32, fmt="e5m2")
    assert np.array_equal(q[:Tp], rq)
    assert np.array_equal(unswizzle_scales(s, cap, 2 * f // 32)[:Tp], rs)
    q = _view(g["bws"], 2, "dhT_q", cfg, precision, True, 2 * f * cap).cpu().numpy().reshape(2 * f, cap)
    assert np.array_equal(q[:, :Tp], mx.quantize_colwise_t(dh32, fmt="e5m2")[0])
    assert rel_err(bf16_np(g["y"]), y) <= TOL[precision]          # the forward is unchanged
    for name, ref in (("dx", gr["dx"]), ("dw1", gr["dw_gate_up"]), ("dw2", gr["dw_down"]), ("dp", gr["d_topk_prob"])):
        got = g[name]
        got = got.float().cpu().numpy() if got.dtype == torch.bfloat16 else got.cpu().numpy()
        parity(f"small_e5m2_grads.{name}", got, ref, TOL[precision])


def test_saved_h_mxfp8_layer():
    """h saved as MXFP8 for the backward (moe_ctx_set_saved_h): the saved buffer holds E4M3 codes
    with one scale per 32 values of h (within tolerance of the oracle's h once dequantised), the
    dSwiGLU epilogue reads g and u from them, and every gradient is within tolerance of the oracle
    run with saved_h='mxfp8'; the dh requantisation stays bit-exact against its dumped input."""
    precision = "mxfp8"
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], T=1024, seed=43)
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    cap = moe.capacity_rows(T, k, E)
    dump_dh = torch.full((cap, 2 * f), float("nan"), dtype=torch.float32, device="cuda")
    moe.set_debug_dump(0, None, dump_dh)
    bws = torch.zeros(moe.sizes(T, d, f, E, k, precision, True)["bwd_ws"], dtype=torch.uint8, device="cuda")
    try:
        y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                           dev["w_down"], precision=precision, training=True, saved_h="mxfp8")
        dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, dev["w_gate_up"], dev["w_down"], workspace=bws)
        moe.get_status(0)
    finally:
        moe.set_debug_dump(0, None, None)
    assert saved.buf.numel() == moe.sizes(T, d, f, E, k, precision, True, "mxfp8")["saved"]
    assert saved.buf.numel() < moe.sizes(T, d, f, E, k, precision, True, "bf16")["saved"]
    np_in = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in inp.items()}
    ry, st = omoe.forward(np_in["x"], np_in["topk_idx"], np_in["topk_prob"], np_in["w_gate_up"], np_in["w_down"],
                          precision, saved_h="mxfp8")
    gr = omoe.backward(np_in["dy"], st, np_in["w_gate_up"], np_in["w_down"])
    Tp = int(st["route"]["poffsets"][E])
    dims = (T, d, f, E, k, precision)
    hq = moe.buffer_view(saved.buf, 0, "h_q", dims, True, cap * 2 * f, saved_h="mxfp8").cpu().numpy()
    hs = moe.buffer_view(saved.buf, 0, "h_s", dims, True, cap * 2 * f // 32, saved_h="mxfp8").cpu().numpy()
    h_deq = mx.dequantize_blocks(hq.reshape(cap, 2 * f)[:Tp], hs.reshape(cap, 2 * f // 32)[:Tp])
    parity("small_saved_h_mxfp8.h", h_deq, mx.fake_quant(st["h"], axis=1), TOL[precision])
    dh32 = dump_dh.cpu().numpy()[:Tp]
    q = moe.buffer_view(bws, 2, "dh_q", dims, True, cap * 2 * f).cpu().numpy().reshape(cap, 2 * f)
    assert np.array_equal(q[:Tp], mx.quantize_rowwise(dh32)[0])
    parity("small_saved_h_mxfp8.dh", dh32, gr["dh_perm"], TOL[precision])
    parity("small_saved_h_mxfp8.y", bf16_np(y), ry, TOL[precision])
    for name, got, ref in (("dx", bf16_np(dx), gr["dx"]), ("dw1", bf16_np(dw1), gr["dw_gate_up"]),
                           ("dw2", bf16_np(dw2), gr["dw_down"]), ("dp", dp.cpu().numpy(), gr["d_topk_prob"])):
        parity(f"small_saved_h_mxfp8.{name}", got, ref, TOL[precision])


@pytest.mark.parametrize("precision", ["mxfp8", "bf16"])
@pytest.mark.parametrize("T", [3, 1500])
def test_fused_forward_matches_two_launches(precision, T):
    """moe_ctx_set_fused_forward: the gate_up and down tiles in one persistent launch (down tiles
    waiting on per-row-block completion counters) compute exactly what the two launches compute:
    the same tiles with the same accumulation order, so every output of the forward and of the
    backward that follows is bit-identical, and within tolerance of the oracle."""
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], precision=precision, T=T, seed=44)
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    res = []
    for fused in (False, True):
        moe.set_fused_forward(0, fused)
        try:
            y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                               dev["w_down"], precision=precision, training=True)
            dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, dev["w_gate_up"], dev["w_down"])
            moe.get_status(0)
        finally:
            moe.set_fused_forward(0, False)
        res.append([t.float().cpu() if t.dtype == torch.bfloat16 else t.cpu() for t in (y, dx, dw1, dw2, dp)])
    for name, a, b in zip(("y", "dx", "dw_gate_up", "dw_down", "d_topk_prob"), *res):
        assert torch.equal(a, b), name
    ref = _oracle(inp, precision, backward=False)
    parity(f"fused_forward_{precision}_T{T}.y", res[1][0].numpy(), ref["y"], TOL[precision])


@pytest.mark.parametrize("precision", ["mxfp8", "bf16"])
def test_recompute_h_matches_saved_h(precision):
    """MOE_SAVED_H_RECOMPUTE: the forward saves x's gate_up operand instead of h, and the backward
    quantises W1 again and re-runs the gate_up GEMM to regenerate h.  Same kernels on the same
    operands: every gradient is bit-identical to the saved-bf16-h backward, with a smaller saved
    buffer; and the regenerated h equals the one the forward saved."""
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], precision=precision, T=1200, seed=45)
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    res, keep = [], {}
    for mode in ("bf16", "recompute"):
        bws = torch.zeros(moe.sizes(T, d, f, E, k, precision, True, mode)["bwd_ws"], dtype=torch.uint8, device="cuda")
        y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                           dev["w_down"], precision=precision, training=True, saved_h=mode)
        dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, dev["w_gate_up"], dev["w_down"], workspace=bws)
        moe.get_status(0)
        keep[mode] = (saved, bws)
        res.append([t.float().cpu() if t.dtype == torch.bfloat16 else t.cpu() for t in (y, dx, dw1, dw2, dp)])
    for name, a, b in zip(("y", "dx", "dw_gate_up", "dw_down", "d_topk_prob"), *res):
        assert torch.equal(a, b), name
    sz = {m: moe.sizes(T, d, f, E, k, precision, True, m)["saved"] for m in ("bf16", "recompute")}
    assert sz["recompute"] < sz["bf16"]
    cap = moe.capacity_rows(T, k, E)
    dims = (T, d, f, E, k, precision)
    h_saved = moe.buffer_view(keep["bf16"][0].buf, 0, "h", dims, True, cap * 2 * f, torch.bfloat16)
    h_again = moe.buffer_view(keep["recompute"][1], 2, "hr", dims, True, cap * 2 * f, torch.bfloat16,
                              saved_h="recompute")
    Tp = int(moe.buffer_view(keep["bf16"][0].buf, 0, "poffsets", dims, True, E + 1, torch.int32)[E])
    assert torch.equal(h_saved[: Tp * 2 * f], h_again[: Tp * 2 * f])
