"""Pin of the oracle's quantised backward (MXFP8 and BF16 modes) against an independent
formulation (CPU only).

The oracle writes the backward of the fused chain out by hand: each of the four backward GEMMs
quantises its own operands along its own K (dgrad: K = the output width; wgrad: K = the expert's
tokens, blocks of 32 starting at the expert's first slot), the SwiGLU gradient reads h as saved
in bf16, and dh, da, dp are held in fp32 (sitech.ge "Memory and quantization overhead": the
fused chain with a matching backward; ai4snews paragraph 3).

The reference here shares no code with the oracle:
* torch fp64 autograd computes every gradient of ScaledSwiGLU (no closed form is written);
* the GEMMs are torch.autograd.Functions whose forward and both backward products fake-quantise
  their operands along that product's K (straight-through: the quantisers pass gradients as
  identity);
* the MXFP8 fake-quantiser is derived here from the scale rule itself: with amax = m * 2**x,
  m in [0.5, 1), the smallest e with amax <= 448 * 2**e is x - 9 + (m > 0.875); elements are
  rounded by torch's own float8_e4m3fn conversion;
* tokens are handled per expert with plain index arithmetic, no padded permuted row space.

Both sides form fp64 products that differ only in summation order before the same fp32 / bf16
roundings and E4M3 codes, so they agree element for element: every output (and the fp32 dh the
dgrad of gate_up quantises) must be identical except for a tiny fraction of elements, and those
within 1e-6 of the largest magnitude.  Inputs get per-row and per-column power-of-two spreads, so
that a wrong quantisation axis, a missing rounding point or a dropped term changes many elements
(an error of that kind mostly moves the small elements of a block, which a max-normalised norm
alone would not see).
"""
import numpy as np
import pytest
import torch

from oracle import moe
from mxfp8_quantize_b200 import workloads

pytestmark = pytest.mark.filterwarnings("ignore:overflow encountered in exp")

REL = 1e-6
MAX_DIFF_FRACTION = 1e-4


# ---------------------------------------------------------------- independent numerics
def _e8m0_exponent(amax: torch.Tensor, rule: str = "ceil") -> torch.Tensor:
    m, x = torch.frexp(amax)                 # amax = m * 2**x, 0.5 <= m < 1 (m = 0 for amax = 0)
    e = x.to(torch.int64) - 9                # floor(log2 amax) - 8: the OCP rule
    if rule == "ceil":                       # one more when amax > 448 * 2**(x - 9), i.e. m > 0.875
        e = e + (m > 0.875).to(torch.int64)
    e = torch.where(amax > 0, e, torch.full_like(e, -127))
    return e.clamp(-127, 127)


def _e8m0_exponent_e5m2(amax: torch.Tensor) -> torch.Tensor:
    """E5M2 elements: the smallest e with amax <= 57344 * 2**e = 0.875 * 2**(16 + e)."""
    m, x = torch.frexp(amax)
    e = x.to(torch.int64) - 16 + (m > 0.875).to(torch.int64)
    e = torch.where(amax > 0, e, torch.full_like(e, -127))
    return e.clamp(-127, 127)


def _fq_mx5(v: torch.Tensor, axis: int) -> torch.Tensor:
    """MXFP8 fake quantisation with E5M2 elements (gradient operands), blocks of 32 along ``axis``."""
    vm = v.movedim(axis, -1)
    n = vm.shape[-1]
    pad = (-n) % 32
    if pad:
        vm = torch.nn.functional.pad(vm, (0, pad))
    blocks = vm.reshape(*vm.shape[:-1], -1, 32)
    scale = torch.ldexp(torch.ones_like(blocks[..., :1]), _e8m0_exponent_e5m2(blocks.abs().amax(dim=-1, keepdim=True)))
    q = (blocks / scale).clamp(-57344.0, 57344.0).to(torch.float8_e5m2).to(torch.float64) * scale
    return q.reshape(vm.shape)[..., :n].movedim(-1, axis)


def _fq_mx(v: torch.Tensor, axis: int, rule: str = "ceil") -> torch.Tensor:
    """MXFP8 fake quantisation with blocks of 32 along ``axis`` (zero-padded to a multiple of 32);
    elements beyond 448 after scaling (floor rule only) saturate."""
    vm = v.movedim(axis, -1)
    n = vm.shape[-1]
    pad = (-n) % 32
    if pad:
        vm = torch.nn.functional.pad(vm, (0, pad))
    blocks = vm.reshape(*vm.shape[:-1], -1, 32)
    e = _e8m0_exponent(blocks.abs().amax(dim=-1, keepdim=True), rule)
    scale = torch.ldexp(torch.ones_like(blocks[..., :1]), e)
    q = (blocks / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).to(torch.float64) * scale
    q = q.reshape(vm.shape)[..., :n]
    return q.movedim(-1, axis)


def _fq_pt(v: torch.Tensor, fmt: str = "e4m3") -> torch.Tensor:
    """Per-tensor FP8 fake quantisation: s = fp32(vmax / amax) (1 for an all-zero tensor, the
    largest fp32 when the quotient overflows), elements by torch's own float8 conversion of the
    fp32 product v * s, value code / s."""
    vmax, dt = (448.0, torch.float8_e4m3fn) if fmt == "e4m3" else (57344.0, torch.float8_e5m2)
    v32 = v.to(torch.float32)
    amax = v32.abs().max()
    if amax > 0:
        s = torch.tensor(vmax, dtype=torch.float32) / amax
        if torch.isinf(s):
            s = torch.tensor(torch.finfo(torch.float32).max, dtype=torch.float32)
    else:
        s = torch.tensor(1.0, dtype=torch.float32)
    q = (v32 * s).clamp(-vmax, vmax).to(dt).to(torch.float64)
    return q / s.to(torch.float64)


def _to_f32(v):
    return v.to(torch.float32).to(torch.float64)


def _to_bf16(v):
    return v.to(torch.float32).to(torch.bfloat16).to(torch.float64)


ROUND = {"f32": _to_f32, "bf16": _to_bf16}


def _operand(v, axis, mode):
    if mode == "bf16":
        return _to_bf16(v)
    if mode.startswith("fp8"):  # one scale for the whole tensor: the axis does not matter
        return _fq_pt(v)
    return _fq_mx(v, axis, "floor" if mode == "mxfp8-floor" else "ceil")


def _grad_operand(v, axis, mode):
    """The gradient operand of a backward product (E5M2 elements in the gradient-format variant)."""
    if mode == "fp8-e5m2grad":
        return _fq_pt(v, "e5m2")
    return _fq_mx5(v, axis) if mode == "mxfp8-e5m2grad" else _operand(v, axis, mode)


class _QuantLinear(torch.autograd.Function):
    """C = A B^T with A [M, K], B [N, K].  Forward: both operands quantised along K.  Backward:
    dA = dC B with dC and B quantised along N; dB = dC^T A with dC and A quantised down the M
    rows (the expert's tokens).  Outputs rounded as the library writes them."""

    @staticmethod
    def forward(ctx, A, B, mode, out_round, da_round):
        ctx.save_for_backward(A, B)
        ctx.mode, ctx.da_round = mode, da_round
        return ROUND[out_round](_operand(A, 1, mode) @ _operand(B, 1, mode).T)

    @staticmethod
    def backward(ctx, dC):
        A, B = ctx.saved_tensors
        mode = ctx.mode
        dA = _grad_operand(dC, 1, mode) @ _operand(B, 0, mode)
        dB = _grad_operand(dC, 0, mode).T @ _operand(A, 0, mode)
        return ROUND[ctx.da_round](dA), _to_bf16(dB), None, None, None


class _ScaledSwiGLU(torch.autograd.Function):
    """a = silu(g) * u * p from fp32 h (result rounded to fp32, then to bf16 in the per-tensor FP8
    mode).  Backward: autograd of the same expression evaluated on h as saved in bf16; dh and dp
    rounded to fp32 (dh then to bf16 in the per-tensor FP8 mode)."""

    @staticmethod
    def forward(ctx, h, p):
        ctx.save_for_backward(h, p)
        f = h.shape[1] // 2
        a = _to_f32(torch.nn.functional.silu(h[:, :f]) * h[:, f:] * p)
        return _to_bf16(a) if _ScaledSwiGLU.act_bf16 else a

    saved_h = "bf16"   # format h is read back in for the backward ("mxfp8": E4M3 blocks of 32 along 2f)
    act_bf16 = False   # a and dh materialised in bf16 before they are quantised (per-tensor FP8)

    @staticmethod
    def backward(ctx, da):
        h, p = ctx.saved_tensors
        f = h.shape[1] // 2
        hs = _fq_mx(h, 1) if _ScaledSwiGLU.saved_h == "mxfp8" else _to_bf16(h)
        hb = hs.detach().requires_grad_(True)
        pp = p.detach().requires_grad_(True)
        with torch.enable_grad():
            a = torch.nn.functional.silu(hb[:, :f]) * hb[:, f:] * pp
            dh, dp = torch.autograd.grad(a, (hb, pp), da)
        dh = _to_bf16(dh) if _ScaledSwiGLU.act_bf16 else _to_f32(dh)
        return dh, _to_f32(dp)


def _reference(x, idx, prob, w1, w2, dy, mode):
    """Forward and gradients of the layer, expert by expert, through torch autograd."""
    T, d = x.shape
    k = idx.shape[1]
    E = w1.shape[0]
    x = torch.tensor(x, dtype=torch.float64)
    dy = torch.tensor(dy, dtype=torch.float64)
    flat_idx = torch.tensor(idx.reshape(-1), dtype=torch.int64)
    flat_p = torch.tensor(prob.reshape(-1), dtype=torch.float64)
    y_slot = torch.zeros(T * k, d, dtype=torch.float64)
    dx_slot = torch.zeros(T * k, d, dtype=torch.float64)
    dp = torch.zeros(T * k, dtype=torch.float64)
    dh = torch.zeros(T * k, w1.shape[1], dtype=torch.float64)
    dw1 = torch.zeros(w1.shape, dtype=torch.float64)
    dw2 = torch.zeros(w2.shape, dtype=torch.float64)
    for e in range(E):
        slots = torch.nonzero(flat_idx == e).reshape(-1)      # ascending slot order
        if slots.numel() == 0:
            continue
        xe = x[slots // k].clone().requires_grad_(True)
        pe = flat_p[slots][:, None].clone().requires_grad_(True)
        W1 = torch.tensor(w1[e], dtype=torch.float64, requires_grad=True)
        W2 = torch.tensor(w2[e], dtype=torch.float64, requires_grad=True)
        h = _QuantLinear.apply(xe, W1, mode, "f32", "bf16")
        h.register_hook(lambda g, slots=slots: dh.__setitem__(slots, g.detach().clone()))
        a = _ScaledSwiGLU.apply(h, pe)
        ye = _QuantLinear.apply(a, W2, mode, "bf16", "f32")
        ye.backward(dy[slots // k])
        y_slot[slots] = ye.detach()
        dx_slot[slots] = xe.grad
        dp[slots] = pe.grad[:, 0]
        dw1[e] = W1.grad
        dw2[e] = W2.grad

    def combine(rows):
        acc = torch.zeros(T, d, dtype=torch.float32)
        for j in range(k):
            acc = acc + rows[j::k].to(torch.float32)
        return acc.to(torch.bfloat16).to(torch.float64)

    return dict(y=combine(y_slot), dx=combine(dx_slot), dw_gate_up=dw1, dw_down=dw2,
                d_topk_prob=dp.reshape(T, k).to(torch.float32).to(torch.float64), dh_slot=dh)


def _spread(a, rng):
    """Multiply every row and every column of the last two axes by its own power of two (exact in
    bf16): blocks of 32 then get different scales along different axes, so a GEMM operand quantised
    along the wrong axis changes the result (with plain Gaussian data almost every block of either
    orientation lands on the same scale)."""
    r = 2.0 ** rng.integers(-4, 5, a.shape[:-1] + (1,))
    c = 2.0 ** rng.integers(-4, 5, a.shape[:-2] + (1, a.shape[-1]))
    return (a * r * c).astype(np.float32)


def _inputs(T, d, f, E, k, seed, routing, empty=None):
    cfg = workloads.MoEConfig("pin", T, d, f, E, k, "mxfp8", True, None, routing, seed, empty_expert=empty)
    inp = workloads.make_inputs(cfg)
    out = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in inp.items()}
    rng = np.random.default_rng(seed + 1000)
    for n in ("x", "dy", "w_gate_up", "w_down"):
        out[n] = _spread(out[n], rng)
    return out


SHAPES = [
    dict(T=40, d=64, f=96, E=3, k=2, seed=11, routing="uniform"),
    dict(T=57, d=96, f=64, E=4, k=2, seed=12, routing="zipf", empty=2),
    dict(T=70, d=64, f=64, E=5, k=3, seed=13, routing="dirichlet"),
]


@pytest.mark.parametrize("mode", ["mxfp8", "bf16", "mxfp8-floor", "mxfp8-e5m2grad", "mxfp8-savedh", "fp8",
                                  "fp8-e5m2grad"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s['T']}_E{s['E']}_k{s['k']}_{s['routing']}")
def test_quantised_backward_matches_straight_through_autograd(shape, mode):
    """mxfp8-floor: the oracle's OCP floor shared-exponent variant, in every quantisation;
    mxfp8-e5m2grad: E5M2 elements for the gradient operand of every backward product;
    mxfp8-savedh: h kept as MXFP8 for the backward (the long-sequence memory variant);
    fp8: per-tensor FP8 (one scale per expert operand, a and dh materialised in bf16);
    fp8-e5m2grad: the same with E5M2 gradient operands."""
    inp = _inputs(**shape)
    args = [inp[n] for n in ("x", "topk_idx", "topk_prob", "w_gate_up", "w_down")]
    if mode == "mxfp8-floor":
        y, st = moe.forward(*args, "mxfp8", scale_rule="floor")
    elif mode == "mxfp8-e5m2grad":
        y, st = moe.forward(*args, "mxfp8", grad_format="e5m2")
    elif mode == "mxfp8-savedh":
        y, st = moe.forward(*args, "mxfp8", saved_h="mxfp8")
    elif mode == "fp8-e5m2grad":
        y, st = moe.forward(*args, "fp8", grad_format="e5m2")
    else:
        y, st = moe.forward(*args, mode)
    got = moe.backward(inp["dy"], st, inp["w_gate_up"], inp["w_down"])
    got["y"] = y
    _ScaledSwiGLU.saved_h = "mxfp8" if mode == "mxfp8-savedh" else "bf16"
    _ScaledSwiGLU.act_bf16 = mode.startswith("fp8")
    try:
        ref = _reference(*args, inp["dy"], "mxfp8" if mode == "mxfp8-savedh" else mode)
    finally:
        _ScaledSwiGLU.saved_h = "bf16"
        _ScaledSwiGLU.act_bf16 = False
    got["dh_slot"] = got["dh_perm"][st["route"]["src_to_sorted"]]
    for name in ("y", "dx", "dw_gate_up", "dw_down", "d_topk_prob", "dh_slot"):
        r = ref[name].numpy()
        g = np.asarray(got[name], dtype=np.float64)
        assert g.shape == r.shape, name
        n_diff = int(np.count_nonzero(g != r))
        assert n_diff <= max(2, MAX_DIFF_FRACTION * g.size), f"{mode} {name}: {n_diff} of {g.size} elements differ"
        err = np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300)
        assert err <= REL, f"{mode} {name}: {err:.3g}"
    if shape.get("empty") is not None:
        assert not got["dw_gate_up"][shape["empty"]].any() and not got["dw_down"][shape["empty"]].any()


def test_fake_quantiser_matches_the_scale_rule_on_hand_values():
    """The reference's own quantiser against values fixed by the format: a block of ones gets
    scale 2**-8 (byte 0x77) and stays exact; amax 1.875 needs e = -7; 450 rounds to 448 after a
    scale of 2."""
    v = torch.ones(1, 32, dtype=torch.float64)
    assert torch.equal(_fq_mx(v, 1), v)
    assert int(_e8m0_exponent(torch.tensor([1.0], dtype=torch.float64))) == -8
    assert int(_e8m0_exponent(torch.tensor([1.875], dtype=torch.float64))) == -7
    assert int(_e8m0_exponent(torch.tensor([448.0], dtype=torch.float64))) == 0
    assert int(_e8m0_exponent(torch.tensor([450.0], dtype=torch.float64))) == 1
    assert int(_e8m0_exponent(torch.tensor([1.875], dtype=torch.float64), "floor")) == -8
    assert int(_e8m0_exponent(torch.tensor([450.0], dtype=torch.float64), "floor")) == 0
    w = torch.zeros(1, 32, dtype=torch.float64)
    w[0, 0] = 450.0
    w[0, 1] = 1.0
    q = _fq_mx(w, 1)
    assert q[0, 0] == 448.0 and q[0, 1] == 1.0
