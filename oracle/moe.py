"""Grouped MoE expert MLP, forward and backward, as a plain per-expert loop.

Test infrastructure only (see the package docstring).

What the layer computes (sitech.ge "Grouped experts instead of a Python loop"
and "Memory and quantization overhead"; ai4snews paragraphs 1-3): every token
t is routed to k experts; for the slot (t, j) with e = topk_idx[t, j] and
p = topk_prob[t, j]

    h      = x_t W1_e^T                  (W1_e = w_gate_up[e], [2f, d])
    g, u   = h[:f], h[f:]                (gate rows first, then up rows)
    a      = silu(g) * u * p             (ScaledSwiGLU; silu(g) = g * sigmoid(g))
    y_slot = a W2_e^T                    (W2_e = w_down[e], [d, f])
    y_t    = sum_j y_slot(t, j)

evaluated the way the pages' baseline does it: one expert at a time over the
tokens routed to it (the loop GroupedLinear replaces).  The backward is the
gradient of that chain (dgrad and wgrad of both linears, the SwiGLU gradient
and the gradient of p).

Precision modes and the readings they encode:

* "mxfp8": every GEMM operand is quantised to MXFP8 with blocks of 32 along
  that GEMM's K (``oracle.mx``); the product of the dequantised operands is
  formed in fp64 and rounded once to fp32.  h stays fp32 in the forward;
  a = silu(g)*u*p is evaluated in fp64 from the fp32 h and rounded to fp32
  before it is quantised (rowwise for the down GEMM, down the token axis for
  the down-weight gradient).  Outputs y, dx, dW and the intermediate
  y / dx rows are rounded to bf16; the k contributions of a token are summed
  in fp32 in order j = 0..k-1.  The backward reads h as saved in bf16.  The
  routing probability is applied once, inside ScaledSwiGLU, so the final
  combine is an unweighted sum.  Straight-through: gradients flow through the
  quantisers as identity; each backward GEMM quantises its own operands along
  its own K (so dgrad uses the weights quantised down the columns).  Variants:
  the OCP floor shared-exponent rule (``scale_rule="floor"``) in every
  quantisation, and E5M2 elements for the gradient operands dy and dh of the
  backward GEMMs (``grad_format="e5m2"``; weights and activations stay E4M3).
  Memory variant for long sequences (andresseo.expert "Memory Pressure From
  Long Sequences"; sitech.ge "Memory and quantization overhead"): h saved as
  MXFP8 instead of bf16 (``saved_h="mxfp8"``: E4M3, blocks of 32 along 2f,
  which never straddle the gate and up halves since f % 32 == 0); the
  backward then reads g and u dequantised from it.
* "fp8": per-tensor FP8 with current scaling (``oracle.fp8``): every GEMM
  operand of every expert is quantised as one tensor with its own fp32 scale;
  E4M3 elements, E5M2 for the gradient operands dy and dh with
  ``grad_format="e5m2"``.  a and dh are rounded to bf16 before they are
  quantised (the tensor is materialised in 16 bits so that its maximum is
  known before any of it is quantised).  Products as for mxfp8; h saved as
  bf16.
* "bf16": the same chain with bf16 GEMM operands (a, dh rounded to bf16) and
  fp32 products.
* "fp64": no quantisation and no rounding anywhere (used to pin the algebra
  against autograd and finite differences).
"""
from __future__ import annotations

import numpy as np

from . import fp8, mx
from .routing import route


def bf16_round(a) -> np.ndarray:
    """Round to the nearest bf16 (ties to even); returns float32 holding bf16 values."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(f.shape)


def f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64).astype(np.float32)


def sigmoid(g):
    g = np.asarray(g, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-g))


def silu(g):
    g = np.asarray(g, dtype=np.float64)
    return g * sigmoid(g)


def gemm(A, B, precision: str, scale_rule: str = "ceil", a_fmt: str = "e4m3") -> np.ndarray:
    """C = A @ B for A [M, K], B [K, N] with operands in the given precision.

    mxfp8: A quantised in blocks of 32 along its axis 1 (K) with elements ``a_fmt``, B along its
           axis 0 (K) with E4M3 elements, both with the shared-exponent rule ``scale_rule``
           (oracle.mx).
    fp8:   A and B each quantised as one tensor (oracle.fp8), A with elements ``a_fmt``, B E4M3.
    bf16:  both operands rounded to bf16.   fp64: used as given.
    The product is formed in fp64 (callers round it).
    """
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    if precision == "mxfp8":
        A = mx.fake_quant(A, axis=1, rule=scale_rule, fmt=a_fmt)
        B = mx.fake_quant(B, axis=0, rule=scale_rule)
    elif precision == "fp8":
        A = fp8.fake_quant(A, a_fmt)
        B = fp8.fake_quant(B)
    elif precision == "bf16":
        A = bf16_round(A).astype(np.float64)
        B = bf16_round(B).astype(np.float64)
    elif precision != "fp64":
        raise ValueError(precision)
    return A @ B


def _round_out(c, precision):
    """Rounding of a GEMM result written as a 16-bit output (fp32 accumulate -> bf16)."""
    if precision == "fp64":
        return np.asarray(c, dtype=np.float64)
    return bf16_round(f32(c))


def _combine(rows_perm, src_to_sorted, T, k, precision):
    """out[t] = sum_j rows_perm[src_to_sorted[t*k + j]] (fp32, j ascending, then bf16)."""
    width = rows_perm.shape[1]
    if precision == "fp64":
        out = np.zeros((T, width))
        for j in range(k):
            out += rows_perm[src_to_sorted[j::k]]
        return out
    acc = np.zeros((T, width), dtype=np.float32)
    for j in range(k):
        acc = acc + rows_perm[src_to_sorted[j::k]].astype(np.float32)
    return bf16_round(acc)


def forward(x, topk_idx, topk_prob, w_gate_up, w_down, precision: str, align: int = 128, scale_rule: str = "ceil",
            grad_format: str = "e4m3", saved_h: str = "bf16"):
    """Returns (y [T, d], state) with the intermediates the backward needs.  ``scale_rule`` is the
    MXFP8 shared-exponent rule of every quantisation (forward and backward); ``grad_format`` the
    element format of the gradient operands (dy, dh) of the four backward GEMMs; ``saved_h`` the
    format h is kept in for the backward ("bf16" or "mxfp8")."""
    if saved_h not in ("bf16", "mxfp8") or (saved_h == "mxfp8" and precision != "mxfp8"):
        raise ValueError(saved_h)
    x = np.asarray(x, dtype=np.float64)
    T, d = x.shape
    E, two_f, _ = w_gate_up.shape
    f = two_f // 2
    k = topk_idx.shape[1]
    r = route(topk_idx, E, align)
    poff, split, s2src = r["poffsets"], r["split_sizes"], r["sorted_to_src"]
    Tp = int(poff[E])
    pflat = np.asarray(topk_prob, dtype=np.float64).reshape(-1)
    hdtype = np.float64 if precision == "fp64" else np.float32

    y_perm = np.zeros((Tp, d))
    h_all = np.zeros((Tp, 2 * f), dtype=hdtype)
    a_all = np.zeros((Tp, f), dtype=hdtype)
    x_perm = np.zeros((Tp, d))
    p_perm = np.zeros(Tp)
    for e in range(E):
        lo, hi = int(poff[e]), int(poff[e + 1])
        if split[e] == 0:
            continue
        slots = s2src[lo:hi]
        valid = slots >= 0
        Xe = np.zeros((hi - lo, d))
        Xe[valid] = x[slots[valid] // k]
        pe = np.zeros(hi - lo)
        pe[valid] = pflat[slots[valid]]
        W1 = np.asarray(w_gate_up[e], dtype=np.float64)
        W2 = np.asarray(w_down[e], dtype=np.float64)
        h = gemm(Xe, W1.T, precision, scale_rule)
        if precision != "fp64":
            h = f32(h)
        g, u = h[:, :f].astype(np.float64), h[:, f:].astype(np.float64)
        a = silu(g) * u * pe[:, None]
        if precision != "fp64":
            a = f32(a)
        if precision == "fp8":
            a = bf16_round(a)
        ye = gemm(a, W2.T, precision, scale_rule)
        y_perm[lo:hi] = _round_out(ye, precision)
        h_all[lo:hi] = h
        a_all[lo:hi] = a
        x_perm[lo:hi] = Xe
        p_perm[lo:hi] = pe
    y = _combine(y_perm, r["src_to_sorted"], T, k, precision)
    state = dict(route=r, x_perm=x_perm, p_perm=p_perm, h=h_all, a=a_all, y_perm=y_perm,
                 T=T, d=d, f=f, E=E, k=k, precision=precision, scale_rule=scale_rule, grad_format=grad_format,
                 saved_h=saved_h)
    return y, state


def backward(dy, state, w_gate_up, w_down):
    """Gradients of the forward in ``state`` for upstream gradient dy [T, d].

    Returns dict(dx [T,d], dw_gate_up [E,2f,d], dw_down [E,d,f], d_topk_prob [T,k]) and the
    per-row intermediates dx_perm, dh_perm (= [dg, du]) and dp_perm of the padded expert rows.
    dW of an expert that received no tokens is exactly zero.
    """
    precision = state["precision"]
    rule = state.get("scale_rule", "ceil")
    gf = state.get("grad_format", "e4m3")   # element format of the gradient operand (A) of each GEMM
    T, d, f, E, k = (state[n] for n in ("T", "d", "f", "E", "k"))
    r = state["route"]
    poff, split, s2src = r["poffsets"], r["split_sizes"], r["sorted_to_src"]
    Tp = int(poff[E])
    dy = np.asarray(dy, dtype=np.float64)

    dx_perm = np.zeros((Tp, d))
    dh_perm = np.zeros((Tp, 2 * f))
    dp_perm = np.zeros(Tp)
    dW1 = np.zeros((E, 2 * f, d))
    dW2 = np.zeros((E, d, f))
    for e in range(E):
        lo, hi = int(poff[e]), int(poff[e + 1])
        if split[e] == 0:
            continue
        slots = s2src[lo:hi]
        valid = slots >= 0
        dYe = np.zeros((hi - lo, d))
        dYe[valid] = dy[slots[valid] // k]
        Xe = state["x_perm"][lo:hi]
        pe = state["p_perm"][lo:hi][:, None]
        a = state["a"][lo:hi].astype(np.float64)
        h = state["h"][lo:hi]
        if precision != "fp64":          # the backward reads h as saved: bf16, or MXFP8 along 2f
            h = bf16_round(h) if state.get("saved_h", "bf16") == "bf16" else mx.fake_quant(h, axis=1, rule=rule)
        g, u = h[:, :f].astype(np.float64), h[:, f:].astype(np.float64)
        W1 = np.asarray(w_gate_up[e], dtype=np.float64)
        W2 = np.asarray(w_down[e], dtype=np.float64)

        # down projection: dgrad (K = d) and wgrad (K = tokens)
        da = gemm(dYe, W2, precision, rule, gf)
        if precision != "fp64":
            da = f32(da)
        da = da.astype(np.float64)
        dW2[e] = _round_out(gemm(dYe.T, a, precision, rule, gf), precision)

        # ScaledSwiGLU gradient
        s = sigmoid(g)
        sg = g * s
        dg = da * pe * u * s * (1.0 + g * (1.0 - s))
        du = da * pe * sg
        dp = np.sum(da * sg * u, axis=1)
        dh = np.concatenate([dg, du], axis=1)
        if precision != "fp64":
            dh = f32(dh)
            dp = f32(dp)
        if precision == "fp8":
            dh = bf16_round(dh)

        # gate_up projection: dgrad (K = 2f) and wgrad (K = tokens)
        dx_perm[lo:hi] = _round_out(gemm(dh, W1, precision, rule, gf), precision)
        dW1[e] = _round_out(gemm(np.asarray(dh, dtype=np.float64).T, Xe, precision, rule, gf), precision)
        dp_perm[lo:hi] = dp
        dh_perm[lo:hi] = dh

    dx = _combine(dx_perm, r["src_to_sorted"], T, k, precision)
    d_prob = dp_perm[r["src_to_sorted"]].reshape(T, k)
    if precision != "fp64":
        d_prob = d_prob.astype(np.float32)
    return dict(dx=dx, dw_gate_up=dW1, dw_down=dW2, d_topk_prob=d_prob, dx_perm=dx_perm, dh_perm=dh_perm,
                dp_perm=dp_perm)


def unpermute(y_perm, src_to_sorted, T, k, probs=None):
    """Standalone combine: y[t] = bf16(sum_j fp32(y_perm[row(t,j)] * p[t,j])) with fp32 products.

    With probs=None the rows are summed unweighted (the fused path's combine).
    """
    y_perm = np.asarray(y_perm, dtype=np.float32)
    acc = np.zeros((T, y_perm.shape[1]), dtype=np.float32)
    for j in range(k):
        rows = y_perm[np.asarray(src_to_sorted)[j::k]]
        if probs is not None:
            rows = rows * np.asarray(probs, dtype=np.float32)[:, j:j + 1]
        acc = acc + rows
    return bf16_round(acc)
