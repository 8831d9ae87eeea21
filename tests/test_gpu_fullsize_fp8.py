"""GPU parity of per-tensor FP8 at the full Mixtral-8x7B layer size (T=8192, d=4096, f=14336, E=8,
top-2), in the fused calls the benchmark times.

Per-tensor scales depend on whole tensors, so the sampled checks are arranged to keep them exact:
* every tensor maximum the library computes is checked in full: x, dy per expert against the
  routed token rows, W1 and W2 per expert, and a and dh per expert against the bf16 rows the
  library wrote before quantising them;
* codes are checked bit-exactly on sampled rows with those (checked) scales;
* rows within tolerance: the oracle runs a one-expert sub-problem made of the first slots of
  expert 0 plus the slots whose rows hold expert 0's largest |x|, |dy|, |a| and |dh|, so that the
  sub-problem's tensors share the full tensors' maxima (exactly for x and dy, whose values are
  inputs; up to the GPU / oracle difference in a and dh, far inside the tolerance).
"""
import numpy as np
import pytest
import torch

from oracle import fp8 as ofp8
from oracle import moe as omoe
from oracle import routing
from tests.gpu_util import has_b200, parity
from mxfp8_quantize_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.slow, pytest.mark.skipif(not has_b200(), reason="needs a B200")]

import mxfp8_quantize_b200 as moe  # noqa: E402

TOL = 2e-2
N_ROWS = 128


def _f(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _amax_rows(t: torch.Tensor) -> np.ndarray:
    """Largest |value| of each row of a bf16 tensor, on the host (exact: a maximum of bf16 values)."""
    return t.cpu().abs().amax(dim=-1).float().numpy()


@pytest.fixture(scope="module")
def full():
    cfg = workloads.CONFIGS["mixtral_fp8"]
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    cap = moe.capacity_rows(T, k, E)
    dims = (T, d, f, E, k, "fp8")
    sz = moe.sizes(T, d, f, E, k, "fp8", True)
    fws = torch.empty(sz["fwd_ws"], dtype=torch.uint8, device="cuda")
    bws = torch.empty(sz["bwd_ws"], dtype=torch.uint8, device="cuda")
    y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"], dev["w_down"],
                                       precision="fp8", training=True, workspace=fws)
    dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, dev["w_gate_up"], dev["w_down"], workspace=bws)
    moe.get_status(0)

    def view(buf, which, name, n, dtype=torch.uint8):
        return moe.buffer_view(buf, which, name, dims, True, n, dtype)

    route = routing.route(inp["topk_idx"].numpy(), E, 128, capacity=cap)
    poff = route["poffsets"]
    a = view(fws, 1, "a", cap * f, torch.bfloat16).view(cap, f)
    dh = view(bws, 2, "dh", cap * 2 * f, torch.bfloat16).view(cap, 2 * f)
    lo0, hi0 = int(poff[0]), int(poff[1])
    g = dict(cfg=cfg, route=route, cap=cap,
             amax=_f(view(saved.buf, 0, "pt_amax", 4 * E, torch.float32)).reshape(4, E),
             amax2=_f(view(bws, 2, "pt_amax", 2 * E, torch.float32)).reshape(2, E),
             # the maxima of the bf16 a and dh rows the library wrote, per row of the permuted space
             a_rowmax=_amax_rows(a), dh_rowmax=_amax_rows(dh),
             a0=_f(a[lo0:hi0]), dh0=_f(dh[lo0:hi0]),
             a_q0=_f(view(fws, 1, "a_q", cap * f).view(cap, f)[lo0:lo0 + N_ROWS]),
             aT_q0=_f(view(saved.buf, 0, "aT_q", f * cap).view(f, cap)[:64, lo0:lo0 + N_ROWS]),
             dh_q0=_f(view(bws, 2, "dh_q", cap * 2 * f).view(cap, 2 * f)[lo0:lo0 + N_ROWS]),
             x_q0=_f(view(fws, 1, "x_q", cap * d).view(cap, d)[lo0:lo0 + N_ROWS]),
             xT_q0=_f(view(saved.buf, 0, "xT_q", d * cap).view(d, cap)[:64, lo0:lo0 + N_ROWS]),
             dy_q0=_f(view(bws, 2, "dy_q", cap * d).view(cap, d)[lo0:lo0 + N_ROWS]),
             w1_q0=_f(view(fws, 1, "w1_q", E * 2 * f * d).view(E, 2 * f, d)[0, :256]),
             w1c_q0=_f(view(saved.buf, 0, "w1c_q", E * d * 2 * f).view(E, d, 2 * f)[0, :64]),
             w2_q7=_f(view(fws, 1, "w2_q", E * d * f).view(E, d, f)[E - 1, :256]),
             h0=_f(view(saved.buf, 0, "h", cap * 2 * f, torch.bfloat16).view(cap, 2 * f)[lo0:hi0]),
             y_perm0=_f(view(fws, 1, "y_perm", cap * d, torch.bfloat16).view(cap, d)[lo0:hi0]),
             dx_perm0=_f(view(bws, 2, "dx_perm", cap * d, torch.bfloat16).view(cap, d)[lo0:hi0]),
             dp=_f(dp))
    g["w_amax"] = (inp["w_gate_up"].abs().amax(dim=(1, 2)).float().numpy(),
                   inp["w_down"].abs().amax(dim=(1, 2)).float().numpy())
    g["x_rowmax"] = _amax_rows(inp["x"])
    g["dy_rowmax"] = _amax_rows(inp["dy"])
    g["np"] = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy())
               for n, t in inp.items() if n not in ("w_gate_up", "w_down")}
    g["np"]["w_gate_up"] = inp["w_gate_up"][0:1].float().numpy()
    g["np"]["w_down0"] = inp["w_down"][0:1].float().numpy()
    g["np"]["w_down7"] = inp["w_down"][E - 1].float().numpy()
    del fws, bws, saved, a, dh, dev, y, dx, dw1, dw2
    torch.cuda.empty_cache()
    return g


def test_full_fp8_maxima_exact(full):
    g = full
    E, k = g["cfg"].E, g["cfg"].k
    r = g["route"]
    poff, s2 = r["poffsets"], r["sorted_to_src"]
    for e in range(E):
        slots = s2[int(poff[e]):int(poff[e + 1])]
        tok = slots[slots >= 0] // k
        assert g["amax"][0, e] == (g["x_rowmax"][tok].max() if tok.size else 0.0), e
        assert g["amax2"][0, e] == (g["dy_rowmax"][tok].max() if tok.size else 0.0), e
        rows = slice(int(poff[e]), int(poff[e + 1]))
        assert g["amax"][3, e] == g["a_rowmax"][rows].max(), e
        assert g["amax2"][1, e] == g["dh_rowmax"][rows].max(), e
    assert np.array_equal(g["amax"][1], g["w_amax"][0]) and np.array_equal(g["amax"][2], g["w_amax"][1])


def test_full_fp8_codes_bit_exact(full):
    g = full
    r = g["route"]
    k = g["cfg"].k
    s = {n: ofp8.scale(g["amax"][i, 0]) for i, n in enumerate(("x", "w1", "w2", "a"))}
    s["dy"] = ofp8.scale(g["amax2"][0, 0])
    s["dh"] = ofp8.scale(g["amax2"][1, 0])
    slots = r["sorted_to_src"][int(r["poffsets"][0]): int(r["poffsets"][0]) + N_ROWS]
    x = g["np"]["x"][slots // k]
    assert np.array_equal(g["x_q0"], ofp8.encode(x, s["x"]))
    assert np.array_equal(g["xT_q0"], ofp8.encode(x, s["x"]).T[:64])
    assert np.array_equal(g["dy_q0"], ofp8.encode(g["np"]["dy"][slots // k], s["dy"]))
    w1 = g["np"]["w_gate_up"][0]
    assert np.array_equal(g["w1_q0"], ofp8.encode(w1[:256], s["w1"]))
    assert np.array_equal(g["w1c_q0"], ofp8.encode(w1[:, :64].T, s["w1"]))
    s_w2_7 = ofp8.scale(g["amax"][2, g["cfg"].E - 1])
    assert np.array_equal(g["w2_q7"], ofp8.encode(g["np"]["w_down7"][:256], s_w2_7))
    a0 = g["a0"][:N_ROWS]
    assert np.array_equal(g["a_q0"], ofp8.encode(a0, s["a"]))
    assert np.array_equal(g["aT_q0"], ofp8.encode(a0, s["a"]).T[:64])
    assert np.array_equal(g["dh_q0"], ofp8.encode(g["dh0"][:N_ROWS], s["dh"]))


def test_full_fp8_expert0_rows_within_tolerance(full):
    g = full
    r = g["route"]
    k = g["cfg"].k
    lo, hi = int(r["poffsets"][0]), int(r["poffsets"][1])
    seg = r["sorted_to_src"][lo:hi]
    n = int(np.count_nonzero(seg >= 0))
    tok = seg[:n] // k
    # rows of expert 0 that hold its largest |x|, |dy|, |a| and |dh|, plus its first N_ROWS rows
    pick = set(range(N_ROWS))
    pick.add(int(np.argmax(g["x_rowmax"][tok])))
    pick.add(int(np.argmax(g["dy_rowmax"][tok])))
    pick.add(int(np.argmax(g["a_rowmax"][lo:lo + n])))
    pick.add(int(np.argmax(g["dh_rowmax"][lo:lo + n])))
    rows = np.array(sorted(pick))
    slots = seg[rows]
    npi = g["np"]
    x = npi["x"][slots // k]
    dy = npi["dy"][slots // k]
    prob = npi["topk_prob"].reshape(-1)[slots][:, None]
    idx = np.zeros((rows.size, 1), dtype=np.int32)
    assert ofp8.amax(x) == g["amax"][0, 0] and ofp8.amax(dy) == g["amax2"][0, 0]
    w1, w2 = npi["w_gate_up"], npi["w_down0"]
    y, st = omoe.forward(x, idx, prob, w1, w2, "fp8")
    gr = omoe.backward(dy, st, w1, w2)
    name, m = "mixtral_fp8", rows.size   # the oracle's permuted rows: the m slots, then padding
    parity(f"{name}.h", g["h0"][rows], st["h"][:m], TOL)
    parity(f"{name}.a", g["a0"][rows], st["a"][:m], TOL)
    parity(f"{name}.y_perm", g["y_perm0"][rows], y, TOL)
    parity(f"{name}.dh", g["dh0"][rows], gr["dh_perm"][:m], TOL)
    parity(f"{name}.dx_perm", g["dx_perm0"][rows], gr["dx_perm"][:m], TOL)
    parity(f"{name}.d_topk_prob", g["dp"].reshape(-1)[slots], gr["d_topk_prob"][:, 0], TOL)
