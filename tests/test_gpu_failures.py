"""Device-side error handling of the fused layer, through the C ABI (no fault, trap or hang).

* An expert index out of range: the routing rejects that slot (it gets no row and contributes
  nothing), the call records MOE_ERR_DEVICE, and every other result equals the oracle's for the
  same routing with that slot's contribution removed.  The oracle cannot take a bad index, so its
  reference routes the slot to a valid expert with probability 0: that slot's a, y and dh rows
  are then exactly zero, and being the last slot it shifts no other row of its expert.
* A caller split_sizes that disagrees with topk_idx: MOE_ERR_DEVICE, results unaffected.
* moe_unpermute skips -1 rows.
* Bounded waits: with the test hook on, every persistent kernel makes one wait on a flag nothing
  sets; it expires after a short limit with operand loads and MMAs in flight, the call reports
  MOE_ERR_TIMEOUT, and the next call on the same context (hook off) matches the oracle.
"""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import routing
from tests.gpu_util import bf16_np, has_b200, rel_err
from mxfp8_quantize_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_b200(), reason="needs a B200")]

import mxfp8_quantize_b200 as moe  # noqa: E402

TOL = {"mxfp8": 2e-2, "bf16": 1e-2}


def _np(inp):
    return {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in inp.items()}


def _layer(dev, precision, split_sizes=None):
    y, saved = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                       dev["w_down"], precision=precision, training=True, split_sizes=split_sizes)
    dx, dw1, dw2, dp = moe.moe_grouped_mlp_bwd(dev["dy"], saved, dev["w_gate_up"], dev["w_down"])
    return dict(y=y, dx=dx, dw1=dw1, dw2=dw2, dp=dp)


def _oracle(npi, precision):
    y, st = omoe.forward(npi["x"], npi["topk_idx"], npi["topk_prob"], npi["w_gate_up"], npi["w_down"], precision)
    g = omoe.backward(npi["dy"], st, npi["w_gate_up"], npi["w_down"])
    return dict(y=y, dx=g["dx"], dw1=g["dw_gate_up"], dw2=g["dw_down"], dp=g["d_topk_prob"])


def _status_code():
    try:
        moe.get_status(0)
    except moe.MoeError as ex:
        return ex.code
    return 0


@pytest.mark.parametrize("precision", ["mxfp8", "bf16"])
def test_bad_expert_index_is_contained(precision):
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], precision=precision, T=1000, seed=21)
    inp = workloads.make_inputs(cfg, with_dy=True)
    T, k, E = cfg.T, cfg.k, cfg.E
    bad = inp["topk_idx"].clone()
    bad[T - 1, k - 1] = E + 3                      # the last slot: out of range
    dev = {n: t.cuda() for n, t in inp.items()}
    dev["topk_idx"] = bad.cuda()
    assert _status_code() == 0
    g = _layer(dev, precision)
    assert _status_code() == 5                    # MOE_ERR_DEVICE, then cleared
    assert _status_code() == 0

    npi = _np(inp)
    npi["topk_idx"][T - 1, k - 1] = npi["topk_idx"][T - 1, 0]   # a valid expert ...
    npi["topk_prob"][T - 1, k - 1] = 0.0                          # ... that contributes nothing
    ref = _oracle(npi, precision)
    for name in ("y", "dx", "dw1", "dw2"):
        assert rel_err(bf16_np(g[name]), ref[name]) <= TOL[precision], name
    dp = g["dp"].cpu().numpy()
    assert dp[T - 1, k - 1] == 0.0                # the rejected slot has no gradient
    valid = np.ones((T, k), dtype=bool)
    valid[T - 1, k - 1] = False
    assert rel_err(dp[valid], ref["dp"][valid]) <= TOL[precision]


def test_split_sizes_mismatch_is_reported():
    precision = "mxfp8"
    cfg = workloads.scaled_config(workloads.CONFIGS["small_mxfp8"], T=700, seed=22)
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    counts = np.bincount(inp["topk_idx"].numpy().reshape(-1), minlength=cfg.E).astype(np.int32)
    wrong = counts.copy()
    wrong[0] += 1
    wrong[1] -= 1
    g = _layer(dev, precision, split_sizes=torch.from_numpy(wrong).cuda())
    assert _status_code() == 5
    ref = _oracle(_np(inp), precision)             # the routing follows topk_idx
    for name in ("y", "dx", "dw1", "dw2", "dp"):
        got = g[name].cpu().numpy() if name == "dp" else bf16_np(g[name])
        assert rel_err(got, ref[name]) <= TOL[precision], name
    g = _layer(dev, precision, split_sizes=torch.from_numpy(counts).cuda())
    assert _status_code() == 0


def test_unpermute_skips_rejected_rows():
    T, E, k, d = 300, 4, 2, 128
    idx, prob = workloads.random_topk(T, E, k, seed=23)
    cap = moe.capacity_rows(T, k, E)
    r = routing.route(idx.numpy(), E, 128, capacity=cap)
    rows = workloads.random_bf16((cap, d), seed=24)
    zero_row = int(np.nonzero(r["sorted_to_src"] < 0)[0][0])   # a padding row, zeroed for the reference
    rows[zero_row] = 0
    s2 = r["src_to_sorted"].astype(np.int32)
    s2[2 * 3 + 1], s2[2 * 50 + 0] = -1, -1        # two rejected slots: (t=3, j=1) and (t=50, j=0)
    s2_ref = np.where(s2 < 0, zero_row, s2)
    for probs in (None, prob):
        y = moe.moe_unpermute(rows.cuda(), torch.from_numpy(s2).cuda(), T, k,
                              probs=None if probs is None else probs.cuda())
        ref = omoe.unpermute(rows.float().numpy(), s2_ref, T, k, probs=None if probs is None else probs.numpy())
        assert np.array_equal(bf16_np(y), ref)
    assert _status_code() == 0


@pytest.mark.parametrize("precision", ["mxfp8", "bf16"])
def test_bounded_waits_expire_and_the_context_recovers(precision):
    cfg = workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision=precision, backward=True)
    inp = workloads.make_inputs(cfg, with_dy=True)
    dev = {n: t.cuda() for n, t in inp.items()}
    torch.cuda.set_device(0)
    moe.set_test_stall(0, True, 200_000)          # about 0.1 ms per wait, on a flag nothing sets
    try:
        _layer(dev, precision)
        assert _status_code() == 6                # MOE_ERR_TIMEOUT
        if precision == "mxfp8":                  # the TMA-fed quantiser alone
            moe.mxfp8_quantize(dev["w_gate_up"][0].contiguous(), rowwise=True, colwise=True, mma_layout=True)
            assert _status_code() == 6
    finally:
        moe.set_test_stall(0, False)
    g = _layer(dev, precision)
    assert _status_code() == 0
    ref = _oracle(_np(inp), precision)
    for name in ("y", "dx", "dw1", "dw2", "dp"):
        got = g[name].cpu().numpy() if name == "dp" else bf16_np(g[name])
        assert rel_err(got, ref[name]) <= TOL[precision], name
