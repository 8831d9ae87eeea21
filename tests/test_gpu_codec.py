"""GPU parity of the HBM-bound kernels against the oracle, through the C ABI.

Bit-exact: E4M3 codes and E8M0 scale bytes (row-wise, column-wise, both scale layouts),
routing arrays, gathered rows and the combine.
"""
import numpy as np
import pytest
import torch

from oracle import mx, routing
from oracle.moe import unpermute as oracle_unpermute
from tests.gpu_util import has_b200, unswizzle_scales
from mxfp8_quantize_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_b200(), reason="needs a B200")]

import mxfp8_quantize_b200 as moe  # noqa: E402


def _spread_bf16(rows, cols, seed):
    """bf16 values whose rows span many binades, plus zero, tiny and negative-zero rows."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * 2.0 ** rng.integers(-24, 24, (rows, 1))
    if rows >= 8:
        x[1] = 0.0
        x[2] = rng.standard_normal(cols) * 2.0 ** -130          # bf16 subnormals
        x[3] = -0.0
        x[4, ::2] = 1e-30
        x[5] = rng.choice([1.0, 1.0625, 1.1875, -448.0, 450.0, 1.875], cols)
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    return t


@pytest.mark.parametrize("rows,cols,colwise,mma", [
    (32, 32, True, False), (64, 128, True, False), (100, 96, False, False), (256, 384, True, False),
    (128, 256, True, True), (384, 1024, True, True), (1000, 4096, False, False), (4096, 512, True, True),
    (256, 512, False, True), (4096, 384, False, True),   # row-wise only through the TMA-fed kernel
])
def test_quantize_bit_exact(rows, cols, colwise, mma):
    x = _spread_bf16(rows, cols, seed=rows + cols)
    out = moe.mxfp8_quantize(x.cuda(), rowwise=True, colwise=colwise, mma_layout=mma)
    torch.cuda.synchronize()
    xf = x.float().numpy()
    q, s = mx.quantize_rowwise(xf)
    assert np.array_equal(out["q_row"].cpu().numpy(), q)
    s_gpu = out["s_row"].cpu().numpy()
    if mma:
        s_gpu = unswizzle_scales(s_gpu, rows, cols // 32)
    assert np.array_equal(s_gpu, s)
    if colwise:
        qc, sc = mx.quantize_colwise_t(xf)
        assert np.array_equal(out["q_colT"].cpu().numpy(), qc)
        sc_gpu = out["s_colT"].cpu().numpy()
        if mma:
            sc_gpu = unswizzle_scales(sc_gpu, cols, rows // 32)
        assert np.array_equal(sc_gpu, sc)


def test_quantize_batched_and_dequantize():
    x = torch.stack([_spread_bf16(128, 256, seed=s) for s in range(3)])
    out = moe.mxfp8_quantize(x.cuda(), rowwise=True, colwise=True, mma_layout=True)
    for b in range(3):
        xf = x[b].float().numpy()
        q, s = mx.quantize_rowwise(xf)
        assert np.array_equal(out["q_row"][b].cpu().numpy(), q)
        assert np.array_equal(unswizzle_scales(out["s_row"][b].cpu().numpy(), 128, 8), s)
        qc, sc = mx.quantize_colwise_t(xf)
        assert np.array_equal(out["q_colT"][b].cpu().numpy(), qc)
        deq = moe.mxfp8_dequantize(out["q_row"][b].contiguous(), out["s_row"][b].contiguous(), mma_layout=True)
        ref = mx.dequantize_blocks(q, s)
        assert np.array_equal(deq.cpu().numpy().astype(np.float64), ref)


def test_golden_hand_vectors_on_gpu():
    import os
    from tests.test_oracle_mx import _golden_cases
    cases = _golden_cases()
    x = np.zeros((len(cases), 32))
    for i, (_, v, _, _) in enumerate(cases):
        x[i] = v
    xt = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    # the hand vectors are exact in bf16 except 1e-7, which rounds but stays below the same threshold
    out = moe.mxfp8_quantize(xt.cuda(), rowwise=True)
    q, s = out["q_row"].cpu().numpy(), out["s_row"].cpu().numpy()
    for i, (name, v, sbyte, codes) in enumerate(cases):
        assert int(s[i, 0]) == sbyte, name
        assert [int(c) for c in q[i, :len(codes)]] == codes, name


def test_quantize_rejects_bad_shapes():
    x = torch.zeros((64, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.mxfp8_quantize(x)
    x = torch.zeros((48, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.mxfp8_quantize(x, colwise=True)


@pytest.mark.parametrize("T,E,k,skew", [(1, 1, 1, "uniform"), (37, 4, 2, "uniform"), (4096, 8, 2, "zipf"),
                                        (3000, 16, 4, "dirichlet"), (16384, 8, 2, "uniform"), (777, 256, 8, "uniform")])
def test_permute_bit_exact(T, E, k, skew):
    idx, prob = workloads.random_topk(T, E, k, seed=T + E, skew=skew)
    d = 64
    x = workloads.random_bf16((T, d), seed=T)
    out = moe.moe_permute(x.cuda(), idx.cuda(), E, topk_prob=prob.cuda())
    torch.cuda.synchronize()
    cap = moe.capacity_rows(T, k, E)
    r = routing.route(idx.numpy(), E, 128, capacity=cap)
    assert np.array_equal(out["split_sizes"].cpu().numpy(), r["split_sizes"])
    assert np.array_equal(out["poffsets"].cpu().numpy(), r["poffsets"])
    assert np.array_equal(out["sorted_to_src"].cpu().numpy(), r["sorted_to_src"])
    assert np.array_equal(out["src_to_sorted"].cpu().numpy(), r["src_to_sorted"])
    assert np.array_equal(out["prob_perm"].cpu().numpy(), routing.permute_probs(prob.numpy(), r["sorted_to_src"]))
    xp = routing.permute_rows(x.float().numpy(), r["sorted_to_src"], k)
    assert np.array_equal(out["x_perm"].float().cpu().numpy(), xp)
    moe.get_status(0)


def test_permute_detects_bad_input():
    idx, _ = workloads.random_topk(64, 4, 2, seed=3)
    wrong = torch.tensor([1, 2, 3, 4], dtype=torch.int32)
    moe.moe_permute(None, idx.cuda(), 4, split_sizes=wrong.cuda())
    with pytest.raises(moe.MoeError) as ei:
        moe.get_status(0)
    assert ei.value.code == 5
    bad = idx.clone()
    bad[5, 1] = 9
    moe.moe_permute(None, bad.cuda(), 4)
    with pytest.raises(moe.MoeError) as ei:
        moe.get_status(0)
    assert ei.value.code == 5
    moe.get_status(0)  # cleared


@pytest.mark.parametrize("with_probs", [False, True])
def test_unpermute_bit_exact(with_probs):
    T, E, k, d = 2000, 8, 2, 256
    idx, prob = workloads.random_topk(T, E, k, seed=11)
    cap = moe.capacity_rows(T, k, E)
    r = routing.route(idx.numpy(), E, 128, capacity=cap)
    rows = workloads.random_bf16((cap, d), seed=12)
    y = moe.moe_unpermute(rows.cuda(), torch.from_numpy(r["src_to_sorted"].astype(np.int32)).cuda(), T, k,
                          probs=prob.cuda() if with_probs else None)
    ref = oracle_unpermute(rows.float().numpy(), r["src_to_sorted"], T, k, probs=prob.numpy() if with_probs else None)
    assert np.array_equal(y.float().cpu().numpy(), ref)


@pytest.mark.parametrize("rows,cols,colwise,mma", [
    (64, 128, True, False), (100, 96, False, False), (128, 256, True, True), (4096, 512, True, True),
])
def test_quantize_floor_rule_bit_exact(rows, cols, colwise, mma):
    """The OCP floor shared-exponent variant (MXFP8_FLAG_SCALE_FLOOR), both quantiser kernels."""
    x = _spread_bf16(rows, cols, seed=7 * rows + cols)
    out = moe.mxfp8_quantize(x.cuda(), rowwise=True, colwise=colwise, mma_layout=mma, scale_rule="floor")
    torch.cuda.synchronize()
    xf = x.float().numpy()
    q, s = mx.quantize_rowwise(xf, rule="floor")
    assert np.array_equal(out["q_row"].cpu().numpy(), q)
    s_gpu = out["s_row"].cpu().numpy()
    assert np.array_equal(unswizzle_scales(s_gpu, rows, cols // 32) if mma else s_gpu, s)
    if colwise:
        qc, sc = mx.quantize_colwise_t(xf, rule="floor")
        assert np.array_equal(out["q_colT"].cpu().numpy(), qc)
        sc_gpu = out["s_colT"].cpu().numpy()
        assert np.array_equal(unswizzle_scales(sc_gpu, cols, rows // 32) if mma else sc_gpu, sc)


def test_golden_floor_vectors_on_gpu():
    from tests.test_oracle_mx import GOLDEN_FLOOR, _golden_cases
    cases = _golden_cases(GOLDEN_FLOOR)
    x = np.zeros((len(cases), 32))
    for i, (_, v, _, _) in enumerate(cases):
        x[i] = v
    out = moe.mxfp8_quantize(torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda(), rowwise=True,
                             scale_rule="floor")
    q, s = out["q_row"].cpu().numpy(), out["s_row"].cpu().numpy()
    for i, (name, v, sbyte, codes) in enumerate(cases):
        assert int(s[i, 0]) == sbyte, name
        assert [int(c) for c in q[i, :len(codes)]] == codes, name


@pytest.mark.parametrize("rule", ["ceil", "floor"])
@pytest.mark.parametrize("rows,cols,colwise,mma", [(64, 128, True, False), (128, 256, True, True), (4096, 512, True, True)])
def test_quantize_e5m2_bit_exact(rows, cols, colwise, mma, rule):
    """E5M2 element codes (MXFP8_FLAG_E5M2, the gradient format), both quantiser kernels, both rules."""
    x = _spread_bf16(rows, cols, seed=3 * rows + cols)
    out = moe.mxfp8_quantize(x.cuda(), rowwise=True, colwise=colwise, mma_layout=mma, scale_rule=rule, fmt="e5m2")
    torch.cuda.synchronize()
    xf = x.float().numpy()
    q, s = mx.quantize_rowwise(xf, rule=rule, fmt="e5m2")
    assert np.array_equal(out["q_row"].cpu().numpy(), q)
    s_gpu = out["s_row"].cpu().numpy()
    assert np.array_equal(unswizzle_scales(s_gpu, rows, cols // 32) if mma else s_gpu, s)
    if colwise:
        qc, sc = mx.quantize_colwise_t(xf, rule=rule, fmt="e5m2")
        assert np.array_equal(out["q_colT"].cpu().numpy(), qc)
        sc_gpu = out["s_colT"].cpu().numpy()
        assert np.array_equal(unswizzle_scales(sc_gpu, cols, rows // 32) if mma else sc_gpu, sc)


def test_golden_e5m2_vectors_on_gpu():
    from tests.test_oracle_mx import GOLDEN_E5M2, _golden_cases
    cases = _golden_cases(GOLDEN_E5M2)
    x = np.zeros((len(cases), 32))
    for i, (_, v, _, _) in enumerate(cases):
        x[i] = v
    out = moe.mxfp8_quantize(torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda(), rowwise=True,
                             fmt="e5m2")
    q, s = out["q_row"].cpu().numpy(), out["s_row"].cpu().numpy()
    for i, (name, v, sbyte, codes) in enumerate(cases):
        assert int(s[i, 0]) == sbyte, name
        assert [int(c) for c in q[i, :len(codes)]] == codes, name
