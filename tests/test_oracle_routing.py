"""Pins for the oracle's routing bookkeeping (CPU only)."""
import numpy as np
import pytest

from oracle import routing
from oracle.moe import bf16_round
from mxfp8_quantize_b200 import workloads


def _random_idx(T, E, k, seed, skew=None):
    rng = np.random.default_rng(seed)
    if skew is None:
        return rng.integers(0, E, (T, k))
    p = np.asarray(skew, dtype=np.float64)
    return rng.choice(E, size=(T, k), p=p / p.sum())


@pytest.mark.parametrize("T,E,k,align,skew", [
    (1, 1, 1, 128, None), (37, 4, 2, 128, None), (300, 8, 2, 32, None),
    (500, 8, 2, 128, [50, 1, 1, 0, 0, 3, 1, 0]), (64, 3, 3, 128, None), (0, 4, 2, 128, None),
])
def test_route_properties(T, E, k, align, skew):
    idx = _random_idx(T, E, k, seed=T + E, skew=skew).astype(np.int32)
    r = routing.route(idx, E, align)
    flat = idx.reshape(-1)
    # counts = histogram; split sizes sum to T*k
    assert np.array_equal(r["split_sizes"], np.bincount(flat, minlength=E))
    assert r["split_sizes"].sum() == T * k
    poff = r["poffsets"]
    assert poff[0] == 0 and np.all(poff % align == 0)
    P = np.diff(poff)
    assert np.all(P >= r["split_sizes"]) and np.all(P - r["split_sizes"] < align)
    assert np.all((P == 0) == (r["split_sizes"] == 0))     # empty experts own no rows
    s2src, src2s = r["sorted_to_src"], r["src_to_sorted"]
    valid = s2src >= 0
    # bijection onto the slots, inverse maps agree
    assert np.array_equal(np.sort(s2src[valid]), np.arange(T * k))
    assert np.array_equal(s2src[src2s], np.arange(T * k))
    # independent formulation of the stable order: sort slots by (expert, slot)
    order = np.lexsort((np.arange(T * k), flat))
    assert np.array_equal(s2src[valid], order)
    # each expert's slots sit at the front of its segment
    for e in range(E):
        seg = s2src[poff[e]:poff[e + 1]]
        m = r["split_sizes"][e]
        assert np.all(seg[:m] >= 0) and np.all(seg[m:] == -1)
        assert np.all(flat[seg[:m]] == e)
        assert np.all(np.diff(seg[:m]) > 0)


def test_capacity_bound_covers_worst_case():
    T, k, E = 10, 2, 8
    for seed in range(20):
        idx = _random_idx(T, E, k, seed)
        r = routing.route(idx, E, 128)
        assert r["poffsets"][E] <= routing.capacity_rows(T, k, E, 128)
    # worst case: every expert gets exactly one slot
    idx = np.arange(8).reshape(4, 2)
    r = routing.route(idx, 8, 128)
    assert r["poffsets"][8] == 8 * 128 <= routing.capacity_rows(4, 2, 8, 128)


def test_out_of_range_rejected():
    with pytest.raises(ValueError):
        routing.route(np.array([[0, 4]]), 4)
    with pytest.raises(ValueError):
        routing.route(np.array([[-1, 0]]), 4)


def test_permute_then_combine_is_identity_for_renormalised_probs():
    cfg = workloads.MoEConfig("t", 64, 32, 32, 4, 2, "bf16", False, None, "uniform", 5)
    inp = workloads.make_inputs(cfg)
    x = inp["x"].float().numpy()
    idx, prob = inp["topk_idx"].numpy(), inp["topk_prob"].numpy()
    r = routing.route(idx, 4, 128)
    xp = routing.permute_rows(x, r["sorted_to_src"], 2)
    # brute force gather per slot
    for s in range(64 * 2):
        assert np.array_equal(xp[r["src_to_sorted"][s]], x[s // 2])
    from oracle.moe import unpermute
    y = unpermute(xp, r["src_to_sorted"], 64, 2, probs=prob)
    # sum_j p_j x = x * (p_0 + p_1) = x up to fp32 rounding of the products and one bf16 rounding
    assert np.max(np.abs(y - x)) <= 2.0 ** -7 * np.max(np.abs(x))
    assert np.allclose(prob.sum(1), 1.0, atol=1e-6)


def test_permute_probs_padding_is_zero():
    idx = np.array([[0, 1], [1, 1], [2, 0]])
    prob = np.array([[0.7, 0.3], [0.5, 0.5], [0.9, 0.1]], dtype=np.float32)
    r = routing.route(idx, 3, 4)
    pp = routing.permute_probs(prob, r["sorted_to_src"])
    assert pp.tolist() == pytest.approx([0.7, 0.1, 0, 0, 0.3, 0.5, 0.5, 0, 0.9, 0, 0, 0])
    assert r["sorted_to_src"].tolist() == [0, 5, -1, -1, 1, 2, 3, -1, 4, -1, -1, -1]


def test_bf16_round_matches_torch():
    import torch
    rng = np.random.default_rng(9)
    v = (rng.standard_normal(100000) * 2.0 ** rng.integers(-30, 30, 100000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    assert np.array_equal(bf16_round(v), ref)
