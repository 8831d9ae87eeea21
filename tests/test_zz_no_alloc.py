"""The allocation-free inference forward (moe_grouped_mlp_fwd_noalloc), called through the C ABI.

It exists for callers that may not allocate device memory when they run the layer (a serving
loop whose memory belongs to its own pool, a host framework whose extensions may not call
cudaMalloc / cudaFree on the hot path).  Its scratch is a static device array, so the checks are:
the output equals the regular entry point's on the same inputs, on two calls in a row (the
array keeps the previous call's contents); no device memory is taken by a call; sizes beyond
the array are refused before anything is enqueued.

This file is collected last so that a run stopping at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import has_b200, rel_err
from mxfp8_quantize_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_b200(), reason="needs a B200")]

import mxfp8_quantize_b200 as moe  # noqa: E402

TOL = {"mxfp8": 2e-2, "bf16": 1e-2}


def _call_noalloc(L, dev, precision, y, status):
    E = dev["w_gate_up"].shape[0]
    T, d = dev["x"].shape
    f = dev["w_down"].shape[2]
    k = dev["topk_idx"].shape[1]
    w1 = (ctypes.c_void_p * E)(*[dev["w_gate_up"][e].data_ptr() for e in range(E)])
    w2 = (ctypes.c_void_p * E)(*[dev["w_down"][e].data_ptr() for e in range(E)])
    return L.moe_grouped_mlp_fwd_noalloc(dev["x"].data_ptr(), dev["topk_idx"].data_ptr(), dev["topk_prob"].data_ptr(),
                                         None, w1, w2, T, d, f, E, k, moe.PRECISIONS[precision], y.data_ptr(),
                                         status.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("precision", ["mxfp8", "bf16"])
def test_noalloc_forward_matches_regular_entry_point(precision):
    L = moe.load_library()
    torch.cuda.set_device(0)
    cfgs = [workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision=precision),
            workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision=precision, T=300, E=3, seed=5,
                                    routing="zipf")]
    for cfg in cfgs:
        inp = workloads.make_inputs(cfg, with_dy=False)
        dev = {n: t.cuda() for n, t in inp.items()}
        ref, _ = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"],
                                         dev["w_down"], precision=precision, training=False)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for call in range(2):
            y = torch.full_like(ref, float("nan"))
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
            rc = _call_noalloc(L, dev, precision, y, status)
            torch.cuda.synchronize()
            assert rc == 0, moe.STATUS.get(rc, rc)
            if call == 1:  # the first call may load the module that holds the static scratch
                assert torch.cuda.mem_get_info()[0] == free_before
            assert int(status.item()) == 0
            got, want = y.float().cpu().numpy(), ref.float().cpu().numpy()
            assert rel_err(got, want) <= TOL[precision]
            assert np.array_equal(got, want)  # same kernels, same inputs


def test_noalloc_rejects_sizes_beyond_the_scratch():
    L = moe.load_library()
    # the small layer's forward needs about 95 MiB of scratch, above the 64 MiB array
    assert L.moe_fwd_workspace_size(4096, 2, 8, 1024, 2048, 1, 0) > moe.NOALLOC_SCRATCH_BYTES
    rc = L.moe_grouped_mlp_fwd_noalloc(None, None, None, None, None, None, 4096, 1024, 2048, 8, 2, 1, None, None,
                                       None)
    assert rc == 7  # MOE_ERR_WORKSPACE, nothing enqueued
