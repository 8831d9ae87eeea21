"""The allocation-free inference forward (moe_grouped_mlp_fwd_noalloc), called through the C ABI.

It exists for callers that may not allocate device memory when they run the layer (a serving
loop whose memory belongs to its own pool, a host framework whose extensions may not call
cudaMalloc / cudaFree on the hot path).  Its scratch is a static device array, so the checks are:
the output equals the regular entry point's on the same inputs, on two calls in a row (the
array keeps the previous call's contents), also at a size just under the array's limit; no
device memory is taken by a call; it works as the first call into the library of a fresh process
(where the per-device set-up happens inside the call); sizes beyond the array are refused before
anything is enqueued.

This file is collected last so that a run stopping at the first failure has run everything else.
"""
import ctypes
import json
import os
import subprocess
import sys
import textwrap

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


def test_noalloc_near_the_scratch_limit():
    """The largest token count whose forward scratch still fits the array (the 1 KiB carving
    alignment is inside the bound): identical to the regular entry point."""
    L = moe.load_library()
    torch.cuda.set_device(0)
    d, f, E, k, prec = 256, 512, 4, 2, "mxfp8"
    lo, hi = 1, 1 << 20
    while hi - lo > 1:  # largest T whose workspace fits
        mid = (lo + hi) // 2
        if L.moe_fwd_workspace_size(mid, k, E, d, f, 1, 0) <= moe.NOALLOC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    T = lo
    assert L.moe_fwd_workspace_size(T + 1, k, E, d, f, 1, 0) > moe.NOALLOC_SCRATCH_BYTES
    cfg = workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision=prec, T=T, seed=9)
    inp = workloads.make_inputs(cfg, with_dy=False)
    dev = {n: t.cuda() for n, t in inp.items()}
    ref, _ = moe.moe_grouped_mlp_fwd(dev["x"], dev["topk_idx"], dev["topk_prob"], dev["w_gate_up"], dev["w_down"],
                                     precision=prec, training=False)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        y = torch.full_like(ref, float("nan"))
        rc = _call_noalloc(L, dev, prec, y, status)
        torch.cuda.synchronize()
        assert rc == 0 and int(status.item()) == 0
        assert torch.equal(y, ref)
    # one token more no longer fits: refused before anything is enqueued
    assert _call_noalloc(L, {**dev, "x": torch.zeros(T + 1, d, dtype=torch.bfloat16, device="cuda"),
                             "topk_idx": torch.zeros(T + 1, k, dtype=torch.int32, device="cuda"),
                             "topk_prob": torch.zeros(T + 1, k, device="cuda")},
                         prec, torch.empty(T + 1, d, dtype=torch.bfloat16, device="cuda"), status) == 7


_FIRST_CALL = textwrap.dedent("""
    import ctypes, json, sys
    sys.path.insert(0, sys.argv[1])
    import numpy as np
    import torch
    import mxfp8_quantize_b200 as moe
    from mxfp8_quantize_b200 import workloads
    from oracle import moe as omoe
    L = moe.load_library()                      # no context, no other call into the library yet
    cfg = workloads.scaled_config(workloads.CONFIGS["tiny_bf16"], precision="mxfp8", T=200, seed=31)
    inp = workloads.make_inputs(cfg, with_dy=False)
    torch.cuda.set_device(0)
    dev = {n: t.cuda() for n, t in inp.items()}
    E, (T, d), f, k = cfg.E, dev["x"].shape, cfg.f, cfg.k
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w1 = (ctypes.c_void_p * E)(*[dev["w_gate_up"][e].data_ptr() for e in range(E)])
    w2 = (ctypes.c_void_p * E)(*[dev["w_down"][e].data_ptr() for e in range(E)])
    rc = L.moe_grouped_mlp_fwd_noalloc(dev["x"].data_ptr(), dev["topk_idx"].data_ptr(), dev["topk_prob"].data_ptr(),
                                       None, w1, w2, T, d, f, E, k, 1, y.data_ptr(), status.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    npi = {n: (t.float().numpy() if t.dtype == torch.bfloat16 else t.numpy()) for n, t in inp.items()}
    ref, _ = omoe.forward(npi["x"], npi["topk_idx"], npi["topk_prob"], npi["w_gate_up"], npi["w_down"], "mxfp8")
    got = y.float().cpu().numpy()
    err = float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))
    print(json.dumps({"rc": rc, "status": int(status.item()), "rel_err": err}))
""")


def test_noalloc_as_the_first_library_call_of_a_fresh_process():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _FIRST_CALL, root], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    out = json.loads(res.stdout.strip().splitlines()[-1])
    assert out["rc"] == 0 and out["status"] == 0
    assert out["rel_err"] <= TOL["mxfp8"]
