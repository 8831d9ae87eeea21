"""Benchmark of the grouped MoE expert MLP (forward + backward) on B200.

A step is one training pass of the whole hot path over one batch of synthetic input: per-step
MXFP8 quantisation of the bf16 master weights, routing, permute + quantise, the gate_up GEMM
with the fused ScaledSwiGLU requantisation, the down GEMM, the combine, and the backward
(dgrad + dSwiGLU, both wgrads, dgrad of gate_up, combine of dx, probability gradient).

Default workload: the Mixtral-8x7B layer shape in MXFP8 (T=8192 tokens, d=4096, f=14336,
E=8 experts, top-2).  ``value`` is algorithmic TFLOP/s (18*T*k*d*f per step, padding excluded)
with inputs resident in HBM; ``e2e`` is the same metric through the public API with host
buffers (inputs copied in from pinned memory and outputs copied back inside the timed region).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

With --gpus N > 1 (under torchrun) every rank runs an independent replica of the layer (the
single-layer path has no exchange step), and the job value is the sum over ranks with the time
taken as the max over ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mxfp8_quantize_b200 import workloads  # noqa: E402

METRIC = "grouped MoE MLP fwd+bwd TFLOP/s and tokens/s (MXFP8, BF16) vs tensor peak"
# the bounded slice of the workload the CPU oracle runs (routed slots of one expert, ffn columns)
ORACLE_SAMPLE = (512, 256)
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------------------ per-kernel work
def kernel_work(cfg, name):
    """(kind, algorithmic amount per launch): FLOPs for GEMMs, bytes for the HBM-bound kernels."""
    Tk, T, d, f, E, k = cfg.Tk, cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    mx = cfg.precision == "mxfp8"
    q8 = cfg.precision in ("mxfp8", "fp8")
    q = (1.0 + 1.0 / 32) if mx else 1.0  # bytes per quantised element (code + its share of a scale)
    gemm = {
        "gemm_gate_up_swiglu": 2.0 * Tk * d * 2 * f,
        "gemm_down": 2.0 * Tk * f * d,
        "gemm_dgrad_down_dswiglu": 2.0 * Tk * d * f,
        "gemm_wgrad_down": 2.0 * Tk * d * f,
        "gemm_dgrad_gate_up": 2.0 * Tk * 2 * f * d,
        "gemm_wgrad_gate_up": 2.0 * Tk * 2 * f * d,
        "gemm_fused_forward": 2.0 * Tk * d * 2 * f + 2.0 * Tk * f * d,
    }
    if name in gemm:
        return "tensor", gemm[name]
    out_b = 2 * q if q8 else 4.0  # row + column outputs per element
    hbm = {
        "quantize_w_gate_up": E * 2 * f * d * (2 + out_b),
        "quantize_w_down": E * d * f * (2 + out_b),
        "permute_quantize_x": T * d * 2 + Tk * d * out_b,
        "permute_x": T * d * 2 + Tk * d * out_b,
        "gather_quantize_dy": T * d * 2 + Tk * d * out_b,
        "transpose_w_gate_up": E * 2 * f * d * 4,
        "transpose_w_down": E * d * f * 4,
        "unpermute_y": Tk * d * 2 + T * d * 2 + Tk * 4,
        "unpermute_dx": Tk * d * 2 + T * d * 2 + Tk * 4,
        "route": Tk * 4 * 3,
        "dprob_reduce": Tk * 4 * 2,
        # per-tensor FP8: the maxima (reads), and the quantisation of the bf16 a / dh rows both ways
        "amax_w_gate_up": E * 2 * f * d * 2,
        "amax_w_down": E * d * f * 2,
        "amax_x": Tk * d * 2,
        "amax_dy": Tk * d * 2,
        "quantize_a": Tk * f * (2 + out_b),
        "quantize_dh": Tk * 2 * f * (2 + out_b),
    }
    return "hbm", hbm.get(name, 0.0)


# ------------------------------------------------------------------------------ clocks
REASON_FIELDS = ["clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                 "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


class ClockSampler:
    def __init__(self, gpu_index: int, out_dir: str):
        self.path = os.path.join(out_dir, f"clocks_gpu{gpu_index}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," + ",".join(REASON_FIELDS)
        try:
            self.f = open(self.path, "w")
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "100",
                                       "-i", str(gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        for line in open(self.path):
            parts = [s.strip() for s in line.split(",")]
            if len(parts) < 5 + len(REASON_FIELDS):
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(REASON_FIELDS, parts[5:]):
                if val.lower().startswith("active"):
                    reasons.add(name.split(".")[1])
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ CPU oracle sample
def oracle_sample(cfg, m_tokens: int, f_slab: int):
    """A bounded slice of the workload for the CPU oracle: expert 0 of the layer with the first
    ``m_tokens`` slots routed to it and a slab of ``f_slab`` ffn columns (gate and up halves),
    forward + backward with the workload's precision.  Returns (callable, flops, description)."""
    from mxfp8_quantize_b200.workloads import _normal_bf16
    rng = np.random.default_rng(cfg.seed)
    d = cfg.d
    std1 = cfg.w_std if cfg.w_std is not None else 1.0 / np.sqrt(d)
    std2 = cfg.w_std if cfg.w_std is not None else 1.0 / np.sqrt(cfg.f)
    x = _normal_bf16(rng, (m_tokens, d), 1.0).float().numpy()
    w1 = _normal_bf16(rng, (1, 2 * f_slab, d), float(std1)).float().numpy()
    w2 = _normal_bf16(rng, (1, d, f_slab), float(std2)).float().numpy()
    dy = _normal_bf16(rng, (m_tokens, d), 1.0).float().numpy()
    prob = rng.uniform(0.05, 0.95, (m_tokens, 1)).astype(np.float32)
    idx = np.zeros((m_tokens, 1), dtype=np.int32)

    def run():
        from oracle import moe as omoe
        y, st = omoe.forward(x, idx, prob, w1, w2, cfg.precision)
        omoe.backward(dy, st, w1, w2)

    flops = 18.0 * m_tokens * d * f_slab
    desc = (f"oracle fwd+bwd ({cfg.precision}) of one expert of the {cfg.name} layer: {m_tokens} routed slots, "
            f"d={d}, a {f_slab}-column ffn slab (gate+up {2 * f_slab} rows), incl. that slab's weight quantisation")
    return run, flops, desc


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(cfg, m_tokens, f_slab, repeats):
    run, flops, desc = oracle_sample(cfg, m_tokens, f_slab)
    ts = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        run()
        ts.append(time.perf_counter() - t0)
    return flops, ts, desc


# ------------------------------------------------------------------------------ tensor-core peak
def tensor_peak(moe, device: int, precision: str, target_ms: float = 100.0, scale_refresh: bool = False):
    """Rate of the library's tensor-core peak loop (tcgen05 MMAs on operands resident in shared
    memory, one CTA per SM) over about ``target_ms`` of back-to-back launches of ~10 ms each.
    Returns (TFLOP/s, ms measured)."""
    dev = torch.device("cuda", device)
    stream = torch.cuda.current_stream(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    iters = 1000
    moe.tensor_peak_loop(device, precision, iters, scale_refresh)      # warm (module load, TMEM)
    e0.record(stream)
    moe.tensor_peak_loop(device, precision, iters, scale_refresh)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    iters = min(1000000, max(100, int(iters * 10.0 / max(e0.elapsed_time(e1), 1e-3))))
    n = max(1, int(round(target_ms / 10.0)))
    flops = 0.0
    e0.record(stream)
    for _ in range(n):
        flops += moe.tensor_peak_loop(device, precision, iters, scale_refresh)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    moe.get_status(device)
    ms = e0.elapsed_time(e1)
    return flops / (ms * 1e-3) / 1e12, ms


def measure_peaks(args):
    """--peaks: burst (about 0.1 s after an idle second) and sustained (about 4 s back to back) rates
    of the tensor-core peak loop, MXFP8 with and without per-step scale copies and BF16, with the
    SM clock sampled during each; plus a torch bf16 matmul burst as a cross-check of the method
    against a library GEMM."""
    import mxfp8_quantize_b200 as moe
    dev = 0
    torch.cuda.set_device(dev)
    out = {}
    for name, prec, refresh in (("mxfp8", "mxfp8", False), ("mxfp8_scale_refresh", "mxfp8", True),
                                ("fp8", "fp8", False), ("bf16", "bf16", False)):
        for regime, ms in (("burst", 100.0), ("sustained", 4000.0)):
            time.sleep(1.0)
            clk = ClockSampler(dev, args.clocks_dir)
            tf, took = tensor_peak(moe, dev, prec, ms, refresh)
            c = clk.stop()
            out[f"{name}_{regime}"] = {"tflops": round(tf, 1), "ms": round(took, 1), "sm_mhz_median": c["sm_mhz"],
                                       "reasons": c["reasons"]}
    a = torch.randn(8192, 8192, device="cuda", dtype=torch.bfloat16)
    b = torch.randn(8192, 8192, device="cuda", dtype=torch.bfloat16)
    for _ in range(3):
        a @ b
    time.sleep(1.0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(10):
        a @ b
    e1.record()
    torch.cuda.synchronize()
    out["torch_bf16_matmul_8192_burst"] = {"tflops": round(10 * 2 * 8192 ** 3 / (e0.elapsed_time(e1) * 1e-3) / 1e12, 1)}
    print(json.dumps(out))


# ------------------------------------------------------------------------------ context: torch loop
def torch_loop_context(cfg, device: int, steps: int = 5, warmup: int = 2):
    """The pages' baseline structure (ai4snews paragraph 1; sitech.ge "Grouped experts instead of a
    Python loop"): a Python loop over experts, each gathering its tokens and running
    gate_up -> SwiGLU * p -> down with plain PyTorch BF16 ops (cuBLAS GEMMs), autograd for the
    backward.  Timed on the same GPU and workload shape as context for the grouped path; it is a
    library path, not this build's kernels.  Returns TFLOP/s and ms per fwd+bwd step."""
    dev = torch.device("cuda", device)
    inp = workloads.make_inputs(cfg, with_dy=True)
    x = inp["x"].to(dev)
    idx = inp["topk_idx"].to(dev).long()
    prob = inp["topk_prob"].to(dev).to(torch.bfloat16)
    dy = inp["dy"].to(dev)
    w1 = inp["w_gate_up"].to(dev).requires_grad_(True)
    w2 = inp["w_down"].to(dev).requires_grad_(True)
    f = cfg.f

    def step():
        xs = x.detach().requires_grad_(True)
        p = prob.detach().requires_grad_(True)
        y = torch.zeros_like(xs)
        for e in range(cfg.E):
            tok, j = torch.where(idx == e)
            if tok.numel() == 0:
                continue
            h = xs[tok] @ w1[e].t()
            a = torch.nn.functional.silu(h[:, :f]) * h[:, f:] * p[tok, j].unsqueeze(1)
            y = y.index_add(0, tok, a @ w2[e].t())
        y.backward(dy)
        w1.grad = None
        w2.grad = None

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    return {"kind": "torch per-expert loop, bf16, autograd (cuBLAS GEMMs)", "tflops": round(cfg.flops_fwd_bwd() / (ms * 1e-3) / 1e12, 1),
            "ms_per_step": round(ms, 3), "steps": steps}


# ------------------------------------------------------------------------------ replicas
def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest ``value`` over all ranks (the job's step time is the slowest replica's)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(cfg, ms_per_step: float, world: int) -> float:
    """Whole-job algorithmic TFLOP/s: every rank runs its own replica of the layer."""
    return world * cfg.flops_fwd_bwd() / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------------------ GPU arm
def run_ours(args, cfg, rank, world, local_rank):
    import mxfp8_quantize_b200 as moe
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    moe.set_fused_forward(local_rank, args.fused_forward)
    inp = workloads.make_inputs(cfg, with_dy=True)
    x = inp["x"].to(dev)
    idx = inp["topk_idx"].to(dev)
    prob = inp["topk_prob"].to(dev)
    dy = inp["dy"].to(dev)
    w1 = inp["w_gate_up"].to(dev)
    w2 = inp["w_down"].to(dev)
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    sz = moe.sizes(T, d, f, E, k, cfg.precision, True, args.saved_h)
    fws = torch.empty(sz["fwd_ws"], dtype=torch.uint8, device=dev)
    bws = torch.empty(sz["bwd_ws"], dtype=torch.uint8, device=dev)
    saved = moe.Saved(torch.empty(sz["saved"], dtype=torch.uint8, device=dev), (T, d, f, E, k, cfg.precision),
                      args.saved_h)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    dx = torch.empty_like(y)
    dw1 = torch.empty_like(w1)
    dw2 = torch.empty_like(w2)
    dp = torch.empty((T, k), dtype=torch.float32, device=dev)

    def step(xi, idxi, probi, dyi, yo=y, dxo=dx, dpo=dp):
        moe.moe_grouped_mlp_fwd(xi, idxi, probi, w1, w2, precision=cfg.precision, training=True, workspace=fws,
                                saved=saved, y=yo, saved_h=args.saved_h)
        moe.moe_grouped_mlp_bwd(dyi, saved, w1, w2, workspace=bws, dx=dxo, dw_gate_up=dw1, dw_down=dw2,
                                d_topk_prob=dpo)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step(x, idx, prob, dy)
    moe.get_status(local_rank)
    # the tensor peak of this GPU, measured live just before the timed region: a 0.1 s burst, and a
    # run as long as the timed region itself (same power-cap and clock regime as the GEMMs in it)
    stream0 = torch.cuda.current_stream(dev)
    est0, est1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    est0.record(stream0)
    step(x, idx, prob, dy)
    est1.record(stream0)
    torch.cuda.synchronize(dev)
    timed_ms_est = est0.elapsed_time(est1) * args.steps
    peak_burst, _ = tensor_peak(moe, local_rank, cfg.precision, 100.0)
    loop_tflops, loop_ms = tensor_peak(moe, local_rank, cfg.precision, min(max(timed_ms_est, 100.0), 4000.0))
    step(x, idx, prob, dy)

    # ---- timed region: device-resident inputs; every kernel bracketed by events on its stream
    records = []
    stream = torch.cuda.current_stream(dev)

    def hook(name, after):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        records.append((name, after, ev))

    clocks = ClockSampler(local_rank if world > 1 else (torch.cuda.current_device()), args.clocks_dir)
    barrier()
    torch.cuda.synchronize(dev)
    moe.set_launch_hook(local_rank, hook)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step(x, idx, prob, dy)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    moe.set_launch_hook(local_rank, None)
    barrier()
    clk = clocks.stop()
    moe.get_status(local_rank)
    ms = t0.elapsed_time(t1) / args.steps
    launches = sum(1 for r in records if not r[1])

    # per-kernel averages
    per = {}
    open_ev = {}
    for name, after, ev in records:
        if not after:
            open_ev[name] = ev
        else:
            per.setdefault(name, []).append(open_ev.pop(name).elapsed_time(ev))
    kern = {}
    peaks, peak_src = load_peaks()
    q8 = cfg.precision in ("mxfp8", "fp8")
    # tensor peak: the peak loop measured live on this GPU (burst); the file's bf16 burst figure
    # (times the nominal fp8/bf16 ratio of 2 for the 8-bit kinds) is reported beside it
    tensor_peak_tf = loop_tflops
    nominal_rule = peaks["bf16_tflops"] * (2.0 if q8 else 1.0)
    mhz = clk.get("sm_mhz")
    for name, v in per.items():
        avg = float(np.mean(v))
        kind, work = kernel_work(cfg, name)
        if kind == "tensor":
            ach = work / (avg * 1e-3) / 1e12
            kern[name] = {"ms": round(avg, 4), "launches": len(v), "tflops": round(ach, 1),
                          "frac": round(ach / tensor_peak_tf, 4)}
        else:
            ach = work / (avg * 1e-3) / 1e9
            kern[name] = {"ms": round(avg, 4), "launches": len(v), "gbs": round(ach, 1),
                          "frac": round(ach / peaks["hbm_gbs"], 4)}
        if mhz:
            kern[name]["ksm_cycles"] = round(avg * mhz, 1)  # ms x median SM MHz = thousands of SM clocks
    dom = max(per, key=lambda n: sum(per[n]))
    kind, work = kernel_work(cfg, dom)
    avg = float(np.mean(per[dom]))
    if kind == "tensor":
        achieved, peak, unit = work / (avg * 1e-3) / 1e12, tensor_peak_tf, "TFLOP/s"
    else:
        achieved, peak, unit = work / (avg * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        import hashlib
        rec = json.load(open(tpath))
        h = hashlib.sha1()
        for fn in rec.get("sources", []):
            h.update(open(os.path.join(ROOT, fn), "rb").read())
        if rec.get("sources") and h.hexdigest()[:12] == rec.get("sources_sha1"):
            traffic = rec.get(cfg.name, {}).get(dom)  # counters taken on this very kernel source
    kind_name = {"mxfp8": "kind::mxf8f6f4 block-scaled", "fp8": "kind::f8f6f4"}.get(cfg.precision, "kind::f16")
    roofline = {"bound": kind, "kernel": dom, "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": unit,
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": (f"measured live: tcgen05 {kind_name} "
                                f"peak loop (operands resident in shared memory, one CTA per SM), run back to back "
                                f"for {round(loop_ms)} ms (the length of the timed region) just before it; its 0.1 s "
                                f"burst was {round(peak_burst, 1)} TFLOP/s (frac {round(achieved / peak_burst, 4)}); "
                                f"{peak_src} bf16 burst {peaks['bf16_tflops']}"
                                f"{' x 2 (nominal fp8/bf16 ratio)' if q8 else ''} = {round(nominal_rule, 1)} TFLOP/s "
                                f"(frac {round(achieved / nominal_rule, 4)})"
                                if kind == "tensor" else f"{peak_src}: HBM copy {peaks['hbm_gbs']} GB/s")}

    # ---- e2e: through the public API with host buffers.  Every step copies its inputs from pinned
    #      host memory and its results (y, dx, d_topk_prob) back, pipelined the way a training loop
    #      feeds a GPU: step i+1's inputs go up on one copy stream and step i-1's results come down on
    #      another while step i computes (device inputs and outputs double-buffered).  The timed
    #      region runs from the first upload to the last download.
    e2e = None
    if not args.no_e2e:
        hin = [inp[n].pin_memory() for n in ("x", "topk_idx", "topk_prob", "dy")]
        din = [[torch.empty_like(t, device=dev) for t in hin] for _ in range(2)]
        hout = [[torch.empty(tuple(t.shape), dtype=t.dtype).pin_memory() for t in (y, dx, dp)] for _ in range(2)]
        dout = [[torch.empty_like(t) for t in (y, dx, dp)] for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in hout[0])
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, in_free, done, out_free = ([ev() for _ in range(2)] for _ in range(4))
        n2 = max(2, min(args.steps, 20))
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(up)

        def upload(i):
            b = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(in_free[b])  # step i-2 has consumed this input buffer
                for dst, src in zip(din[b], hin):
                    dst.copy_(src, non_blocking=True)
                in_ready[b].record(up)

        upload(0)
        for i in range(n2):
            b = i % 2
            if i + 1 < n2:
                upload(i + 1)
            stream.wait_event(in_ready[b])
            if i >= 2:
                stream.wait_event(out_free[b])  # step i-2's results have left this output buffer
            step(*din[b], *dout[b])
            in_free[b].record(stream)
            done[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(done[b])
                for dst, src in zip(hout[b], dout[b]):
                    dst.copy_(src, non_blocking=True)
                out_free[b].record(down)
        e1.record(down)
        torch.cuda.synchronize(dev)
        barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / n2, world, dev)
        e2e = {"value": round(job_tflops(cfg, ms_e2e, world), 2), "unit": "TFLOP/s",
               "ms_per_step": round(ms_e2e, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "tokens_per_s": round(world * T / (ms_e2e * 1e-3), 1),
               "pipelining": "uploads of step i+1 and downloads of step i-1 overlap step i (two copy streams)"}

    ms = max_over_ranks(ms, world, dev)
    tensor_peaks = {"matched_tflops": round(loop_tflops, 1), "matched_ms": round(loop_ms, 1),
                    "burst_tflops": round(peak_burst, 1), "nominal_rule_tflops": round(nominal_rule, 1)}
    return dict(ms=ms, kernels=kern, roofline=roofline, clocks=clk, e2e=e2e, launches=launches,
                tensor_peaks=tensor_peaks, fused_forward=bool(args.fused_forward),
                memory={"saved_h": args.saved_h, "saved_bytes": sz["saved"],
                                                   "fwd_workspace_bytes": sz["fwd_ws"], "bwd_workspace_bytes": sz["bwd_ws"]})


def config_desc(cfg):
    return {"workload": f"{cfg.name}: T={cfg.T} d={cfg.d} f={cfg.f} E={cfg.E} top-{cfg.k}, {cfg.precision} "
                        f"fwd+bwd incl. per-step weight quantisation, {cfg.routing} routing",
            "tokens": cfg.T, "d": cfg.d, "f": cfg.f, "experts": cfg.E, "top_k": cfg.k,
            "l2": "inputs larger than L2 (bf16 master weights and their MXFP8 copies are GBs)",
            "parallelism": "replicas (one independent layer per GPU)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="mixtral_mxfp8", choices=sorted(workloads.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling cases)")
    ap.add_argument("--experts", type=int, default=None, help="override E (profiling cases)")
    ap.add_argument("--clocks-dir", default=tempfile.gettempdir(), help="where the nvidia-smi clock samples go")
    ap.add_argument("--peaks", action="store_true", help="measure the tensor-core peak loop (burst and sustained)")
    ap.add_argument("--fused-forward", action="store_true", help="both forward GEMMs in one persistent launch")
    ap.add_argument("--saved-h", default="bf16", choices=["bf16", "mxfp8", "recompute"],
                    help="format h is saved in for the backward (long-sequence memory mode)")
    ap.add_argument("--context-torch-loop", action="store_true",
                    help="also time a plain PyTorch per-expert loop (BF16, autograd) on the same workload shape")
    args = ap.parse_args()
    if args.peaks:
        measure_peaks(args)
        return
    cfg = workloads.CONFIGS[args.config]
    if args.tokens or args.experts:
        cfg = workloads.scaled_config(cfg, T=args.tokens or cfg.T, E=args.experts or cfg.E,
                                      name=f"{cfg.name}[T={args.tokens or cfg.T},E={args.experts or cfg.E}]")
    if not cfg.backward:
        cfg = workloads.scaled_config(cfg, backward=True)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        # per step: a bounded slice (the same one the cpu_baseline leg times) so that the whole
        # run stays within a few minutes
        m, fs = ORACLE_SAMPLE
        for _ in range(args.warmup):
            time_oracle(cfg, m, fs, 1)
        flops, ts, desc = time_oracle(cfg, m, fs, args.steps)
        sec = float(np.sum(ts))
        val = flops * args.steps / sec / 1e12
        line = {"metric": METRIC, "value": round(val, 5), "unit": "TFLOP/s", "impl": "reference",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * sec / args.steps, 2), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_desc(cfg),
                "cpu_baseline": {"value": round(val, 5), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": round(val, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    res = run_ours(args, cfg, rank, world, local_rank)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    tflops = job_tflops(cfg, res["ms"], world)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        flops, ts, desc = time_oracle(cfg, *ORACLE_SAMPLE, 3)
        cpu = {"value": round(flops / float(np.median(ts)) / 1e12, 5), "unit": "TFLOP/s", "cores": cpu_threads(),
               "kind": "oracle", "sample": desc + f"; median of {len(ts)} runs of {float(np.median(ts)):.1f} s"}
    line = {"metric": METRIC, "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(res["ms"], 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": {"mxfp8": "mxfp8-e4m3 (fp32 accumulate)",
                                                      "fp8": "fp8-e4m3 per-tensor (fp32 accumulate)"}.get(cfg.precision,
                                                                                                          "bf16"),
            "data": "synthetic", "config": config_desc(cfg),
            "tokens_per_s": round(world * cfg.T / (res["ms"] * 1e-3), 1),
            "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"], "gpu_launches": res["launches"],
            "clocks": res["clocks"], "tensor_peaks": res["tensor_peaks"], "memory": res["memory"],
            "fused_forward": res["fused_forward"],
            "kernels": res["kernels"]}
    if args.context_torch_loop and world == 1:
        line["context_torch_loop"] = torch_loop_context(workloads.scaled_config(cfg, precision="bf16"), local_rank)
    print(json.dumps(line))


if __name__ == "__main__":
    main()
