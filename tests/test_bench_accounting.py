"""The benchmark's accounting (host logic, no GPU): the algorithmic work it divides by.

The six GEMMs' FLOPs must add up to the step's FLOPs the headline metric uses (18 Tk d f), and
the weight quantisers' bytes are one bf16 read plus row-wise and column-wise codes with their
scale bytes.
"""
import bench
from mxfp8_quantize_b200 import workloads

GEMMS = ["gemm_gate_up_swiglu", "gemm_down", "gemm_dgrad_down_dswiglu", "gemm_wgrad_down", "gemm_dgrad_gate_up",
         "gemm_wgrad_gate_up"]


def test_gemm_flops_add_up_to_the_step():
    for name in ("mixtral_mxfp8", "mixtral_bf16", "longseq_mxfp8", "small_mxfp8"):
        cfg = workloads.CONFIGS[name]
        kinds = [bench.kernel_work(cfg, g) for g in GEMMS]
        assert all(kind == "tensor" for kind, _ in kinds)
        total = sum(w for _, w in kinds)
        assert total == 18.0 * cfg.Tk * cfg.d * cfg.f
        assert abs(total - cfg.flops_fwd_bwd()) <= 1e-9 * total


def test_weight_quantiser_bytes():
    cfg = workloads.CONFIGS["mixtral_mxfp8"]
    kind, b = bench.kernel_work(cfg, "quantize_w_gate_up")
    n = cfg.E * 2 * cfg.f * cfg.d
    assert kind == "hbm" and b == n * 2 + 2 * (n + n / 32)   # bf16 in; two code copies + scales out
    assert abs(b - 3.82e9) < 0.01e9
    kind, b = bench.kernel_work(workloads.CONFIGS["mixtral_bf16"], "transpose_w_down")
    assert kind == "hbm" and b == cfg.E * cfg.d * cfg.f * 4  # bf16 in, bf16 transposed out


def test_fused_forward_work_is_both_forward_gemms():
    cfg = workloads.CONFIGS["mixtral_mxfp8"]
    kind, w = bench.kernel_work(cfg, "gemm_fused_forward")
    assert kind == "tensor"
    assert w == bench.kernel_work(cfg, "gemm_gate_up_swiglu")[1] + bench.kernel_work(cfg, "gemm_down")[1]
    assert w == cfg.flops_fwd()


def test_oracle_sample_is_shared_by_both_cpu_legs():
    """The cpu_baseline object and the --impl reference arm time the same bounded slice."""
    import inspect
    src = inspect.getsource(bench.main)
    assert src.count("ORACLE_SAMPLE") >= 2


def test_fp8_kernel_bytes():
    """Per-tensor FP8: codes without scale bytes, the maxima passes read their tensor once, and the
    quantisation of the bf16 a / dh rows reads them and writes codes both ways."""
    cfg = workloads.CONFIGS["mixtral_fp8"]
    n = cfg.E * 2 * cfg.f * cfg.d
    assert bench.kernel_work(cfg, "quantize_w_gate_up") == ("hbm", n * 2 + 2 * n)
    assert bench.kernel_work(cfg, "amax_w_gate_up") == ("hbm", n * 2)
    assert bench.kernel_work(cfg, "amax_w_down") == ("hbm", cfg.E * cfg.d * cfg.f * 2)
    assert bench.kernel_work(cfg, "quantize_a") == ("hbm", cfg.Tk * cfg.f * 4)
    assert bench.kernel_work(cfg, "quantize_dh") == ("hbm", cfg.Tk * 2 * cfg.f * 4)
    total = sum(bench.kernel_work(cfg, g)[1] for g in GEMMS)
    assert total == 18.0 * cfg.Tk * cfg.d * cfg.f
