"""Python binding of libmoemx: the grouped MoE expert MLP with MXFP8 / per-tensor FP8 / BF16
operands on B200.

Argument marshalling only.  Every step of the computation runs in the CUDA kernels of
``libmoemx.so`` behind the C ABI declared in ``include/moemx.h``; PyTorch provides device
memory (outputs, workspaces) and the current CUDA stream.  There is no CPU fallback: if the
library is not built, or the device is not an sm_100 GPU, the calls raise.

Names follow the C ABI: ``mxfp8_quantize``, ``mxfp8_dequantize``, ``fp8_quantize``,
``moe_permute``, ``moe_unpermute``, ``moe_grouped_mlp_fwd``, ``moe_grouped_mlp_bwd``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Union

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoemx.so")

MOE_ROW_ALIGN = 128
MXFP8_ROWWISE, MXFP8_COLWISE_T, MXFP8_SF_MMA_LAYOUT, MXFP8_FLAG_SCALE_FLOOR, MXFP8_FLAG_E5M2 = 1, 2, 4, 8, 16
GRAD_FORMATS = {"e4m3": 0, "e5m2": 1}
SAVED_H = {"bf16": 0, "mxfp8": 1, "recompute": 2}
SCALE_RULES = {"ceil": 0, "floor": 1}
PRECISIONS = {"bf16": 0, "mxfp8": 1, "fp8": 2}
FP8_ROWWISE, FP8_COLWISE_T, FP8_FLAG_E5M2 = 1, 2, 16
STATUS = {0: "ok", 1: "invalid argument", 2: "shape", 3: "unsupported", 4: "cuda", 5: "device", 6: "timeout",
          7: "workspace"}

# every symbol include/moemx.h declares
EXPORTS = ["moe_ctx_create", "moe_ctx_destroy", "moe_get_status", "moe_ctx_set_debug_dump", "moe_status_string",
           "mxfp8_quantize", "mxfp8_dequantize", "moe_capacity_rows", "moe_permute", "moe_unpermute",
           "moe_saved_size", "moe_fwd_workspace_size", "moe_bwd_workspace_size", "moe_grouped_mlp_fwd",
           "moe_grouped_mlp_bwd", "moe_buffer_address", "moe_ctx_set_launch_hook", "moe_grouped_mlp_fwd_noalloc",
           "moe_ctx_set_test_stall", "moe_tensor_peak_loop", "moe_tensor_peak_flops", "moe_ctx_set_scale_rule",
           "moe_ctx_set_grad_format", "moe_ctx_set_saved_h", "moe_saved_size_ex", "moe_buffer_address_ex",
           "moe_ctx_set_fused_forward", "moe_bwd_workspace_size_ex", "fp8_quantize"]

LAUNCH_HOOK = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_char_p, ctypes.c_int, ctypes.c_void_p)


class MoeError(RuntimeError):
    def __init__(self, where: str, code: int):
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")
        self.code = code


_lib = None
_ctx = {}

c_vp, c_i64, c_int, c_size = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoemx.so and declare its signatures (no GPU needed)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libmoemx.so is not built ({path}); run mxfp8_quantize_b200.build.build()")
    L = ctypes.CDLL(path)
    sig = {
        "moe_ctx_create": (c_int, [ctypes.POINTER(c_vp), c_int]),
        "moe_ctx_destroy": (c_int, [c_vp]),
        "moe_get_status": (c_int, [c_vp, c_vp]),
        "moe_ctx_set_debug_dump": (c_int, [c_vp, c_vp, c_vp]),
        "moe_ctx_set_test_stall": (c_int, [c_vp, c_int, c_i64]),
        "moe_ctx_set_scale_rule": (c_int, [c_vp, c_int]),
        "moe_ctx_set_grad_format": (c_int, [c_vp, c_int]),
        "moe_ctx_set_saved_h": (c_int, [c_vp, c_int]),
        "moe_ctx_set_fused_forward": (c_int, [c_vp, c_int]),
        "moe_saved_size_ex": (c_size, [c_i64, c_int, c_int, c_i64, c_i64, c_int, c_int]),
        "moe_bwd_workspace_size_ex": (c_size, [c_i64, c_int, c_int, c_i64, c_i64, c_int, c_int]),
        "moe_buffer_address_ex": (c_vp, [c_i64, c_int, c_int, c_i64, c_i64, c_int, c_int, c_int, c_int, c_vp,
                                         ctypes.c_char_p]),
        "moe_tensor_peak_loop": (c_int, [c_vp, c_int, c_i64, c_int, c_vp]),
        "moe_tensor_peak_flops": (ctypes.c_double, [c_vp, c_int, c_i64]),
        "moe_status_string": (ctypes.c_char_p, [c_int]),
        "mxfp8_quantize": (c_int, [c_vp, c_vp, c_i64, c_i64, c_i64, c_int, c_vp, c_vp, c_vp, c_vp, c_vp]),
        "mxfp8_dequantize": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_int, c_vp, c_vp]),
        "fp8_quantize": (c_int, [c_vp, c_vp, c_i64, c_i64, c_i64, c_int, c_vp, c_vp, c_vp, c_vp]),
        "moe_capacity_rows": (c_i64, [c_i64, c_int, c_int]),
        "moe_permute": (c_int, [c_vp, c_vp, c_vp, c_vp, c_i64, c_int, c_int, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp,
                                c_vp, c_vp, c_vp]),
        "moe_unpermute": (c_int, [c_vp, c_vp, c_vp, c_vp, c_i64, c_int, c_i64, c_vp, c_vp]),
        "moe_saved_size": (c_size, [c_i64, c_int, c_int, c_i64, c_i64, c_int]),
        "moe_fwd_workspace_size": (c_size, [c_i64, c_int, c_int, c_i64, c_i64, c_int, c_int]),
        "moe_bwd_workspace_size": (c_size, [c_i64, c_int, c_int, c_i64, c_i64, c_int]),
        "moe_grouped_mlp_fwd": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_int, c_int,
                                        c_int, c_int, c_vp, c_vp, c_size, c_vp, c_size, c_vp]),
        "moe_grouped_mlp_bwd": (c_int, [c_vp, c_vp, c_vp, c_size, c_vp, c_vp, c_i64, c_i64, c_i64, c_int, c_int,
                                        c_int, c_vp, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
        "moe_ctx_set_launch_hook": (c_int, [c_vp, LAUNCH_HOOK, c_vp]),
        "moe_grouped_mlp_fwd_noalloc": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_int, c_int,
                                                c_int, c_vp, c_vp, c_vp]),
        "moe_buffer_address": (c_vp, [c_i64, c_int, c_int, c_i64, c_i64, c_int, c_int, c_int, c_vp,
                                      ctypes.c_char_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(where: str, code: int):
    if code != 0:
        raise MoeError(where, code)


def _device_index(t: torch.Tensor) -> int:
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    return t.device.index if t.device.index is not None else torch.cuda.current_device()


def context(device: int) -> int:
    """The library context of a CUDA device (created on first use)."""
    if device not in _ctx:
        L = load_library()
        h = c_vp()
        _check("moe_ctx_create", L.moe_ctx_create(ctypes.byref(h), device))
        _ctx[device] = h.value
    return _ctx[device]


def _stream(device: int) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def get_status(device: int = 0):
    """Synchronise the current stream and raise if a kernel recorded a device-side error."""
    L = load_library()
    _check("moe_get_status", L.moe_get_status(context(device), _stream(device)))


def set_debug_dump(device: int, a_f32: Optional[torch.Tensor], dh_f32: Optional[torch.Tensor]):
    L = load_library()
    _check("moe_ctx_set_debug_dump", L.moe_ctx_set_debug_dump(context(device), _ptr(a_f32), _ptr(dh_f32)))


def set_test_stall(device: int, stall: bool, limit_cycles: int = 0):
    """Test hook for the bounded in-kernel waits (see moe_ctx_set_test_stall in moemx.h)."""
    L = load_library()
    _check("moe_ctx_set_test_stall", L.moe_ctx_set_test_stall(context(device), int(stall), int(limit_cycles)))


_hooks = {}


def set_launch_hook(device: int, fn):
    """fn(kernel_name: str, after: bool) is called around every kernel the library enqueues on
    ``device`` (None switches it off).  Used to time kernels with CUDA events."""
    L = load_library()
    if fn is None:
        _hooks.pop(device, None)
        _check("moe_ctx_set_launch_hook", L.moe_ctx_set_launch_hook(context(device), LAUNCH_HOOK(), None))
        return
    cb = LAUNCH_HOOK(lambda user, name, after, stream: fn(name.decode(), bool(after)))
    _hooks[device] = cb
    _check("moe_ctx_set_launch_hook", L.moe_ctx_set_launch_hook(context(device), cb, None))


def capacity_rows(T: int, k: int, E: int) -> int:
    return int(load_library().moe_capacity_rows(T, k, E))


def set_scale_rule(device: int, rule: str):
    """MXFP8 shared-exponent rule of the fused layer on ``device``: "ceil" (default) or "floor" (OCP)."""
    L = load_library()
    _check("moe_ctx_set_scale_rule", L.moe_ctx_set_scale_rule(context(device), SCALE_RULES[rule]))


def set_fused_forward(device: int, on: bool):
    """Run the forward's two GEMMs as one persistent launch on ``device`` (see moemx.h)."""
    L = load_library()
    _check("moe_ctx_set_fused_forward", L.moe_ctx_set_fused_forward(context(device), int(on)))


def set_grad_format(device: int, fmt: str):
    """Element format of the MXFP8 gradient operands of the backward on ``device``: "e4m3" or "e5m2"."""
    L = load_library()
    _check("moe_ctx_set_grad_format", L.moe_ctx_set_grad_format(context(device), GRAD_FORMATS[fmt]))


def mxfp8_quantize(x: torch.Tensor, rowwise: bool = True, colwise: bool = False, mma_layout: bool = False,
                   scale_rule: str = "ceil", fmt: str = "e4m3"):
    """x bf16 [..., rows, cols] -> dict(q_row, s_row, q_colT, s_colT) (uint8; absent parts are None)."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() >= 2
    dev = _device_index(x)
    rows, cols = x.shape[-2], x.shape[-1]
    lead = tuple(x.shape[:-2])
    batch = 1
    for s in lead:
        batch *= s
    out = dict(q_row=None, s_row=None, q_colT=None, s_colT=None)
    flags = (MXFP8_ROWWISE if rowwise else 0) | (MXFP8_COLWISE_T if colwise else 0) | (MXFP8_SF_MMA_LAYOUT if mma_layout else 0)
    flags |= MXFP8_FLAG_SCALE_FLOOR if scale_rule == "floor" else 0
    flags |= MXFP8_FLAG_E5M2 if fmt == "e5m2" else 0
    if rowwise:
        out["q_row"] = torch.empty(lead + (rows, cols), dtype=torch.uint8, device=x.device)
        out["s_row"] = torch.empty(lead + (rows, cols // 32), dtype=torch.uint8, device=x.device)
    if colwise:
        out["q_colT"] = torch.empty(lead + (cols, rows), dtype=torch.uint8, device=x.device)
        out["s_colT"] = torch.empty(lead + (cols, rows // 32), dtype=torch.uint8, device=x.device)
    L = load_library()
    _check("mxfp8_quantize", L.mxfp8_quantize(context(dev), x.data_ptr(), batch, rows, cols, flags,
                                              _ptr(out["q_row"]), _ptr(out["s_row"]), _ptr(out["q_colT"]),
                                              _ptr(out["s_colT"]), _stream(dev)))
    return out


def mxfp8_dequantize(q: torch.Tensor, s: torch.Tensor, mma_layout: bool = False) -> torch.Tensor:
    dev = _device_index(q)
    rows, cols = q.shape[-2], q.shape[-1]
    out = torch.empty((rows, cols), dtype=torch.float32, device=q.device)
    L = load_library()
    _check("mxfp8_dequantize", L.mxfp8_dequantize(context(dev), q.data_ptr(), s.data_ptr(), rows, cols,
                                                  int(mma_layout), out.data_ptr(), _stream(dev)))
    return out


def fp8_quantize(x: torch.Tensor, colwise: bool = False, fmt: str = "e4m3"):
    """x bf16 [..., rows, cols], each [rows, cols] matrix one tensor -> dict(q_row, q_colT, scale):
    per-tensor FP8 codes (uint8; q_colT transposed, None unless ``colwise``) and the fp32 scale of
    each tensor."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() >= 2
    dev = _device_index(x)
    rows, cols = x.shape[-2], x.shape[-1]
    lead = tuple(x.shape[:-2])
    batch = 1
    for s in lead:
        batch *= s
    flags = FP8_ROWWISE | (FP8_COLWISE_T if colwise else 0) | (FP8_FLAG_E5M2 if fmt == "e5m2" else 0)
    out = dict(q_row=torch.empty(lead + (rows, cols), dtype=torch.uint8, device=x.device),
               q_colT=torch.empty(lead + (cols, rows), dtype=torch.uint8, device=x.device) if colwise else None,
               scale=torch.empty(lead if lead else (1,), dtype=torch.float32, device=x.device))
    L = load_library()
    _check("fp8_quantize", L.fp8_quantize(context(dev), x.data_ptr(), batch, rows, cols, flags,
                                          out["q_row"].data_ptr(), _ptr(out["q_colT"]), out["scale"].data_ptr(),
                                          _stream(dev)))
    return out


def moe_permute(x: Optional[torch.Tensor], topk_idx: torch.Tensor, E: int, topk_prob: Optional[torch.Tensor] = None,
                split_sizes: Optional[torch.Tensor] = None):
    """Routing bookkeeping (+ the gathered bf16 rows when x is given); see moe_permute in moemx.h."""
    assert topk_idx.dtype == torch.int32 and topk_idx.is_contiguous()
    dev = _device_index(topk_idx)
    T, k = topk_idx.shape
    cap = capacity_rows(T, k, E)
    kw = dict(dtype=torch.int32, device=topk_idx.device)
    out = dict(split_sizes=torch.empty(E, **kw), poffsets=torch.empty(E + 1, **kw),
               sorted_to_src=torch.empty(cap, **kw), src_to_sorted=torch.empty(T * k, **kw),
               prob_perm=None, x_perm=None)
    if topk_prob is not None:
        out["prob_perm"] = torch.empty(cap, dtype=torch.float32, device=topk_idx.device)
    d = 0
    if x is not None:
        d = x.shape[1]
        out["x_perm"] = torch.empty((cap, d), dtype=torch.bfloat16, device=x.device)
    L = load_library()
    _check("moe_permute", L.moe_permute(context(dev), _ptr(x), topk_idx.data_ptr(), _ptr(topk_prob), T, k, E, d,
                                        _ptr(split_sizes), out["split_sizes"].data_ptr(), out["poffsets"].data_ptr(),
                                        out["sorted_to_src"].data_ptr(), out["src_to_sorted"].data_ptr(),
                                        _ptr(out["prob_perm"]), _ptr(out["x_perm"]), _stream(dev)))
    return out


def moe_unpermute(y_perm: torch.Tensor, src_to_sorted: torch.Tensor, T: int, k: int,
                  probs: Optional[torch.Tensor] = None) -> torch.Tensor:
    dev = _device_index(y_perm)
    d = y_perm.shape[1]
    y = torch.empty((T, d), dtype=torch.bfloat16, device=y_perm.device)
    L = load_library()
    _check("moe_unpermute", L.moe_unpermute(context(dev), y_perm.data_ptr(), src_to_sorted.data_ptr(), _ptr(probs),
                                            T, k, d, y.data_ptr(), _stream(dev)))
    return y


def tensor_peak_loop(device: int, precision: str, iters: int, scale_refresh: bool = False) -> float:
    """Enqueue the tensor-core peak loop on the current stream of ``device``; returns its FLOPs."""
    L = load_library()
    ctx = context(device)
    _check("moe_tensor_peak_loop", L.moe_tensor_peak_loop(ctx, PRECISIONS[precision], int(iters), int(scale_refresh),
                                                          _stream(device)))
    return float(L.moe_tensor_peak_flops(ctx, PRECISIONS[precision], int(iters)))


Weights = Union[torch.Tensor, Sequence[torch.Tensor]]


def _ptr_array(ws: Weights, E: int):
    ts = [ws[e] for e in range(E)]
    for t in ts:
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    return (c_vp * E)(*[t.data_ptr() for t in ts])


class Saved:
    """Opaque buffer a training forward leaves for the backward, plus the call's dimensions and the
    format h was saved in."""

    def __init__(self, buf: torch.Tensor, dims: tuple, saved_h: str = "bf16"):
        self.buf = buf
        self.dims = dims
        self.saved_h = saved_h


def sizes(T: int, d: int, f: int, E: int, k: int, precision: str, training: bool, saved_h: str = "bf16"):
    L = load_library()
    p = PRECISIONS[precision]
    return dict(saved=int(L.moe_saved_size_ex(T, k, E, d, f, p, SAVED_H[saved_h])),
                fwd_ws=int(L.moe_fwd_workspace_size(T, k, E, d, f, p, int(training))),
                bwd_ws=int(L.moe_bwd_workspace_size_ex(T, k, E, d, f, p, SAVED_H[saved_h])))


def buffer_view(buf: torch.Tensor, which: int, name: str, dims: tuple, training: bool, nbytes: int,
                dtype=torch.uint8, saved_h: str = "bf16") -> torch.Tensor:
    """A view of the named intermediate inside ``buf`` (a saved / workspace buffer); tests only."""
    T, d, f, E, k, precision = dims
    L = load_library()
    p = L.moe_buffer_address_ex(T, k, E, d, f, PRECISIONS[precision], int(training), SAVED_H[saved_h], which,
                                buf.data_ptr(), name.encode())
    if not p:
        raise KeyError(name)
    off = p - buf.data_ptr()
    esz = torch.empty((), dtype=dtype).element_size()
    return buf[off:off + nbytes * esz].view(dtype)


def moe_grouped_mlp_fwd(x: torch.Tensor, topk_idx: torch.Tensor, topk_prob: torch.Tensor, w_gate_up: Weights,
                        w_down: Weights, precision: str = "mxfp8", training: bool = False,
                        split_sizes: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        saved: Optional[Saved] = None, y: Optional[torch.Tensor] = None, saved_h: str = "bf16"):
    """y = sum_j p_j * W2_e (silu(W1g_e x) * W1u_e x) over each token's k experts.

    Returns (y, saved) where saved is a Saved for the backward when ``training`` else None.
    ``saved_h``: the format h is saved in for the backward ("bf16" or "mxfp8").
    """
    dev = _device_index(x)
    T, d = x.shape
    E = len(w_gate_up)
    f = w_down[0].shape[1]
    k = topk_idx.shape[1]
    sz = sizes(T, d, f, E, k, precision, training, saved_h)
    if sz["fwd_ws"] == 0:
        raise MoeError("moe_grouped_mlp_fwd (sizes)", 2)
    if workspace is None:
        workspace = torch.empty(sz["fwd_ws"], dtype=torch.uint8, device=x.device)
    if training and saved is None:
        saved = Saved(torch.empty(sz["saved"], dtype=torch.uint8, device=x.device), (T, d, f, E, k, precision),
                      saved_h)
    if training:
        saved.saved_h = saved_h
    if y is None:
        y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device)
    L = load_library()
    _check("moe_ctx_set_saved_h", L.moe_ctx_set_saved_h(context(dev), SAVED_H[saved_h] if training else 0))
    _check("moe_grouped_mlp_fwd", L.moe_grouped_mlp_fwd(
        context(dev), x.data_ptr(), topk_idx.data_ptr(), topk_prob.data_ptr(), _ptr(split_sizes),
        _ptr_array(w_gate_up, E), _ptr_array(w_down, E), T, d, f, E, k, PRECISIONS[precision], int(training),
        y.data_ptr(), _ptr(saved.buf) if training else None, saved.buf.numel() if training else 0,
        workspace.data_ptr(), workspace.numel(), _stream(dev)))
    return y, (saved if training else None)


NOALLOC_SCRATCH_BYTES = 64 << 20


def moe_grouped_mlp_fwd_noalloc(x: torch.Tensor, topk_idx: torch.Tensor, topk_prob: torch.Tensor,
                                w_gate_up: Weights, w_down: Weights, precision: str = "mxfp8",
                                y: Optional[torch.Tensor] = None, device_status: Optional[torch.Tensor] = None,
                                split_sizes: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Inference forward that allocates no device memory inside the call (scratch is a static
    device array of NOALLOC_SCRATCH_BYTES; see include/moemx.h).  ``y`` may be preallocated."""
    dev = _device_index(x)
    T, d = x.shape
    E = len(w_gate_up)
    f = w_down[0].shape[1]
    k = topk_idx.shape[1]
    if y is None:
        y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device)
    L = load_library()
    with torch.cuda.device(dev):
        _check("moe_grouped_mlp_fwd_noalloc", L.moe_grouped_mlp_fwd_noalloc(
            x.data_ptr(), topk_idx.data_ptr(), topk_prob.data_ptr(), _ptr(split_sizes), _ptr_array(w_gate_up, E),
            _ptr_array(w_down, E), T, d, f, E, k, PRECISIONS[precision], y.data_ptr(), _ptr(device_status),
            _stream(dev)))
    return y


def moe_grouped_mlp_bwd(dy: torch.Tensor, saved: Saved, w_gate_up: Weights, w_down: Weights,
                        workspace: Optional[torch.Tensor] = None, dx: Optional[torch.Tensor] = None,
                        dw_gate_up: Optional[Weights] = None, dw_down: Optional[Weights] = None,
                        d_topk_prob: Optional[torch.Tensor] = None):
    """Gradients (dx, dw_gate_up [E,2f,d], dw_down [E,d,f], d_topk_prob [T,k]) for upstream dy."""
    T, d, f, E, k, precision = saved.dims
    dev = _device_index(dy)
    sz = sizes(T, d, f, E, k, precision, True, saved.saved_h)
    if workspace is None:
        workspace = torch.empty(sz["bwd_ws"], dtype=torch.uint8, device=dy.device)
    if dx is None:
        dx = torch.empty((T, d), dtype=torch.bfloat16, device=dy.device)
    if dw_gate_up is None:
        dw_gate_up = torch.empty((E, 2 * f, d), dtype=torch.bfloat16, device=dy.device)
    if dw_down is None:
        dw_down = torch.empty((E, d, f), dtype=torch.bfloat16, device=dy.device)
    if d_topk_prob is None:
        d_topk_prob = torch.empty((T, k), dtype=torch.float32, device=dy.device)
    L = load_library()
    _check("moe_ctx_set_saved_h", L.moe_ctx_set_saved_h(context(dev), SAVED_H[saved.saved_h]))
    _check("moe_grouped_mlp_bwd", L.moe_grouped_mlp_bwd(
        context(dev), dy.data_ptr(), saved.buf.data_ptr(), saved.buf.numel(), _ptr_array(w_gate_up, E),
        _ptr_array(w_down, E), T, d, f, E, k, PRECISIONS[precision], dx.data_ptr(), _ptr_array(dw_gate_up, E),
        _ptr_array(dw_down, E), d_topk_prob.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(dev)))
    return dx, dw_gate_up, dw_down, d_topk_prob
