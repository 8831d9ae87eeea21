"""Helpers for the GPU parity tests (test-side code; shares nothing with the CUDA library)."""
import json
import os

import numpy as np
import torch


def has_b200() -> bool:
    if not torch.cuda.is_available():
        return False
    return torch.cuda.get_device_capability(0) == (10, 0)


def unswizzle_scales(buf: np.ndarray, R: int, KB: int) -> np.ndarray:
    """Plain [R, KB] view of a scale matrix stored in the tensor-core tile layout documented in
    include/moemx.h: 512-byte tiles of 128 rows x 4 scale columns, row-block major; inside a
    tile S[r][kb] at 16*(r%32) + 4*((r//32)%4) + kb%4."""
    buf = np.asarray(buf).reshape(-1)
    r = np.arange(R)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r // 128) * (KB // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    return buf[off]


def rel_err(got, ref) -> float:
    """max |got - ref| / max |ref| (the tolerance metric of the parity tests)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    if den == 0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref)) / den)


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def p99_rel_err(got, ref) -> float:
    """99th percentile of the element-wise relative error |got - ref| / max(|ref|, 1e-3 max|ref|)
    (the floor keeps elements near zero from dominating)."""
    got = np.asarray(got, dtype=np.float64).reshape(-1)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1)
    den = np.maximum(np.abs(ref), 1e-3 * max(float(np.max(np.abs(ref))), 1e-300))
    return float(np.percentile(np.abs(got - ref) / den, 99))


def parity(name: str, got, ref, tol: float) -> float:
    """Assert max|got - ref| / max|ref| <= tol and return it; the figure and the element-wise p99
    relative error are appended as a JSON line to the file named by MOE_PARITY_REPORT, if set."""
    err = rel_err(got, ref)
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        with open(path, "a") as fh:
            fh.write(json.dumps({"case": name, "max_rel": err, "p99_rel": p99_rel_err(got, ref), "tol": tol}) + "\n")
    assert err <= tol, f"{name}: {err:.3g} > {tol}"
    return err
