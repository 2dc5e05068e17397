"""Shared comparison helpers for the GPU parity tests."""
import numpy as np
import torch

# Linear outputs: max |Y - Y_ref| / max |Y_ref| <= 1e-2 (bf16 output, fp32 accumulation).
LINEAR_RTOL = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a device/host tensor as a numpy array of its unsigned type."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.int32,):
        return t.numpy().view(np.uint32)
    if t.dtype in (torch.float16, torch.bfloat16, torch.int16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.uint8:
        return t.numpy()
    if t.dtype == torch.float32:
        return t.numpy().view(np.uint32)
    raise TypeError(t.dtype)


def rel_linf(y, ref) -> float:
    y = y.detach().float().cpu().numpy().astype(np.float64) if isinstance(y, torch.Tensor) else np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-30))


def assert_linear_close(y, ref, tol=LINEAR_RTOL, what=""):
    r = rel_linf(y, ref)
    assert np.isfinite(r) and r <= tol, f"{what}: max|Y-Yref|/max|Yref| = {r:.3e} > {tol}"
    return r
