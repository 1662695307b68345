"""Shared parity bar for the CUDA path against the CPU oracle.

Tolerances (fixed for this kernel): O max-abs <= 2e-2 and relative L2 <= 5e-3,
LSE max-abs <= 1e-3, both against the oracle's float64 result on the same
bf16-rounded inputs.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def to_f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def errors(o, lse, o_ref, lse_ref):
    o, lse = to_f64(o), to_f64(lse)
    o_ref, lse_ref = np.asarray(o_ref, np.float64), np.asarray(lse_ref, np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), "non-finite output"
    max_abs = float(np.abs(o - o_ref).max())
    rel = float(np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    lse_abs = float(np.abs(lse - lse_ref).max())
    return max_abs, rel, lse_abs


def assert_parity(o, lse, o_ref, lse_ref, tag=""):
    max_abs, rel, lse_abs = errors(o, lse, o_ref, lse_ref)
    msg = f"{tag}: O max-abs {max_abs:.3e}, O rel-L2 {rel:.3e}, LSE max-abs {lse_abs:.3e}"
    assert max_abs <= O_MAX_ABS and rel <= O_REL_L2 and lse_abs <= LSE_MAX_ABS, msg
    return max_abs, rel, lse_abs
