"""Shared helpers for the GPU tests: device copies of generated workloads and
the tolerance checks used everywhere.

Tolerances (fixed by the method's accuracy targets):
  fp32 io:   |out - ref| <= 1e-4 * (1 + |ref|)  element-wise
  bf16 io:   |out - ref| <= 2e-2 * (1 + |ref|)  element-wise
  gradients: ||g - ref|| / ||ref|| <= 1e-3 per tensor, and element-wise
             |g - ref| <= 1e-2 * (|ref| + rms(ref))
"""
import numpy as np
import torch

from selective_state_space_50_b200.workloads import to_torch

TOL = {"f32": 1e-4, "bf16": 2e-2}
GRAD_NORM_TOL = 1e-3
GRAD_ELEM_TOL = 1e-2


def to_device(inp, w, device="cuda"):
    return to_torch(inp, w, device)


def subset_channels(inp, channels):
    """Restricts the per-channel arrays of a generated workload to `channels`."""
    out = {}
    for k, v in inp.items():
        base = k[:-4] if k.endswith("_f64") else k
        if base in ("u", "delta", "z", "dout"):
            out[k] = np.ascontiguousarray(v[:, channels])
        elif base in ("A", "D", "delta_bias"):
            out[k] = np.ascontiguousarray(v[channels])
        else:
            out[k] = v
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_close_io(got: np.ndarray, ref: np.ndarray, io_dtype: str, what: str = "out"):
    tol = TOL[io_dtype]
    err = np.abs(got - ref)
    bound = tol * (1.0 + np.abs(ref))
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside {tol}*(1+|ref|); worst at "
                             f"{i}: got {got[i]!r} ref {ref[i]!r}")
    return float((err / (1.0 + np.abs(ref))).max())


def assert_close_grad(got: np.ndarray, ref: np.ndarray, what: str):
    nrm = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / max(nrm, 1e-300)
    assert rel <= GRAD_NORM_TOL, f"{what}: normwise rel err {rel:.3e}"
    rms = nrm / np.sqrt(max(ref.size, 1))
    err = np.abs(got - ref)
    bound = GRAD_ELEM_TOL * (np.abs(ref) + rms) + 1e-30
    if (err > bound).any():
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: element {i} got {got[i]!r} ref {ref[i]!r} (rms {rms:.3e})")
    return float(rel)
