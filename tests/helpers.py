"""Shared helpers for the parity tests: marshal torch tensors to the oracle's
input format and compute the tolerance metric."""
import numpy as np
import torch

# max |err| / max |ref| per (request, tensor); the bar depends on the input dtype
TOL = {"f32": 1e-4, "bf16": 2e-2}


def oracle_view(t: torch.Tensor) -> np.ndarray:
    """Exact bytes of a tensor as the oracle takes them: float32 values or bf16 bits."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.max(np.abs(ref))
    if denom == 0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref)) / denom)


def per_request_state_err(got, ref):
    """Largest per-request relative error of [B, H, dk, dv] states."""
    return max(rel_err(got[b], ref[b]) for b in range(ref.shape[0])) if ref.shape[0] else 0.0


def per_request_rows_err(got, ref, cu):
    """Largest per-request relative error of packed [rows, H, d] outputs."""
    errs = [rel_err(got[cu[b]:cu[b + 1]], ref[cu[b]:cu[b + 1]])
            for b in range(len(cu) - 1) if cu[b + 1] > cu[b]]
    return max(errs) if errs else 0.0
