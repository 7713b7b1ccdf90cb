"""Shared helpers for the GPU parity tests (tensor conversion and the tolerance rule).

Tolerances (stated for this method's parity contract):
  fp32 path:                         max|gpu - oracle| <= 1e-5 * max|oracle|
  bf16 inputs, fp32 accumulation:    max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3
Index / CSR handling is checked bit-exactly with probe inputs.
"""
import numpy as np
import torch

import rocs_inputs as ri


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy fp32 or bf16-bits (uint16) -> CUDA tensor (fp32 or bf16)."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return ri.bf16_to_f32(t.view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    return t.numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def assert_close(got, ref, kind: str, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    scale = float(np.abs(ref).max())
    err = float(np.abs(got - ref).max())
    tol = 1e-5 * scale if kind == "f32" else 1e-2 * scale + 1e-3
    assert err <= tol, f"{what}: max|gpu-oracle| = {err:.3e} > tol {tol:.3e} (max|oracle| = {scale:.3e})"
    return err, tol
