"""Shared helpers for the GPU parity tests.

Tolerance (from the stated accuracy target for bf16 inputs with fp32
accumulation): max |gpu - oracle| <= 2e-3 and max rel <= 1e-2, where
rel_i = |gpu_i - ref_i| / max(|ref_i|, 0.2); the 0.2 floor is atol / rtol, so
below it the relative bound is the absolute bound.  A bf16 output is compared
against the oracle value rounded to bf16: within 2e-3 or within one bf16 ulp.
"""

from __future__ import annotations

import numpy as np
import torch

ATOL = 2e-3
RTOL = 1e-2
REL_FLOOR = ATOL / RTOL


def errors(gpu: np.ndarray, ref: np.ndarray):
    err = np.abs(gpu.astype(np.float64) - ref)
    rel = err / np.maximum(np.abs(ref), REL_FLOOR)
    return float(err.max(initial=0.0)), float(rel.max(initial=0.0))


def assert_parity(gpu_out: torch.Tensor, ref: np.ndarray, what: str = ""):
    """Element-by-element comparison of a GPU result with the fp64 oracle."""
    g = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    if gpu_out.dtype == torch.bfloat16:
        rb = torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16).double().numpy()
        ulp = np.spacing(np.abs(rb).astype(np.float32)).astype(np.float64) * 65536.0  # bf16 ulp
        diff = np.abs(g - rb)
        bad = (diff > ATOL) & (diff > ulp)
        assert not bad.any(), f"{what}: {int(bad.sum())} bf16 outputs off (max diff {diff.max():.3g})"
        return
    err, rel = errors(g, ref)
    assert err <= ATOL and rel <= RTOL, f"{what}: max abs {err:.3g}, max rel {rel:.3g}"


def to_device(inputs: dict, device) -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}
