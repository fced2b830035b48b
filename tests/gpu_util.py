"""Helpers shared by the GPU parity tests (no attention arithmetic here)."""

import numpy as np
import torch

# Tolerances: max-abs 1e-2 on fp32 outputs for bf16 inputs with fp32
# accumulation; log-sum-exp within 1e-3 relative (absolute below |lse| = 1).
O_ATOL = 1e-2
LSE_RTOL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_o(got: torch.Tensor, ref: np.ndarray, what: str = "o") -> float:
    g = f64(got)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = float(np.abs(g - ref).max()) if g.size else 0.0
    if got.dtype == torch.bfloat16:
        # bf16 storage adds up to half an ulp of the reference value
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
        bound = O_ATOL + half_ulp
        assert (np.abs(g - ref) <= bound).all(), f"{what}: max err {err}"
    else:
        assert err <= O_ATOL, f"{what}: max abs err {err}"
    return err


def check_lse(got: torch.Tensor, ref: np.ndarray, what: str = "lse") -> float:
    g = f64(got)
    assert np.isfinite(g).all(), f"{what}: non-finite lse"
    rel = np.abs(g - ref) / np.maximum(1.0, np.abs(ref))
    assert (rel <= LSE_RTOL).all(), f"{what}: max rel err {rel.max()}"
    return float(rel.max()) if rel.size else 0.0


def to_dev_i32(a, device="cuda") -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.int32), device=device)
