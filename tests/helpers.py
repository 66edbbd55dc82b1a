"""Shared helpers of the GPU parity tests: oracle inputs built from the same seeded
bf16 tensors that the CUDA path gets, and the tolerance of the comparisons."""
import numpy as np
import torch

from oracle import quant

# Floating-point outputs and gradients: max |gpu - oracle| <= TOL * max |oracle|;
# loss: relative 1e-3 (the tolerances the target states).
TOL = 2e-2
LOSS_RTOL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def close(gpu, ref, tol=TOL, what=""):
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.max(np.abs(g - r)) if g.size else 0.0
    scale = np.max(np.abs(r)) if r.size else 0.0
    assert err <= tol * scale, f"{what}: max|diff| {err:.3e} > {tol} * max|ref| {scale:.3e}"
    return err / scale if scale else 0.0


def oracle_weights(w: dict) -> dict:
    """Dequantised float64 weights of a layer, by the oracle, from the bf16 tensors."""
    out = {}
    for name in ("q", "k", "v", "o", "gate", "up", "down"):
        t = w[name]
        q = quant.quantize(t.float().cpu().numpy().reshape(-1))
        out[name] = quant.dequantize(q).reshape(t.shape)
    out["norm_in"] = f64(w["norm_in"])
    out["norm_post"] = f64(w["norm_post"])
    return out


def oracle_lora(lo: dict) -> dict:
    return {k: f64(v) for k, v in lo.items()}
