"""Shared helpers of the GPU parity tests: inputs from `synth`, comparison
metrics, and the tolerances the kernels are held to.

Tolerances (bf16 in, fp32 accumulation; the oracle is float64 on the same
bf16-rounded inputs, so input quantisation is not counted):
  forward   max |dO| <= 2e-2, mean |dO| <= 2e-3, max |dLSE| <= 1e-3
  backward  relative Frobenius error <= 1e-2 for each of dQ, dK, dV
"""
import numpy as np

FWD_MAX_ABS = 2e-2
FWD_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
BWD_REL_FRO = 1e-2


def to_dev(x, dtype, device):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(device=device, dtype=dtype)


def fwd_errors(o_gpu, lse_gpu, o_ref, lse_ref):
    do = np.abs(np.asarray(o_gpu, np.float64) - o_ref)
    dl = np.abs(np.asarray(lse_gpu, np.float64) - lse_ref)
    return {"max_abs_o": float(do.max()) if do.size else 0.0,
            "mean_abs_o": float(do.mean()) if do.size else 0.0,
            "max_abs_lse": float(dl.max()) if dl.size else 0.0}


def assert_fwd_ok(err, label=""):
    assert err["max_abs_o"] <= FWD_MAX_ABS, (label, err)
    assert err["mean_abs_o"] <= FWD_MEAN_ABS, (label, err)
    assert err["max_abs_lse"] <= LSE_MAX_ABS, (label, err)


def rel_fro(x, ref):
    """||x - ref||_F / ||ref||_F. Where the exact gradient vanishes (N = 1 gives
    dS = 0, hence dQ = dK = 0), the denominator is floored at an RMS of 1e-3
    per element, so only rounding-level noise passes."""
    ref = np.asarray(ref, np.float64)
    den = max(np.linalg.norm(ref), 1e-3 * np.sqrt(max(ref.size, 1)))
    return float(np.linalg.norm(np.asarray(x, np.float64) - ref) / den)
