"""Shared helpers of the GPU parity tests: inputs from `synth`, comparison
metrics, and the tolerances the kernels are held to.

Tolerances (bf16 in, fp32 accumulation; the oracle is float64 on the same
bf16-rounded inputs, so input quantisation is not counted):
  forward   max |dO| <= 2e-2, mean |dO| <= 2e-3, max |dLSE| <= 1e-3
  backward  relative Frobenius error <= 1e-2 for each of dQ, dK, dV

FP8 forward (the oracle runs on the dequantised E4M3 or E5M2 inputs, so again only
the kernel's own rounding counts; the figures below are E4M3's, E5M2 has 2^-3 relative
and 2^-17 absolute in place of 2^-4 and 2^-10). S is exact E4M3 products summed in fp32, so LSE
keeps the 1e-3 bound. The one coarse step is P: the kernel rounds
e_j = exp(s_j - m_ref) (m_ref <= the row max) to E4M3 before P V but divides by
L = sum_j e_j unrounded. E4M3 rounding moves e by at most 2^-4 e (normal range)
or 2^-10 (subnormal step 2^-9), and L >= 1 / pi_max, with pi the exact softmax
row. Hence, per output element,
  |dO_id| <= 2^-4 sum_j pi_ij |v_jd| + 2^-10 n_i pi_max,i max_j |v_jd|
             + 2^-8 |O_id| (bf16 output) + 1e-5,
with n_i the keys row i sees. For the mean, the rounding errors are modelled as
independent and uniform over one E4M3 step (variance step^2 / 12; values that
flush to zero count e^2), which gives a standard deviation sigma_id per element;
E|X| <= sigma (Jensen), and the test allows 10% over the model plus the bf16
output rounding (mean <= 2^-9 |O|).
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


# FP8 formats: mantissa bits and the smallest normal exponent
FP8_FORMATS = {"e4m3": (3, -6), "e5m2": (2, -14)}


def fp8_step(e, fmt="e4m3"):
    """Spacing of the format's values around e >= 0 (constant in the subnormal range)."""
    mant, emin = FP8_FORMATS[fmt]
    e = np.asarray(e, np.float64)
    ex = np.floor(np.log2(np.where(e > 0, e, 1.0)))
    return np.exp2(np.maximum(ex, float(emin)) - mant)


def e4m3_step(e):
    return fp8_step(e, "e4m3")


def fp8_fwd_model(p_rows, v, o_ref, fmt="e4m3"):
    """Per-element error bound and the modelled mean |dO| for the E4M3 forward.

    p_rows [R, N]: exact softmax rows (oracle.head_probs64); v [N, d] the
    dequantised V; o_ref [R, d] the oracle output. Returns (bound [R, d], mean)."""
    p = np.asarray(p_rows, np.float64)
    v = np.asarray(v, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    pmax = p.max(axis=1)
    n = (p > 0).sum(axis=1)
    vmax = np.abs(v).max(axis=0)
    mant, emin = FP8_FORMATS[fmt]
    rel, flush = 2.0 ** -(mant + 1), 2.0 ** (emin - mant - 1)   # half a step: relative, and absolute below normals
    bound = rel * (p @ np.abs(v)) + flush * (n * pmax)[:, None] * vmax[None, :] \
        + (2.0 ** -8) * np.abs(o_ref) + 1e-5
    e = p / pmax[:, None]                                   # kernel units with m_ref = row max
    var_unit = np.where(e >= flush, fp8_step(e, fmt) ** 2 / 12.0, e * e)
    sigma = np.sqrt(var_unit @ (v * v)) * pmax[:, None]     # divided by L = 1 / pmax
    mean = 1.1 * float(sigma.mean()) + (2.0 ** -9) * float(np.abs(o_ref).mean()) + 1e-6
    return bound, mean


def assert_fp8_fwd_ok(o_gpu, lse_gpu, o_ref, lse_ref, p_rows, v, label="", fmt="e4m3"):
    """o_gpu, o_ref, p_rows: rows of ONE head; v [N, d] that head's dequantised V."""
    o_gpu = np.asarray(o_gpu, np.float64)
    err = np.abs(o_gpu - o_ref)
    bound, mean = fp8_fwd_model(p_rows, v, o_ref, fmt)
    worst = float((err / bound).max()) if err.size else 0.0
    dl = float(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref).max()) if err.size else 0.0
    stats = {"max_abs_o": float(err.max()) if err.size else 0.0, "mean_abs_o": float(err.mean()) if err.size else 0.0,
             "mean_model": mean, "max_err_over_bound": worst, "max_abs_lse": dl}
    assert worst <= 1.0, (label, stats)
    assert stats["mean_abs_o"] <= mean, (label, stats)
    assert dl <= LSE_MAX_ABS, (label, stats)
    return stats
