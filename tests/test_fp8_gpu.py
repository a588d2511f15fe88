"""FP8 forward parity (fa_fwd_fp8 with E4M3 inputs, fa_fwd_e5m2 with E5M2): against the float64 oracle run on the
dequantised inputs (code * descale), with the error model of tests/parity.py:
every output element within its rounding bound, the mean error within the
modelled mean, and LSE within 1e-3.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from tests.parity import assert_fp8_fwd_ok, to_dev

pytestmark = pytest.mark.gpu


def fp8_dev(codes, device, fmt="e4m3"):
    import torch
    dt = torch.float8_e5m2 if fmt == "e5m2" else torch.float8_e4m3fn
    return torch.from_numpy(np.ascontiguousarray(codes, np.float32)).to(dt).to(device)


def e4m3_dev(codes, device):
    return fp8_dev(codes, device, "e4m3")


def run_fp8(qc, kc, vc, dq, dk, dv, causal, scale, device, fmt="e4m3"):
    import exact_io_aware_44_b200 as fa
    o, lse = fa.fwd_fp8(fp8_dev(qc, device, fmt), fp8_dev(kc, device, fmt), fp8_dev(vc, device, fmt), dq, dk, dv,
                        causal=causal, scale=scale)
    assert fa.get_status() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def check_heads(qc, kc, vc, dq, dk, dv, causal, scale, o, lse, heads=None, rows_of=None, label="", fmt="e4m3"):
    """Compare the given (b, h) heads (all by default), each on `rows_of(b, h)` rows (all by default)."""
    B, Hq, N, _ = qc.shape
    g = Hq // kc.shape[1]
    heads = heads or [(b, h) for b in range(B) for h in range(Hq)]
    worst = {}
    for (b, h) in heads:
        rows = np.arange(N) if rows_of is None else rows_of(b, h)
        q64 = qc[b, h].astype(np.float64) * dq
        k64 = kc[b, h // g].astype(np.float64) * dk
        v64 = vc[b, h // g].astype(np.float64) * dv
        o_ref, lse_ref = oracle.head_fwd64(q64, k64, v64, causal, scale, rows=rows)
        p = oracle.head_probs64(q64, k64, causal, scale, rows=rows)
        st = assert_fp8_fwd_ok(o[b, h, rows], lse[b, h, rows], o_ref, lse_ref, p, v64, f"{label} head {(b, h)}", fmt)
        for key, val in st.items():
            worst[key] = max(worst.get(key, 0.0), val)
    return worst


def check_workload(w, device, causal=None):
    causal = w.causal if causal is None else causal
    qc, kc, vc = (synth.tensor(w, t) for t in (synth.TID_Q, synth.TID_K, synth.TID_V))
    ds = w.descale
    o, lse = run_fp8(qc, kc, vc, ds, ds, ds, causal, w.scale, device, w.dtype)
    return check_heads(qc, kc, vc, ds, ds, ds, causal, w.scale, o, lse, label=w.name, fmt=w.dtype)


SHAPES = [
    # B, Hq, Hkv, N (d = 128)
    (1, 1, 1, 1),
    (1, 2, 1, 17),
    (1, 1, 1, 127),
    (1, 1, 1, 128),
    (2, 2, 2, 129),
    (1, 2, 2, 256),
    (1, 4, 1, 300),
    (2, 4, 2, 640),
    (1, 2, 1, 1000),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fp8_fwd_small(cuda_device, shape, causal):
    B, Hq, Hkv, N = shape
    w = synth.small(B, Hq, Hkv, N, 128, causal, seed=500 + N, dtype="e4m3")
    check_workload(w, cuda_device)


def test_fp8_fwd_distinct_descales(cuda_device):
    """Three different, non-power-of-two descales and code ranges."""
    rng = np.random.default_rng(21)
    B, Hq, Hkv, N, d = 1, 4, 2, 700, 128
    qc = synth.round_to_e4m3(rng.standard_normal((B, Hq, N, d)).astype(np.float32) * 90)
    kc = synth.round_to_e4m3(rng.standard_normal((B, Hkv, N, d)).astype(np.float32) * 30)
    vc = synth.round_to_e4m3(rng.standard_normal((B, Hkv, N, d)).astype(np.float32) * 150)
    dq, dk, dv = 0.0123, 0.0371, 0.0057
    for causal in (True, False):
        o, lse = run_fp8(qc, kc, vc, dq, dk, dv, causal, 1 / math.sqrt(d), cuda_device)
        check_heads(qc, kc, vc, dq, dk, dv, causal, 1 / math.sqrt(d), o, lse, label=f"descales{causal}")


def test_fp8_fwd_sharp_rows_rescale_and_flush(cuda_device):
    """Large scores: rows whose max keeps growing (rescales) and whose small
    probabilities fall into E4M3's subnormal and flushed range."""
    rng = np.random.default_rng(22)
    N, d = 1024, 128
    qc = synth.round_to_e4m3(np.abs(rng.standard_normal((1, 2, N, d))).astype(np.float32) * 60)
    ramp = np.linspace(0.2, 3.0, N, dtype=np.float32)[:, None]
    kc = synth.round_to_e4m3((np.abs(rng.standard_normal((1, 2, N, d))) * ramp * 60).astype(np.float32))
    vc = synth.round_to_e4m3(rng.standard_normal((1, 2, N, d)).astype(np.float32) * 100)
    ds = 8.0 / 448.0
    for causal in (True, False):
        o, lse = run_fp8(qc, kc, vc, ds, ds, ds, causal, 1 / math.sqrt(d), cuda_device)
        check_heads(qc, kc, vc, ds, ds, ds, causal, 1 / math.sqrt(d), o, lse, label=f"sharp{causal}")


def test_fp8_fwd_closed_forms(cuda_device):
    """Q = 0: every P is exactly 1, so O is the running mean of V and LSE = ln(i + 1)."""
    rng = np.random.default_rng(23)
    N, d, dv = 600, 128, 0.02
    kc = synth.round_to_e4m3(rng.standard_normal((1, 1, N, d)).astype(np.float32) * 50)
    vc = synth.round_to_e4m3(rng.standard_normal((1, 1, N, d)).astype(np.float32) * 50)
    qc = np.zeros((1, 1, N, d), np.float32)
    o, lse = run_fp8(qc, kc, vc, 0.01, 0.01, dv, True, 1 / math.sqrt(d), cuda_device)
    cmean = np.cumsum(vc[0, 0].astype(np.float64) * dv, 0) / np.arange(1, N + 1)[:, None]
    assert np.abs(o[0, 0] - cmean).max() <= 2.0 ** -8 * np.abs(cmean).max() + 1e-5
    assert np.abs(lse[0, 0] - np.log(np.arange(1, N + 1))).max() <= 1e-4


def test_fp8_fwd_repeatable_and_bounded_writes(cuda_device):
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.small(1, 2, 1, 333, 128, True, seed=24, dtype="e4m3")
    q, k, v = (e4m3_dev(synth.tensor(w, t), cuda_device) for t in (0, 1, 2))
    n_o = q.numel()
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device=cuda_device)
    l_buf = torch.full((2 * 333 + 1024,), 7.0, dtype=torch.float32, device=cuda_device)
    ds = w.descale
    fa.fwd_fp8(q, k, v, ds, ds, ds, out=o_buf[:n_o].view(q.shape), lse=l_buf[:666].view(1, 2, 333))
    o2, l2 = fa.fwd_fp8(q, k, v, ds, ds, ds)
    torch.cuda.synchronize()
    assert torch.all(o_buf[n_o:] == 7.0) and torch.all(l_buf[666:] == 7.0)
    assert torch.equal(o_buf[:n_o].view(q.shape), o2) and torch.equal(l_buf[:666].view(1, 2, 333), l2)


@pytest.mark.parametrize("name", ["f3", "f4"])
def test_fp8_fwd_full_size_sampled(cuda_device, name):
    w = synth.WORKLOADS[name]
    qc, kc, vc = (synth.tensor(w, t) for t in (synth.TID_Q, synth.TID_K, synth.TID_V))
    ds = w.descale
    o, lse = run_fp8(qc, kc, vc, ds, ds, ds, w.causal, w.scale, cuda_device)
    check_heads(qc, kc, vc, ds, ds, ds, w.causal, w.scale, o, lse, heads=list(w.sample_heads),
                rows_of=lambda b, h: synth.sample_rows(w, b, h), label=w.name)


# ------------------------------------------------------------------ E5M2 (fa_fwd_e5m2)

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_e5m2_fwd_small(cuda_device, shape, causal):
    B, Hq, Hkv, N = shape
    w = synth.small(B, Hq, Hkv, N, 128, causal, seed=700 + N, dtype="e5m2")
    check_workload(w, cuda_device)


def test_e5m2_fwd_distinct_descales_and_rescales(cuda_device):
    """Different descales per tensor and keys whose scores grow along the sequence."""
    rng = np.random.default_rng(41)
    N, d = 1100, 128
    qc = synth.round_to_e5m2(np.abs(rng.standard_normal((1, 2, N, d))).astype(np.float32) * 3000)
    ramp = np.linspace(0.2, 3.0, N, dtype=np.float32)[:, None]
    kc = synth.round_to_e5m2((np.abs(rng.standard_normal((1, 1, N, d))) * ramp * 2000).astype(np.float32))
    vc = synth.round_to_e5m2(rng.standard_normal((1, 1, N, d)).astype(np.float32) * 5000)
    dq, dk, dv = 3.1e-4, 4.7e-4, 1.3e-4
    for causal in (True, False):
        o, lse = run_fp8(qc, kc, vc, dq, dk, dv, causal, 1 / math.sqrt(d), cuda_device, "e5m2")
        check_heads(qc, kc, vc, dq, dk, dv, causal, 1 / math.sqrt(d), o, lse, label=f"e5m2 {causal}", fmt="e5m2")


def test_e5m2_fwd_full_size_sampled(cuda_device):
    w = synth.WORKLOADS["f5"]
    qc, kc, vc = (synth.tensor(w, t) for t in (synth.TID_Q, synth.TID_K, synth.TID_V))
    ds = w.descale
    o, lse = run_fp8(qc, kc, vc, ds, ds, ds, w.causal, w.scale, cuda_device, "e5m2")
    check_heads(qc, kc, vc, ds, ds, ds, w.causal, w.scale, o, lse, heads=list(w.sample_heads),
                rows_of=lambda b, h: synth.sample_rows(w, b, h), label=w.name, fmt="e5m2")
