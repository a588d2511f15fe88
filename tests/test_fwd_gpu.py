"""Forward parity: the CUDA kernels against the float64 oracle, element by element.

Small shapes cover several tiles and ragged tails in both dimensions; the
large workloads are checked on sampled heads and query rows (each sampled row
is evaluated by the oracle over its full key row).
"""
import math

import numpy as np
import pytest

import oracle
import synth
from tests.parity import assert_fwd_ok, fwd_errors, to_dev

pytestmark = pytest.mark.gpu


def run_fwd(w, device, causal=None):
    import torch
    import exact_io_aware_44_b200 as fa
    causal = w.causal if causal is None else causal
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q = synth.tensor(w, synth.TID_Q)
    k = synth.tensor(w, synth.TID_K)
    v = synth.tensor(w, synth.TID_V)
    o, lse = fa.fwd(to_dev(q, dt, device), to_dev(k, dt, device), to_dev(v, dt, device), causal=causal,
                    scale=w.scale)
    assert fa.get_status() == 0
    return q, k, v, o.float().cpu().numpy(), lse.cpu().numpy()


def check_full(w, device, causal=None):
    causal = w.causal if causal is None else causal
    q, k, v, o, lse = run_fwd(w, device, causal)
    o_ref, lse_ref = oracle.attention_fwd64(q, k, v, causal, w.scale)
    err = fwd_errors(o, lse, o_ref, lse_ref)
    assert_fwd_ok(err, w.name)
    return err


SHAPES = [
    # B, Hq, Hkv, N, d
    (1, 1, 1, 1, 64),
    (1, 2, 1, 17, 64),
    (1, 1, 1, 127, 128),
    (1, 1, 1, 128, 128),
    (2, 2, 2, 129, 64),
    (1, 2, 2, 256, 128),
    (1, 4, 1, 300, 128),
    (2, 4, 2, 640, 64),
    (1, 2, 1, 1000, 128),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_fwd_small(cuda_device, shape, causal):
    B, Hq, Hkv, N, d = shape
    w = synth.small(B, Hq, Hkv, N, d, causal, seed=7 + N + d)
    check_full(w, cuda_device)


# More work units (query blocks x heads) than SMs, so that each CTA of the
# persistent grid runs several units in a row, among them units whose second
# query tile lies past N (N = 800 and 300: the last block holds one tile).
PERSISTENT_SHAPES = [
    # B, Hq, Hkv, N, d
    (2, 40, 8, 800, 64),
    (2, 40, 8, 800, 128),
    (1, 160, 160, 300, 256),
    (3, 64, 16, 520, 128),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", PERSISTENT_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_fwd_many_units_per_cta(cuda_device, shape, causal):
    B, Hq, Hkv, N, d = shape
    w = synth.small(B, Hq, Hkv, N, d, causal, seed=1300 + N + d)
    check_full(w, cuda_device)


D256_SHAPES = [
    # B, Hq, Hkv, N (d = 256: one 128-row query tile per CTA)
    (1, 1, 1, 1),
    (1, 2, 1, 129),
    (2, 2, 2, 300),
    (1, 4, 2, 1000),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", D256_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_fwd_d256(cuda_device, shape, causal):
    B, Hq, Hkv, N = shape
    w = synth.small(B, Hq, Hkv, N, 256, causal, seed=900 + N)
    check_full(w, cuda_device)


@pytest.mark.parametrize("d", [64, 256])
def test_bf16_fwd_spiked_rows_force_rescales(cuda_device, d):
    """Query rows x20 make late key tiles raise the running max far above the
    lazy-rescale threshold."""
    w = synth.small(1, 4, 4, 1024, d, True, seed=99, spike_frac=0.05, spike_mul=20.0)
    check_full(w, cuda_device)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_bf16_fwd_increasing_scores_rescale_every_tile(cuda_device, d):
    """Keys that grow along the sequence raise every row's max at each new tile
    (at d = 256 the rescale waits for the previous P V product, which runs beside
    the softmax)."""
    import torch
    import exact_io_aware_44_b200 as fa
    N = 1024
    rng = np.random.default_rng(5)
    q = synth.round_to_bf16(np.abs(rng.standard_normal((1, 1, N, d))).astype(np.float32))
    ramp = np.linspace(0.0, 3.0, N, dtype=np.float32)[:, None]
    k = synth.round_to_bf16((np.abs(rng.standard_normal((1, 1, N, d))) * ramp).astype(np.float32))
    v = synth.round_to_bf16(rng.standard_normal((1, 1, N, d)).astype(np.float32))
    for causal in (True, False):
        o, lse = fa.fwd(*(to_dev(x, torch.bfloat16, cuda_device) for x in (q, k, v)), causal=causal)
        o_ref, lse_ref = oracle.attention_fwd64(q, k, v, causal, 1 / math.sqrt(d))
        assert_fwd_ok(fwd_errors(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref), f"ramp{causal}")


def test_bf16_fwd_closed_forms(cuda_device):
    """Q = 0 gives running means of V and LSE = ln(i + 1); constant V returns V."""
    import torch
    import exact_io_aware_44_b200 as fa
    N, d = 384, 64
    rng = np.random.default_rng(11)
    k = synth.round_to_bf16(rng.standard_normal((1, 1, N, d)).astype(np.float32))
    v = synth.round_to_bf16(rng.standard_normal((1, 1, N, d)).astype(np.float32))
    q0 = np.zeros((1, 1, N, d), np.float32)
    dev = lambda x: to_dev(x, torch.bfloat16, cuda_device)
    o, lse = fa.fwd(dev(q0), dev(k), dev(v), causal=True)
    cmean = np.cumsum(v[0, 0].astype(np.float64), 0) / np.arange(1, N + 1)[:, None]
    assert np.abs(o.float().cpu().numpy()[0, 0] - cmean).max() <= 2e-2
    assert np.abs(lse.cpu().numpy()[0, 0] - np.log(np.arange(1, N + 1))).max() <= 1e-3
    vc = np.broadcast_to(synth.round_to_bf16(rng.standard_normal(d).astype(np.float32)), (1, 1, N, d)).copy()
    qr = synth.round_to_bf16(rng.standard_normal((1, 1, N, d)).astype(np.float32) * 4)
    o, _ = fa.fwd(dev(qr), dev(k), dev(vc), causal=False)
    assert np.abs(o.float().cpu().numpy() - vc).max() <= 2e-2


def test_bf16_fwd_leaves_memory_past_the_outputs_untouched(cuda_device):
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.small(1, 2, 2, 200, 128, True, seed=3)
    q, k, v = (to_dev(synth.tensor(w, t), torch.bfloat16, cuda_device) for t in (0, 1, 2))
    n_o = q.numel()
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device=cuda_device)
    l_buf = torch.full((2 * 200 + 1024,), 7.0, dtype=torch.float32, device=cuda_device)
    fa.fwd(q, k, v, causal=True, out=o_buf[:n_o].view_as(q), lse=l_buf[:400].view(1, 2, 200))
    torch.cuda.synchronize()
    assert torch.all(o_buf[n_o:] == 7.0)
    assert torch.all(l_buf[400:] == 7.0)


def test_bf16_fwd_repeatable(cuda_device):
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.small(1, 2, 1, 700, 128, True, seed=4)
    q, k, v = (to_dev(synth.tensor(w, t), torch.bfloat16, cuda_device) for t in (0, 1, 2))
    o1, l1 = fa.fwd(q, k, v)
    o2, l2 = fa.fwd(q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------------------------ fp32 path

def test_f32_fwd_c1_workload(cuda_device):
    """fp32, B=1 H=1 N=128 d=64, non-causal: the small exact-check workload."""
    err = check_full(synth.WORKLOADS["c1"], cuda_device)
    # fp32 arithmetic throughout: far inside the bf16 bounds
    assert err["max_abs_o"] < 1e-5 and err["max_abs_lse"] < 1e-5, err


@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 4), (1, 2, 1, 33, 32), (2, 4, 2, 100, 64), (1, 1, 1, 257, 128)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [True, False])
def test_f32_fwd_small(cuda_device, shape, causal):
    B, Hq, Hkv, N, d = shape
    w = synth.small(B, Hq, Hkv, N, d, causal, seed=100 + N, dtype="f32")
    err = check_full(w, cuda_device)
    assert err["max_abs_o"] < 1e-5 and err["max_abs_lse"] < 1e-5, err


# ------------------------------------------------------------------ full-size workloads (sampled)

def sampled_fwd_check(w, device):
    import torch
    import exact_io_aware_44_b200 as fa
    q = synth.tensor(w, synth.TID_Q)
    k = synth.tensor(w, synth.TID_K)
    v = synth.tensor(w, synth.TID_V)
    qd, kd, vd = (to_dev(x, torch.bfloat16, device) for x in (q, k, v))
    o, lse = fa.fwd(qd, kd, vd, causal=w.causal, scale=w.scale)
    assert fa.get_status() == 0
    worst = {"max_abs_o": 0.0, "mean_abs_o": 0.0, "max_abs_lse": 0.0}
    for (b, h) in w.sample_heads:
        rows = synth.sample_rows(w, b, h)
        kvh = h // w.group
        o_ref, lse_ref = oracle.head_fwd64(q[b, h], k[b, kvh], v[b, kvh], w.causal, w.scale, rows=rows)
        o_g = o[b, h, torch.from_numpy(rows).to(device)].float().cpu().numpy()
        l_g = lse[b, h, torch.from_numpy(rows).to(device)].cpu().numpy()
        err = fwd_errors(o_g, l_g, o_ref, lse_ref)
        assert_fwd_ok(err, f"{w.name} head {(b, h)}")
        for key in worst:
            worst[key] = max(worst[key], err[key])
    return worst


@pytest.mark.parametrize("name", ["c3", "c3n", "c4", "c5", "c6"])
def test_bf16_fwd_full_size_sampled(cuda_device, name):
    sampled_fwd_check(synth.WORKLOADS[name], cuda_device)


def test_bf16_fwd_c2_full(cuda_device):
    """B=4 H=16 N=2048 d=64 causal with spiked rows: every output checked."""
    check_full(synth.WORKLOADS["c2"], cuda_device)


def test_bounded_wait_reports_timeout(cuda_device):
    """A barrier nothing completes: the bounded wait must give up, record
    FA_ERR_DEVICE_TIMEOUT and return (no trap, no hang)."""
    import exact_io_aware_44_b200 as fa
    assert fa.selftest_wait_timeout(5_000_000) == -5
    assert fa.get_status() == 0   # the status word was cleared


def test_progress_record_counts_each_ctas_work(cuda_device):
    """The per-CTA progress words after a launch equal the work each CTA was
    given: P V products in the forward, query tiles in the backward."""
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.small(1, 2, 1, 300, 128, True, seed=4)
    q, k, v, do = (to_dev(synth.tensor(w, t), torch.bfloat16, cuda_device)
                   for t in (synth.TID_Q, synth.TID_K, synth.TID_V, synth.TID_DO))
    o, lse = fa.fwd(q, k, v, causal=True)
    # 2 heads x 2 blocks of 256 query rows; each block issues 3 P V products
    # (rows 0-255: 1 + 2 key tiles; rows 256-299: 3 key tiles)
    assert fa.get_progress(4) == [3, 3, 3, 3]
    fa.bwd(q, k, v, o, lse, do, causal=True)
    # key tiles 0, 1, 2 of the one kv head see 3, 2, 1 query tiles of each of 2 query heads
    assert sorted(fa.get_progress(3)) == [2, 4, 6]
    assert fa.get_status() == 0


def test_progress_record_d256(cuda_device):
    """d = 256 runs one 128-row query tile per CTA: each CTA issues as many P V
    products as its tile visits key tiles."""
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.small(1, 2, 1, 300, 256, True, seed=5)
    q, k, v = (to_dev(synth.tensor(w, t), torch.bfloat16, cuda_device)
               for t in (synth.TID_Q, synth.TID_K, synth.TID_V))
    fa.fwd(q, k, v, causal=True)
    # 2 heads x 3 query tiles, which visit 1, 2 and 3 key tiles
    assert sorted(fa.get_progress(6)) == [1, 1, 2, 2, 3, 3]
    assert fa.get_status() == 0
