"""Backward parity: the CUDA backward (fed the CUDA forward's O and LSE, as a
user would) against the float64 oracle's gradients of L = sum(O o dO).

Bound: relative Frobenius error <= 1e-2 for each of dQ, dK, dV. Small shapes
are compared in full; the long workloads on sampled heads and rows (dQ on
sampled query rows, dK/dV on sampled key rows, each exact in float64).
"""
import numpy as np
import pytest

import oracle
import synth
from tests.parity import BWD_REL_FRO, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def gpu_fwd_bwd(w, device, workspace_fill=None):
    import torch
    import exact_io_aware_44_b200 as fa
    arrs = [synth.tensor(w, t) for t in (synth.TID_Q, synth.TID_K, synth.TID_V, synth.TID_DO)]
    q, k, v, do = (to_dev(x, torch.bfloat16, device) for x in arrs)
    o, lse = fa.fwd(q, k, v, causal=w.causal, scale=w.scale)
    ws = None
    if workspace_fill is not None:
        n = fa.workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d)
        ws = torch.empty(n // 4 + 64, dtype=torch.float32, device=device).fill_(workspace_fill)
    dq, dk, dv = fa.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, workspace=ws)
    assert fa.get_status() == 0
    return arrs, (dq, dk, dv)


def check_full(w, device, **kw):
    (q, k, v, do), grads = gpu_fwd_bwd(w, device, **kw)
    refs = oracle.attention_bwd64(q, k, v, do, w.causal, w.scale)
    errs = {}
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        errs[name] = rel_fro(g.float().cpu().numpy(), r)
        assert errs[name] <= BWD_REL_FRO, (w.name, name, errs)
    return errs


SHAPES = [
    # B, Hq, Hkv, N, d
    (1, 1, 1, 1, 64),
    (1, 1, 1, 17, 128),
    (1, 2, 1, 64, 128),
    (1, 1, 1, 127, 64),
    (1, 1, 1, 128, 128),
    (2, 2, 2, 129, 64),
    (1, 2, 2, 200, 128),
    (1, 4, 1, 300, 128),
    (2, 4, 2, 640, 64),
    (1, 2, 1, 1000, 128),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_bwd_small(cuda_device, shape, causal):
    B, Hq, Hkv, N, d = shape
    w = synth.small(B, Hq, Hkv, N, d, causal, seed=31 + N + d)
    check_full(w, cuda_device)


D256_SHAPES = [
    # B, Hq, Hkv, N (d = 256: 64-row query tiles, two passes over the head dim)
    (1, 1, 1, 1),
    (1, 2, 1, 65),
    (1, 1, 1, 128),
    (2, 2, 2, 300),
    (1, 4, 2, 1000),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", D256_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_bwd_d256(cuda_device, shape, causal):
    B, Hq, Hkv, N = shape
    w = synth.small(B, Hq, Hkv, N, 256, causal, seed=950 + N)
    check_full(w, cuda_device)


def test_bf16_bwd_workspace_contents_do_not_matter(cuda_device):
    w = synth.small(1, 2, 1, 333, 128, True, seed=8)
    check_full(w, cuda_device, workspace_fill=float("nan"))


def test_bf16_bwd_spiked_rows(cuda_device):
    w = synth.small(1, 4, 2, 1024, 128, True, seed=77, spike_frac=0.02, spike_mul=20.0)
    check_full(w, cuda_device)


def test_bf16_bwd_dk_dv_deterministic(cuda_device):
    w = synth.small(1, 4, 2, 512, 128, True, seed=5)
    _, (dq1, dk1, dv1) = gpu_fwd_bwd(w, cuda_device)
    _, (dq2, dk2, dv2) = gpu_fwd_bwd(w, cuda_device)
    import torch
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    # dQ is accumulated with fp32 atomics: equal up to rounding
    assert rel_fro(dq2.float().cpu().numpy(), dq1.float().cpu().numpy()) < 1e-3


def test_bf16_bwd_c2_full(cuda_device):
    """B=4 H=16 N=2048 d=64 causal with 1% of query rows x20: every gradient checked."""
    check_full(synth.WORKLOADS["c2"], cuda_device)


def sampled_bwd_check(w, device):
    import torch
    (q, k, v, do), (dq, dk, dv) = gpu_fwd_bwd(w, device)
    kv_heads = sorted({(b, h // w.group) for (b, h) in w.sample_heads})
    worst = {}
    for (b, kvh) in kv_heads:
        heads = list(range(kvh * w.group, (kvh + 1) * w.group))
        q_rows = synth.sample_rows(w, b, heads[0])
        k_rows = synth.sample_rows(w, b, kvh, count=w.sample_rows)
        rq, rk, rv = oracle.group_bwd_sampled64(q[b, heads], k[b, kvh], v[b, kvh], do[b, heads], w.causal, w.scale,
                                               q_rows, k_rows)
        qi = torch.from_numpy(q_rows).to(device)
        ki = torch.from_numpy(k_rows).to(device)
        g_q = dq[b, heads][:, qi].float().cpu().numpy()
        g_k = dk[b, kvh, ki].float().cpu().numpy()
        g_v = dv[b, kvh, ki].float().cpu().numpy()
        for name, g, r in (("dq", g_q, rq), ("dk", g_k, rk), ("dv", g_v, rv)):
            e = rel_fro(g, r)
            worst[name] = max(worst.get(name, 0.0), e)
            assert e <= BWD_REL_FRO, (w.name, (b, kvh), name, e)
    return worst


@pytest.mark.parametrize("name", ["c3", "c3n", "c5", "c6b"])
def test_bf16_bwd_full_size_sampled(cuda_device, name):
    sampled_bwd_check(synth.WORKLOADS[name], cuda_device)


def test_bwd_equals_its_three_phases(cuda_device):
    """fa_bwd is fa_bwd_preprocess, fa_bwd_main and fa_bwd_convert in order."""
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.small(1, 4, 2, 384, 128, True, seed=21)
    q, k, v, do = (to_dev(synth.tensor(w, t), torch.bfloat16, cuda_device) for t in range(4))
    o, lse = fa.fwd(q, k, v)
    dq1, dk1, dv1 = fa.bwd(q, k, v, o, lse, do)
    dq2, dk2, dv2 = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.workspace_bytes(1, 4, 2, 384, 128), dtype=torch.uint8, device=cuda_device)
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: t.data_ptr()
    rc = fa.bwd_phases_raw(ptr(q), ptr(k), ptr(v), ptr(o), ptr(lse), ptr(do), ptr(dq2), ptr(dk2), ptr(dv2), ptr(ws),
                           1, 4, 2, 384, 128, True, w.scale, stream)
    assert rc == 0 and fa.get_status() == 0
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert rel_fro(dq2.float().cpu().numpy(), dq1.float().cpu().numpy()) < 1e-3
