"""Decode parity: fa_decode (queries at the end of a longer key/value cache,
split along the keys and merged) against the float64 oracle, element by
element, with the bf16 forward tolerances."""
import math

import numpy as np
import pytest

import oracle
import synth
from tests.parity import assert_fwd_ok, fwd_errors, to_dev

pytestmark = pytest.mark.gpu


def run_decode(w, device, num_splits=0, causal=None):
    import torch
    import exact_io_aware_44_b200 as fa
    causal = w.causal if causal is None else causal
    q, k, v = synth.decode_inputs(w)
    o, lse = fa.decode(*(to_dev(x, torch.bfloat16, device) for x in (q, k, v)), causal=causal, scale=w.scale,
                       num_splits=num_splits)
    assert fa.get_status() == 0
    return q, k, v, o.float().cpu().numpy(), lse.cpu().numpy()


def check(w, device, num_splits=0, causal=None):
    causal = w.causal if causal is None else causal
    q, k, v, o, lse = run_decode(w, device, num_splits, causal)
    o_ref, lse_ref = oracle.decode_fwd64(q, k, v, causal, w.scale)
    err = fwd_errors(o, lse, o_ref, lse_ref)
    assert_fwd_ok(err, f"{w.name} splits={num_splits} causal={causal}")
    return err


SHAPES = [
    # B, Hq, Hkv, Nq, Nk
    (1, 8, 1, 1, 1),
    (1, 8, 1, 1, 127),
    (1, 8, 1, 1, 128),
    (1, 8, 1, 1, 129),
    (2, 8, 2, 1, 1000),
    (1, 4, 1, 4, 700),      # 16 query rows per CTA
    (2, 16, 1, 1, 3000),    # a 16-head group
    (1, 2, 2, 3, 333),      # no GQA, 3 new tokens
    (1, 4, 4, 2, 4097),
    (1, 8, 1, 3, 900),      # 24 rows: the 32-row kernel, 8 rows unused
    (2, 32, 4, 4, 2500),    # GQA group 8 x 4 new tokens = 32 rows
    (1, 32, 1, 1, 513),     # a 32-head group
    (1, 2, 1, 16, 640),     # 16 new tokens per head, 32 rows, the causal edge spans 16 keys
    (1, 1, 1, 17, 17),      # square, 17 rows
    (3, 8, 2, 1, 7000),     # 330 chunks over 148 CTAs: slices cross group boundaries
    (1, 32, 4, 4, 9000),    # the same with 32 rows
    (64, 16, 8, 1, 200),    # 1024 chunks of short caches: about 4 segments per CTA
    (32, 32, 4, 3, 300),    # 24 rows, 3 chunks a group, segments across groups
    # more than 32 rows a group: 128-row blocks with the rows as the MMA's M
    (1, 8, 1, 5, 900),      # 40 rows, one block, 88 rows unused
    (2, 64, 1, 1, 3000),    # a 64-head group (MQA)
    (1, 16, 2, 8, 1000),    # GQA group 8 x 8 new tokens = 64 rows, the causal edge spans 8 keys
    (2, 32, 2, 8, 2500),    # 128 rows: one full block
    (1, 16, 1, 9, 700),     # 144 rows: a full block and a block of 16
    (1, 4, 1, 100, 640),    # 400 rows: four blocks, the causal edge spans 100 keys
    (1, 1, 1, 200, 200),    # square, 200 rows
    (8, 32, 4, 5, 3000),    # 40 rows, 24 chunks a block over 148 CTAs: segments across blocks
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("splits", [0, 1, 7])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_decode_small(cuda_device, shape, splits, causal):
    B, Hq, Hkv, Nq, Nk = shape
    w = synth.DecodeWorkload(f"d{'x'.join(map(str, shape))}", B, Hq, Hkv, Nq, Nk, 128, causal, 2000 + Nk + Nq)
    check(w, cuda_device, splits)


D64_SHAPES = [
    # B, Hq, Hkv, Nq, Nk: d = 64 takes 128-row blocks for every group size
    (1, 8, 1, 1, 1),
    (2, 8, 2, 1, 1000),
    (1, 32, 4, 4, 2500),    # 32 rows
    (2, 16, 2, 8, 1300),    # 64 rows
    (1, 16, 1, 9, 700),     # 144 rows: a full block and a block of 16
    (3, 8, 2, 1, 7000),     # segments across units
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("splits", [0, 3])
@pytest.mark.parametrize("shape", D64_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_decode_d64(cuda_device, shape, splits, causal):
    B, Hq, Hkv, Nq, Nk = shape
    w = synth.DecodeWorkload(f"d64_{'x'.join(map(str, shape))}", B, Hq, Hkv, Nq, Nk, 64, causal, 2600 + Nk + Nq)
    check(w, cuda_device, splits)


def test_decode_square_matches_the_forward(cuda_device):
    """Nq = Nk: the decode mask is fa_fwd's causal mask; both within tolerance of each other."""
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.DecodeWorkload("sq", 1, 4, 1, 4, 4, 128, True, 77)
    q, k, v = synth.decode_inputs(w)
    dev = lambda x: to_dev(x, torch.bfloat16, cuda_device)
    o1, l1 = fa.decode(dev(q), dev(k), dev(v), causal=True)
    o2, l2 = fa.fwd(dev(q), dev(k).repeat_interleave(4, 1).contiguous(), dev(v).repeat_interleave(4, 1).contiguous(),
                    causal=True)
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_decode_spiked_scores_rescale(cuda_device):
    """Keys whose scores grow along the cache force reference-max raises in later chunks."""
    import torch
    import exact_io_aware_44_b200 as fa
    rng = np.random.default_rng(31)
    B, Hq, Hkv, Nq, Nk, d = 1, 8, 2, 2, 2500, 128
    q = synth.round_to_bf16(np.abs(rng.standard_normal((B, Hq, Nq, d))).astype(np.float32))
    ramp = np.linspace(0.0, 4.0, Nk, dtype=np.float32)[:, None]
    k = synth.round_to_bf16((np.abs(rng.standard_normal((B, Hkv, Nk, d))) * ramp).astype(np.float32))
    v = synth.round_to_bf16(rng.standard_normal((B, Hkv, Nk, d)).astype(np.float32))
    dev = lambda x: to_dev(x, torch.bfloat16, cuda_device)
    for causal in (True, False):
        for splits in (0, 1, 5):
            o, lse = fa.decode(dev(q), dev(k), dev(v), causal=causal, num_splits=splits)
            o_ref, lse_ref = oracle.decode_fwd64(q, k, v, causal, 1 / math.sqrt(d))
            assert_fwd_ok(fwd_errors(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref),
                          f"ramp causal={causal} splits={splits}")


def test_decode_repeatable_and_bounded_writes(cuda_device):
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.DecodeWorkload("rep", 2, 8, 2, 1, 1500, 128, True, 78)
    q, k, v = (to_dev(x, torch.bfloat16, cuda_device) for x in synth.decode_inputs(w))
    n_o = q.numel()
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device=cuda_device)
    l_buf = torch.full((16 + 1024,), 7.0, dtype=torch.float32, device=cuda_device)
    fa.decode(q, k, v, out=o_buf[:n_o].view_as(q), lse=l_buf[:16].view(2, 8, 1))
    o2, l2 = fa.decode(q, k, v)
    torch.cuda.synchronize()
    assert torch.all(o_buf[n_o:] == 7.0) and torch.all(l_buf[16:] == 7.0)
    assert torch.equal(o_buf[:n_o].view_as(q), o2) and torch.equal(l_buf[:16].view(2, 8, 1), l2)


@pytest.mark.parametrize("shape", [(3, 8, 2, 1, 7000), (1, 16, 1, 9, 700), (2, 32, 4, 4, 2500)],
                         ids=lambda s: "x".join(map(str, s)))
def test_decode_workspace_reused_with_garbage(cuda_device, shape):
    """One workspace, filled with garbage and reused across calls and split counts:
    nothing in it carries over, so each result equals the oracle."""
    import torch
    import exact_io_aware_44_b200 as fa
    B, Hq, Hkv, Nq, Nk = shape
    w = synth.DecodeWorkload("ws" + "x".join(map(str, shape)), B, Hq, Hkv, Nq, Nk, 128, True, 3000 + Nk)
    q, k, v = synth.decode_inputs(w)
    dev = lambda x: to_dev(x, torch.bfloat16, cuda_device)
    qd, kd, vd = dev(q), dev(k), dev(v)
    nbytes = max(fa.decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, 128, s) for s in (0, 3, 7))
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device=cuda_device)
    o_ref, lse_ref = oracle.decode_fwd64(q, k, v, True, w.scale)
    for splits in (0, 7, 3, 0):
        o, lse = fa.decode(qd, kd, vd, causal=True, num_splits=splits, workspace=ws)
        assert fa.get_status() == 0
        assert_fwd_ok(fwd_errors(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref),
                      f"reused workspace splits={splits}")


@pytest.mark.parametrize("name", ["dec", "dec4", "dec8", "dec64"])
def test_decode_full_size_workload(cuda_device, name):
    """The benchmark's decode steps (B=16 against 32768 cached keys: Hq=32 Hkv=8 with
    one new query at d = 128 and at d = 64, Hq=32 Hkv=4 with four, Hq=64 Hkv=8 with
    eight), in the launch configuration the benchmark times (automatic splits); every
    output computed, sampled heads checked against the oracle."""
    w = synth.DECODE_WORKLOADS[name]
    q, k, v, o, lse = run_decode(w, cuda_device)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    for (b, h) in ((0, 0), (3, 9), (7, 31), (15, 16), (15, w.Hq - 1)):
        kvh = h // w.group
        o_ref, lse_ref = oracle.decode_fwd64(q[b:b + 1, h:h + 1], k[b:b + 1, kvh:kvh + 1], v[b:b + 1, kvh:kvh + 1],
                                             w.causal, w.scale)
        assert_fwd_ok(fwd_errors(o[b, h], lse[b, h], o_ref[0, 0], lse_ref[0, 0]), f"dec head {(b, h)}")
