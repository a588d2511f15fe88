"""Seeded random shapes against the oracle: forward and backward over every head
dim and GQA ratio, decode over every kernel (16 and 32 rows a group, 128-row
blocks with a partial last block; d = 64 and 128), with ragged lengths that do not line up with
the 128-row tiles. The shapes are drawn once from a fixed seed, so every run
checks the same cases; each case uses the same parity bounds as the targeted
tests.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.parity import BWD_REL_FRO, assert_fwd_ok, fwd_errors, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def _attention_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        d = int(rng.choice([64, 128, 256]))
        hkv = int(rng.integers(1, 4))
        g = int(rng.choice([1, 2, 4]))
        B = int(rng.integers(1, 3))
        N = int(rng.integers(1, 1400))
        causal = bool(rng.integers(0, 2))
        cases.append((B, hkv * g, hkv, N, d, causal, 7000 + i))
    return cases


def _decode_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        hkv = int(rng.integers(1, 4))
        g = int(rng.choice([1, 2, 4, 8, 16]))
        nq = int(rng.choice([1, 2, 3, 5, 8, 13, 40]))
        B = int(rng.integers(1, 4))
        nk = int(rng.integers(nq, 5000))
        causal = bool(rng.integers(0, 2))
        splits = int(rng.choice([0, 0, 1, 5]))
        d = int(rng.choice([64, 128, 128]))
        cases.append((B, hkv * g, hkv, nq, nk, causal, splits, d, 8000 + i))
    return cases


@pytest.mark.parametrize("case", _attention_cases(24, 20261203), ids=lambda c: "x".join(map(str, c[:6])))
def test_random_attention_fwd_bwd(cuda_device, case):
    import torch

    import exact_io_aware_44_b200 as fa
    B, Hq, Hkv, N, d, causal, seed = case
    w = synth.small(B, Hq, Hkv, N, d, causal, seed=seed)
    arrs = [synth.tensor(w, t) for t in (synth.TID_Q, synth.TID_K, synth.TID_V, synth.TID_DO)]
    q, k, v, do = (to_dev(x, torch.bfloat16, cuda_device) for x in arrs)
    o, lse = fa.fwd(q, k, v, causal=causal)
    dq, dk, dv = fa.bwd(q, k, v, o, lse, do, causal=causal)
    assert fa.get_status() == 0
    o_ref, lse_ref = oracle.attention_fwd64(arrs[0], arrs[1], arrs[2], causal, w.scale)
    assert_fwd_ok(fwd_errors(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref), str(case))
    refs = oracle.attention_bwd64(arrs[0], arrs[1], arrs[2], arrs[3], causal, w.scale)
    for name, a, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        assert rel_fro(a.float().cpu().numpy(), ref) <= BWD_REL_FRO, (name, case)


@pytest.mark.parametrize("case", _decode_cases(24, 20261204), ids=lambda c: "x".join(map(str, c[:8])))
def test_random_decode(cuda_device, case):
    import torch

    import exact_io_aware_44_b200 as fa
    B, Hq, Hkv, Nq, Nk, causal, splits, d, seed = case
    w = synth.DecodeWorkload("fz", B, Hq, Hkv, Nq, Nk, d, causal, seed)
    q, k, v = synth.decode_inputs(w)
    o, lse = fa.decode(*(to_dev(x, torch.bfloat16, cuda_device) for x in (q, k, v)), causal=causal,
                       num_splits=splits)
    assert fa.get_status() == 0
    o_ref, lse_ref = oracle.decode_fwd64(q, k, v, causal, w.scale)
    assert_fwd_ok(fwd_errors(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref), str(case))
