"""fa_bwd_noalloc, the backward pass for callers that cannot allocate device
memory (plugins whose host owns every allocation, loops that must avoid
cudaMalloc's implicit synchronisation, fixed-budget deployments).

Its scratch is a static device array inside the library rather than a
caller-provided workspace. These tests call it through the C ABI and compare
it with fa_bwd on the same inputs, twice in a row, because every call reuses
the array the previous call left behind. The file is named to run after all
other tests and also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import synth
from tests.parity import BWD_REL_FRO, rel_fro, to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def _noalloc(fa, q, k, v, o, lse, do, dq, dk, dv, w, stream):
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    return fa.lib.fa_bwd_noalloc(P(q), P(k), P(v), P(o), P(lse), P(do), P(dq), P(dk), P(dv), w.B, w.Hq, w.Hkv,
                                 w.N, w.d, int(w.causal), float(w.scale), ctypes.c_void_p(stream))


@pytest.mark.parametrize("d", [128, 64])
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row(cuda_device, d):
    import torch
    import exact_io_aware_44_b200 as fa
    w = synth.small(2, 4, 2, 700, d, True, seed=4242 + d)
    assert fa.workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d) <= SCRATCH_BYTES
    q, k, v, do = (to_dev(synth.tensor(w, t), torch.bfloat16, cuda_device) for t in range(4))
    o, lse = fa.fwd(q, k, v, causal=w.causal, scale=w.scale)
    ref = fa.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)   # the existing entry point
    assert fa.get_status() == 0
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rc = _noalloc(fa, q, k, v, o, lse, do, dq, dk, dv, w, stream)
        assert rc == 0, (call, rc)
        assert fa.get_status() == 0
        for name, got, exp in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
            err = rel_fro(got.float().cpu().numpy(), exp.float().cpu().numpy())
            assert err <= BWD_REL_FRO, (call, name, err)
        # the same kernels on the same inputs: dK and dV are bit-identical
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2]), call


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    import torch
    import exact_io_aware_44_b200 as fa
    B, Hq, Hkv, N, d = 1, 32, 8, 8192, 128       # needs ~135 MB of scratch
    assert fa.workspace_bytes(B, Hq, Hkv, N, d) > SCRATCH_BYTES
    dk = torch.full((B, Hkv, 128, d), 3.0, dtype=torch.bfloat16, device=cuda_device)
    p = ctypes.c_void_p(dk.data_ptr())
    rc = fa.lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, Hq, Hkv, N, d, 1, 0.088, ctypes.c_void_p(0))
    assert rc == -2                               # FA_ERR_UNSUPPORTED, nothing launched
    torch.cuda.synchronize()
    assert torch.all(dk == 3.0)
