"""Head-sharded problems through the CUDA kernels, on one GPU.

A problem split across GPUs by heads gives each rank a contiguous slice of the
flattened [B * H] head axis, cut at GQA group boundaries (`head_shard`): a
problem of its own with B = 1. Every (batch, kv-head) group is independent in
both passes, so running the kernels on each rank's slice and concatenating the
slices must reproduce the unsharded call: O, LSE, dK and dV bit for bit (each
of their elements is computed by one CTA whose arithmetic does not depend on
the launch it belongs to), dQ within the run-to-run spread of its fp32
atomics, and everything within the oracle bounds. The ranks run one after
another on the same device; no collective is involved.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.parity import BWD_REL_FRO, assert_fwd_ok, fwd_errors, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def _flat(t):
    """[B, H, N, d] (or [B, H, N]) -> [1, B*H, ...] view of the same memory."""
    return t.reshape((1, t.shape[0] * t.shape[1]) + tuple(t.shape[2:]))


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("world", [2, 3, 8])
def test_sharded_heads_equal_the_whole_problem(cuda_device, world, causal):
    import torch

    import exact_io_aware_44_b200 as fa
    w = synth.small(2, 16, 4, 1000, 128, causal, seed=4242 + world)
    arrs = [synth.tensor(w, t) for t in (synth.TID_Q, synth.TID_K, synth.TID_V, synth.TID_DO)]
    q, k, v, do = (to_dev(x, torch.bfloat16, cuda_device) for x in arrs)
    o, lse = fa.fwd(q, k, v, causal=causal)
    dq, dk, dv = fa.bwd(q, k, v, o, lse, do, causal=causal)
    assert fa.get_status() == 0

    fq, fk, fv, fdo = (_flat(t) for t in (q, k, v, do))
    parts = {n: [] for n in ("o", "lse", "dq", "dk", "dv")}
    for rank in range(world):
        q0, q1, k0, k1 = fa.head_shard(w.B, w.Hq, w.Hkv, rank, world)
        if k1 == k0:
            continue
        sq, sk, sv, sdo = (x[:, a:b].contiguous() for x, (a, b) in
                           ((fq, (q0, q1)), (fk, (k0, k1)), (fv, (k0, k1)), (fdo, (q0, q1))))
        so, slse = fa.fwd(sq, sk, sv, causal=causal)
        sdq, sdk, sdv = fa.bwd(sq, sk, sv, so, slse, sdo, causal=causal)
        assert fa.get_status() == 0
        for n, t in (("o", so), ("lse", slse), ("dq", sdq), ("dk", sdk), ("dv", sdv)):
            parts[n].append(t)
    cat = {n: torch.cat(ts, dim=1) for n, ts in parts.items()}

    assert torch.equal(cat["o"], _flat(o))
    assert torch.equal(cat["lse"], _flat(lse))
    assert torch.equal(cat["dk"], _flat(dk))
    assert torch.equal(cat["dv"], _flat(dv))
    dq_whole = _flat(dq).float().cpu().numpy()
    assert rel_fro(cat["dq"].float().cpu().numpy(), dq_whole) <= 1e-3

    o_ref, lse_ref = oracle.attention_fwd64(*arrs[:3], causal, w.scale)
    err = fwd_errors(cat["o"].float().cpu().numpy().reshape(o_ref.shape),
                     cat["lse"].cpu().numpy().reshape(lse_ref.shape), o_ref, lse_ref)
    assert_fwd_ok(err, f"world {world}")
    refs = oracle.attention_bwd64(*arrs, causal, w.scale)
    for n, r in zip(("dq", "dk", "dv"), refs):
        g = cat[n].float().cpu().numpy().reshape(r.shape)
        assert rel_fro(g, r) <= BWD_REL_FRO, (n, world)


def test_more_ranks_than_groups_leave_the_extra_ranks_empty(cuda_device):
    import exact_io_aware_44_b200 as fa
    shards = [fa.head_shard(1, 8, 2, r, 3) for r in range(3)]
    assert [s[3] - s[2] for s in shards] == [1, 1, 0]
    assert shards[-1][0] == shards[-1][1]
