"""The entry points inside a CUDA graph.

A serving or training loop captures its kernels once and replays them: every
entry point only enqueues work on the caller's stream (no host synchronisation,
no allocation), so fa_fwd, fa_bwd and fa_decode can be captured with
torch.cuda.graph after one eager call has loaded the kernels. Replays must give
what eager calls give on the same buffers: O, LSE, dK, dV and the decode outputs
bit for bit (each element is computed by one CTA, in an order that does not
depend on the launch), dQ within the spread of its fp32 atomics; the oracle
bounds hold for all of them. New inputs copied into the captured buffers between
replays must be picked up.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.parity import BWD_REL_FRO, assert_fwd_ok, fwd_errors, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [True, False])
def test_fwd_bwd_decode_captured_and_replayed(cuda_device, causal, d):
    import torch

    import exact_io_aware_44_b200 as fa
    w = synth.small(1, 8, 2, 700, d, causal, seed=9100 + causal + d)
    arrs = [synth.tensor(w, t) for t in (synth.TID_Q, synth.TID_K, synth.TID_V, synth.TID_DO)]
    q, k, v, do = (to_dev(x, torch.bfloat16, cuda_device) for x in arrs)
    dd = 64 if d == 64 else 128  # decode runs d = 64 and 128
    dw = synth.DecodeWorkload("graph_dec", 2, 16, 2, 4, 1500, dd, causal, 9200 + causal)  # 32 rows a group
    dq_np, dk_np, dv_np = synth.decode_inputs(dw)
    qd, kd, vd = (to_dev(x, torch.bfloat16, cuda_device) for x in (dq_np, dk_np, dv_np))

    # captured buffers
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=cuda_device)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    ws = torch.empty(fa.workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d), dtype=torch.uint8, device=cuda_device)
    od = torch.empty_like(qd)
    lsed = torch.empty(qd.shape[:3], dtype=torch.float32, device=cuda_device)
    wsd = torch.empty(fa.decode_workspace_bytes(dw.B, dw.Hq, dw.Hkv, dw.Nq, dw.Nk, dd), dtype=torch.uint8,
                      device=cuda_device)

    def step(stream=None):
        fa.fwd(q, k, v, causal=causal, out=o, lse=lse, stream=stream)
        fa.bwd(q, k, v, o, lse, do, causal=causal, workspace=ws, out=grads, stream=stream)
        fa.decode(qd, kd, vd, causal=causal, out=od, lse=lsed, workspace=wsd, stream=stream)

    step()  # eager: loads the kernels and sets their shared-memory limits
    assert fa.get_status() == 0
    eager = [t.clone() for t in (o, lse, *grads, od, lsed)]

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device=cuda_device)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step(stream=s)
    torch.cuda.current_stream().wait_stream(s)

    for t in (o, lse, *grads, od, lsed):
        t.fill_(float("nan"))
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    o_g, lse_g, dq_g, dk_g, dv_g, od_g, lsed_g = (t.clone() for t in (o, lse, *grads, od, lsed))
    for name, a, b in (("o", o_g, eager[0]), ("lse", lse_g, eager[1]), ("dk", dk_g, eager[3]),
                       ("dv", dv_g, eager[4]), ("decode o", od_g, eager[5]), ("decode lse", lsed_g, eager[6])):
        assert torch.equal(a, b), f"{name}: replay differs from the eager call"
    assert rel_fro(dq_g.float().cpu().numpy(), eager[2].float().cpu().numpy()) <= 1e-3

    # the replays against the oracle
    o_ref, lse_ref = oracle.attention_fwd64(arrs[0], arrs[1], arrs[2], causal, w.scale)
    assert_fwd_ok(fwd_errors(o_g.float().cpu().numpy(), lse_g.cpu().numpy(), o_ref, lse_ref), "graph fwd")
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd64(arrs[0], arrs[1], arrs[2], arrs[3], causal, w.scale)
    for name, a, ref in (("dq", dq_g, dq_ref), ("dk", dk_g, dk_ref), ("dv", dv_g, dv_ref)):
        assert rel_fro(a.float().cpu().numpy(), ref) <= BWD_REL_FRO, name
    od_ref, lsed_ref = oracle.decode_fwd64(dq_np, dk_np, dv_np, causal, dw.scale)
    assert_fwd_ok(fwd_errors(od_g.float().cpu().numpy(), lsed_g.cpu().numpy(), od_ref, lsed_ref), "graph decode")

    # new inputs in the captured buffers: the next replay computes on them
    q2 = synth.round_to_bf16((arrs[0] * np.float32(0.5)).astype(np.float32))
    q.copy_(to_dev(q2, torch.bfloat16, cuda_device))
    g.replay()
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    o2_ref, lse2_ref = oracle.attention_fwd64(q2, arrs[1], arrs[2], causal, w.scale)
    assert_fwd_ok(fwd_errors(o.float().cpu().numpy(), lse.cpu().numpy(), o2_ref, lse2_ref), "graph fwd, new q")
    del g
