"""Pins for the float64 oracle, checked against what the pages and mathematics fix.

None of these re-types the oracle's own formulas: each compares it with an
independent route (pure-Python loops, SciPy, closed forms, invariants, finite
differences, a hand-derived trace). The last group plants plausible mistakes in
copies of the oracle and checks that some pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
from oracle import attention64 as A
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- pin helpers
# Each takes a forward (and backward) implementation so mutants can be fed in.

def pin_bruteforce(fwd, seed=0):
    for causal in (False, True):
        for (N, d) in ((1, 1), (3, 2), (5, 3), (6, 2)):
            q, k, v = rand((1, 1, N, d), seed), rand((1, 1, N, d), seed + 1), rand((1, 1, N, d), seed + 2)
            scale = 0.7
            o, lse = fwd(q, k, v, causal, scale)
            o_ref, lse_ref = A.attention_naive_loops(q[0, 0].tolist(), k[0, 0].tolist(),
                                                     v[0, 0].tolist(), causal, scale)
            np.testing.assert_allclose(o[0, 0], np.array(o_ref), rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse[0, 0], np.array(lse_ref), rtol=1e-12, atol=1e-12)


def pin_scipy(fwd, seed=3):
    B, H, N, d = 1, 2, 40, 8
    q, k, v = rand((B, H, N, d), seed), rand((B, H, N, d), seed + 1), rand((B, H, N, d), seed + 2)
    scale = 1 / math.sqrt(d)
    for causal in (False, True):
        o, lse = fwd(q, k, v, causal, scale)
        for h in range(H):
            s = scale * np.einsum("id,jd->ij", q[0, h], k[0, h])
            if causal:
                s = np.where(np.tri(N, dtype=bool), s, -np.inf)
            np.testing.assert_allclose(lse[0, h], scipy.special.logsumexp(s, axis=1), rtol=1e-12)
            p = scipy.special.softmax(s, axis=1)
            np.testing.assert_allclose(o[0, h], p @ v[0, h], rtol=1e-10, atol=1e-12)


def pin_closed_forms(fwd, seed=5):
    N, d = 17, 4
    k, v = rand((1, 1, N, d), seed), rand((1, 1, N, d), seed + 1)
    scale = 0.5
    # Q = 0: every score is 0, so attention is a plain mean over the visible keys.
    q0 = np.zeros((1, 1, N, d))
    o, lse = fwd(q0, k, v, True, scale)
    cmean = np.cumsum(v[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(o[0, 0], cmean, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, N + 1)), rtol=1e-12, atol=1e-14)
    o, lse = fwd(q0, k, v, False, scale)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (N, d)), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.full(N, math.log(N)), rtol=1e-12)
    # constant V returns V
    q = rand((1, 1, N, d), seed + 2, 3.0)
    vc = np.broadcast_to(np.array([1.5, -2.0, 0.25, 7.0]), (1, 1, N, d)).copy()
    for causal in (False, True):
        o, _ = fwd(q, k, vc, causal, scale)
        np.testing.assert_allclose(o, vc, rtol=1e-12)
    # causal rows 0 and 1: one- and two-term softmax
    o, lse = fwd(q, k, v, True, scale)
    s00 = scale * q[0, 0, 0] @ k[0, 0, 0]
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], rtol=1e-12)
    np.testing.assert_allclose(lse[0, 0, 0], s00, rtol=1e-12, atol=1e-14)
    s10, s11 = scale * q[0, 0, 1] @ k[0, 0, 0], scale * q[0, 0, 1] @ k[0, 0, 1]
    w1 = 1.0 / (1.0 + math.exp(s10 - s11))
    np.testing.assert_allclose(o[0, 0, 1], (1 - w1) * v[0, 0, 0] + w1 * v[0, 0, 1], rtol=1e-12)
    np.testing.assert_allclose(lse[0, 0, 1], np.logaddexp(s10, s11), rtol=1e-12)


def pin_invariances(fwd, seed=7):
    N, d = 23, 5
    q, k, v = rand((1, 1, N, d), seed), rand((1, 1, N, d), seed + 1), rand((1, 1, N, d), seed + 2)
    scale = 0.4
    u = rand((d,), seed + 3)
    for causal in (False, True):
        o, lse = fwd(q, k, v, causal, scale)
        # adding u to every key shifts row i by scale q_i.u: P unchanged, LSE shifted
        o2, lse2 = fwd(q, k + u, v, causal, scale)
        np.testing.assert_allclose(o2, o, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse2[0, 0], lse[0, 0] + scale * q[0, 0] @ u, rtol=1e-10, atol=1e-12)
    perm = np.random.default_rng(seed).permutation(N)
    o, lse = fwd(q, k, v, False, scale)
    o3, lse3 = fwd(q, k[:, :, perm], v[:, :, perm], False, scale)
    np.testing.assert_allclose(o3, o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse3, lse, rtol=1e-12)


def pin_gqa(fwd, seed=11):
    """Query head h reads kv head h // g: compare with each head run on its own."""
    B, Hq, Hkv, N, d = 2, 4, 2, 9, 3
    q, k, v = rand((B, Hq, N, d), seed), rand((B, Hkv, N, d), seed + 1), rand((B, Hkv, N, d), seed + 2)
    o, lse = fwd(q, k, v, True, 0.6)
    for b in range(B):
        for h in range(Hq):
            ref, rl = A.attention_naive_loops(q[b, h].tolist(), k[b, h // 2].tolist(),
                                              v[b, h // 2].tolist(), True, 0.6)
            np.testing.assert_allclose(o[b, h], np.array(ref), rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse[b, h], np.array(rl), rtol=1e-12, atol=1e-13)


def pin_finite_diff(fwd, bwd, seed=13):
    cases = [(1, 1, 1, 6, 4, False), (1, 1, 1, 7, 4, True), (1, 2, 1, 5, 8, True), (2, 2, 2, 4, 4, False)]
    for i, (B, Hq, Hkv, N, d, causal) in enumerate(cases):
        q = rand((B, Hq, N, d), seed + 4 * i)
        k = rand((B, Hkv, N, d), seed + 4 * i + 1)
        v = rand((B, Hkv, N, d), seed + 4 * i + 2)
        do = rand((B, Hq, N, d), seed + 4 * i + 3)
        scale = 1 / math.sqrt(d)
        dq, dk, dv = bwd(q, k, v, do, causal, scale)
        # finite differences taken through the forward under test
        saved = A.attention_fwd64
        A.attention_fwd64 = fwd
        try:
            fq, fk, fv = A.finite_diff_grads64(q, k, v, do, causal, scale)
        finally:
            A.attention_fwd64 = saved
        for g_an, g_fd in ((dq, fq), (dk, fk), (dv, fv)):
            err = np.linalg.norm(g_an - g_fd) / max(np.linalg.norm(g_fd), 1e-30)
            assert err <= 1e-6, err


# ---------------------------------------------------------------- the pins

def test_bruteforce_loops():
    pin_bruteforce(A.attention_fwd64)


def test_scipy_softmax_logsumexp():
    pin_scipy(A.attention_fwd64)


def test_closed_forms():
    pin_closed_forms(A.attention_fwd64)


def test_invariances():
    pin_invariances(A.attention_fwd64)


def test_gqa_head_map():
    pin_gqa(A.attention_fwd64)


def test_finite_difference_gradients():
    pin_finite_diff(A.attention_fwd64, A.attention_bwd64)


def test_probabilities_are_distributions():
    N, d = 33, 6
    q, k = rand((N, d), 21, 2.0), rand((N, d), 22)
    v = rand((N, d), 23)
    for causal in (False, True):
        _, lse = A.head_fwd64(q, k, v, causal, 0.3)
        p = A._probs(q, k, lse, 0.3, 0, causal)
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-12)
        if causal:
            assert np.all(p[np.triu_indices(N, 1)] == 0.0)


def test_delta_identity():
    """D_i = sum_c dO_ic O_ic equals sum_j P_ij dP_ij (what makes dS = P o (dP - D) exact)."""
    N, d = 19, 4
    q, k, v, do = (rand((N, d), s) for s in (31, 32, 33, 34))
    o, lse = A.head_fwd64(q, k, v, True, 0.5)
    p = A._probs(q, k, lse, 0.5, 0, True)
    dp = do @ v.T
    np.testing.assert_allclose((do * o).sum(1), (p * dp).sum(1), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 3, 32, 64])
def test_online_equals_one_pass(chunk):
    rng = np.random.default_rng(41)
    N, d = 64, 5
    v = rng.standard_normal((N, d))
    rows = [rng.standard_normal(N) * 4,
            np.sort(rng.standard_normal(N)) * 10,           # increasing: rescale every chunk
            -np.sort(rng.standard_normal(N)) * 10,          # decreasing: no rescale after the first
            np.where(np.arange(N) == 40, 1000.0, rng.standard_normal(N))]  # one huge spike
    for s in rows:
        o_on, lse_on, trace = A.online_softmax_trace64(s, v, chunk)
        assert len(trace) == -(-N // chunk)
        m = s.max()
        p = np.exp(s - m)
        ref_o = (p @ v) / p.sum()
        ref_lse = m + math.log(p.sum())
        np.testing.assert_allclose(o_on, ref_o, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse_on, ref_lse, rtol=1e-12)
        # the running max is non-decreasing
        ms = [t[0] for t in trace]
        assert all(b >= a for a, b in zip(ms, ms[1:]))


def test_four_block_trace_golden():
    g = json.load(open(os.path.join(GOLDEN, "four_block_trace.json")))
    s = np.array([0.0, math.log(2), math.log(4), 0.0])
    v = np.array(g["values"])[:, None]
    o, lse, trace = A.online_softmax_trace64(s, v, 1)
    np.testing.assert_allclose([t[1] for t in trace], g["trace_l"], rtol=1e-15)
    np.testing.assert_allclose([t[2][0] for t in trace], g["trace_O"], rtol=1e-15)
    np.testing.assert_allclose([t[0] for t in trace], [0, math.log(2), math.log(4), math.log(4)], rtol=1e-15)
    assert abs(o[0] - g["final_O"]) < 1e-15
    assert abs(lse - math.log(8)) < 1e-15


def test_c1_four_chunk_trace_matches_one_pass():
    """The fp32 workload's rows {0, 1, 63, 127}, streamed in 4 chunks of 32 keys."""
    w = synth.WORKLOADS["c1"]
    q, k, v = (synth.head_slice(w, t, 0, 0).astype(np.float64) for t in (0, 1, 2))
    o, lse = A.head_fwd64(q, k, v, False, w.scale)
    for i in (0, 1, 63, 127):
        s = w.scale * (k @ q[i])
        o_on, lse_on, trace = A.online_softmax_trace64(s, v, 32)
        assert len(trace) == 4
        np.testing.assert_allclose(o_on, o[i], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse_on, lse[i], rtol=1e-12)


def test_sampled_rows_equal_full(monkeypatch):
    monkeypatch.setattr(A, "ROW_BLOCK", 16)  # exercise the row blocking
    N, d, g = 70, 4, 2
    qg = rand((g, N, d), 51)
    kh, vh = rand((N, d), 52), rand((N, d), 53)
    dog = rand((g, N, d), 54)
    rows = np.array([0, 1, 15, 16, 17, 40, 69])
    for causal in (False, True):
        o, lse = A.attention_fwd64(qg[None], kh[None, None], vh[None, None], causal, 0.5)
        o_s, lse_s = A.head_fwd64(qg[1], kh, vh, causal, 0.5, rows=rows)
        np.testing.assert_allclose(o_s, o[0, 1, rows], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse_s, lse[0, 1, rows], rtol=1e-12)
        dq, dk, dv = A.attention_bwd64(qg[None], kh[None, None], vh[None, None], dog[None], causal, 0.5)
        sq, sk, sv = A.group_bwd_sampled64(qg, kh, vh, dog, causal, 0.5, rows, rows)
        np.testing.assert_allclose(sq, dq[0][:, rows], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sk, dk[0, 0, rows], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sv, dv[0, 0, rows], rtol=1e-10, atol=1e-12)


def test_row_blocking_is_invisible(monkeypatch):
    q, k, v, do = (rand((1, 1, 50, 3), s) for s in (61, 62, 63, 64))
    ref = A.attention_fwd64(q, k, v, True, 0.5) + A.attention_bwd64(q, k, v, do, True, 0.5)
    monkeypatch.setattr(A, "ROW_BLOCK", 7)
    got = A.attention_fwd64(q, k, v, True, 0.5) + A.attention_bwd64(q, k, v, do, True, 0.5)
    for a, b in zip(ref, got):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_finite_difference_on_a_closed_form():
    """The FD helper itself: L = sum(O dO) with Q = 0 is linear in V with gradient mean weights."""
    N, d = 5, 2
    q = np.zeros((1, 1, N, d))
    k, v, do = rand((1, 1, N, d), 71), rand((1, 1, N, d), 72), rand((1, 1, N, d), 73)
    _, _, fv = A.finite_diff_grads64(q, k, v, do, True, 1.0)
    # O_i = mean_{j<=i} V_j  =>  dL/dV_j = sum_{i>=j} dO_i / (i + 1)
    exp = np.array([sum(do[0, 0, i] / (i + 1) for i in range(j, N)) for j in range(N)])
    np.testing.assert_allclose(fv[0, 0], exp, rtol=1e-8, atol=1e-9)


def test_synth_bf16_rounding_matches_torch():
    import torch
    x = np.random.default_rng(5).standard_normal(10000).astype(np.float32) * 50
    x[:4] = [1.00390625, 1.01171875, -3.0078125, 65504.0]  # exact ties and a large value
    ours = synth.round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours, ref)


def test_head_probs_are_the_softmax_of_brute_force_scores():
    N, d, scale = 37, 8, 0.4
    q, k, v = rand((N, d), 41), rand((N, d), 42), rand((N, d), 43)
    for causal in (False, True):
        rows = np.array([0, 1, 5, 36]) if causal else None
        p = oracle.head_probs64(q, k, causal, scale, rows=rows)
        sel = np.arange(N) if rows is None else rows
        s = scale * np.einsum("id,jd->ij", q[sel], k)
        if causal:
            s = np.where(np.arange(N)[None, :] <= sel[:, None], s, -np.inf)
            assert np.all(p[np.arange(N)[None, :] > sel[:, None]] == 0.0)
        np.testing.assert_allclose(p, scipy.special.softmax(s, axis=1), rtol=1e-12, atol=1e-15)
        o_ref, _ = A.attention_naive_loops([q[i].tolist() for i in range(N)], k.tolist(), v.tolist(), causal, scale)
        np.testing.assert_allclose(p @ v, np.array(o_ref)[sel], rtol=1e-10, atol=1e-12)


def pin_decode(dec):
    """Pins for a decode implementation dec(q, k, v, causal, scale) -> (O, LSE)."""
    scale = 0.35
    # brute force on tiny shapes, GQA, causal and not
    for causal in (True, False):
        for (Nq, Nk) in ((1, 1), (1, 5), (3, 7), (4, 4)):
            q, k, v = rand((1, 4, Nq, 3), 51), rand((1, 2, Nk, 3), 52), rand((1, 2, Nk, 3), 53)
            o, lse = dec(q, k, v, causal, scale)
            for h in range(4):
                ob, lb = oracle.decode_naive_loops(q[0, h].tolist(), k[0, h // 2].tolist(), v[0, h // 2].tolist(),
                                                    causal, scale)
                np.testing.assert_allclose(o[0, h], np.array(ob), rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(lse[0, h], np.array(lb), rtol=1e-12, atol=1e-12)
    # a whole 32-row group (8 query heads on one kv head x 4 new tokens; 16 x 2), as one CTA serves it
    for causal in (True, False):
        for (g, Nq, Nk) in ((8, 4, 6), (16, 2, 9)):
            q, k, v = rand((1, g, Nq, 3), 57), rand((1, 1, Nk, 3), 58), rand((1, 1, Nk, 3), 59)
            o, lse = dec(q, k, v, causal, scale)
            for h in range(g):
                ob, lb = oracle.decode_naive_loops(q[0, h].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), causal, scale)
                np.testing.assert_allclose(o[0, h], np.array(ob), rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(lse[0, h], np.array(lb), rtol=1e-12, atol=1e-12)
    # Nq = Nk is the square attention; the last Nq rows of a causal sequence are a causal decode
    N, d = 37, 8
    q, k, v = rand((2, 2, N, d), 54), rand((2, 1, N, d), 55), rand((2, 1, N, d), 56)
    for causal in (True, False):
        o, lse = dec(q, k, v, causal, scale)
        o2, lse2 = A.attention_fwd64(q, k, v, causal, scale)
        np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, lse2, rtol=1e-12)
    o, lse = dec(q[:, :, -5:], k, v, True, scale)
    o2, lse2 = A.attention_fwd64(q, k, v, True, scale)
    np.testing.assert_allclose(o, o2[:, :, -5:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse2[:, :, -5:], rtol=1e-12)
    # a single causal query is the last position: it sees every key
    oc, lc = dec(q[:, :, :1], k, v, True, scale)
    on, ln = dec(q[:, :, :1], k, v, False, scale)
    np.testing.assert_allclose(oc, on, rtol=1e-12)
    np.testing.assert_allclose(lc, ln, rtol=1e-12)


def test_decode_oracle_pins():
    pin_decode(oracle.decode_fwd64)


def _mut_decode_top_left(q, k, v, causal, scale=None):
    """Queries aligned to the start of the cache (query i sees keys j <= i)."""
    q, k, v = (np.asarray(x, float) for x in (q, k, v))
    B, Hq, Nq, d = q.shape
    Nk = k.shape[2]
    g = Hq // k.shape[1]
    o = np.empty_like(q)
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, h] @ k[b, h // g].T
            if causal:
                s = np.where(np.arange(Nk)[None, :] <= np.arange(Nq)[:, None], s, -np.inf)
            m = s.max(1, keepdims=True)
            l = np.exp(s - m).sum(1, keepdims=True)
            o[b, h] = (np.exp(s - m) / l) @ v[b, h // g]
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


def _mut_decode_gqa_modulo(q, k, v, causal, scale=None):
    Hq, Hkv = np.asarray(q).shape[1], np.asarray(k).shape[1]
    idx = [h % Hkv for h in range(Hq)]
    return oracle.decode_fwd64(q, np.asarray(k)[:, idx], np.asarray(v)[:, idx], causal, scale)


def _mut_decode_lse_log2(q, k, v, causal, scale=None):
    o, lse = oracle.decode_fwd64(q, k, v, causal, scale)
    return o, lse / math.log(2)


@pytest.mark.parametrize("mutant", [_mut_decode_top_left, _mut_decode_gqa_modulo, _mut_decode_lse_log2])
def test_planted_decode_mistakes_are_caught(mutant):
    assert _fails(pin_decode, mutant), mutant.__name__


def test_synth_e4m3_rounding_matches_torch():
    import torch
    x = np.random.default_rng(6).standard_normal(20000).astype(np.float32)
    x *= np.repeat(np.float32([1e-3, 0.05, 1.0, 40.0]), 5000)
    x[:6] = [2.0 ** -10, 3 * 2.0 ** -11, 1.0625, 1.1875, 448.0, -440.0]  # ties (to even) and the top
    ours = synth.round_to_e4m3(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(ours, ref)
    assert synth.round_to_e4m3(np.float32([1000.0, -1e6]))[0] == 448.0   # saturates
    assert synth.round_to_e4m3(np.float32([-1e6]))[0] == -448.0


def test_synth_e5m2_rounding_matches_torch():
    import torch
    x = np.random.default_rng(7).standard_normal(20000).astype(np.float32)
    x *= np.repeat(np.float32([1e-5, 0.05, 1.0, 5000.0]), 5000)
    x[:6] = [2.0 ** -17, 3 * 2.0 ** -18, 1.125, 1.375, 57344.0, -50000.0]  # ties (to even) and the top
    ours = synth.round_to_e5m2(x)
    ref = torch.from_numpy(x).to(torch.float8_e5m2).to(torch.float32).numpy()
    assert np.array_equal(ours, ref)
    assert synth.round_to_e5m2(np.float32([1e6]))[0] == 57344.0   # saturates


def test_synth_e4m3_workload_codes():
    w = synth.WORKLOADS["f3"]
    x = synth.head_slice(w, synth.TID_K, 1, 5, n=2048)
    assert np.array_equal(x, synth.round_to_e4m3(x))          # stored values are E4M3 codes
    deq = x.astype(np.float64) * w.descale
    assert abs(deq.std() - w.std) < 0.02 and np.abs(x).max() <= 448.0


def test_synth_spiked_rows():
    w = synth.WORKLOADS["c2"]
    q = synth.head_slice(w, synth.TID_Q, 1, 3)
    rows = synth.spiked_rows(w, 1, 3)
    assert rows.size == 20
    norms = np.linalg.norm(q, axis=1)
    assert norms[rows].min() > 3 * np.median(norms)


# ------------------------------------------------------ planted mistakes caught

def _mut_scale(q, k, v, causal, scale=None):
    return A.attention_fwd64(q, k, v, causal, (scale or 1.0) * 1.0001 if scale else None)


def _mut_mask_off_by_one(q, k, v, causal, scale=None):
    """Causal mask that lets each query see one key too many (j <= i + 1)."""
    if not causal:
        return A.attention_fwd64(q, k, v, causal, scale)
    q, k, v = (np.asarray(x, float) for x in (q, k, v))
    B, Hq, N, d = q.shape
    g = Hq // k.shape[1]
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N))
    vis = np.tri(N, k=1, dtype=bool)
    for b in range(B):
        for h in range(Hq):
            s = np.where(vis, scale * q[b, h] @ k[b, h // g].T, -np.inf)
            m = s.max(1, keepdims=True)
            l = np.exp(s - m).sum(1, keepdims=True)
            o[b, h] = (np.exp(s - m) / l) @ v[b, h // g]
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


def _mut_swap_kv(q, k, v, causal, scale=None):
    return A.attention_fwd64(q, v, k, causal, scale)


def _mut_log2(q, k, v, causal, scale=None):
    o, lse = A.attention_fwd64(q, k, v, causal, scale)
    return o, lse / math.log(2)


def _mut_gqa_modulo(q, k, v, causal, scale=None):
    q = np.asarray(q, float)
    B, Hq = q.shape[:2]
    Hkv = k.shape[1]
    idx = [h % Hkv for h in range(Hq)]
    return A.attention_fwd64(q, np.asarray(k)[:, idx], np.asarray(v)[:, idx], causal, scale)


def _mut_bwd_no_delta(q, k, v, do, causal, scale=None):
    o, lse = A.attention_fwd64(q, k, v, causal, scale)
    return A.attention_bwd64(q, k, v, do, causal, scale, o=np.zeros_like(o), lse=lse)


def _mut_bwd_dk_unscaled(q, k, v, do, causal, scale=None):
    dq, dk, dv = A.attention_bwd64(q, k, v, do, causal, scale)
    return dq, dk / scale, dv


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("mutant", [_mut_scale, _mut_mask_off_by_one, _mut_swap_kv, _mut_log2, _mut_gqa_modulo])
def test_planted_forward_mistakes_are_caught(mutant):
    pins = [pin_bruteforce, pin_scipy, pin_closed_forms, pin_invariances, pin_gqa]
    assert any(_fails(p, mutant) for p in pins), mutant.__name__


@pytest.mark.parametrize("mutant", [_mut_bwd_no_delta, _mut_bwd_dk_unscaled])
def test_planted_backward_mistakes_are_caught(mutant):
    assert _fails(pin_finite_diff, A.attention_fwd64, mutant), mutant.__name__
