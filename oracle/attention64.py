"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE. Only the test suite, the package entry's smoke check and the
CPU-baseline leg of the benchmark may import this module. The CUDA product path
never calls it, and it shares no code with that path.

What it follows (page titles and passages):
  * "Walk through what FlashAttention does differently from standard attention"
    (zenaique short answer), first paragraph: Attn(Q,K,V) = softmax(QK^T/sqrt(d_k)) V.
    FlashAttention computes the same output; only floating-point rounding differs.
  * "FlashAttention Kernel & Online Softmax" (airsota card), first paragraph: the
    running-max update m_new = max(m, x), l_new = l*e^(m-m_new) + e^(x-m_new), the
    output rescaled by e^(m-m_new) and normalised by 1/l at the end.
  * "FlashAttention" (akshathtiwari blog): the running max m, normaliser ell and
    output accumulator O, each rescaled by exp(m - m_new) when a block arrives;
    the four-block streaming-softmax widget; the backward pass recomputes blocks.
  * Same short answer, second paragraph: the backward pass recomputes attention from
    the saved Q, K, V and softmax statistics (m, l) instead of storing the scores.

Readings (the pages leave these open):
  * The saved statistics are LSE = m + ln(l) (natural log), which is m and l folded.
  * scale defaults to 1/sqrt(d).
  * Causal: square N x N, key j is visible to query i iff j <= i.
  * Grouped-query attention: query head h reads key/value head h // (Hq/Hkv).
  * Backward of L = sum(O * dO): D_i = sum_c dO_ic O_ic, dS = P o (dP - D),
    dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO (summed over a GQA group).

The forward is the one-pass definition on full rows (max, log-sum-exp, P, P V),
processed ROW_BLOCK query rows at a time only to bound memory. It is not the
online softmax: `online_softmax_trace64` implements that separately, and the
tests pin the two against each other.
"""
from __future__ import annotations

import numpy as np

ROW_BLOCK = 1024


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _scores(q_rows, k, scale, row0, causal):
    """scale * q_rows k^T with the causal mask; keys past the last row are all masked."""
    n_rows = q_rows.shape[0]
    n_keys = k.shape[0]
    kcols = min(n_keys, row0 + n_rows) if causal else n_keys
    s = np.full((n_rows, n_keys), -np.inf)
    s[:, :kcols] = scale * (q_rows @ k[:kcols].T)
    if causal:
        i = np.arange(row0, row0 + n_rows)[:, None]
        j = np.arange(kcols)[None, :]
        s[:, :kcols][j > i] = -np.inf
    return s


def _softmax_rows(s):
    """One-pass softmax of each full row; returns P and the natural-log LSE."""
    m = s.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(s - m).sum(axis=1, keepdims=True))
    p = np.exp(s - lse)
    return p, lse[:, 0]


def head_fwd64(qh, kh, vh, causal, scale, rows=None):
    """Forward for one head. qh [N, d], kh/vh [N, d] -> (O [R, d], LSE [R]).

    With `rows` given, only those query rows are evaluated (each still over its
    full key row), which is how the large workloads are sampled.
    """
    qh, kh, vh = _f64(qh), _f64(kh), _f64(vh)
    if rows is None:
        rows = np.arange(qh.shape[0])
    rows = np.asarray(rows, dtype=np.int64)
    o = np.empty((rows.size, vh.shape[1]))
    lse = np.empty(rows.size)
    for r0 in range(0, rows.size, ROW_BLOCK):
        sel = rows[r0:r0 + ROW_BLOCK]
        if sel.size and np.all(np.diff(sel) == 1):
            s = _scores(qh[sel], kh, scale, int(sel[0]), causal)
        else:
            s = np.vstack([_scores(qh[i:i + 1], kh, scale, int(i), causal) for i in sel])
        p, l = _softmax_rows(s)
        o[r0:r0 + sel.size] = p @ vh
        lse[r0:r0 + sel.size] = l
    return o, lse


def head_probs64(qh, kh, causal, scale, rows=None):
    """The attention probabilities P = softmax(scale q k^T) of one head, for the
    given query rows ([R, N]; masked keys are 0). Used to model the rounding of
    low-precision kernels, whose error depends on the individual P_ij."""
    qh, kh = _f64(qh), _f64(kh)
    if rows is None:
        rows = np.arange(qh.shape[0])
    rows = np.asarray(rows, dtype=np.int64)
    s = np.vstack([_scores(qh[i:i + 1], kh, scale, int(i), causal) for i in rows]) if rows.size else \
        np.zeros((0, kh.shape[0]))
    return _softmax_rows(s)[0]


def attention_fwd64(q, k, v, causal, scale=None):
    """Exact attention. q [B, Hq, N, d]; k, v [B, Hkv, N, d] -> O [B, Hq, N, d], LSE [B, Hq, N]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            o[b, h], lse[b, h] = head_fwd64(q[b, h], k[b, h // g], v[b, h // g], causal, scale)
    return o, lse


def decode_fwd64(q, k, v, causal, scale=None):
    """Attention of Nq new queries against a cache of Nk >= Nq keys (decode).

    q [B, Hq, Nq, d]; k, v [B, Hkv, Nk, d] -> O [B, Hq, Nq, d], LSE [B, Hq, Nq].
    The queries are the last Nq positions of the sequence: query i sits at
    position Nk - Nq + i and, when causal, sees keys j <= Nk - Nq + i (with
    Nq = Nk this is the square causal mask of attention_fwd64). One-pass softmax
    over each full key row, as in head_fwd64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if causal and Nq > Nk:
        raise ValueError("causal decode needs Nq <= Nk")
    g = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            s = scale * (q[b, h] @ k[b, h // g].T)          # [Nq, Nk]
            if causal:
                pos = Nk - Nq + np.arange(Nq)[:, None]
                s = np.where(np.arange(Nk)[None, :] <= pos, s, -np.inf)
            p, lse[b, h] = _softmax_rows(s)
            o[b, h] = p @ v[b, h // g]
    return o, lse


def decode_naive_loops(q, k, v, causal, scale):
    """Pure-Python brute force of decode_fwd64 for one head (lists of rows)."""
    import math
    nq, nk = len(q), len(k)
    out, lses = [], []
    for i in range(nq):
        keys = range(nk - nq + i + 1) if causal else range(nk)
        s = [scale * sum(a * b for a, b in zip(q[i], k[j])) for j in keys]
        mx = max(s)
        z = sum(math.exp(x - mx) for x in s)
        out.append([sum(math.exp(s[t] - mx) / z * v[j][c] for t, j in enumerate(keys)) for c in range(len(v[0]))])
        lses.append(mx + math.log(z))
    return out, lses


def _probs(q_rows, kh, lse_rows, scale, row0, causal):
    """P recomputed from Q, K and the saved LSE (the backward's recomputation)."""
    s = _scores(q_rows, kh, scale, row0, causal)
    return np.exp(s - lse_rows[:, None])


def attention_bwd64(q, k, v, do, causal, scale=None, o=None, lse=None):
    """Gradients of L = sum(O * dO) -> (dQ, dK, dV), all float64.

    O and LSE are computed by `attention_fwd64` unless given.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    if o is None or lse is None:
        o, lse = attention_fwd64(q, k, v, causal, scale)
    o, lse = _f64(o), _f64(lse)
    D = (do * o).sum(axis=-1)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kh, vh = k[b, h // g], v[b, h // g]
            for r0 in range(0, N, ROW_BLOCK):
                r1 = min(N, r0 + ROW_BLOCK)
                p = _probs(q[b, h, r0:r1], kh, lse[b, h, r0:r1], scale, r0, causal)
                dv[b, h // g] += p.T @ do[b, h, r0:r1]
                dp = do[b, h, r0:r1] @ vh.T
                ds = p * (dp - D[b, h, r0:r1, None])
                dq[b, h, r0:r1] = scale * (ds @ kh)
                dk[b, h // g] += scale * (ds.T @ q[b, h, r0:r1])
    return dq, dk, dv


def online_softmax_trace64(s_row, v, chunk):
    """Online softmax over one score row, streamed in key chunks of size `chunk`.

    Follows the running-max update of "FlashAttention Kernel & Online Softmax" and
    the m / ell / O rescaling of the "FlashAttention" blog: for each new chunk,
    m' = max(m, max chunk), alpha = e^(m - m'), ell' = alpha ell + sum e^(s - m'),
    O' = alpha O + sum e^(s - m') v. The short snippet on the zenaique MCQ page never
    adds the values into its numerator; this follows the blog's full update.

    Returns (O / ell, m + ln ell, trace) with trace = [(m, ell, O copy) per chunk].
    """
    s_row = _f64(s_row)
    v = _f64(v)
    m = -np.inf
    ell = 0.0
    acc = np.zeros(v.shape[1])
    trace = []
    for c0 in range(0, s_row.size, chunk):
        s = s_row[c0:c0 + chunk]
        m_new = max(m, float(s.max()))
        if m_new == -np.inf:  # nothing visible yet: nothing to rescale
            trace.append((m, ell, acc.copy()))
            continue
        alpha = np.exp(m - m_new)
        e = np.exp(s - m_new)
        ell = alpha * ell + e.sum()
        acc = alpha * acc + e @ v[c0:c0 + chunk]
        m = m_new
        trace.append((m, ell, acc.copy()))
    return acc / ell, m + np.log(ell), trace


# ---------------------------------------------------------------------------
# Sampled evaluation for the long sequences: the same definitions restricted to
# a subset of query rows (for O, LSE, dQ) or key rows (for dK, dV).
# ---------------------------------------------------------------------------

def group_bwd_sampled64(qg, kh, vh, dog, causal, scale, q_rows, k_rows):
    """Backward for one GQA group on sampled rows.

    qg, dog: [g, N, d] (the q-heads sharing kv head kh/vh), kh, vh: [N, d].
    Returns dQ [g, |q_rows|, d] and dK, dV [|k_rows|, d], each the exact float64
    value of the full gradient at those rows. Every query row's O and LSE are
    computed in full, since dK_j and dV_j depend on all of them.
    """
    qg, kh, vh, dog = _f64(qg), _f64(kh), _f64(vh), _f64(dog)
    g, N, d = qg.shape
    q_rows = np.asarray(q_rows, dtype=np.int64)
    k_rows = np.asarray(k_rows, dtype=np.int64)
    dq = np.empty((g, q_rows.size, d))
    dk = np.zeros((k_rows.size, d))
    dv = np.zeros((k_rows.size, d))
    kj, vj = kh[k_rows], vh[k_rows]
    for h in range(g):
        o, lse = head_fwd64(qg[h], kh, vh, causal, scale)
        D = (dog[h] * o).sum(axis=1)
        # dQ rows: full key rows of P, dP
        for r0 in range(0, q_rows.size, ROW_BLOCK):
            sel = q_rows[r0:r0 + ROW_BLOCK]
            s = np.vstack([_scores(qg[h, i:i + 1], kh, scale, int(i), causal) for i in sel])
            p = np.exp(s - lse[sel, None])
            dp = dog[h, sel] @ vh.T
            ds = p * (dp - D[sel, None])
            dq[h, r0:r0 + sel.size] = scale * (ds @ kh)
        # dK, dV rows: columns j of P over every query row
        for r0 in range(0, N, ROW_BLOCK):
            r1 = min(N, r0 + ROW_BLOCK)
            s = scale * (qg[h, r0:r1] @ kj.T)
            if causal:
                i = np.arange(r0, r1)[:, None]
                s = np.where(k_rows[None, :] > i, -np.inf, s)
            p = np.exp(s - lse[r0:r1, None])
            dv += p.T @ dog[h, r0:r1]
            dp = dog[h, r0:r1] @ vj.T
            ds = p * (dp - D[r0:r1, None])
            dk += scale * (ds.T @ qg[h, r0:r1])
    return dq, dk, dv


def finite_diff_grads64(q, k, v, do, causal, scale=None, h=1e-6):
    """Central differences of L = sum(attention(q,k,v) * do) w.r.t. every input element.

    Tiny shapes only (N <= 16): one pair of forward evaluations per element.
    """
    q, k, v, do = _f64(q).copy(), _f64(k).copy(), _f64(v).copy(), _f64(do)

    def loss():
        o, _ = attention_fwd64(q, k, v, causal, scale)
        return float((o * do).sum())

    grads = []
    for x in (q, k, v):
        gx = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = x[idx]
            x[idx] = x0 + h
            lp = loss()
            x[idx] = x0 - h
            lm = loss()
            x[idx] = x0
            gx[idx] = (lp - lm) / (2 * h)
        grads.append(gx)
    return tuple(grads)


def attention_naive_loops(q, k, v, causal, scale):
    """Pure-Python brute force for one head (q, k, v: lists of rows). Tiny inputs only.

    Written with plain loops and math.exp, independent of NumPy, as a pin for
    the vectorised oracle.
    """
    import math
    n = len(q)
    d = len(q[0])
    out, lses = [], []
    for i in range(n):
        keys = range(i + 1) if causal else range(len(k))
        s = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in keys]
        mx = max(s)
        z = sum(math.exp(x - mx) for x in s)
        out.append([sum(math.exp(s[t] - mx) / z * v[j][c] for t, j in enumerate(keys))
                    for c in range(len(v[0]))])
        lses.append(mx + math.log(z))
    return out, lses
