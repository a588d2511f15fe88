"""Float64 CPU oracle for exact attention (test infrastructure only).

Only the tests, the package entry's smoke check and the benchmark's CPU-baseline
leg may import this package. The CUDA product path never does.

Parity status per function (what pins it; see tests/test_oracle.py):
  attention_fwd64         pinned: pure-Python brute force, SciPy softmax/logsumexp,
                          closed forms (Q = 0, constant V, causal rows 0 and 1),
                          shift and permutation invariance, online == one-pass.
  attention_bwd64         pinned: central finite differences (N <= 16, GQA too),
                          the identity D_i = sum_j P_ij dP_ij.
  online_softmax_trace64  pinned: equals the one-pass softmax on adversarial rows.
  head_fwd64 / group_bwd_sampled64
                          pinned: equal the full oracle restricted to the sampled rows.
  head_probs64            pinned: SciPy softmax of brute-force scores, zero above the
                          causal diagonal, P V reproduces the brute-force output.
  decode_fwd64            pinned: pure-Python brute force (decode_naive_loops), equals
                          attention_fwd64 when Nq = Nk, equals the last rows of the square
                          causal attention when the queries are the sequence's last rows,
                          and a single causal query sees every key.
  finite_diff_grads64     pinned: exact gradients of closed-form cases.
The pages print no worked numeric example, so no value is pinned to a printed number.
"""
from .attention64 import (  # noqa: F401
    ROW_BLOCK,
    attention_bwd64,
    attention_fwd64,
    attention_naive_loops,
    decode_fwd64,
    decode_naive_loops,
    finite_diff_grads64,
    group_bwd_sampled64,
    head_fwd64,
    head_probs64,
    online_softmax_trace64,
)
