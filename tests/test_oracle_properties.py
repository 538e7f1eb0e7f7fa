"""Property-based pins of the oracle (no GPU): generated inputs, independent references.

* top-k: the oracle's selection equals repeatedly taking the best remaining key (higher score, then smaller
  index; -0 and +0 equal), on rows drawn from a handful of values so that ties are the rule.
* sparse attention: the oracle's attention over an index row equals torch's softmax attention over the
  explicit set of distinct in-range keys of that row, whatever the duplicates, INVALID and out-of-range
  entries (metrale: the index row is a set; fak note: dot * scale, softmax, weighted sum of V).
"""
import numpy as np
import torch
from hypothesis import given, settings, strategies as st

from oracle import dsa_oracle as O

SCORES = st.sampled_from([-2.0, -1.0, -0.0, 0.0, 0.25, 1.0, 3.0])


def _brute(cand, scores, k):
    left = list(zip(cand, scores))
    out = []
    while left and len(out) < k:
        best = min(left, key=lambda cs: (-(cs[1] + 0.0), cs[0]))
        out.append(best[0])
        left.remove(best)
    return out + [O.INVALID] * (k - len(out))


@settings(max_examples=300, deadline=None)
@given(st.lists(SCORES, max_size=30), st.integers(1, 34), st.integers(0, 50))
def test_topk_row_is_repeated_argmax(scores, k, offset):
    cand = np.arange(offset, offset + len(scores), dtype=np.int64)
    got = O.topk_row(cand, np.array(scores, dtype=np.float64), k).tolist()
    assert got == _brute(cand.tolist(), scores, k)


@settings(max_examples=150, deadline=None)
@given(st.lists(st.integers(-3, 12), min_size=1, max_size=24), st.integers(0, 2 ** 16))
def test_attention_over_an_index_row_is_softmax_over_its_distinct_valid_keys(row, seed):
    n_kv, kd, vd, scale = 9, 5, 3, 0.7
    rng = np.random.default_rng(seed)
    q = rng.standard_normal(kd)
    K = rng.standard_normal((n_kv, kd))
    V = rng.standard_normal((n_kv, vd))
    o, l = O.sparse_attend_row(q[None, :], K[:, None, :], V[:, None, :], np.array(row), scale)
    keys = sorted({i for i in row if 0 <= i < n_kv})
    if not keys:
        assert np.all(o == 0) and np.all(np.isneginf(l))
        return
    logits = torch.tensor(K[keys] @ q * scale)
    ref = torch.softmax(logits, 0).numpy() @ V[keys]
    np.testing.assert_allclose(o[0], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l[0], torch.logsumexp(logits, 0).item(), rtol=1e-12, atol=1e-12)
