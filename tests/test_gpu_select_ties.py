"""Selection on rows whose cut falls inside more than 2048 near-equal scores.

The selection kernel sorts the crossing bin of a value histogram exactly only
when it holds at most 2048 members; larger bins are binned again.  These rows
are built so that value bins cannot separate them (thousands of distinct
scores spread over many binades close to zero, the cut among the smallest),
or so that thousands of scores are exactly equal.  Method §3 ranks key blocks
by P_ij = softmax of the scores, which orders them exactly like the scores,
with ties broken by index (R13); k decides the cut here (p is tiny), so the
expected set is the first k of that ranking, written out directly.  The
oracle's own selection is compared too (its float64 probabilities merge
scores closer than about 1e-16, which the near-tie rule accepts).
"""

import numpy as np
import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
from oracle import prism_oracle as po
from tests.helpers import selection_row_ok

pytestmark = pytest.mark.gpu


def _geometric_scores(rng, per_binade=40):
    """Distinct float32 scores: per_binade values in each binade 2^-1 .. 2^-126,
    plus two negative ones, shuffled."""
    e = np.repeat(np.arange(1, 127), per_binade)
    m = rng.integers(0, 1 << 22, len(e))
    g = np.ldexp(1.0 + m / 2.0 ** 22, -e).astype(np.float32)
    g = np.concatenate([g, np.float32([-1.0, -2.0])])
    g = g[rng.permutation(len(g))]
    assert len(np.unique(g)) == len(g)
    return g


def _first_k(scores, k):
    order = sorted(range(len(scores)), key=lambda j: (-float(scores[j]), j))
    return np.sort(np.array(order[:k], dtype=np.int64))


@pytest.mark.parametrize("cut_from_end", [100, 3000])
def test_cut_inside_thousands_of_tightly_packed_scores(cut_from_end):
    rng = np.random.default_rng(40)
    g = _geometric_scores(rng)
    n = len(g)                                    # 5042 key blocks
    k = n - cut_from_end
    # 640 zones of 8 blocks: room for n rows; one head, head_dim 64, scale 1 so
    # that s_ij = qbar_i[0] * kbar_j[0] exactly in float32
    att = PrismSparseAttention(8, 8 * 20, 8 * 32, 1, 64, k, 1e-6, scale=1.0, col_capacity=n * n)
    assert att.cap >= n
    # row patterns: qbar_i[0] = 1 (the scores), 2 (doubled, same order),
    # -1 (reversed order), 0 (every score equal: the first k by index)
    coef = np.array([1.0, 2.0, -1.0, 0.0], dtype=np.float32)
    att.qbar.zero_()
    att.kbar.zero_()
    att.qbar[0, :n, 0] = torch.from_numpy(coef[np.arange(n) % 4]).cuda()
    att.kbar[0, :n, 0] = torch.from_numpy(g).cuda()
    att.nblk.fill_(n)
    att.select()
    P.prism_device_status()                       # no capacity, bounds or timeout error
    rp, cols = att.host_csr()
    expect = {}
    for c in coef:
        s = (np.float32(c) * g).astype(np.float32)
        expect[float(c)] = (s, _first_k(s, k))
    for i in range(n):
        s, e = expect[float(coef[i % 4])]
        got = cols[0][rp[0, i]:rp[0, i + 1]]
        np.testing.assert_array_equal(got, e, err_msg=f"row {i} (coefficient {coef[i % 4]})")
    # the oracle on one row of each pattern
    for i in range(4):
        s, e = expect[float(coef[i])]
        prob = po.block_probabilities(s.astype(np.float64))
        sel_o = po.select_row(prob, k, 1e-6)
        _, ok = selection_row_ok(prob, e, sel_o, k, 1e-6)
        assert ok, f"pattern {coef[i]}: the exact ranking is not a valid selection for the oracle's row"
        if coef[i] == 0.0:
            np.testing.assert_array_equal(e, sel_o)   # all equal: the oracle takes the first k by index too


def test_cut_inside_a_run_of_equal_scores_longer_than_the_sort_buffer():
    """3000 exactly equal scores below ten distinct larger ones; the cut takes
    the first of the equal ones by index (R13), matching the oracle exactly."""
    rng = np.random.default_rng(41)
    n = 3010
    s = np.full(n, 0.25, dtype=np.float32)
    top = rng.choice(n, 10, replace=False)
    s[top] = rng.uniform(1.0, 2.0, 10).astype(np.float32)
    k = 2500
    att = PrismSparseAttention(8, 8 * 20, 8 * 32, 1, 64, k, 1e-6, scale=1.0, col_capacity=n * k)
    att.qbar.zero_()
    att.kbar.zero_()
    att.qbar[0, :n, 0] = 1.0
    att.kbar[0, :n, 0] = torch.from_numpy(s).cuda()
    att.nblk.fill_(n)
    att.select()
    P.prism_device_status()
    rp, cols = att.host_csr()
    e = _first_k(s, k)
    sel_o = po.select_row(po.block_probabilities(s.astype(np.float64)), k, 1e-6)
    np.testing.assert_array_equal(e, sel_o)
    for i in (0, 1, n // 2, n - 1):
        np.testing.assert_array_equal(cols[0][rp[0, i]:rp[0, i + 1]], e)
