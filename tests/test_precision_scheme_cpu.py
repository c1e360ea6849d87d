"""The attention's consistent-rounding scheme, emulated in float32 on the CPU.

The forward turns each score x (log2 units) into p = t(2^(x - m)), t() the
truncation to 11 significant bits, with an integer running maximum m moved
lazily (rescales are exact powers of two), and normalises O by l = sum p.  The
backward knows only L = m_final + log2(l); it takes m' = ceil(L) - 15 and forms
P = t(2^(x - m')) 2^(m' - L).  Truncation commutes with scaling by a power of
two, so this P is the one that formed O (up to the rare element whose
2^(x - m) and 2^(x - m') differ in a last bit of the float32 subtraction), D =
rowsum(dO o O) equals sum_c P_c dP_c, and the rows of dS = P (dP - D) sum to
zero to float32 precision.  With the backward's P rounded independently (the
scheme this replaces) the rows keep a sum of the order of 2^-11 |D|.
"""

import numpy as np

F = np.float32


def _t11(x):
    return (np.asarray(x, dtype=F).view(np.uint32) & np.uint32(0xFFFFE000)).view(F)


def _exp2(y):
    # float32 of 2^y, correctly rounded from float64 (y itself a float32)
    return np.exp2(np.asarray(y, dtype=F).astype(np.float64)).astype(F)


def _forward(x_tiles, v_tiles):
    """Per row: (O, l, m) of the forward's lazily rescaled softmax."""
    l = np.zeros(x_tiles[0].shape[0], dtype=F)
    o = np.zeros((x_tiles[0].shape[0], v_tiles[0].shape[1]), dtype=F)
    m = np.full(x_tiles[0].shape[0], -np.inf, dtype=F)
    for x, v in zip(x_tiles, v_tiles):
        mx = x.max(axis=1)
        grow = mx > m + F(8)
        m_new = np.where(grow, np.ceil(mx).astype(F), m)
        alpha = np.where(np.isfinite(m), np.exp2((m - m_new).astype(np.float64)).astype(F), F(0))
        alpha = np.where(grow, alpha, F(1))
        l = (l * alpha).astype(F)
        o = (o * alpha[:, None]).astype(F)
        m = m_new
        p = _t11(_exp2((x - m[:, None]).astype(F)))
        l = (l + p.sum(axis=1, dtype=np.float64)).astype(F)
        o = (o + (p.astype(np.float64) @ v.astype(np.float64))).astype(F)
    return o / l[:, None], l, m


def _case(seed, n_tiles=6, rows=32, keys=128, d=16):
    rng = np.random.default_rng(seed)
    # scores whose maximum grows by 3 per tile along the row, so that the lazy rescale
    # (threshold 8) runs at least once in every row
    x = [(rng.normal(0, 2.0, (rows, keys)) + 3.0 * t).astype(F) for t in range(n_tiles)]
    v = [rng.normal(0, 1, (keys, d)).astype(F) for _ in range(n_tiles)]
    do = rng.normal(0, 1, (rows, d)).astype(np.float64)
    return x, v, do


def test_backward_rebuilds_the_forward_probabilities_from_the_lse():
    mismatched = total = 0
    for seed in range(4):
        x, v, do = _case(seed)
        o, l, m = _forward(x, v)
        L = (m.astype(np.float64) + np.log2(l.astype(np.float64))).astype(F)
        mb = (np.ceil(L) - 15).astype(F)
        inv = np.exp2((mb - L).astype(np.float64))
        xs = np.concatenate(x, axis=1)
        p_b = _t11(_exp2((xs - mb[:, None]).astype(F))).astype(np.float64) * inv[:, None]
        # the forward's own P, relative to its final max: t(2^(x - m)) / l
        p_f = _t11(_exp2((xs - m[:, None]).astype(F))).astype(np.float64) / l.astype(np.float64)[:, None]
        rel = np.abs(p_b - p_f) / np.maximum(p_f, 1e-30)
        mismatched += int((rel > 1e-5).sum())
        total += rel.size
        np.testing.assert_allclose(p_b.sum(axis=1), 1.0, rtol=1e-5)
    assert mismatched <= 0.001 * total, f"{mismatched} of {total} probabilities differ from the forward's"


def test_rows_of_ds_sum_to_zero_only_with_the_rebuilt_probabilities():
    worst_rebuilt = worst_independent = 0.0
    for seed in range(4):
        x, v, do = _case(seed)
        o, l, m = _forward(x, v)
        L = (m.astype(np.float64) + np.log2(l.astype(np.float64))).astype(F)
        xs = np.concatenate(x, axis=1)
        vs = np.concatenate(v, axis=0).astype(np.float64)
        dp = do @ vs.T
        D = (do * o.astype(np.float64)).sum(axis=1)
        mb = (np.ceil(L) - 15).astype(F)
        p_b = _t11(_exp2((xs - mb[:, None]).astype(F))).astype(np.float64) * np.exp2((mb - L).astype(np.float64))[:, None]
        # the replaced scheme: the backward's own P, exp2(x - L) in float32, not truncated
        p_i = _exp2((xs - L[:, None]).astype(F)).astype(np.float64)
        scale = np.abs(D).max()
        worst_rebuilt = max(worst_rebuilt, np.abs((p_b * (dp - D[:, None])).sum(axis=1)).max() / scale)
        worst_independent = max(worst_independent, np.abs((p_i * (dp - D[:, None])).sum(axis=1)).max() / scale)
    # float32 O (the forward stores O at that precision here) bounds the rebuilt rows' sums
    assert worst_rebuilt < 1e-6, worst_rebuilt
    assert worst_independent > 100 * worst_rebuilt, (worst_independent, worst_rebuilt)


def test_truncation_commutes_with_powers_of_two():
    rng = np.random.default_rng(3)
    y = rng.uniform(-20, 15, 100000).astype(F)
    p = _exp2(y)
    for k in (-9, -1, 1, 7, 15):
        scaled = (p * F(2.0 ** k)).astype(F)
        assert np.array_equal(_t11(scaled), (_t11(p) * F(2.0 ** k)).astype(F))
