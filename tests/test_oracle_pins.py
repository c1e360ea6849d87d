"""Pins for the fp64 oracle: closed forms, invariants, brute force and library routines.

Each test fixes one part of the oracle to something other than itself, so that
a dropped term, a wrong axis, sign or index fails here before any GPU parity
test trusts the oracle.  CPU only.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import prism_oracle as po

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _grid(T, H, W, C, fn):
    """[N, 1, C] natural-layout tensor from fn(t, y, x) -> [C]."""
    out = np.zeros((T, H, W, C))
    for t in range(T):
        for y in range(H):
            for x in range(W):
                out[t, y, x] = fn(t, y, x)
    return out.reshape(T * H * W, 1, C)


# ---------------------------------------------------------------- indicator --

def test_variance_of_one_period_sinusoid_along_each_axis():
    """A channel A cos(2 pi u/8 + phi) along one axis: its 8 samples have mean 0 and
    mean square A^2/2, so sigma^2 on that axis is the channel average of A^2/2 and 0
    on the two others; r is one-hot."""
    amps = np.array([0.5, 1.0, 2.0])
    phis = np.array([0.1, 1.3, 2.9])
    for axis in range(3):
        def fn(t, y, x, axis=axis):
            u = (t, y, x)[axis]
            return amps * np.cos(2 * math.pi * u / 8 + phis)
        V = _grid(8, 8, 8, 3, fn)
        ind = po.zone_indicator(V, 8, 8, 8)
        expect = np.zeros(3)
        expect[axis] = np.mean(amps ** 2 / 2)
        np.testing.assert_allclose(ind["sigma2_v"][0], expect, atol=1e-12)
        onehot = np.zeros(3)
        onehot[axis] = 1.0
        np.testing.assert_allclose(ind["r_v"][0], onehot, atol=1e-12)


def test_separable_field_variances_are_the_axis_variances():
    """For V = f(t) + g(y) + h(x), pooling over two axes removes their terms, so
    sigma^2_T is the population variance of f over the zone's 8 samples, etc."""
    rng = np.random.default_rng(3)
    f, g, h = rng.standard_normal((3, 16, 2))
    V = _grid(16, 8, 8, 2, lambda t, y, x: f[t] + g[y] + h[x])
    ind = po.zone_indicator(V, 16, 8, 8)
    for m, zt in enumerate(range(2)):
        sl = slice(8 * zt, 8 * zt + 8)
        exp = [np.var(f[sl], axis=0).mean(), np.var(g[:8], axis=0).mean(), np.var(h[:8], axis=0).mean()]
        np.testing.assert_allclose(ind["sigma2_v"][m], exp, rtol=1e-12, atol=1e-14)
        assert abs(ind["r_v"][m].sum() - 1.0) < 1e-12


def test_indicator_invariances():
    """Shifts per channel do not change sigma^2; scaling by c multiplies it by c^2 and
    leaves r; swapping the T and H axes of the grid swaps sigma^2_T and sigma^2_H."""
    rng = np.random.default_rng(4)
    V = rng.standard_normal((8 * 16 * 8, 2, 3))
    base = po.zone_indicator(V, 8, 16, 8)
    shifted = po.zone_indicator(V + rng.standard_normal((1, 2, 3)), 8, 16, 8)
    np.testing.assert_allclose(shifted["sigma2_v"], base["sigma2_v"], rtol=1e-10)
    scaled = po.zone_indicator(3.0 * V, 8, 16, 8)
    np.testing.assert_allclose(scaled["sigma2_v"], 9.0 * base["sigma2_v"], rtol=1e-10)
    np.testing.assert_allclose(scaled["r_v"], base["r_v"], rtol=1e-10)
    Vc = V.reshape(8, 16, 8, 6)[:, :8]                     # one zone, T = H = 8
    swapped = np.ascontiguousarray(Vc.transpose(1, 0, 2, 3)).reshape(-1, 2, 3)
    a = po.zone_indicator(Vc.reshape(-1, 2, 3), 8, 8, 8)["sigma2_v"][0]
    b = po.zone_indicator(swapped, 8, 8, 8)["sigma2_v"][0]
    np.testing.assert_allclose(b, a[[1, 0, 2]], rtol=1e-12)


def test_audio_terms():
    """Constant audio: abar = 1 (zone mean = global max), vhat = 0, so g = r + eps.
    Audio varying along W only: vhat = (0, 0, 1).  Zero audio: abar = vhat = 0."""
    rng = np.random.default_rng(5)
    V = rng.standard_normal((8 * 8 * 16, 1, 4))
    const = po.zone_indicator(V, 8, 8, 16, np.full(8 * 8 * 16, 0.7))
    np.testing.assert_allclose(const["abar"], 1.0)
    np.testing.assert_allclose(const["vhat_a"], 0.0)
    np.testing.assert_allclose(const["g"], const["r_v"] + po.EPS, rtol=1e-14)
    aw = np.tile(np.cos(2 * math.pi * np.arange(16) / 8) + 2.0, 8 * 8)
    ind = po.zone_indicator(V, 8, 8, 16, aw)
    np.testing.assert_allclose(ind["vhat_a"], [[0, 0, 1], [0, 0, 1]], atol=1e-12)
    np.testing.assert_allclose(ind["abar"], [2.0 / 3.0, 2.0 / 3.0], rtol=1e-12)
    zero = po.zone_indicator(V, 8, 8, 16, np.zeros(8 * 8 * 16))
    np.testing.assert_allclose(zero["abar"], 0.0)
    np.testing.assert_allclose(zero["g"], zero["r_v"] + po.EPS)


def test_density_threshold_rule():
    """Method §2 thresholds: rho >= 0.5 -> 64, 0.25 <= rho < 0.5 -> 128, rho < 0.25 -> 256."""
    rho = np.array([1.0, 0.5, np.nextafter(0.5, 0), 0.25, np.nextafter(0.25, 0), 0.0])
    np.testing.assert_array_equal(po.block_volume(rho), [64, 64, 128, 128, 256, 256])


# ------------------------------------------------------------------ shapes --

def test_log2_edges_sum_and_isotropic():
    rng = np.random.default_rng(6)
    g = rng.uniform(1e-4, 2.0, size=(50, 3))
    for B in (64, 128, 256):
        ell = po.optimal_log2_edges(g, np.full(50, B))
        np.testing.assert_allclose(ell.sum(axis=1), math.log2(B), rtol=1e-12)
        iso = po.optimal_log2_edges(np.array([[0.3, 0.3, 0.3]]), np.array([B]))
        np.testing.assert_allclose(iso[0], math.log2(B) / 3, rtol=1e-12)


def test_log2_edges_minimise_the_stated_loss():
    """l* must minimise sum_d g_d (b_d^2 - 1) on prod b_d = B (Method §2), found here
    by a generic constrained minimiser over two free log-edges."""
    from scipy.optimize import minimize
    rng = np.random.default_rng(7)
    for _ in range(20):
        g = rng.uniform(0.01, 3.0, size=3)
        B = int(rng.choice([64, 128, 256]))
        S = math.log2(B)

        def loss(u):
            ell = np.array([u[0], u[1], S - u[0] - u[1]])
            return float(np.sum(g * (4.0 ** ell - 1)))

        res = minimize(loss, x0=[S / 3, S / 3], method="Nelder-Mead",
                       options=dict(xatol=1e-10, fatol=1e-14, maxiter=20000))
        num = np.array([res.x[0], res.x[1], S - res.x[0] - res.x[1]])
        np.testing.assert_allclose(po.optimal_log2_edges(g, B), num, atol=1e-5)


def test_candidate_set_is_every_power_of_two_box_of_edge_at_least_two():
    """The 16 candidates are exactly the boxes with edges in {2,4,8} and volume in
    {64,128,256}; every edge divides the zone edge 8."""
    boxes = sorted((b for b in itertools.product([1, 2, 4, 8], repeat=3)
                    if b[0] * b[1] * b[2] in (64, 128, 256) and min(b) >= 2),
                   key=lambda b: (b[0] * b[1] * b[2], b))
    assert tuple(boxes) == po.SHAPES
    assert len(po.SHAPES) == 16


def test_golden_shape_cases():
    cases = 0
    with open(os.path.join(GOLDEN, "shape_cases.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].split()
            if not line:
                continue
            gT, gH, gW, B, bT, bH, bW = map(float, line)
            ell = po.optimal_log2_edges(np.array([gT, gH, gW]), B)
            sid = po.quantise_shape(ell, B)
            assert po.SHAPES[sid] == (int(bT), int(bH), int(bW)), line
            cases += 1
    assert cases == 8


def test_quantisation_matches_enumeration_and_volume():
    rng = np.random.default_rng(8)
    for _ in range(300):
        g = rng.uniform(1e-4, 2.0, size=3)
        B = int(rng.choice([64, 128, 256]))
        ell = po.optimal_log2_edges(g, B)
        sid = po.quantise_shape(ell, B)
        bT, bH, bW = po.SHAPES[sid]
        assert bT * bH * bW == B
        best = min(sum((ell[d] - math.log2(c[d])) ** 2 for d in range(3))
                   for c in po.SHAPES if c[0] * c[1] * c[2] == B)
        got = sum((ell[d] - math.log2(po.SHAPES[sid][d])) ** 2 for d in range(3))
        assert got <= best + 1e-9


# ------------------------------------------------------------- permutation --

def _random_layout(T, H, W, seed):
    rng = np.random.default_rng(seed)
    Z = (T // 8) * (H // 8) * (W // 8)
    g = rng.uniform(1e-4, 1.0, size=(Z, 3))
    rho = rng.uniform(0, 1, size=Z)
    return po.assign_blocks(g, rho, T, H, W)


def test_permutation_is_a_box_tiling_of_each_zone():
    T, H, W = 16, 8, 24
    shape_id, base, blocks = _random_layout(T, H, W, 9)
    perm = po.permutation(T, H, W, shape_id)
    assert sorted(perm.tolist()) == list(range(T * H * W))
    assert base[-1] == len(blocks)
    ZY, ZX = H // 8, W // 8
    for j, (start, size, m, sid) in enumerate(blocks):
        bT, bH, bW = po.SHAPES[sid]
        assert size == bT * bH * bW and sid == shape_id[m]
        assert base[m] <= j < base[m + 1]
        n = perm[start:start + size]
        t, y, x = n // (H * W), (n // W) % H, n % W
        zt, zy, zx = m // (ZY * ZX), (m // ZX) % ZY, m % ZX
        assert t.min() // 8 == zt and y.min() // 8 == zy and x.min() // 8 == zx
        assert (t.max() - t.min() + 1, y.max() - y.min() + 1, x.max() - x.min() + 1) == (bT, bH, bW)
        assert t.min() % bT == 0 and y.min() % bH == 0 and x.min() % bW == 0
        assert len(set(n.tolist())) == size
        assert start // 512 == m


def test_permute_round_trip_and_pooling():
    T, H, W = 8, 16, 16
    shape_id, base, blocks = _random_layout(T, H, W, 10)
    perm = po.permutation(T, H, W, shape_id)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((T * H * W, 3, 4))
    xp = po.permute(x, perm)
    np.testing.assert_array_equal(po.unpermute(xp, perm), x)
    pooled = po.pool_blocks(xp, blocks)
    grid = x.reshape(T, H, W, 3, 4)
    for j, (start, size, m, sid) in enumerate(blocks):
        n0 = perm[start]
        t0, y0, x0 = n0 // (H * W), (n0 // W) % H, n0 % W
        bT, bH, bW = po.SHAPES[sid]
        box = grid[t0:t0 + bT, y0:y0 + bH, x0:x0 + bW].reshape(-1, 3, 4).mean(axis=0)
        np.testing.assert_allclose(pooled[:, j, :], box, rtol=1e-12)


# --------------------------------------------------------------- selection --

def test_select_against_subset_brute_force():
    """n_p is the smallest n for which SOME n-subset reaches mass p; the chosen set is
    a max-mass subset of its size, and |S| = max(k, n_p)."""
    rng = np.random.default_rng(12)
    for trial in range(200):
        n = int(rng.integers(1, 8))
        P = po.block_probabilities(rng.standard_normal(n) * rng.uniform(0.1, 4))
        assert abs(P.sum() - 1) < 1e-12
        k = int(rng.integers(1, 9))
        p = float(rng.uniform(0.05, 1.0))
        best_np = n
        for size in range(1, n + 1):
            if max(sum(P[list(c)]) for c in itertools.combinations(range(n), size)) >= p:
                best_np = size
                break
        sel = po.select_row(P, k, p)
        assert len(sel) == max(min(k, n), best_np)
        top = max(sum(P[list(c)]) for c in itertools.combinations(range(n), len(sel)))
        assert abs(P[sel].sum() - top) < 1e-12
        assert list(sel) == sorted(sel)


def test_select_edge_cases():
    P = np.array([0.1, 0.4, 0.1, 0.4])
    assert po.select_row(P, 10, 0.5).tolist() == [0, 1, 2, 3]        # k clamps to nblk
    assert po.select_row(P, 1, 1e-9).tolist() == [1]                  # exactly k; tie -> lower index
    assert po.select_row(P, 1, 0.5).tolist() == [1, 3]                # 0.4 + 0.4 >= 0.5
    assert po.select_row(P, 1, 0.85).tolist() == [0, 1, 3]            # next tie -> index 0
    assert po.select_row(P, 1, 1.0).tolist() == [0, 1, 2, 3]


# --------------------------------------------------------------- attention --

def _tiny_problem(seed, T=8, H=8, W=16, heads=2, d=8):
    rng = np.random.default_rng(seed)
    N = T * H * W
    Z = N // 512
    g = rng.uniform(1e-4, 1.0, size=(Z, 3))
    rho = rng.uniform(0, 1, size=Z)
    shape_id, base, blocks = po.assign_blocks(g, rho, T, H, W)
    perm = po.permutation(T, H, W, shape_id)
    q, k, v, do = (rng.standard_normal((N, heads, d)) for _ in range(4))
    return dict(N=N, heads=heads, d=d, blocks=blocks, perm=perm,
                qp=po.permute(q, perm), kp=po.permute(k, perm), vp=po.permute(v, perm),
                dop=po.permute(do, perm))


def _mask(blocks, row_ptr, cols, h, N):
    m = np.zeros((N, N), dtype=bool)
    for i, (s, z, _, _) in enumerate(blocks):
        for j in cols[h][row_ptr[h, i]:row_ptr[h, i + 1]]:
            m[s:s + z, blocks[j][0]:blocks[j][0] + blocks[j][1]] = True
    return m


def _random_csr(blocks, heads, seed, density):
    rng = np.random.default_rng(seed)
    nb = len(blocks)
    row_ptr = np.zeros((heads, nb + 1), dtype=np.int64)
    cols = []
    for h in range(heads):
        hc = []
        for i in range(nb):
            sel = np.flatnonzero(rng.random(nb) < density)
            if len(sel) == 0:
                sel = np.array([int(rng.integers(nb))])
            hc.append(sel)
            row_ptr[h, i + 1] = row_ptr[h, i] + len(sel)
        cols.append(np.concatenate(hc))
    return row_ptr, cols


@pytest.mark.parametrize("density", [1.0, 0.3])
def test_forward_equals_masked_sdpa(density):
    """At k = all (density 1) the sparse forward is dense softmax attention; for a
    partial selection it equals SDPA with the block mask (torch, float64)."""
    pb = _tiny_problem(13)
    row_ptr, cols = _random_csr(pb["blocks"], pb["heads"], 14, density)
    scale = 1 / math.sqrt(pb["d"])
    O, L = po.bsa_forward(pb["qp"], pb["kp"], pb["vp"], pb["blocks"], row_ptr, cols, scale)
    for h in range(pb["heads"]):
        mask = torch.from_numpy(_mask(pb["blocks"], row_ptr, cols, h, pb["N"]))
        q, k, v = (torch.from_numpy(t[h]) for t in (pb["qp"], pb["kp"], pb["vp"]))
        ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask[None])
        np.testing.assert_allclose(O[h], ref[0].numpy(), rtol=1e-10, atol=1e-12)
        logits = (q @ k.T) * scale
        lse = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), dim=1)
        np.testing.assert_allclose(L[h], lse.numpy(), rtol=1e-12)


def test_backward_equals_autograd_of_masked_sdpa():
    pb = _tiny_problem(15)
    row_ptr, cols = _random_csr(pb["blocks"], pb["heads"], 16, 0.4)
    scale = 1 / math.sqrt(pb["d"])
    dq, dk, dv = po.bsa_backward(pb["qp"], pb["kp"], pb["vp"], pb["dop"], pb["blocks"], row_ptr, cols, scale)
    for h in range(pb["heads"]):
        mask = torch.from_numpy(_mask(pb["blocks"], row_ptr, cols, h, pb["N"]))
        q, k, v = (torch.from_numpy(t[h]).clone().requires_grad_(True) for t in (pb["qp"], pb["kp"], pb["vp"]))
        out = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask[None])
        out.backward(torch.from_numpy(pb["dop"][h])[None])
        np.testing.assert_allclose(dq[h], q.grad.numpy(), rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dk[h], k.grad.numpy(), rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dv[h], v.grad.numpy(), rtol=1e-9, atol=1e-12)


def test_block_restricted_gradients_equal_autograd_of_masked_sdpa():
    """dQ of chosen query blocks and dK, dV of chosen key blocks (the forms used
    for sampled checks on large grids) against torch autograd of SDPA with the
    block mask, on the rows of those blocks."""
    pb = _tiny_problem(25)
    row_ptr, cols = _random_csr(pb["blocks"], pb["heads"], 26, 0.4)
    scale = 1 / math.sqrt(pb["d"])
    nb = len(pb["blocks"])
    for h in range(pb["heads"]):
        mask = torch.from_numpy(_mask(pb["blocks"], row_ptr, cols, h, pb["N"]))
        q, k, v = (torch.from_numpy(t[h]).clone().requires_grad_(True) for t in (pb["qp"], pb["kp"], pb["vp"]))
        out = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask[None])
        out.backward(torch.from_numpy(pb["dop"][h])[None])
        picks = [0, nb // 2, nb - 1]
        dq = po.bsa_query_block_dq(pb["qp"], pb["kp"], pb["vp"], pb["dop"], pb["blocks"], row_ptr, cols, scale,
                                   picks, h=h)
        kv = po.bsa_key_block_dkdv(pb["qp"], pb["kp"], pb["vp"], pb["dop"], pb["blocks"], row_ptr, cols, scale,
                                   picks, h=h)
        for i in picks:
            s0, sz = pb["blocks"][i][0], pb["blocks"][i][1]
            np.testing.assert_allclose(dq[i], q.grad.numpy()[s0:s0 + sz], rtol=1e-9, atol=1e-12)
            dk_j, dv_j = kv[i]
            np.testing.assert_allclose(dk_j, k.grad.numpy()[s0:s0 + sz], rtol=1e-9, atol=1e-12)
            np.testing.assert_allclose(dv_j, v.grad.numpy()[s0:s0 + sz], rtol=1e-9, atol=1e-12)


def test_backward_against_finite_differences():
    """Central differences of L = sum(dO * O) on a few entries of q, k, v."""
    pb = _tiny_problem(17, T=8, H=8, W=8, heads=1, d=4)
    row_ptr, cols = _random_csr(pb["blocks"], 1, 18, 0.6)
    scale = 0.5
    args = [pb["qp"].copy(), pb["kp"].copy(), pb["vp"].copy()]
    grads = po.bsa_backward(*args, pb["dop"], pb["blocks"], row_ptr, cols, scale)
    rng = np.random.default_rng(19)
    eps = 1e-6
    for which in range(3):
        for _ in range(6):
            r, c = int(rng.integers(pb["N"])), int(rng.integers(4))
            vals = []
            for sgn in (+1, -1):
                a = [x.copy() for x in args]
                a[which][0, r, c] += sgn * eps
                O, _ = po.bsa_forward(*a, pb["blocks"], row_ptr, cols, scale)
                vals.append(np.sum(O * pb["dop"]))
            fd = (vals[0] - vals[1]) / (2 * eps)
            an = grads[which][0, r, c]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, r, c, fd, an)


def test_pipeline_runs_end_to_end_with_every_volume():
    """Zone amplitudes 1, 0.8, 0.1.. give info ratios 1, 0.64, 0.01 and (no audio)
    rho = 0.5, 0.32, 0.005: volumes 64, 128 and 256 all occur."""
    rng = np.random.default_rng(20)
    T, H, W = 8, 16, 24
    N = T * H * W
    n = np.arange(N)
    zone = ((n // (H * W)) // 8 * 2 + (n // W) % H // 8) * 3 + (n % W) // 8
    amp = np.array([1.0, 0.8, 0.1, 0.1, 0.1, 0.1])[zone]
    q, k = (rng.standard_normal((N, 2, 8)) for _ in range(2))
    v = amp[:, None, None] * rng.standard_normal((N, 2, 8))
    out = po.pipeline(q, k, v, T, H, W, None, 2, 0.5)
    B = [int(b[1]) for b in out["blocks"]]
    assert B[:8] == [64] * 8 and B[8:12] == [128] * 4 and set(B[12:]) == {256}
    assert out["O"].shape == (N, 2, 8) and np.isfinite(out["O"]).all()
    assert out["zone_blk_base"][-1] == len(out["blocks"])


def test_bf16_half_ulp_helper():
    """The tolerance helper is half the bf16 spacing: rounding any value to bf16
    moves it by at most that much, and consecutive bf16 values above a
    representable x differ by twice that."""
    from tests.helpers import bf16_half_ulp
    rng = np.random.default_rng(40)
    x = rng.standard_normal(10000) * np.exp(rng.uniform(-5, 5, 10000))
    r = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(r - x) <= bf16_half_ulp(x) * (1 + 1e-12))
    for v in (1.0, 1.5, 3.0, 8.0, 9.5):
        b = torch.tensor(v, dtype=torch.bfloat16)
        nxt = torch.tensor(v + 2 * bf16_half_ulp(v), dtype=torch.bfloat16)
        assert float(nxt) - float(b) == 2 * bf16_half_ulp(v)


def test_pooling_from_natural_layout_equals_pooling_of_the_permuted_copy():
    T, H, W = 8, 16, 16
    shape_id, base, blocks = _random_layout(T, H, W, 41)
    perm = po.permutation(T, H, W, shape_id)
    x = np.random.default_rng(42).standard_normal((T * H * W, 3, 4)).astype(np.float32)
    a = po.pool_blocks(po.permute(x, perm), blocks)
    b = po.pool_blocks_natural(x, perm, blocks)
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(po.pool_blocks_natural(x, perm, blocks, heads=[2]), a[2:3], rtol=1e-12, atol=1e-12)


# ------------------------------------------------- audio norms and variants --

def test_audio_norms_closed_forms():
    """a = ||h||_2 per token: a 3-4-5 row gives 5, a constant row c over C channels
    gives |c| sqrt(C), a zero row 0; scaling by alpha scales a by |alpha|, an
    orthogonal mixing of the channels leaves a unchanged, and a random matrix
    agrees with numpy's own vector norm."""
    h = np.zeros((4, 16))
    h[0, 3], h[0, 9] = 3.0, -4.0
    h[1, :] = -0.25
    np.testing.assert_allclose(po.audio_norms(h), [5.0, 0.25 * 4.0, 0.0, 0.0], rtol=0, atol=1e-15)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((64, 48))
    a = po.audio_norms(x)
    np.testing.assert_allclose(po.audio_norms(-2.5 * x), 2.5 * a, rtol=1e-14)
    q, _ = np.linalg.qr(rng.standard_normal((48, 48)))
    np.testing.assert_allclose(po.audio_norms(x @ q), a, rtol=1e-12)
    np.testing.assert_allclose(a, np.linalg.norm(x, axis=1), rtol=1e-14)


def test_top_k_from_sparsity_follows_the_readme_ratio():
    """The README's bsa_sparsity 0.75 means each query block attends to a quarter of
    the key blocks: k = nblk/4 whenever 4 divides nblk; a share that is not a whole
    block rounds up; sparsity 0 keeps every block and k never drops below 1."""
    for nblk in (8, 240, 960, 15360):
        assert po.top_k_from_sparsity(0.75, nblk) == nblk // 4
        assert po.top_k_from_sparsity(0.5, nblk) == nblk // 2
        assert po.top_k_from_sparsity(0.0, nblk) == nblk
    assert po.top_k_from_sparsity(0.75, 9) == 3            # 2.25 -> 3
    assert po.top_k_from_sparsity(0.999, 10) == 1          # 0.01 -> 1
    assert po.top_k_from_sparsity(1.0, 10) == 1            # never empty
    # float32 parameter width: 0.93 is 0.93000000715..., so 960 * 0.06999999285 = 67.2 -> 68
    assert po.top_k_from_sparsity(0.93, 960) == 68


def test_select_with_sparsity_ratio_equals_select_with_its_k():
    rng = np.random.default_rng(3)
    qb, kb = rng.standard_normal((2, 12, 8)), rng.standard_normal((2, 12, 8))
    k = po.top_k_from_sparsity(0.75, 12)
    a = po.block_select(qb, kb, 1, 0.5, 0.4, sparsity=0.75)
    b = po.block_select(qb, kb, k, 0.5, 0.4)
    np.testing.assert_array_equal(a[0], b[0])
    for x, y in zip(a[1], b[1]):
        np.testing.assert_array_equal(x, y)
    assert all(np.diff(a[0][h]).min() >= k for h in range(2))


def test_fixed_shape_mode_is_the_uniform_444_tiling():
    """enable_ivpq_dynamic_block off: every zone is cut into eight 4x4x4 boxes, in
    raster order, whatever g and rho are; on zones where the dynamic rule itself
    lands on 4x4x4 (isotropic g, rho >= tau_128) the two layouts coincide."""
    T, H, W = 16, 8, 16
    Z = (T // 8) * (H // 8) * (W // 8)
    rng = np.random.default_rng(11)
    g = rng.uniform(1e-4, 1.0, (Z, 3))
    rho = rng.uniform(0, 1, Z)
    sid, base, blocks = po.assign_blocks(g, rho, T, H, W, fixed_shape=3)
    assert (sid == 3).all() and po.SHAPES[3] == (4, 4, 4)
    np.testing.assert_array_equal(base, 8 * np.arange(Z + 1))
    assert (blocks[:, 1] == 64).all()
    np.testing.assert_array_equal(blocks[:, 0], 64 * np.arange(8 * Z))
    perm = po.permutation(T, H, W, sid)
    for b in range(8 * Z):
        n = perm[64 * b: 64 * b + 64]
        t, y, x = n // (H * W), (n // W) % H, n % W
        for c in (t, y, x):
            assert c.max() - c.min() == 3 and c.min() % 4 == 0
    iso = np.full((Z, 3), 0.3)
    dyn = po.assign_blocks(iso, np.full(Z, 0.9), T, H, W)
    fix = po.assign_blocks(iso, np.full(Z, 0.9), T, H, W, fixed_shape=3)
    for u, v in zip(dyn, fix):
        np.testing.assert_array_equal(u, v)
    # other fixed shapes keep their own volume
    sid, base, blocks = po.assign_blocks(None, None, T, H, W, fixed_shape=13)
    assert (blocks[:, 1] == 256).all() and (np.diff(base) == 2).all()


def test_top_p_one_keeps_every_block_even_where_float_sums_reach_one_early():
    """p = 1: every softmax probability is positive, so no proper prefix has mass 1
    in exact arithmetic and Top-p is the whole row.  Softmax rows whose float64
    running sum (in ranking order) reaches 1.0 before the end are common; on such a
    row the selection must still be the whole row, and p just below 1 stops early."""
    rng = np.random.default_rng(0)
    early = None
    for _ in range(2000):
        n = int(rng.integers(3, 40))
        P = po.block_probabilities(rng.normal(0, 1, n) * rng.uniform(0.1, 20))
        acc = 0.0
        for pos, j in enumerate(sorted(range(n), key=lambda j: (-P[j], j))):
            acc += P[j]
            if acc >= 1.0:
                if pos + 1 < n:
                    early = P
                break
        if early is not None:
            break
    assert early is not None
    np.testing.assert_array_equal(po.select_row(early, 1, 1.0), np.arange(len(early)))
    assert len(po.select_row(early, 1, 1.0 - 1e-9)) < len(early)


# ------------------------------------------------------------ block scores --

def test_block_scores_and_probabilities_hand_derived():
    """Method §3: each pooled query block is scored against every pooled key
    block of its head, s_ij = scale * Qbar_i . Kbar_j (R10, R11), and P_i is the
    softmax of row i over the key blocks.  Two query blocks and three key blocks
    (so a transposed product has the wrong shape), scale 1/2, worked by hand:
      Qbar_0 = (1, 0): dots with Kbar = (1,1), (2,0), (0,1) are 1, 2, 0
      Qbar_1 = (0, 2): dots are 2, 0, 2
    so s_0 = (1/2, 1, 0), s_1 = (1, 0, 1), and
      P_0 = (e^{1/2}, e, 1) / (1 + e^{1/2} + e),  P_1 = (e, 1, e) / (1 + 2e)."""
    qbar = np.array([[1.0, 0.0], [0.0, 2.0]])
    kbar = np.array([[1.0, 1.0], [2.0, 0.0], [0.0, 1.0]])
    s = po.block_scores(qbar, kbar, 0.5)
    assert s.shape == (2, 3)
    np.testing.assert_array_equal(s, [[0.5, 1.0, 0.0], [1.0, 0.0, 1.0]])
    e = math.e
    r = math.sqrt(e)
    P0 = po.block_probabilities(s[0])
    P1 = po.block_probabilities(s[1])
    np.testing.assert_allclose(P0, np.array([r, e, 1.0]) / (1.0 + r + e), rtol=1e-15)
    np.testing.assert_allclose(P1, np.array([e, 1.0, e]) / (1.0 + 2.0 * e), rtol=1e-15)
    # the softmax runs along the key blocks of one query row: that row sums to 1,
    # while a column of the first key block does not
    assert abs(P0.sum() - 1.0) < 1e-15 and abs(P1.sum() - 1.0) < 1e-15
    assert abs(P0[0] + P1[0] - 1.0) > 0.1
    # dropping the scale (or doubling it) changes the hand values
    assert not np.allclose(po.block_probabilities(po.block_scores(qbar, kbar, 1.0)[0]), P0)
    # the whole-head selection uses the same rows: k = 1, p = 0.5 keeps the most
    # probable key block of each row (index 1 for row 0; indices 0 and 2 tie for
    # row 1, and 0 + 2 together pass 0.5, so both are kept)
    rp, cols, probs = po.block_select(qbar[None], kbar[None], 1, 0.5, 0.5)
    np.testing.assert_allclose(probs[0], np.stack([P0, P1]), rtol=1e-15)
    np.testing.assert_array_equal(rp[0], [0, 1, 3])
    np.testing.assert_array_equal(cols[0], [1, 0, 2])


def test_block_probabilities_ignore_a_common_shift_of_the_key_blocks():
    """Adding one vector u to every pooled key block adds scale * Qbar_i . u to the
    whole row i, which a softmax over that row's key blocks ignores.  The added
    amount differs between rows, so a softmax over the wrong axis, or scores built
    as Kbar Qbar^T, would move.  Rectangular case (5 query blocks, 9 key blocks)."""
    rng = np.random.default_rng(21)
    qbar = rng.standard_normal((5, 6))
    kbar = rng.standard_normal((9, 6))
    u = 3.0 * rng.standard_normal(6)
    scale = 0.37
    s = po.block_scores(qbar, kbar, scale)
    s_shift = po.block_scores(qbar, kbar + u, scale)
    assert s.shape == (5, 9)
    row_shift = s_shift - s
    np.testing.assert_allclose(row_shift, np.repeat((scale * qbar @ u)[:, None], 9, axis=1), atol=1e-12)
    assert np.ptp(row_shift[:, 0]) > 1.0      # rows move by different amounts
    for i in range(5):
        np.testing.assert_allclose(po.block_probabilities(s_shift[i]), po.block_probabilities(s[i]),
                                   rtol=1e-12, atol=1e-15)


def test_block_probabilities_match_the_library_softmax():
    """The probability rows against torch's softmax of the same fp64 scores, on rows
    with large spreads (the max subtraction keeps them finite)."""
    rng = np.random.default_rng(22)
    for n in (1, 2, 7, 300):
        s = rng.standard_normal(n) * 40.0
        ref = torch.softmax(torch.from_numpy(s), dim=0).numpy()
        np.testing.assert_allclose(po.block_probabilities(s), ref, rtol=1e-12, atol=1e-300)
