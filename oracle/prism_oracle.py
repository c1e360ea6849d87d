"""Plain fp64 CPU oracle for Prism's dynamic block-sparse video self-attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this file; only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
leg of ``bench.py`` use it.  It shares no code, header or table with the CUDA
library: every constant below is written out here on its own.

Source: "Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio
Generation Model Training" (arXiv 2610.05416 reading guide), sections
"Key ideas" and "Method" §1 (variation indicator), §2 (block volume and shape
quantisation) and §3 (hybrid top-k / top-p attention).  Where the text leaves a
step open, the reading taken is named inline as R1..R20; the same list is kept
with the design notes of the repository.

Layouts (all numpy, float64 unless stated):
  natural token index   n = (t*H + y)*W + x
  Q, K, V, dO (natural) [N, heads, d]
  permuted tensors      [heads, N, d]   (zone-major, block-major, in-block raster)
  zones                 m = (zt*(H/8) + zy)*(W/8) + zx, each 8x8x8 tokens

Parity status per function (pins live in tests/test_oracle_pins.py):
  audio_norms             pinned (closed forms, scaling, a library norm)
  zone_indicator          pinned (closed forms, invariants)
  block_volume            parity unpinned: the density rho(m) is a reading (R6);
                          only its threshold rule is fixed by the pages
  optimal_log2_edges      pinned (sum = S, independent constrained minimisation)
  quantise_shape          pinned (hand-derived cases, product = B, enumeration)
  permutation / pooling   pinned (bijection, box tiling, round trip)
  block_scores /          pinned (a hand-worked 2x3 case, invariance of each row
  block_probabilities       under a common shift of the key blocks, torch softmax)
  block_select            pinned (subset brute force, invariants, the hand case)
  top_k_from_sparsity     pinned (the README's worked ratio: 0.75 keeps 25%)
  assign_blocks (fixed)   pinned (every zone the 4x4x4 box; equals dynamic
                          assignment wherever that picks 4x4x4)
  bsa_forward / backward  pinned (dense attention at k = all via torch SDPA,
                          finite differences, autograd of a dense masked form)
  bsa_query_block_dq /    pinned (autograd of the dense masked form, on the
  bsa_key_block_dkdv        rows of the blocks they return)
"""

from __future__ import annotations

import math

import numpy as np

ZONE = 8                      # macro-zone edge, Key ideas: Z_T x Z_H x Z_W = 8x8x8
ZONE_TOKENS = ZONE ** 3       # 512 tokens per zone
TAU_128 = 0.5                 # Method §2 thresholds
TAU_256 = 0.25
EPS = 1e-4                    # R5: the epsilon of the composite indicator
TIE_TOL = 1e-9                # R8: distance ties in the shape quantisation

# R7: the 16-shape candidate set.  Edges are powers of two in {2,4,8} whose
# product is the block volume; that gives 7 + 6 + 3 = 16 shapes, the count the
# Key ideas state.  Canonical order: volume ascending, then (bT,bH,bW)
# lexicographic ascending.  Listed by hand so the list can be read off.
SHAPES = (
    (2, 4, 8), (2, 8, 4), (4, 2, 8), (4, 4, 4), (4, 8, 2), (8, 2, 4), (8, 4, 2),   # B = 64
    (2, 8, 8), (4, 4, 8), (4, 8, 4), (8, 2, 8), (8, 4, 4), (8, 8, 2),              # B = 128
    (4, 8, 8), (8, 4, 8), (8, 8, 4),                                                # B = 256
)


def audio_norms(h):
    """Method §1: the audio coupling input a = ||h_hat||_2 per video token.

    h : [N, C], the audio-to-video cross-attention output of each video token
    over all of its channels (heads * head_dim).  Returns [N] float64: the
    Euclidean norm of each row (R20: the norm is taken over every channel of
    the token, all heads together).
    """
    h = np.asarray(h, dtype=np.float64)
    out = np.empty(h.shape[0])
    for n in range(h.shape[0]):
        out[n] = math.sqrt(float(np.dot(h[n], h[n])))
    return out


def zone_grid(T, H, W):
    """Number of zones along each axis; every axis must be a multiple of 8."""
    if T % ZONE or H % ZONE or W % ZONE or min(T, H, W) <= 0:
        raise ValueError("token grid must be a positive multiple of 8 on every axis")
    return T // ZONE, H // ZONE, W // ZONE


def _zone_cube(x, T, H, W, zt, zy, zx):
    """Return the zone's tokens as an array [8(t), 8(y), 8(x), channels]."""
    grid = x.reshape(T, H, W, -1)
    return grid[zt * ZONE:(zt + 1) * ZONE, zy * ZONE:(zy + 1) * ZONE, zx * ZONE:(zx + 1) * ZONE, :]


def directional_variance(cube):
    """Method §1: sigma^2_d for d in (T, H, W) of one zone.

    ``cube`` is [8, 8, 8, C].  For axis d, the zone is mean-pooled over the two
    other axes, giving Z_d = 8 vectors Vbar_{i,c}.  mu_c is the mean of those 8
    vectors (the zone mean).  sigma^2_d is the channel average (1/D sum_c) of
    the population variance (1/Z_d sum_i) of Vbar_{i,c} about mu_c.
    """
    cube = np.asarray(cube, dtype=np.float64)
    out = np.zeros(3)
    for axis in range(3):
        others = tuple(a for a in range(3) if a != axis)
        pooled = cube.mean(axis=others)              # [8, C]
        mu = pooled.mean(axis=0)                     # [C]
        var_c = ((pooled - mu) ** 2).mean(axis=0)    # population variance, [C]
        out[axis] = var_c.mean()                     # 1/D sum over channels
    return out


def _normalise(v):
    """v / sum(v); R3/R2: a zone with zero total variance gives all zeros."""
    s = v.sum()
    return v / s if s > 0 else np.zeros_like(v)


def zone_indicator(V, T, H, W, audio=None, eps=EPS):
    """Method §1 + §2 (density): per-zone indicator g_d(m) and density rho(m).

    V      : [N, heads, d] value features (all heads*d channels form D, R2)
    audio  : [N] cached audio-to-video cross-attention output norms, or None (R16)
    Returns a dict of float64 arrays:
      sigma2_v [Z,3], r_v [Z,3], abar [Z], vhat_a [Z,3], g [Z,3], info [Z], rho [Z]
    Readings:
      R2  r_{v,d} = 0 on all axes when the zone's video variance is zero
      R3  vhat_{a,d}: the audio norms pooled exactly like V (one channel), its
          directional variances normalised to sum 1 (0 when they are all 0)
      R4  abar(m) = mean of a over the zone / max of a over the whole grid
      R6  rho(m) = (info(m)/max_m' info(m') + abar(m)) / 2 with
          info(m) = sum_d sigma^2_{v,d}(m); a zero max gives a zero first term
    """
    ZT, ZY, ZX = zone_grid(T, H, W)
    N = T * H * W
    V = np.asarray(V).reshape(N, -1)      # each zone is converted to float64 on its own
    Z = ZT * ZY * ZX
    sigma2_v = np.zeros((Z, 3))
    sigma2_a = np.zeros((Z, 3))
    amean = np.zeros(Z)
    a = None if audio is None else np.asarray(audio, dtype=np.float64).reshape(N, 1)
    for zt in range(ZT):
        for zy in range(ZY):
            for zx in range(ZX):
                m = (zt * ZY + zy) * ZX + zx
                sigma2_v[m] = directional_variance(_zone_cube(V, T, H, W, zt, zy, zx))
                if a is not None:
                    acube = _zone_cube(a, T, H, W, zt, zy, zx)
                    sigma2_a[m] = directional_variance(acube)
                    amean[m] = acube.mean()
    r_v = np.stack([_normalise(s) for s in sigma2_v])
    amax = 0.0 if a is None else float(a.max())
    if amax > 0:
        abar = amean / amax
        vhat = np.stack([_normalise(s) for s in sigma2_a])
    else:
        abar = np.zeros(Z)
        vhat = np.zeros((Z, 3))
    g = r_v + abar[:, None] * vhat + eps
    info = sigma2_v.sum(axis=1)
    imax = info.max()
    rho = 0.5 * ((info / imax if imax > 0 else np.zeros(Z)) + abar)
    return dict(sigma2_v=sigma2_v, r_v=r_v, abar=abar, vhat_a=vhat, g=g, info=info, rho=rho)


def block_volume(rho, tau128=TAU_128, tau256=TAU_256):
    """Method §2: B(m) from the density rho(m) and the thresholds tau_128, tau_256.

    A dense zone (rho >= tau_128) keeps the finest volume 64; tau_256 <= rho <
    tau_128 gives 128; a sparse zone (rho < tau_256) takes 256.
    """
    rho = np.asarray(rho, dtype=np.float64)
    return np.where(rho >= tau128, 64, np.where(rho >= tau256, 128, 256)).astype(np.int64)


def optimal_log2_edges(g, B):
    """Method §2: l*_d = -1/2 log2 g_d + 1/3 (S + 1/2 sum_d' log2 g_d'), S = log2 B.

    g : [Z, 3] (or [3]); B : [Z] (or scalar).  Returns l* with the same leading shape.
    """
    g = np.asarray(g, dtype=np.float64)
    S = np.log2(np.asarray(B, dtype=np.float64))
    lg = np.log2(g)
    return -0.5 * lg + (1.0 / 3.0) * (S + 0.5 * lg.sum(axis=-1))[..., None]


def quantise_shape(ell, B):
    """Method §2: the candidate of volume B nearest to l* in log2 space (Euclidean).

    R8: squared distances are compared in float64; every candidate within
    TIE_TOL of the minimum counts as tied and the lowest canonical index wins.
    Returns the canonical shape index (into SHAPES).
    """
    ell = np.asarray(ell, dtype=np.float64)
    cands = [i for i, s in enumerate(SHAPES) if s[0] * s[1] * s[2] == int(B)]
    dist = [sum((ell[d] - math.log2(SHAPES[i][d])) ** 2 for d in range(3)) for i in cands]
    best = min(dist)
    for i, dd in zip(cands, dist):
        if dd <= best + TIE_TOL:
            return i
    raise AssertionError("unreachable")


def assign_blocks(g, rho, T, H, W, tau128=TAU_128, tau256=TAU_256, fixed_shape=None):
    """Method §2 end to end, plus the block table of the zone-local layout (R9).

    Returns (shape_id [Z] int, zone_blk_base [Z+1] int, blocks) where blocks is
    an int64 array [nblk, 4] of (start, size, zone, shape_id): block b of zone m
    starts at permuted position 512*m + b*B(m) and holds B(m) tokens.

    fixed_shape: the repository README's mode with the dynamic block-shape
    assignment switched off (``enable_ivpq_dynamic_block`` false, R19): every
    zone takes the one canonical shape given (the README's 4x4x4 chunk is
    index 3) and g, rho are not read.
    """
    ZT, ZY, ZX = zone_grid(T, H, W)
    Z = ZT * ZY * ZX
    if fixed_shape is not None:
        bT, bH, bW = SHAPES[int(fixed_shape)]
        Bv = np.full(Z, bT * bH * bW, dtype=np.int64)
        shape_id = np.full(Z, int(fixed_shape), dtype=np.int64)
    else:
        g = np.asarray(g, dtype=np.float64).reshape(Z, 3)
        Bv = block_volume(np.asarray(rho, dtype=np.float64).reshape(Z), tau128, tau256)
        ell = optimal_log2_edges(g, Bv)
        shape_id = np.array([quantise_shape(ell[m], Bv[m]) for m in range(Z)], dtype=np.int64)
    per_zone = ZONE_TOKENS // Bv
    base = np.zeros(Z + 1, dtype=np.int64)
    base[1:] = np.cumsum(per_zone)
    blocks = []
    for m in range(Z):
        for b in range(per_zone[m]):
            blocks.append((ZONE_TOKENS * m + b * Bv[m], Bv[m], m, shape_id[m]))
    return shape_id, base, np.array(blocks, dtype=np.int64).reshape(-1, 4)


def permutation(T, H, W, shape_id):
    """R9: permuted position p -> natural token n.

    Zones in raster order; zone m owns positions [512m, 512m+512).  Inside a
    zone the blocks of shape (bT,bH,bW) follow raster order over the
    (8/bT, 8/bH, 8/bW) block grid, and inside a block the tokens follow raster
    order (t, y, x).
    """
    ZT, ZY, ZX = zone_grid(T, H, W)
    perm = np.empty(T * H * W, dtype=np.int64)
    p = 0
    for zt in range(ZT):
        for zy in range(ZY):
            for zx in range(ZX):
                m = (zt * ZY + zy) * ZX + zx
                bT, bH, bW = SHAPES[int(shape_id[m])]
                for it in range(ZONE // bT):
                    for iy in range(ZONE // bH):
                        for ix in range(ZONE // bW):
                            for lt in range(bT):
                                for ly in range(bH):
                                    for lx in range(bW):
                                        t = zt * ZONE + it * bT + lt
                                        y = zy * ZONE + iy * bH + ly
                                        x = zx * ZONE + ix * bW + lx
                                        perm[p] = (t * H + y) * W + x
                                        p += 1
    return perm


def permute(x, perm):
    """[N, heads, d] natural -> [heads, N, d] permuted (x_perm[h, p] = x[perm[p], h])."""
    x = np.asarray(x)
    return np.ascontiguousarray(x[perm].transpose(1, 0, 2))


def unpermute(x_perm, perm):
    """Inverse of permute: [heads, N, d] permuted -> [N, heads, d] natural."""
    x_perm = np.asarray(x_perm)
    out = np.empty((x_perm.shape[1], x_perm.shape[0], x_perm.shape[2]), dtype=x_perm.dtype)
    out[perm] = x_perm.transpose(1, 0, 2)
    return out


def pool_blocks_natural(x, perm, blocks, heads=None):
    """pool_blocks(permute(x, perm), blocks) without building the permuted copy:
    each block's rows are gathered from the natural layout [N, heads, d].
    Returns [len(heads), nblk, d] float64."""
    x = np.asarray(x)
    hs = list(range(x.shape[1])) if heads is None else list(heads)
    out = np.empty((len(hs), len(blocks), x.shape[2]))
    for j, (start, size, _, _) in enumerate(blocks):
        rows = np.asarray(x[perm[start:start + size]][:, hs, :], dtype=np.float64)
        out[:, j, :] = rows.mean(axis=0)
    return out


def pool_blocks(x_perm, blocks):
    """Method §3: block representatives, the mean of each block's rows, per head (R10).

    x_perm [heads, N, d] -> [heads, nblk, d] float64.
    """
    x_perm = np.asarray(x_perm, dtype=np.float64)
    out = np.empty((x_perm.shape[0], len(blocks), x_perm.shape[2]))
    for j, (start, size, _, _) in enumerate(blocks):
        out[:, j, :] = x_perm[:, start:start + size, :].mean(axis=1)
    return out


def block_scores(qbar, kbar, scale):
    """Method §3 (R10, R11): s_ij = scale * Qbar_i . Kbar_j for one head."""
    return scale * (np.asarray(qbar, dtype=np.float64) @ np.asarray(kbar, dtype=np.float64).T)


def block_probabilities(s_row):
    """Method §3: P_i = softmax over all key blocks j of the same head."""
    s_row = np.asarray(s_row, dtype=np.float64)
    e = np.exp(s_row - s_row.max())
    return e / e.sum()


def select_row(P_row, top_k, top_p):
    """Method §3: S_i = Top-k(P_i, k) U Top-p(P_i, p) for one query block.

    R13: key blocks are ranked by (P descending, index ascending).  Top-p is the
    shortest prefix of that ranking whose mass, summed in ranking order,
    reaches p (the whole row if it never does); top-k is the first min(k, nblk)
    entries.  Both are prefixes of one ranking, so the union is the longer one.
    Returns the selected indices in ascending order.
    """
    P_row = np.asarray(P_row, dtype=np.float64)
    n = len(P_row)
    order = sorted(range(n), key=lambda j: (-P_row[j], j))
    n_p = n
    acc = 0.0
    # With p >= 1 only the whole row reaches p in exact arithmetic (every
    # softmax probability is positive); a float64 running sum can round up to
    # 1 a few blocks early, so that case is taken as the whole row directly.
    for pos, j in enumerate(order if top_p < 1.0 else ()):
        acc += P_row[j]
        if acc >= top_p:
            n_p = pos + 1
            break
    count = max(min(top_k, n), n_p)
    return np.sort(np.array(order[:count], dtype=np.int64))


def top_k_from_sparsity(sparsity, nblk):
    """The repository README's ratio form of k (``bsa_sparsity``, R15).

    A sparsity s means each query block skips the share s of the key blocks
    (0.75 keeps a quarter), so k = ceil((1 - s) * nblk), at least 1.  s is
    taken at float32 (the width the library's parameter has) and the product
    is formed in float64.
    """
    s = float(np.float32(sparsity))
    return max(1, int(math.ceil((1.0 - s) * nblk)))


def block_select(qbar, kbar, top_k, top_p, scale, sparsity=None):
    """Method §3 for all heads.  qbar, kbar: [heads, nblk, d].

    Returns (row_ptr [heads, nblk+1], cols) as a CSR per head, cols ascending
    within a row, plus the list of per-head probability matrices.  With a
    sparsity ratio, k comes from top_k_from_sparsity instead of top_k.
    """
    heads, nblk, _ = np.asarray(qbar).shape
    if sparsity:
        top_k = top_k_from_sparsity(sparsity, nblk)
    row_ptr = np.zeros((heads, nblk + 1), dtype=np.int64)
    cols = []
    probs = []
    for h in range(heads):
        s = block_scores(qbar[h], kbar[h], scale)
        P = np.stack([block_probabilities(s[i]) for i in range(nblk)])
        probs.append(P)
        hc = []
        for i in range(nblk):
            sel = select_row(P[i], top_k, top_p)
            hc.append(sel)
            row_ptr[h, i + 1] = row_ptr[h, i] + len(sel)
        cols.append(np.concatenate(hc) if hc else np.zeros(0, dtype=np.int64))
    return row_ptr, cols, probs


def _key_rows(blocks, sel):
    """Permuted token rows covered by the selected key blocks, in block order."""
    return np.concatenate([np.arange(blocks[j][0], blocks[j][0] + blocks[j][1]) for j in sel])


def bsa_forward(q, k, v, blocks, row_ptr, cols, scale, query_blocks=None, heads=None):
    """Method §3: attention of each query block i restricted to the key blocks in S_i.

    q, k, v : [heads, N, d] permuted.  For every query row r of block i,
      O_r = sum_c softmax_c(scale * q_r . k_c) v_c over the tokens c of S_i,
      LSE_r = log sum_c exp(scale * q_r . k_c)   (natural log).
    R14: bidirectional, no mask inside a selected block.
    query_blocks / heads restrict the work to a sample (other rows stay NaN).
    Returns O [heads, N, d] and LSE [heads, N].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Hh, N, d = q.shape
    O = np.full((Hh, N, d), np.nan)
    L = np.full((Hh, N), np.nan)
    for h in (range(Hh) if heads is None else heads):
        for i in (range(len(blocks)) if query_blocks is None else query_blocks):
            start, size = blocks[i][0], blocks[i][1]
            sel = cols[h][row_ptr[h, i]:row_ptr[h, i + 1]]
            rows = _key_rows(blocks, sel)
            logits = scale * (q[h, start:start + size] @ k[h, rows].T)
            mx = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - mx)
            z = e.sum(axis=1, keepdims=True)
            O[h, start:start + size] = (e / z) @ v[h, rows]
            L[h, start:start + size] = (mx + np.log(z))[:, 0]
    return O, L


def bsa_backward(q, k, v, dout, blocks, row_ptr, cols, scale, query_blocks=None, heads=None):
    """Exact gradient of bsa_forward with respect to q, k, v for fixed S_i.

    The selection carries no gradient (it is discrete).  With
    P = softmax(scale q k^T) over the selected keys:
      dV_c += sum_r P_rc dO_r,  dP_rc = dO_r . v_c,  D_r = sum_c P_rc dP_rc,
      dS_rc = P_rc (dP_rc - D_r),  dQ_r = scale sum_c dS_rc k_c,
      dK_c += scale sum_r dS_rc q_r.
    All arrays [heads, N, d] permuted; returns (dq, dk, dv) in float64.
    query_blocks / heads restrict the sum to a sample of query blocks (dK, dV
    then hold only those blocks' contributions).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    Hh = q.shape[0]
    for h in (range(Hh) if heads is None else heads):
        for i in (range(len(blocks)) if query_blocks is None else query_blocks):
            start, size = blocks[i][0], blocks[i][1]
            sel = cols[h][row_ptr[h, i]:row_ptr[h, i + 1]]
            rows = _key_rows(blocks, sel)
            qi = q[h, start:start + size]
            logits = scale * (qi @ k[h, rows].T)
            e = np.exp(logits - logits.max(axis=1, keepdims=True))
            P = e / e.sum(axis=1, keepdims=True)
            dOi = dout[h, start:start + size]
            dv[h, rows] += P.T @ dOi
            dP = dOi @ v[h, rows].T
            D = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[h, start:start + size] += scale * (dS @ k[h, rows])
            dk[h, rows] += scale * (dS.T @ qi)
    return dq, dk, dv


def bsa_query_block_dq(q, k, v, dout, blocks, row_ptr, cols, scale, query_blocks, h=0):
    """dQ of a few query blocks of head h, the gradient of bsa_forward with respect
    to those blocks' query rows (for sampled checks on large grids, without
    whole-grid arrays).  Same algebra as bsa_backward, rows of block i only:
      P = softmax(scale q_i k_S^T), dP = dO_i v_S^T, D_r = sum_c P_rc dP_rc,
      dQ_i = scale (P (dP - D)) k_S   over the tokens of S_i.
    Returns {i: dQ_i [B_i, d] float64}."""
    out = {}
    for i in query_blocks:
        start, size = blocks[i][0], blocks[i][1]
        sel = cols[h][row_ptr[h, i]:row_ptr[h, i + 1]]
        rows = _key_rows(blocks, sel)
        qi = np.asarray(q[h, start:start + size], dtype=np.float64)
        ks = np.asarray(k[h, rows], dtype=np.float64)
        logits = scale * (qi @ ks.T)
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        P = e / e.sum(axis=1, keepdims=True)
        dP = np.asarray(dout[h, start:start + size], dtype=np.float64) @ np.asarray(v[h, rows], dtype=np.float64).T
        D = (P * dP).sum(axis=1, keepdims=True)
        out[i] = scale * ((P * (dP - D)) @ ks)
    return out


def bsa_key_block_dkdv(q, k, v, dout, blocks, row_ptr, cols, scale, key_blocks, h=0):
    """dK and dV of a few key blocks of head h: every query block i whose S_i
    holds key block j adds
      dV_j += P[:, j]^T dO_i,   dK_j += scale dS[:, j]^T q_i,
    with P, dS of query block i formed over all of S_i (the softmax and D_r need
    the whole row).  Returns {j: (dK_j, dV_j)}, each [B_j, d] float64."""
    want = {int(j) for j in key_blocks}
    acc = {j: (np.zeros((blocks[j][1], q.shape[2])), np.zeros((blocks[j][1], q.shape[2]))) for j in want}
    nb = row_ptr.shape[1] - 1
    for i in range(nb):
        sel = [int(j) for j in cols[h][row_ptr[h, i]:row_ptr[h, i + 1]]]
        hit = [j for j in sel if j in want]
        if not hit:
            continue
        start, size = blocks[i][0], blocks[i][1]
        rows = _key_rows(blocks, sel)
        qi = np.asarray(q[h, start:start + size], dtype=np.float64)
        dOi = np.asarray(dout[h, start:start + size], dtype=np.float64)
        logits = scale * (qi @ np.asarray(k[h, rows], dtype=np.float64).T)
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        P = e / e.sum(axis=1, keepdims=True)
        dP = dOi @ np.asarray(v[h, rows], dtype=np.float64).T
        D = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        col0 = 0
        for j in sel:
            bj = blocks[j][1]
            if j in want:
                dk, dv = acc[j]
                dv += P[:, col0:col0 + bj].T @ dOi
                dk += scale * (dS[:, col0:col0 + bj].T @ qi)
            col0 += bj
    return acc


def pipeline(Q, K, V, T, H, W, audio, top_k, top_p, scale=None, eps=EPS,
             tau128=TAU_128, tau256=TAU_256, fixed_shape=None, sparsity=None):
    """The whole forward path on natural-layout inputs, in the Method's order.

    Returns a dict with every intermediate: indicator dict, shape_id,
    zone_blk_base, blocks, perm, permuted q/k/v, pooled q/k, CSR, O (permuted
    and natural) and LSE.  fixed_shape and sparsity select the README's
    variants (see assign_blocks and top_k_from_sparsity).
    """
    d = np.asarray(Q).shape[2]
    scale = 1.0 / math.sqrt(d) if not scale else scale
    ind = zone_indicator(V, T, H, W, audio, eps)
    shape_id, base, blocks = assign_blocks(ind["g"], ind["rho"], T, H, W, tau128, tau256, fixed_shape)
    perm = permutation(T, H, W, shape_id)
    qp, kp, vp = permute(Q, perm), permute(K, perm), permute(V, perm)
    qbar, kbar = pool_blocks(qp, blocks), pool_blocks(kp, blocks)
    row_ptr, cols, _ = block_select(qbar, kbar, top_k, top_p, scale, sparsity)
    O, L = bsa_forward(qp, kp, vp, blocks, row_ptr, cols, scale)
    return dict(ind=ind, shape_id=shape_id, zone_blk_base=base, blocks=blocks, perm=perm,
                qp=qp, kp=kp, vp=vp, qbar=qbar, kbar=kbar, row_ptr=row_ptr, cols=cols,
                O_perm=O, O=unpermute(O, perm), lse=L, scale=scale)
