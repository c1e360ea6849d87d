"""Shared test utilities: comparisons, CSR conversion, near-tie analysis."""

import math
import os

import numpy as np
import torch

# Attention tolerance (bf16 storage, fp32 accumulation) against fp64:
# relative RMS error <= 1e-2 and max absolute error <= 3e-2.  A result stored
# in bf16 cannot be nearer to the exact value than half a bf16 ulp of it
# (0.03125 already for |x| in [8, 16)), so the max-abs bound applies to the
# error beyond that half ulp, i.e. to the error before the final rounding.
REL_RMS_TOL = 1e-2
MAX_ABS_TOL = 3e-2


def bf16_half_ulp(x):
    """Half the bf16 spacing at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 0.5 * 2.0 ** (e - 7)


def f64(t):
    """Exact float64 copy of a (CPU or GPU) tensor."""
    return t.detach().to("cpu", torch.float64).numpy()


def rel_rms(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.sqrt(np.mean((a - b) ** 2)) / max(np.sqrt(np.mean(b ** 2)), 1e-30))


# Below this magnitude half a bf16 ulp is at most 2^-8, and the max-abs bound
# is also applied to the raw error.
RAW_MAX_ABS_BELOW = 2.0


def _max_err_below(err, ref, bound):
    small = np.abs(ref) < bound
    return float(np.max(err[small])) if small.any() else 0.0


def assert_close_attn(got, ref, what):
    """rel-RMS <= 1e-2; max-abs <= 3e-2 beyond half a bf16 ulp of the exact
    value, and raw max-abs <= 3e-2 over the entries with |ref| < 2.  With
    PRISM_PARITY_LOG set, one line per comparison is appended to that file
    (with the raw max-abs below 2 and below 4)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rr = rel_rms(got, ref)
    err = np.abs(got - ref)
    ma = float(np.max(err))
    beyond = float(np.max(err - bf16_half_ulp(ref)))
    raw2 = _max_err_below(err, ref, RAW_MAX_ABS_BELOW)
    log = os.environ.get("PRISM_PARITY_LOG")
    if log:
        with open(log, "a") as fh:
            fh.write(f"{what}\trel_rms={rr:.3e}\tmax_abs={ma:.3e}\tbeyond_half_ulp={beyond:.3e}\t"
                     f"max_abs(|ref|<2)={raw2:.3e}\tmax_abs(|ref|<4)={_max_err_below(err, ref, 4.0):.3e}\t"
                     f"max|ref|={float(np.max(np.abs(ref))):.3e}\n")
    assert rr <= REL_RMS_TOL and beyond <= MAX_ABS_TOL and raw2 <= MAX_ABS_TOL, \
        f"{what}: rel_rms={rr:.3e} max_abs={ma:.3e} beyond half-ulp={beyond:.3e} max_abs(|ref|<2)={raw2:.3e}"
    return rr, ma


def csr_to_device(row_ptr_h, cols_h, cap, device):
    """Per-head CSR (oracle form) -> the library's global row_ptr [heads*cap+1] and col."""
    heads, nb1 = row_ptr_h.shape
    nb = nb1 - 1
    rp = np.zeros(heads * cap + 1, dtype=np.int64)
    cols = []
    off = 0
    for h in range(heads):
        r = row_ptr_h[h]
        rp[h * cap: h * cap + nb + 1] = off + r
        rp[h * cap + nb + 1: (h + 1) * cap + 1] = off + r[-1]
        off += int(r[-1])
        cols.append(np.asarray(cols_h[h], dtype=np.int64))
    col = np.concatenate(cols) if cols else np.zeros(0, dtype=np.int64)
    return (torch.from_numpy(rp.astype(np.int32)).to(device),
            torch.from_numpy(col.astype(np.int32)).to(device),
            torch.tensor([off], dtype=torch.int64, device=device))


def blocks_to_device(blocks, cap, device):
    b = np.zeros((cap, 4), dtype=np.int32)
    b[:len(blocks)] = blocks
    return torch.from_numpy(b).to(device)


def selection_row_ok(P_row, gpu_sel, ora_sel, top_k, top_p, score_tol=1e-4, mass_tol=1e-5):
    """Exact match, or a valid alternative when the oracle's row is near a tie.

    Returns (exact, valid).  A row is near a tie if two blocks straddling the
    cut have probabilities within a relative score_tol, or the cumulative mass
    at the cut is within mass_tol of p.  A valid alternative keeps every block
    clearly above the cut, no block clearly below it, at least min(k, nblk)
    blocks, and mass >= p - mass_tol.
    """
    gpu_sel = np.asarray(gpu_sel)
    ora_sel = np.asarray(ora_sel)
    if len(gpu_sel) == len(ora_sel) and np.array_equal(gpu_sel, ora_sel):
        return True, True
    n = len(P_row)
    logp = np.log(np.maximum(P_row, 1e-300))
    cut = len(ora_sel)
    order = sorted(range(n), key=lambda j: (-P_row[j], j))
    lo = logp[order[cut - 1]]
    hi_thr = lo + score_tol * max(1.0, abs(lo))
    lo_thr = lo - score_tol * max(1.0, abs(lo))
    must = {j for j in range(n) if logp[j] > hi_thr}
    never = {j for j in range(n) if logp[j] < lo_thr and j not in must}
    gs = set(gpu_sel.tolist())
    cum = P_row[gpu_sel].sum() if len(gpu_sel) else 0.0
    valid = (must <= gs and not (gs & never) and len(gs) >= min(top_k, n)
             and cum >= top_p - mass_tol and list(gpu_sel) == sorted(gs))
    # also allow a boundary move of the top-p prefix by one element when the
    # cumulative mass at the cut is within mass_tol of p
    if not valid:
        csum = np.cumsum(P_row[order])
        near = abs(csum[cut - 1] - top_p) < mass_tol or (cut >= 2 and abs(csum[cut - 2] - top_p) < mass_tol)
        if near and abs(len(gs) - cut) <= 1:
            pref = set(order[:len(gs)])
            valid = gs == pref
    return False, valid


def check_whole_path(wl, inp, att_kw=None, ora_kw=None, audio=None, zero_grads=()):
    """Run the whole GPU path (forward + backward) on the CPU inputs `inp` and
    compare it with the oracle run in the same mode: block layout bit for bit,
    every selection row exact or a valid near-tie alternative (>= 99% exact),
    O and dQ, dK, dV within the attention tolerance.  Gradients named in
    `zero_grads` are exactly zero (the oracle's reference must be zero to
    rounding); a relative error has no meaning there, so they are held to the
    max-abs bound alone.  Returns (att, ora, out)."""
    from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
    from dynamic_block_sparse_variance_b200 import prism as P
    from oracle import prism_oracle as po
    att_kw, ora_kw = dict(att_kw or {}), dict(ora_kw or {})
    a = inp["audio"] if audio is None else audio
    a64 = None if a is None else a.numpy().astype(np.float64)
    ora = po.pipeline(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), wl.T, wl.H, wl.W, a64, wl.top_k, wl.top_p,
                      **ora_kw)
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p, **att_kw)
    cu = lambda t: None if t is None else t.cuda()
    out = att.forward(cu(inp["q"]), cu(inp["k"]), cu(inp["v"]), cu(a))
    P.prism_device_status()
    lay = att.host_layout()
    np.testing.assert_array_equal(lay["shape_id"], ora["shape_id"])
    np.testing.assert_array_equal(lay["blocks"], ora["blocks"])
    nb = len(ora["blocks"])
    k_eff = po.top_k_from_sparsity(ora_kw["sparsity"], nb) if ora_kw.get("sparsity") else wl.top_k
    rp_g, cols_g = att.host_csr()
    scale = ora["scale"]
    exact = total = 0
    for h in range(wl.heads):
        s = po.block_scores(ora["qbar"][h], ora["kbar"][h], scale)
        for i in range(nb):
            g = cols_g[h][rp_g[h, i]:rp_g[h, i + 1]]
            o = ora["cols"][h][ora["row_ptr"][h, i]:ora["row_ptr"][h, i + 1]]
            ex, ok = selection_row_ok(po.block_probabilities(s[i]), g, o, k_eff, wl.top_p)
            assert ok, (h, i, g, o)
            assert len(g) >= min(k_eff, nb)
            exact += ex
            total += 1
    assert exact >= 0.99 * total, f"{exact}/{total} rows bit-exact"
    bf = lambda t: f64(t.to(torch.bfloat16))
    pm = {n: po.permute(bf(inp[n]), ora["perm"]) for n in ("q", "k", "v", "dout")}
    O, _ = po.bsa_forward(pm["q"], pm["k"], pm["v"], ora["blocks"], rp_g, cols_g, scale)
    assert_close_attn(f64(out), po.unpermute(O, ora["perm"]), "O")
    dq, dk, dv = att.backward(cu(inp["dout"]))
    P.prism_device_status()
    gq, gk, gv = po.bsa_backward(pm["q"], pm["k"], pm["v"], pm["dout"], ora["blocks"], rp_g, cols_g, scale)
    for got, ref, w in ((dq, gq, "dQ"), (dk, gk, "dK"), (dv, gv, "dV")):
        if w in zero_grads:
            assert np.abs(ref).max() < 1e-12, f"{w}: the reference is not zero"
            assert np.abs(f64(got)).max() <= MAX_ABS_TOL, f"{w}: max-abs {np.abs(f64(got)).max():.3e}"
        else:
            assert_close_attn(f64(got), po.unpermute(ref, ora["perm"]), w)
    return att, ora, out


def assert_dq_consistent(got, ref, what="dQ", rel=1e-3, frac=1e-2):
    """Two dQ results that may differ in the order of their fp32 additions
    (the tensor-core backward sums dQ partials by atomic reductions): rel-RMS
    of the difference <= rel and no entry further than frac of the largest
    |ref| (each result is also held to the oracle tolerance by the parity
    tests)."""
    g = got.double().cpu()
    r = ref.double().cpu()
    d = (g - r)
    rr = float(d.norm() / r.norm().clamp_min(1e-30))
    ma = float(d.abs().max())
    scale = float(r.abs().max())
    assert rr <= rel and ma <= frac * scale, f"{what}: rel_rms diff {rr:.3e}, max |diff| {ma:.3e} (max |ref| {scale:.3e})"
