"""Head-sharded Prism sparse attention over several GPUs.

A sequence-parallel DiT keeps each rank's share of the tokens: here a T-slab
of the grid (T/R frames, whole 8-frame zone layers) for all heads.  The
attention of a head needs all of its tokens, so the layer runs as

  1. zone records of the local slab (indicator, first half)      local kernels
  2. all-gather of the records (9 doubles per zone)               collective
  3. g, rho of the whole grid; block layout of the whole grid and
     of the local slab (identical on every rank)                  local kernels
  4. permutation + block pooling of the local Q, K, V             local kernels
  5. sequence -> heads: every rank gets all tokens of its
     heads / R heads (permuted rows, pooled rows)                 point-to-point
  6. block selection and sparse attention of the head group       local kernels
  7. heads -> sequence of O, inverse permutation                  point-to-point

and the backward permutes dO locally, moves it sequence -> heads, runs the
attention backward of the head group and moves dQ, dK, dV back.  A slab is a
grid of its own and its zones are the whole grid's zones in the same order,
so the permutation of a slab writes exactly the rows of the whole grid's
permuted tensor that belong to it: the exchanges only move contiguous
[tokens, head_dim] runs, with no reordering.

The stages are methods, and the exchanges go through an object with
``all_gather``, ``seq_to_heads`` and ``heads_to_seq`` (``TorchDistExchange``
for torch.distributed), so that the same stages can be driven for every rank
in one process when checking the decomposition against the unsharded layer.

Stage 3 reads the slab boundaries of the block table back to the host (R + 1
integers, one synchronisation per forward) to size the pooled-row exchange.
"""

from __future__ import annotations

import torch

from . import prism as P
from .attention import PrismSparseAttention


class TorchDistExchange:
    """The three exchanges over torch.distributed (NCCL between GPUs, gloo on CPU).

    Every rank calls every method with the same arguments' shapes, in the same
    order.  Transfers are point-to-point of contiguous runs; a rank's share to
    itself is a local copy.
    """

    def __init__(self, rank, world, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.rank, self.world, self.group = rank, world, group

    def all_gather(self, local, out):
        """out [R * n, ...] = the ranks' local [n, ...] in rank order."""
        if self.world == 1:
            out.copy_(local)
        else:
            self.dist.all_gather_into_tensor(out, local, group=self.group)

    def _run(self, ops, local_copies):
        for dst, src in local_copies:
            dst.copy_(src)
        if ops:
            for req in self.dist.batch_isend_irecv(ops):
                req.wait()

    def seq_to_heads(self, x_loc, x_h, rows_of):
        """x_loc [heads, n_loc_rows, d] (this rank's rows of every head) ->
        x_h [heads/R, n_rows, d] (every rank's rows of this rank's heads).
        rows_of(s) = (first row, row count) of rank s in x_h's row space; rank
        s's rows sit at x_loc rows [0, count) on rank s."""
        hpr = x_h.shape[0]
        ops, local = [], []
        for g in range(self.world):          # send my rows of group g's heads
            cnt = rows_of(self.rank)[1]
            for hh in range(hpr):
                src = x_loc[g * hpr + hh, :cnt]
                if g == self.rank:
                    r0 = rows_of(self.rank)[0]
                    local.append((x_h[hh, r0:r0 + cnt], src))
                else:
                    ops.append(self.dist.P2POp(self.dist.isend, src, g, group=self.group))
        for s in range(self.world):          # receive rank s's rows of my heads
            if s == self.rank:
                continue
            r0, cnt = rows_of(s)
            for hh in range(hpr):
                ops.append(self.dist.P2POp(self.dist.irecv, x_h[hh, r0:r0 + cnt], s, group=self.group))
        self._run(ops, local)

    def heads_to_seq(self, x_h, x_loc, rows_of):
        """Inverse of seq_to_heads."""
        hpr = x_h.shape[0]
        ops, local = [], []
        for s in range(self.world):          # send rank s its rows of my heads
            r0, cnt = rows_of(s)
            for hh in range(hpr):
                src = x_h[hh, r0:r0 + cnt]
                if s == self.rank:
                    local.append((x_loc[self.rank * hpr + hh, :cnt], src))
                else:
                    ops.append(self.dist.P2POp(self.dist.isend, src, s, group=self.group))
        for g in range(self.world):          # receive my rows of group g's heads
            if g == self.rank:
                continue
            cnt = rows_of(self.rank)[1]
            for hh in range(hpr):
                ops.append(self.dist.P2POp(self.dist.irecv, x_loc[g * hpr + hh, :cnt], g, group=self.group))
        self._run(ops, local)


class ShardedPrismAttention:
    """One rank's part of a head-sharded Prism attention layer.

    T x H x W is the whole grid; this rank holds frames [rank*T/R, (rank+1)*T/R)
    of Q, K, V (natural layout [N/R, heads, head_dim]) and computes the
    attention of heads [rank*heads/R, (rank+1)*heads/R).  T must be a multiple
    of 8R and heads a multiple of R.  Other keywords as PrismSparseAttention.
    """

    def __init__(self, T, H, W, heads, head_dim, top_k, top_p, *, rank, world, exchange=None, device="cuda",
                 **kw):
        if T % (8 * world) or heads % world:
            raise ValueError("T must be a multiple of 8 * world and heads a multiple of world")
        self.rank, self.world = rank, world
        self.T, self.H, self.W, self.heads, self.D = T, H, W, heads, head_dim
        self.Tl = T // world
        self.Nl = self.Tl * H * W
        self.Zl = self.Nl // 512
        self.hpr = heads // world
        self.dev = torch.device(device)
        self._ex = exchange
        fixed = kw.get("fixed_shape", P.PRISM_DYNAMIC_SHAPES)
        extra = {k: kw[k] for k in ("tau128", "tau256", "eps", "scale") if k in kw}
        self.p_loc = P.make_params(self.Tl, H, W, heads, head_dim, top_k, top_p, fixed_shape=fixed,
                                   sparsity=kw.get("sparsity", 0.0), **extra)
        # the head group's layer over the whole grid: selection, attention and their buffers
        self.inner = PrismSparseAttention(T, H, W, self.hpr, head_dim, top_k, top_p, device=self.dev, **kw)
        f64, i32, f32, bf16 = torch.float64, torch.int32, torch.float32, torch.bfloat16
        Z, Zl, d = self.inner.Z, self.Zl, head_dim
        self.rec_loc = torch.empty(Zl, P.PRISM_ZONE_RECORD, dtype=f64, device=self.dev)
        self.rec_all = torch.empty(Z, P.PRISM_ZONE_RECORD, dtype=f64, device=self.dev)
        ind, _ = P.prism_workspace_size(self.p_loc, P.PRISM_WS_INDICATOR)
        self.ws_ind = torch.empty(max(ind, 256), dtype=torch.uint8, device=self.dev)
        self.shape_loc = torch.empty(Zl, dtype=torch.uint8, device=self.dev)
        self.zbb_loc = torch.empty(Zl + 1, dtype=i32, device=self.dev)
        self.blocks_loc = torch.empty(8 * Zl, 4, dtype=i32, device=self.dev)
        self.nblk_loc = torch.empty(1, dtype=i32, device=self.dev)
        self.qp = torch.empty(heads, self.Nl, d, dtype=bf16, device=self.dev)
        self.kp = torch.empty_like(self.qp)
        self.vp = torch.empty_like(self.qp)
        self.qbar = torch.empty(heads, 8 * Zl, d, dtype=f32, device=self.dev)
        self.kbar = torch.empty_like(self.qbar)
        self.has_audio = False
        self.slab_rows = self.slab_blocks = None

    # -- rows of each rank in the whole grid's permuted row / block spaces
    def _token_rows(self, s):
        return s * self.Nl, self.Nl

    def _block_rows(self, s):
        return self.slab_blocks[s]

    # -- forward stages ------------------------------------------------------
    def stage_records(self, v_loc, audio_loc=None):
        self.has_audio = audio_loc is not None
        P.prism_zone_records(self.p_loc, v_loc, audio_loc, self.rec_loc, self.ws_ind)

    def stage_layout(self):
        """g, rho and the block layout of the whole grid (from rec_all, which
        holds every rank's records), and the local slab's layout."""
        inn = self.inner
        if inn.fixed_shape == P.PRISM_DYNAMIC_SHAPES:
            P.prism_zone_finalize(inn.p, self.rec_all, self.has_audio, inn.g, inn.rho, inn.debug)
        inn.assign()
        m0, m1 = self.rank * self.Zl, (self.rank + 1) * self.Zl
        P.prism_assign_blocks(self.p_loc, inn.g[m0:m1], inn.rho[m0:m1], self.shape_loc, self.zbb_loc,
                              self.blocks_loc, self.nblk_loc)
        bounds = inn.zone_blk_base[::self.Zl].to("cpu", torch.int64).tolist()   # R + 1 slab boundaries
        self.slab_blocks = [(bounds[s], bounds[s + 1] - bounds[s]) for s in range(self.world)]

    def stage_permute(self, q_loc, k_loc, v_loc):
        P.prism_permute(self.p_loc, self.shape_loc, self.zbb_loc, q_loc, self.qp, self.qbar)
        P.prism_permute(self.p_loc, self.shape_loc, self.zbb_loc, k_loc, self.kp, self.kbar)
        P.prism_permute(self.p_loc, self.shape_loc, self.zbb_loc, v_loc, self.vp, None)

    def stage_attend(self):
        self.inner.select()
        self.inner.attend()

    def stage_unpermute(self, x_loc_perm, out):
        P.prism_unpermute(self.p_loc, self.shape_loc, x_loc_perm, out)

    # -- backward stages -----------------------------------------------------
    def stage_permute_dout(self, dout_loc, dop_loc):
        P.prism_permute(self.p_loc, self.shape_loc, self.zbb_loc, dout_loc, dop_loc, None)

    # -- the whole layer through the exchange ----------------------------------
    @property
    def ex(self):
        """The exchange: the one given, else torch.distributed's (which must be initialised
        when there is more than one rank)."""
        if self._ex is None:
            if self.world > 1:
                import torch.distributed as dist
                if not dist.is_initialized():
                    raise RuntimeError("ShardedPrismAttention over several ranks needs torch.distributed "
                                       "initialised (or an explicit exchange)")
            self._ex = TorchDistExchange(self.rank, self.world)
        return self._ex

    def forward(self, q_loc, k_loc, v_loc, audio_loc=None, out=None):
        """Natural-layout O of this rank's tokens, all heads: [N/R, heads, d] bf16."""
        ex, inn = self.ex, self.inner
        if inn.fixed_shape == P.PRISM_DYNAMIC_SHAPES:
            self.stage_records(v_loc, audio_loc)
            ex.all_gather(self.rec_loc, self.rec_all)
        self.stage_layout()
        self.stage_permute(q_loc, k_loc, v_loc)
        for x_loc, x_h in ((self.qp, inn.qp), (self.kp, inn.kp), (self.vp, inn.vp)):
            ex.seq_to_heads(x_loc, x_h, self._token_rows)
        for x_loc, x_h in ((self.qbar, inn.qbar), (self.kbar, inn.kbar)):
            ex.seq_to_heads(x_loc, x_h, self._block_rows)
        self.stage_attend()
        ex.heads_to_seq(inn.op, self.qp, self._token_rows)      # qp is free again: O lands there
        if out is None:
            out = torch.empty(self.Nl, self.heads, self.D, dtype=torch.bfloat16, device=self.dev)
        self.stage_unpermute(self.qp, out)
        return out

    def backward(self, dout_loc, dq=None, dk=None, dv=None):
        """dQ, dK, dV of this rank's tokens, all heads, natural layout."""
        ex, inn = self.ex, self.inner
        bw = inn._bwd_buffers()
        self.stage_permute_dout(dout_loc, self.kp)               # kp is free after the forward's exchange
        ex.seq_to_heads(self.kp, bw["dop"], self._token_rows)
        inn.attend_backward()
        outs = []
        for src, dst in ((bw["dqp"], dq), (bw["dkp"], dk), (bw["dvp"], dv)):
            ex.heads_to_seq(src, self.vp, self._token_rows)
            if dst is None:
                dst = torch.empty(self.Nl, self.heads, self.D, dtype=torch.bfloat16, device=self.dev)
            self.stage_unpermute(self.vp, dst)
            outs.append(dst)
        return tuple(outs)
