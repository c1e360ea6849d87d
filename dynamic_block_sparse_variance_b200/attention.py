"""PrismSparseAttention: the whole forward/backward path through the C ABI.

PyTorch only allocates device memory and supplies the stream; each step is
one call into libprism_b200.so:

  forward : zone_indicator(V) -> assign_blocks -> permute(Q, K, V) (+ block
            pooling of Q, K) -> block_select -> bsa_fwd -> unpermute(O)
  backward: permute(dO) -> bsa_bwd -> unpermute(dQ, dK, dV)
"""

from __future__ import annotations

import torch

from . import prism as P


class PrismSparseAttention:
    """Dynamic block-sparse self-attention over a T x H x W token grid.

    Inputs are natural-layout [N, heads, head_dim] tensors (bf16, or f32 which
    the permutation rounds to bf16), N = T*H*W in raster order (t, y, x).
    ``col_capacity`` bounds the number of selected (query block, key block)
    pairs over all heads; the default allows every pair on small grids and a
    quarter of them on large ones.  With ``training`` the forward also keeps
    the bf16 rounding residual of O for the backward's row sums.
    ``select_ws_bytes`` bounds the block-score workspace (heads are processed
    in passes that fit).  The Prism README's variants: ``fixed_shape`` (0 =
    dynamic shapes; ``P.PRISM_FIXED_444`` = every zone in 4x4x4 blocks, and the
    indicator is skipped) and ``sparsity`` (k from the ratio instead of top_k).
    """

    def __init__(self, T, H, W, heads, head_dim, top_k, top_p, *, tau128=0.5, tau256=0.25, eps=1e-4,
                 scale=0.0, col_capacity=None, select_ws_bytes=4 << 30, training=True, device="cuda",
                 fixed_shape=P.PRISM_DYNAMIC_SHAPES, sparsity=0.0):
        self.p = P.make_params(T, H, W, heads, head_dim, top_k, top_p, tau128, tau256, eps, scale,
                               fixed_shape, sparsity)
        self.fixed_shape = fixed_shape
        self.T, self.H, self.W, self.heads, self.D = T, H, W, heads, head_dim
        self.N = T * H * W
        self.Z = self.N // 512
        self.cap = 8 * self.Z
        dev = torch.device(device)
        self.device = dev
        i32, f32, bf16 = torch.int32, torch.float32, torch.bfloat16
        Z, cap, N, D = self.Z, self.cap, self.N, head_dim
        self.g = torch.empty(Z, 3, dtype=f32, device=dev)
        self.rho = torch.empty(Z, dtype=f32, device=dev)
        self.debug = torch.empty(Z, 8, dtype=f32, device=dev)
        self.shape_id = torch.empty(Z, dtype=torch.uint8, device=dev)
        self.zone_blk_base = torch.empty(Z + 1, dtype=i32, device=dev)
        self.blocks = torch.empty(cap, 4, dtype=i32, device=dev)
        self.nblk = torch.empty(1, dtype=i32, device=dev)
        self.qp = torch.empty(heads, N, D, dtype=bf16, device=dev)
        self.kp = torch.empty_like(self.qp)
        self.vp = torch.empty_like(self.qp)
        self.op = torch.empty_like(self.qp)
        self.op_res = torch.empty_like(self.qp) if training else None
        self.qbar = torch.empty(heads, cap, D, dtype=f32, device=dev)
        self.kbar = torch.empty_like(self.qbar)
        self.lse = torch.empty(heads, N, dtype=f32, device=dev)
        self.row_ptr = torch.empty(heads * cap + 1, dtype=i32, device=dev)
        if col_capacity is None:
            pairs = heads * cap * cap
            col_capacity = min(pairs, max(1 << 24, pairs // 4), 2**31 - 1)
        self.col = torch.empty(int(col_capacity), dtype=i32, device=dev)
        self.nnz = torch.empty(1, dtype=torch.int64, device=dev)
        ind, _ = P.prism_workspace_size(self.p, P.PRISM_WS_INDICATOR)
        self.ws_ind = torch.empty(max(ind, 256), dtype=torch.uint8, device=dev)
        sel_min, sel_all = P.prism_workspace_size(self.p, P.PRISM_WS_SELECT)
        self.ws_sel = torch.empty(max(sel_min, min(sel_all, select_ws_bytes)), dtype=torch.uint8, device=dev)
        fwd_ws, _ = P.prism_workspace_size(self.p, P.PRISM_WS_FWD)
        self.ws_fwd = torch.empty(max(fwd_ws, 256), dtype=torch.uint8, device=dev)
        self._bwd = None

    # -- forward ------------------------------------------------------------
    def indicator(self, v, audio=None):
        P.prism_zone_indicator(self.p, v, audio, self.g, self.rho, self.debug, self.ws_ind)

    def assign(self):
        P.prism_assign_blocks(self.p, self.g, self.rho, self.shape_id, self.zone_blk_base, self.blocks, self.nblk)

    def permute(self, q, k, v):
        P.prism_permute(self.p, self.shape_id, self.zone_blk_base, q, self.qp, self.qbar)
        P.prism_permute(self.p, self.shape_id, self.zone_blk_base, k, self.kp, self.kbar)
        P.prism_permute(self.p, self.shape_id, self.zone_blk_base, v, self.vp, None)

    def select(self):
        P.prism_block_select(self.p, self.nblk, self.qbar, self.kbar, self.row_ptr, self.col, self.nnz,
                             self.ws_sel)

    def attend(self):
        P.prism_bsa_fwd(self.p, self.blocks, self.zone_blk_base, self.nblk, self.qp, self.kp, self.vp,
                        self.row_ptr, self.col, self.op, self.lse, o_res=self.op_res, workspace=self.ws_fwd)

    def forward(self, q, k, v, audio=None, out=None):
        """Natural-layout output O [N, heads, head_dim] bf16."""
        if self.fixed_shape == P.PRISM_DYNAMIC_SHAPES:
            self.indicator(v, audio)
        self.assign()
        self.permute(q, k, v)
        self.select()
        self.attend()
        if out is None:
            out = torch.empty(self.N, self.heads, self.D, dtype=torch.bfloat16, device=self.device)
        P.prism_unpermute(self.p, self.shape_id, self.op, out)
        return out

    def forward_reuse(self, q, k, v, out=None):
        """Inference across diffusion steps: attention over new Q, K, V with the
        block layout and the selection of the last forward() (no indicator,
        assignment, pooling or selection).  Natural-layout output."""
        P.prism_permute(self.p, self.shape_id, self.zone_blk_base, q, self.qp, None)
        P.prism_permute(self.p, self.shape_id, self.zone_blk_base, k, self.kp, None)
        P.prism_permute(self.p, self.shape_id, self.zone_blk_base, v, self.vp, None)
        P.prism_bsa_fwd(self.p, self.blocks, self.zone_blk_base, self.nblk, self.qp, self.kp, self.vp,
                        self.row_ptr, self.col, self.op, self.lse, o_res=None, workspace=self.ws_fwd)
        if out is None:
            out = torch.empty(self.N, self.heads, self.D, dtype=torch.bfloat16, device=self.device)
        P.prism_unpermute(self.p, self.shape_id, self.op, out)
        return out

    # -- backward -----------------------------------------------------------
    def _bwd_buffers(self):
        if self._bwd is None:
            ws, _ = P.prism_workspace_size(self.p, P.PRISM_WS_BWD, self.col.numel())
            self._bwd = dict(
                dop=torch.empty_like(self.qp), dqp=torch.empty_like(self.qp), dkp=torch.empty_like(self.qp),
                dvp=torch.empty_like(self.qp), ws=torch.empty(ws, dtype=torch.uint8, device=self.device))
        return self._bwd

    def attend_backward(self):
        b = self._bwd_buffers()
        P.prism_bsa_bwd(self.p, self.blocks, self.zone_blk_base, self.nblk, self.qp, self.kp, self.vp, self.op,
                        self.op_res, b["dop"], self.lse, self.row_ptr, self.col, self.nnz, b["dqp"], b["dkp"], b["dvp"],
                        b["ws"])

    def backward(self, dout, dq=None, dk=None, dv=None):
        """Gradients (dQ, dK, dV) in natural layout for the last forward's selection."""
        b = self._bwd_buffers()
        P.prism_permute(self.p, self.shape_id, self.zone_blk_base, dout, b["dop"], None)
        self.attend_backward()
        outs = []
        for src, dst in ((b["dqp"], dq), (b["dkp"], dk), (b["dvp"], dv)):
            if dst is None:
                dst = torch.empty(self.N, self.heads, self.D, dtype=torch.bfloat16, device=self.device)
            P.prism_unpermute(self.p, self.shape_id, src, dst)
            outs.append(dst)
        return tuple(outs)

    # -- host views (for tests and reports) ---------------------------------
    def host_layout(self):
        nb = int(self.nblk.item())
        return dict(nblk=nb, shape_id=self.shape_id.cpu().numpy(), zone_blk_base=self.zone_blk_base.cpu().numpy(),
                    blocks=self.blocks[:nb].cpu().numpy())

    def host_csr(self):
        """Per-head CSR (row_ptr [heads, nblk+1] relative to each head, cols list)."""
        nb = int(self.nblk.item())
        rp = self.row_ptr.cpu().numpy().astype("int64")
        col = self.col.cpu().numpy()
        out_rp, out_cols = [], []
        for h in range(self.heads):
            r = rp[h * self.cap: h * self.cap + nb + 1]
            out_rp.append(r - r[0])
            out_cols.append(col[r[0]:r[-1]].astype("int64"))
        import numpy as np
        return np.stack(out_rp), out_cols


class HostStepper:
    """Forward + backward steps on inputs that live in pinned host memory.

    The same C-ABI calls as PrismSparseAttention.forward/backward run on the
    current stream; the host<->device copies run on two copy streams, ordered
    by CUDA events so that each one overlaps kernels instead of bracketing the
    step: step i+1's Q, K, V and audio upload as soon as step i has read them
    (after its permutation), its dO as soon as step i's backward has permuted
    dO, O downloads while the backward runs, and dQ, dK, dV download while the
    next step's forward runs.  One device copy of each input and output is
    enough; nothing waits on the host.

    run(host_inputs, host_outputs): lists (one entry per step) of dicts of
    pinned host tensors, inputs {q, k, v, audio (or None), dout} and outputs
    {o, dq, dk, dv}; returns after enqueueing everything (synchronize the
    current stream, then the copy streams' work is complete too).
    ``device_buffers`` (optional): the device tensors to stage through, a dict
    with the same keys (natural layout, the host tensors' shapes and dtypes);
    by default the stepper allocates its own on the first run.
    """

    def __init__(self, att: PrismSparseAttention, device_buffers=None):
        self.att = att
        self.dev = att.device
        self.up = torch.cuda.Stream(self.dev)
        self.down = torch.cuda.Stream(self.dev)
        self.buf = dict(device_buffers) if device_buffers is not None else None

    def _buffers(self, first):
        if self.buf is None:
            shp = (self.att.N, self.att.heads, self.att.D)
            b = {n: torch.empty(first[n].shape, dtype=first[n].dtype, device=self.dev)
                 for n in ("q", "k", "v", "dout")}
            b["audio"] = None if first.get("audio") is None else torch.empty(first["audio"].shape,
                                                                          dtype=first["audio"].dtype,
                                                                          device=self.dev)
            for n in ("o", "dq", "dk", "dv"):
                b[n] = torch.empty(shp, dtype=torch.bfloat16, device=self.dev)
            self.buf = b
        return self.buf

    def _upload(self, host, names, after):
        with torch.cuda.stream(self.up):
            if after is not None:
                self.up.wait_event(after)
            for n in names:
                if host.get(n) is not None:
                    self.buf[n].copy_(host[n], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(self.up)
        return ev

    def _download(self, names, host, after):
        with torch.cuda.stream(self.down):
            self.down.wait_event(after)
            for n in names:
                host[n].copy_(self.buf[n], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(self.down)
        return ev

    def run(self, host_inputs, host_outputs):
        att = self.att
        comp = torch.cuda.current_stream(self.dev)
        b = self._buffers(host_inputs[0])
        # the first uploads overwrite the device inputs: after everything already
        # queued on the caller's stream (an earlier run may still be reading them)
        start = torch.cuda.Event()
        start.record(comp)
        ready_in = self._upload(host_inputs[0], ("q", "k", "v", "audio"), start)
        ready_do = self._upload(host_inputs[0], ("dout",), start)
        o_free = grads_free = None
        for i, (hin, hout) in enumerate(zip(host_inputs, host_outputs)):
            nxt = host_inputs[i + 1] if i + 1 < len(host_inputs) else None
            # forward: read the uploaded inputs, then release them for step i+1
            comp.wait_event(ready_in)
            if att.fixed_shape == P.PRISM_DYNAMIC_SHAPES:
                att.indicator(b["v"], b["audio"])
            att.assign()
            att.permute(b["q"], b["k"], b["v"])
            in_free = torch.cuda.Event()
            in_free.record(comp)
            if nxt is not None:
                ready_in = self._upload(nxt, ("q", "k", "v", "audio"), in_free)
            att.select()
            att.attend()
            if o_free is not None:
                comp.wait_event(o_free)
            P.prism_unpermute(att.p, att.shape_id, att.op, b["o"])
            o_ready = torch.cuda.Event()
            o_ready.record(comp)
            o_free = self._download(("o",), hout, o_ready)
            # backward
            bw = att._bwd_buffers()
            comp.wait_event(ready_do)
            P.prism_permute(att.p, att.shape_id, att.zone_blk_base, b["dout"], bw["dop"], None)
            do_free = torch.cuda.Event()
            do_free.record(comp)
            if nxt is not None:
                ready_do = self._upload(nxt, ("dout",), do_free)
            att.attend_backward()
            if grads_free is not None:
                comp.wait_event(grads_free)
            for src, n in ((bw["dqp"], "dq"), (bw["dkp"], "dk"), (bw["dvp"], "dv")):
                P.prism_unpermute(att.p, att.shape_id, src, b[n])
            g_ready = torch.cuda.Event()
            g_ready.record(comp)
            grads_free = self._download(("dq", "dk", "dv"), hout, g_ready)
        # the caller's stream covers the last downloads
        comp.wait_event(o_free)
        comp.wait_event(grads_free)
