#!/usr/bin/env python
"""Benchmark of the whole Prism sparse-attention step (forward + backward).

One step = indicator -> block assignment -> permutation (Q, K, V) -> block
selection -> sparse attention forward -> unpermute(O) -> permute(dO) ->
sparse attention backward -> unpermute(dQ, dK, dV), on one synthetic batch
already resident in HBM.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2k]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Multi-GPU runs (torchrun) are independent replicas, one layer per GPU (weak
scaling); there is no data-path collective.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "block-sparse attn fwd+bwd ms & executed TFLOP/s (% bf16 peak) at 2K-like grid"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = dict(bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, hbm_gbs=6650.0)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="prism", choices=["prism", "reference"])
    ap.add_argument("--workload", default="2k")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-attention comparator")
    ap.add_argument("--no-norms", action="store_true", help="skip the audio-norm producer measurement")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi samples of this GPU's SM clock and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.lines = []
        try:
            pr = torch.cuda.get_device_properties(device)
            self.target = ["-i", "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)]
        except Exception:
            self.target = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.target, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"])
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        if not rows:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["no samples"])
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[4 + k].lower().startswith("active")})
        load = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return dict(sm_mhz=statistics.median(load) if load else None, sm_max_mhz=max(mx) if mx else None,
                    reasons=reasons, samples=len(rows))


# ------------------------------------------------------------- counting --
def executed_pairs(att):
    """sum over heads, query blocks i and selected key blocks j of B_i * B_j
    (in total, and for query blocks of 256 tokens alone)."""
    nb = int(att.nblk.item())
    sizes = att.blocks[:nb, 1].to(torch.int64)
    nnz = int(att.nnz.item())
    total = big = 0
    for h in range(att.heads):
        rp = att.row_ptr[h * att.cap: h * att.cap + nb + 1].to(torch.int64)
        cnt = rp[1:] - rp[:-1]
        cols = att.col[int(rp[0]): int(rp[-1])].to(torch.int64)
        rows = torch.repeat_interleave(torch.arange(nb, device=cols.device), cnt)
        prod = sizes[rows] * sizes[cols]
        total += int(prod.sum().item())
        big += int(prod[sizes[rows] == 256].sum().item())
    return total, nnz, nb, sizes, big


# Algorithmic tensor-core FLOPs of each attention kernel, in units of
# P = sum_h sum_i sum_{j in S_i} B_i B_j d: forward 4P (QK^T, PV); the
# tensor-core backward 10P (S, dP, dV, dK, dQ); in the warp-MMA backward the
# key-side kernel 8P (S, dP, dV, dK) and the query-side one 2P (dQ; its S and
# dP recomputation is extra work and not counted).
KERNEL_FLOP_UNITS = {"bsa_fwd_mma_kernel": 4, "bsa_fwd_tc_kernel": 4, "bsa_fwd_tc2_kernel": 4,
                     "bsa_dkdv_mma_kernel": 8, "bsa_dq_mma_kernel": 2, "bsa_bwd_tc_kernel": 10}
FWD_KERNELS = ("bsa_fwd_mma_kernel", "bsa_fwd_tc_kernel", "bsa_fwd_tc2_kernel")

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# kernel from one ncu capture on a smaller grid, as bytes per algorithmic FLOP.
# The backward's record is the 2K grid with 2 heads (the same selection
# density and per-head working set as the 24-head grid; one launch, counters
# dram__bytes_read.sum + dram__bytes_write.sum).  The full-size figure is
# scaled by the launch's algorithmic FLOPs (the heads are independent
# problems), and reported only while the kernel's sources hash to the value
# they had when the counters were taken.
ATTN_SOURCES = ("attn_common.cuh", "attn_tc_bwd.cuh", "attn_tc_fwd.cuh", "tc_common.cuh", "v16.cuh")
PROFILED_TRAFFIC = {
    "bsa_bwd_tc_kernel": dict(bytes=547118283264 + 287245915648, flops=205282664775680.0,
                              grid="2K-like with 2 heads (64x96x160)",
                              sha256="dab8a993bc9c686b18e82b110934f8c4ffc15e90b3defb0551e1f6dcb315378e"),
}


def profiled_traffic(kernel, flops_per_launch):
    rec = PROFILED_TRAFFIC.get(kernel)
    if rec is None:
        return None, None
    import hashlib
    csrc = os.path.join(ROOT, "dynamic_block_sparse_variance_b200", "csrc")
    hsh = hashlib.sha256()
    for f in ATTN_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            hsh.update(fh.read())
    if hsh.hexdigest() != rec["sha256"]:
        return None, "kernel changed since the ncu capture"
    return rec["bytes"] / rec["flops"] * flops_per_launch, (f"ncu capture on the {rec['grid']} grid, scaled by "
                                                            "algorithmic FLOPs per launch")
BWD_KERNELS = ("bsa_dkdv_mma_kernel", "bsa_dq_mma_kernel", "bsa_bwd_tc_kernel", "dq_convert_kernel")


def hbm_kernel_bytes(wl, nblk, heads_per_pass_launches):
    """Algorithmic bytes per step of the HBM-bound kernels (each tensor read or
    written once; bf16 inputs), for achieved GB/s.  Returns {kernel: bytes}."""
    t = wl.N * wl.heads * wl.head_dim * 2          # one [N, heads, d] bf16 tensor
    scores = wl.heads * float(nblk) ** 2 * 4        # one fp32 score matrix per head
    return {
        "zone_stats_kernel": t,                      # reads V once
        "permute_kernel": 4 * 2 * t,                 # Q, K, V, dO: read natural + write permuted
        "unpermute_kernel": 4 * 2 * t,               # O, dQ, dK, dV
        "bwd_delta_kernel": 3 * t + wl.N * wl.heads * 4,   # dO, O, O residual in; D out
        "bwd_stats_tc_kernel": 3 * t + wl.N * wl.heads * 16,   # dO, O, O residual, LSE in; D, m, inv out
        "v_to_f16_kernel": 2 * t,                    # V in, fp16 copy out
        "head_absmax2_kernel": 2 * t,                # V, dO read once
        "to_f16x2_kernel": 4 * t,                    # V, dO in, fp16 copies out
        "dq_convert_kernel": 3 * t,                  # fp32 dQ accumulator in, bf16 dQ out
        "block_scores_kernel": scores * heads_per_pass_launches,   # score rows written
        "row_cut_kernel": scores,                    # score rows read once
        "emit_kernel": scores,                       # score rows read once
    }


def measure_dense(wl, dev, steps=1):
    """Dense softmax attention (torch SDPA, bf16) on one head of the same grid,
    forward + backward, as the comparator for the speedup ratio (measurement
    only; extrapolated to all heads)."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    import torch.nn.functional as F
    g = torch.Generator(device=dev).manual_seed(9)
    q, k, v = (torch.randn(1, 1, wl.N, wl.head_dim, device=dev, dtype=torch.bfloat16, generator=g)
               .requires_grad_(True) for _ in range(3))
    do = torch.randn(1, 1, wl.N, wl.head_dim, device=dev, dtype=torch.bfloat16, generator=g)
    for backend in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION):
        try:
            with sdpa_kernel([backend]):
                def once():
                    o = F.scaled_dot_product_attention(q, k, v)
                    o.backward(do)
                once()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(steps):
                    once()
                e1.record()
                torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
            flops = 14.0 * float(wl.N) ** 2 * wl.head_dim
            return dict(backend=str(backend).split(".")[-1], heads_timed=1, ms_per_head=ms,
                        ms_all_heads=ms * wl.heads, tflops=flops / (ms * 1e-3) / 1e12)
        except Exception as exc:  # backend unavailable for this size: try the next
            err = f"{backend}: {type(exc).__name__}: {str(exc)[:120]}"
    return dict(unavailable=err)


def measure_inference(att, inputs, out, fwd_flops, steps=3):
    """Inference across diffusion steps: a forward that reuses the last step's
    block layout and selection (permute Q, K, V; attention; unpermute O)."""
    from dynamic_block_sparse_variance_b200 import prism as P
    att.forward_reuse(inputs["q"], inputs["k"], inputs["v"], out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with P.KernelTrace() as tr:
        e0.record()
        for _ in range(steps):
            att.forward_reuse(inputs["q"], inputs["k"], inputs["v"], out=out)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    summ = tr.summary()
    attn_ms = sum(summ.get(k, (0, 0.0))[1] for k in FWD_KERNELS) / steps
    return dict(ms_per_forward=ms, attn_fwd_ms=attn_ms, executed_tflops=fwd_flops / (ms * 1e-3) / 1e12,
                attn_executed_tflops=fwd_flops / (attn_ms * 1e-3) / 1e12 if attn_ms else None,
                gpu_launches=sum(n for n, _ in summ.values()) // steps)


def measure_norms(wl, dev, steps=3):
    """The audio-norm producer (prism_audio_norms) on [N, heads*d] bf16."""
    from dynamic_block_sparse_variance_b200 import prism as P
    C = wl.heads * wl.head_dim
    g = torch.Generator(device=dev).manual_seed(8)
    h = torch.randn(wl.N, C, device=dev, dtype=torch.bfloat16, generator=g)
    a = torch.empty(wl.N, device=dev)
    P.prism_audio_norms(h, a)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        P.prism_audio_norms(h, a)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del h
    return dict(ms=ms, bytes=wl.N * C * 2, gbs=wl.N * C * 2 / (ms * 1e-3) / 1e9)


# ------------------------------------------------------------ CPU oracle --
def oracle_sample(inputs, wl, budget_s, seed=0, steps=1):
    """Time the fp64 oracle on a bounded sample of the same workload.

    The sample is the first 8-frame slab (one zone layer: 8 x H x W tokens,
    all heads) of the benchmark's own inputs.  The indicator, block
    assignment, permutation and pooling run in full on the slab; selection,
    forward and backward run on query blocks drawn at random (seeded) until
    the time budget is spent.  Returns executed attention TFLOP/s of the
    sampled query blocks and the details.
    """
    from oracle import prism_oracle as po

    plane = wl.H * wl.W
    n_s = 8 * plane
    f = lambda t: t[:n_s].detach().to("cpu", torch.float32).numpy()
    q, k, v, do = (f(inputs[n]) for n in ("q", "k", "v", "dout"))
    audio = None if inputs["audio"] is None else inputs["audio"][:n_s].cpu().numpy().astype(np.float64)
    t0 = time.perf_counter()
    ind = po.zone_indicator(v, 8, wl.H, wl.W, audio)
    shape_id, base, blocks = po.assign_blocks(ind["g"], ind["rho"], 8, wl.H, wl.W)
    perm = po.permutation(8, wl.H, wl.W, shape_id)
    qp, kp, vp, dop = (po.permute(x, perm) for x in (q, k, v, do))
    qbar, kbar = po.pool_blocks(qp, blocks), po.pool_blocks(kp, blocks)
    t_prep = time.perf_counter() - t0
    nb = len(blocks)
    scale = 1.0 / math.sqrt(wl.head_dim)
    rng = np.random.default_rng(seed)
    heads = sorted(rng.choice(wl.heads, size=min(2, wl.heads), replace=False).tolist())
    per_head = {h: tuple(np.ascontiguousarray(x[h:h + 1], dtype=np.float64) for x in (qp, kp, vp, dop))
                for h in heads}
    step_vals = []
    rows_done = 0
    flops_total = 0.0
    t_total = 0.0
    per_step_budget = budget_s / max(1, steps)
    for _ in range(steps):
        t_step = 0.0
        f_step = 0.0
        while t_step < per_step_budget:
            h, i = heads[int(rng.integers(len(heads)))], int(rng.integers(nb))
            hq, hk, hv, hdo = per_head[h]
            t1 = time.perf_counter()
            s = po.block_scores(qbar[h][i:i + 1], kbar[h], scale)[0]
            sel = po.select_row(po.block_probabilities(s), wl.top_k, wl.top_p)
            row_ptr = np.zeros((1, nb + 1), dtype=np.int64)
            row_ptr[0, i + 1:] = len(sel)
            po.bsa_forward(hq, hk, hv, blocks, row_ptr, [sel], scale, query_blocks=[i])
            po.bsa_backward(hq, hk, hv, hdo, blocks, row_ptr, [sel], scale, query_blocks=[i])
            dt = time.perf_counter() - t1
            t_step += dt
            f_step += 14.0 * blocks[i][1] * float(blocks[sel, 1].sum()) * wl.head_dim
            rows_done += 1
        step_vals.append(f_step / t_step / 1e12)
        flops_total += f_step
        t_total += t_step
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return dict(value=flops_total / t_total / 1e12, unit=UNIT, cores=cores, kind="oracle",
                sample=(f"first 8-frame slab (8x{wl.H}x{wl.W}, {wl.heads} heads) of the {wl.name} inputs: "
                        f"indicator/assign/permute/pool in full ({t_prep:.1f} s, not in the rate); "
                        f"select+fwd+bwd on {rows_done} random query blocks of heads {heads}, fp64 numpy"),
                step_values=step_vals, prep_s=t_prep, seconds=t_total)


# ----------------------------------------------------------------- ranks --
def setup_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ GPU bench --
def run_prism(args, rank, world):
    from dynamic_block_sparse_variance_b200 import prism as P
    from dynamic_block_sparse_variance_b200 import synth
    from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention

    P.lib()
    wl = synth.get_workload(args.workload)
    dev = torch.device("cuda", torch.cuda.current_device())
    inputs = synth.make_inputs(wl, dev, with_dout=True)
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p, device=dev)
    shp = (wl.N, wl.heads, wl.head_dim)
    O = torch.empty(shp, dtype=torch.bfloat16, device=dev)
    dq, dk, dv = (torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(3))

    def step():
        att.forward(inputs["q"], inputs["k"], inputs["v"], inputs["audio"], out=O)
        att.backward(inputs["dout"], dq, dk, dv)

    for _ in range(args.warmup):
        step()
    P.prism_device_status()
    pairs, nnz, nb, sizes, pairs256 = executed_pairs(att)
    Punit = float(pairs) * wl.head_dim
    # work of each forward kernel: the paired kernel takes the 256-token query blocks
    unit_of = {"bsa_fwd_tc2_kernel": float(pairs256) * wl.head_dim,
               "bsa_fwd_tc_kernel": float(pairs - pairs256) * wl.head_dim}
    exec_flops = 14.0 * Punit
    # the products the attention kernels run, in the same units: 4 P forward and 14 P backward (the
    # tensor-core backward's second dK and dQ products on the low halves of dS, or the warp-MMA
    # backward's recomputed S and dP), against the 14 P of the algorithm
    product_flops = 18.0 * Punit
    dense_flops = 14.0 * float(wl.N) ** 2 * wl.head_dim * wl.heads

    clocks = ClockSampler(dev)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    with P.KernelTrace() as tr:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    P.prism_device_status()
    ms_local = ev0.elapsed_time(ev1) / args.steps
    ms = max_over_ranks(ms_local, world)
    summ = tr.summary()
    launches = sum(n for n, _ in summ.values())

    # dominant kernel and its roofline
    peaks, peak_src = load_peaks()
    dom = max(summ.items(), key=lambda kv: kv[1][1])
    dom_name, (dom_n, dom_ms) = dom
    if dom_name in KERNEL_FLOP_UNITS:
        split = "bsa_fwd_tc2_kernel" in summ
        per_launch = KERNEL_FLOP_UNITS[dom_name] * (unit_of[dom_name] if split and dom_name in unit_of else Punit)
        achieved = per_launch / (dom_ms / dom_n * 1e-3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        traffic, traffic_src = profiled_traffic(dom_name, per_launch)
        roof = dict(kernel=dom_name, bound="tensor", achieved=achieved, peak=peak, unit="TFLOP/s",
                    frac=achieved / peak, traffic=traffic, traffic_source=traffic_src,
                    peak_source=f"{peak_src} sustained bf16 (cuBLAS)",
                    flops_per_launch=per_launch, ms_per_launch=dom_ms / dom_n)
    else:
        roof = dict(kernel=dom_name, bound="hbm", achieved=None, peak=peaks.get("hbm_gbs"), unit="GB/s",
                    frac=None, traffic=None)
    t_fwd = sum(summ.get(k, (0, 0.0))[1] for k in FWD_KERNELS) / args.steps
    t_bwd = sum(summ.get(k, (0, 0.0))[1] for k in BWD_KERNELS) / args.steps
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    n_scores = summ.get("block_scores_kernel", (0, 0.0))[0] // max(1, args.steps)
    n_cut = max(1, summ.get("row_cut_kernel", (0, 0.0))[0] // max(1, args.steps))
    hbm_bytes = hbm_kernel_bytes(wl, nb, n_scores / n_cut)
    kernels = {}
    for k, (n, t) in sorted(summ.items()):
        rec = dict(launches=n, ms_per_step=t / args.steps)
        if k in hbm_bytes and t > 0:
            gbs = hbm_bytes[k] / (t / args.steps * 1e-3) / 1e9
            rec.update(algorithmic_gb_per_step=hbm_bytes[k] / 1e9, achieved_gbs=gbs, hbm_frac=gbs / hbm_peak)
        kernels[k] = rec
    value = world * exec_flops / (ms * 1e-3) / 1e12
    out = dict(
        metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=ms, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
        data="synthetic",
        config=workload_config(wl, world),
        roofline=roof,
        attention=dict(fwd_ms=t_fwd, bwd_ms=t_bwd, executed_tflop=exec_flops / 1e12,
                       dense_equiv_tflop=dense_flops / 1e12,
                       attn_executed_tflops=exec_flops / ((t_fwd + t_bwd) * 1e-3) / 1e12 if t_fwd + t_bwd else None,
                       product_tflop=product_flops / 1e12,
                       attn_product_tflops=product_flops / ((t_fwd + t_bwd) * 1e-3) / 1e12 if t_fwd + t_bwd else None,
                       step_executed_pct_of_burst_peak=100.0 * exec_flops / (ms * 1e-3) / 1e12 / burst,
                       dense_equiv_tflops=dense_flops / (ms * 1e-3) / 1e12,
                       flop_density=pairs / (wl.heads * float(wl.N) ** 2),
                       block_density=nnz / (wl.heads * float(nb) ** 2), nblk=nb, nnz=nnz,
                       B_hist={int(b): int((sizes == b).sum().item()) for b in (64, 128, 256)}),
        kernels=kernels,
        gpu_launches=launches,
        clocks=clk,
    )
    # the measurements below are extras around the step: a failure in one is
    # recorded in its key and never costs the line
    def extra(key, fn):
        try:
            out[key] = fn()
        except Exception as exc:  # e.g. out of memory on a busier device
            out[key] = dict(error=f"{type(exc).__name__}: {str(exc)[:200]}")
            torch.cuda.empty_cache()

    if world == 1:
        extra("inference", lambda: measure_inference(att, inputs, O, 4.0 * Punit))
    if not args.no_norms and world == 1:
        def norms():
            nm = measure_norms(wl, dev)
            nm.update(hbm_frac=nm["gbs"] / hbm_peak, shape=f"[{wl.N}, {wl.heads * wl.head_dim}] bf16")
            return nm
        extra("audio_norms", norms)
    if not args.no_dense and world == 1:
        def dense():
            dn = measure_dense(wl, dev)
            if "ms_all_heads" in dn:
                dn["speedup_vs_dense"] = dn["ms_all_heads"] / ms
            return dn
        extra("dense_attention", dense)
    # end-to-end through the public API with host buffers (every rank takes the
    # same collective steps inside, so a failure there is left to raise)
    if not args.no_e2e:
        out["e2e"] = run_e2e(att, inputs, (O, dq, dk, dv), wl, exec_flops, args, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = {k: v for k, v in oracle_sample(inputs, wl, args.cpu_budget_s).items()
                               if k in ("value", "unit", "cores", "kind", "sample", "prep_s", "seconds")}
    return out


def run_e2e(att, inputs, outs, wl, exec_flops, args, world):
    """Same step with inputs in pinned host memory, through the public
    HostStepper: the H2D of Q, K, V, audio, dO and the D2H of O, dQ, dK, dV of
    every step are inside the timed region, overlapped with the kernels of
    the neighbouring steps (the first upload and the last download are not)."""
    from dynamic_block_sparse_variance_b200.attention import HostStepper
    names = ["q", "k", "v", "audio", "dout"]
    host_in = {n: (None if inputs[n] is None else torch.empty(inputs[n].shape, dtype=inputs[n].dtype,
                                                              pin_memory=True).copy_(inputs[n]))
               for n in names}
    host_out = {n: torch.empty((wl.N, wl.heads, wl.head_dim), dtype=torch.bfloat16, pin_memory=True)
                for n in ("o", "dq", "dk", "dv")}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values() if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    dev_buf = {n: inputs[n] for n in names}
    dev_buf.update(o=outs[0], dq=outs[1], dk=outs[2], dv=outs[3])
    stepper = HostStepper(att, device_buffers=dev_buf)
    stepper.run([host_in], [host_out])
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    stepper.run([host_in] * args.e2e_steps, [host_out] * args.e2e_steps)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.e2e_steps, world)
    return dict(value=world * exec_flops / (ms * 1e-3) / 1e12, unit=UNIT, ms_per_step=ms,
                h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, steps=args.e2e_steps,
                overlap="copies of step i+1's inputs and step i's outputs overlap kernels (HostStepper)")


# ----------------------------------------------------- reference (oracle) --
def workload_config(wl, world):
    """The workload both arms name: grid, heads, selection knobs, L2 regime, ranks."""
    return dict(workload=f"{wl.name}-like grid {wl.T}x{wl.H}x{wl.W}", T=wl.T, H=wl.H, W=wl.W, N=wl.N,
                heads=wl.heads, head_dim=wl.head_dim, top_k=wl.top_k, top_p=wl.top_p,
                l2="inputs larger than L2 (each Q/K/V tensor %.2f GB)" % (wl.N * wl.heads * wl.head_dim * 2 / 1e9),
                parallelism=f"replicas x{world}")


def run_reference(args, rank, world):
    """The fp64 CPU oracle on the host cores, on a bounded sample of the workload."""
    if rank != 0:
        return None
    from dynamic_block_sparse_variance_b200 import synth

    wl = synth.get_workload(args.workload)
    gdev = "cuda" if torch.cuda.is_available() else "cpu"
    inputs = synth.make_inputs(wl, gdev, with_dout=True)
    budget = min(args.cpu_budget_s * max(1, args.steps), 150.0)
    cb = oracle_sample(inputs, wl, budget, steps=max(1, args.steps))
    value = cb["value"]
    return dict(
        metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=cb["seconds"] * 1e3 / max(1, args.steps), higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
        config=workload_config(wl, world),
        cpu_baseline=dict(kind="oracle", cores=cb["cores"], sample=cb["sample"], value=value, unit=UNIT),
        e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0),
        gpu_launches=0,
    )


def main():
    args = parse_args()
    rank, world, _ = setup_dist(args)
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        else:
            res = run_prism(args, rank, world)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
