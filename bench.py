"""Benchmark: one layer of Prism dynamic sparse video self-attention at the 2K grid.

A step is the whole hot path on one batch: plan (zone statistics, volumes and
shapes, block-contiguous permutation, pooled scoring, Top-k U Top-p CSR),
sparse attention forward, and sparse attention backward (dQ, dK, dV).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  `value` is effective TFLOP/s over the
selected blocks (forward 4*D and backward 10*D FLOP per selected
query-key token pair), summed over ranks; `ms_per_step` is ms per layer.
Multi-GPU runs are independent replicas (the path has no exchange step).
The reference arm times the fp64 CPU oracle on a bounded sample.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn ms/layer fwd+bwd & effective TFLOP/s (selected blocks) at 2K grid"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
SLOWDOWN_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def smi_device_id(device_index: int) -> str:
    """nvidia-smi's name for torch's device `device_index`: CUDA_VISIBLE_DEVICES
    renumbers the GPUs a process sees (its entries are indices or UUIDs, both
    of which nvidia-smi --id accepts); nvidia-smi does not renumber them."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    return ids[device_index] if device_index < len(ids) else str(device_index)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"prism_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={smi_device_id(self.idx)}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sms, watts, mx, reasons = [], [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sms.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                try:
                    watts.append(float(parts[3]))
                except ValueError:
                    pass
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "power_w": statistics.median(watts) if watts else None, "samples": len(sms)}


# --------------------------------------------------------------------------
def selected_pairs(view, D):
    """sum over rows of |B_i| * sum_{j in S_i} |B_j| (token pairs), per sample."""
    import torch
    blk = view["blk_off"].long()
    nbmax = view["nbmax"]
    rp = view["row_ptr"].long()
    col = view["col_idx"].long()
    B = blk.shape[0]
    rows = rp.numel() - 1
    counts = rp[1:] - rp[:-1]
    row_ids = torch.repeat_interleave(torch.arange(rows, device=rp.device), counts)
    sample = row_ids // (rows // B)
    i = row_ids % nbmax
    sizes = blk[:, 1:] - blk[:, :-1]                     # [B, nbmax]
    si = sizes[sample, i]
    sj = sizes[sample, col]
    return int((si * sj).sum().item())


def pooled_pairs(view):
    """sum over rows of |B_i| * (N_b - |S_i|): (query token, pooled key block)
    pairs of the Taylor term, per sample."""
    import torch
    blk = view["blk_off"].long()
    nbmax = view["nbmax"]
    rp = view["row_ptr"].long()
    B = blk.shape[0]
    nbs = torch.as_tensor([int(x) for x in view["n_blocks"]], device=rp.device)
    rows = torch.arange(rp.numel() - 1, device=rp.device)
    counts = rp[1:] - rp[:-1]
    sample = rows // (rows.numel() // B)
    i = rows % nbmax
    valid = i < nbs[sample]
    sizes = blk[:, 1:] - blk[:, :-1]
    si = torch.where(valid, sizes[sample, i.clamp(max=nbmax - 1)], torch.zeros_like(i))
    return int((si * (nbs[sample] - counts) * valid).sum().item())


def kernel_bytes(name, w, nb, pairs_unused):
    """Algorithmic HBM bytes of one launch of the plan kernels (one sample)."""
    N, C, D, h = w.N, w.heads * w.head_dim, w.head_dim, w.heads
    if name == "zone_stats_v":
        return N * C * 2
    if name == "permute_pool":
        return 6 * N * C * 2 + 2 * h * nb * D * 8 + N * 4
    if name == "attn_bwd_pre":
        return 2 * N * C * 2 + N * C * 2 + h * N * 4
    if name == "dq_finalize":
        return h * N * D * 4 + N * C * 2
    if name == "taylor_pool":  # read V (permuted) and the fp64 pooled keys, write two bf16 pooled copies
        return N * C * 2 + h * nb * D * 8 + 2 * h * nb * D * 2
    return None


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of x over all ranks (timings are taken as the slowest
    rank's).  The only collective of the benchmark: replicas never exchange
    data."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(flops_per_step: float, steps: int, world: int, ms_max: float) -> float:
    """Whole-job TFLOP/s: every rank runs `steps` steps of the same workload
    (weak scaling), timed by the slowest rank."""
    return flops_per_step * steps * world / (ms_max * 1e-3) / 1e12


L2_BYTES = 128 << 20  # B200 L2: 126 MB


def steps_or_1(args):
    return max(args.steps, 1)


def workload_of(args):
    from dynamic_block_sparse_zone_b200.synth import WORKLOADS, scaled
    w = WORKLOADS[args.workload]
    return scaled(w, heads=args.heads) if args.heads else w


def run_ours(args, rank, world, dev):
    import torch
    import torch.distributed as dist
    import dynamic_block_sparse_zone_b200 as P
    from dynamic_block_sparse_zone_b200.synth import WORKLOADS, make_inputs

    w = workload_of(args)
    P.load_library()
    inp = make_inputs(w, seed=0, device=dev, with_grad_output=True)
    plan = P.PrismPlan(P.params_for(w, hilbert_block=args.hilbert))
    shp = inp.Q.shape
    O = torch.empty(shp, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.heads, w.N), dtype=torch.float32, device=dev)
    dQ, dK, dV = (torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(3))

    def step(Q, K, V, a, dO):
        plan.build(Q, K, V, a)
        plan.fwd(O, lse, taylor=args.taylor)
        if not args.fwd_only:
            plan.bwd(O, dO, dQ, dK, dV)

    for _ in range(args.warmup):
        step(inp.Q, inp.K, inp.V, inp.a, inp.dO)
    torch.cuda.synchronize()
    plan.check()
    view = plan.view()
    pairs = selected_pairs(view, w.head_dim)
    nb = view["n_blocks"][0]
    tpairs = pooled_pairs(view) if args.taylor else 0
    flops_fwd = 4.0 * w.head_dim * (pairs + tpairs)
    flops_bwd = 10.0 * w.head_dim * pairs
    flops_step = flops_fwd + (0.0 if args.fwd_only else flops_bwd)

    def barrier():
        if world > 1:
            dist.barrier()


    # ---- device-resident timed region ----
    # Inputs larger than L2 stream from HBM every step; smaller ones would stay
    # in L2 between steps, so then L2 is flushed (a 256 MB write) before each
    # step and the steps are timed one by one, the flush outside the events.
    in_bytes = sum(x.numel() * x.element_size() for x in (inp.Q, inp.K, inp.V, inp.a)) + (
        0 if args.fwd_only else inp.dO.numel() * inp.dO.element_size())
    flush = None if in_bytes > L2_BYTES else torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    l2_note = (f"inputs larger than L2 ({in_bytes / 1e9:.2f} GB per step vs 126 MB)" if flush is None else
               f"L2 flushed (256 MB write) before each timed step, steps timed one by one (inputs {in_bytes / 1e6:.1f} MB)")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(run, sample_clocks=True):
        """Device time of args.steps calls of run(), max over ranks, with clocks sampled."""
        clocks = ClockSampler(torch.cuda.current_device())
        barrier()
        torch.cuda.synchronize()
        if sample_clocks:
            clocks.start()
        if flush is None:
            e0.record(stream)
            for _ in range(args.steps):
                run()
            e1.record(stream)
            torch.cuda.synchronize()
            total = e0.elapsed_time(e1)
        else:
            pairs = []
            for _ in range(args.steps):
                flush.fill_(1)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                run()
                b.record(stream)
                pairs.append((a, b))
            torch.cuda.synchronize()
            total = sum(a.elapsed_time(b) for a, b in pairs)
        barrier()
        return max_over_ranks(total, world, dev), clocks.stop()

    # the headline: no instrumentation inside the timed region
    plan.set_timing(False)
    ms, clk = timed(lambda: step(inp.Q, inp.K, inp.V, inp.a, inp.dO))
    plan.check()
    # a run that saw a hardware or thermal slowdown on any rank is measured
    # once more (every rank takes the same steps), and the line says so
    slow = 1.0 if clk and any(r in SLOWDOWN_REASONS for r in clk["reasons"]) else 0.0
    if max_over_ranks(slow, world, dev) > 0:
        first = clk
        ms, clk = timed(lambda: step(inp.Q, inp.K, inp.V, inp.a, inp.dO))
        plan.check()
        if clk is not None:
            clk["remeasured_after"] = first["reasons"] if first else "a slowdown on another rank"
    # the per-kernel split: a second pass of the same steps with the plan's
    # event timers on (two event records around each launch), timed apart
    plan.set_timing(True)
    plan.read_timing()
    ms_split, _ = timed(lambda: step(inp.Q, inp.K, inp.V, inp.a, inp.dO), sample_clocks=False)
    timing = plan.read_timing()
    plan.set_timing(False)
    plan.check()

    # ---- the same step captured once in a CUDA graph and replayed ----
    # (the per-kernel times above come from the eager loop: event timers do
    # not run inside a graph; the kernels are the same)
    launch = "eager"
    if args.graph:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step(inp.Q, inp.K, inp.V, inp.a, inp.dO)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(inp.Q, inp.K, inp.V, inp.a, inp.dO)
        for _ in range(args.warmup):
            graph.replay()
        ms, clk = timed(graph.replay)
        plan.check()
        del graph
        launch = "cuda graph (one step captured, replayed)"

    # ---- end to end through the C ABI with page-locked host buffers ----
    # prism_step_host: every step copies its inputs host->device, runs the
    # plan and the attention kernels, and copies its outputs back; the plan
    # overlaps one step's copies with its neighbours' kernels on three streams.
    e2e = None
    if not args.no_e2e:
        host_in = [x.cpu().pin_memory() for x in (inp.Q, inp.K, inp.V, inp.a)]
        host_dO = None if args.fwd_only else inp.dO.cpu().pin_memory()
        host_out = [torch.empty(shp, dtype=torch.bfloat16).pin_memory() for _ in range(1 if args.fwd_only else 4)]
        h2d = sum(x.numel() * x.element_size() for x in host_in) + (
            0 if host_dO is None else host_dO.numel() * host_dO.element_size())
        d2h = sum(x.numel() * x.element_size() for x in host_out)

        def e2e_step():
            if args.fwd_only:
                return plan.step_host(*host_in, host_out[0], taylor=args.taylor)
            return plan.step_host(*host_in, host_out[0], dO=host_dO, dQ=host_out[1], dK=host_out[2], dV=host_out[3])

        for _ in range(max(1, args.warmup // 2)):
            plan.step_wait(e2e_step())
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        last = None
        for _ in range(args.steps):
            last = e2e_step()
        plan.step_join(last)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        plan.step_wait(last)
        plan.check()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": round(aggregate_value(flops_step, args.steps, world, ms_e2e), 3),
               "unit": "TFLOP/s", "ms_per_step": round(ms_e2e / args.steps, 3),
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "prism_step_host (copies and kernels of consecutive steps overlap on three streams)"}
        del host_in, host_out, host_dO

    peaks, peak_src = load_peaks()
    fp64_peak = measure_fp64_peak(dev) if not args.no_fp64_peak else None
    kernels = {}
    total_k = sum(v[0] for v in timing.values()) or 1.0
    for name, (tms, n) in timing.items():
        if n == 0:
            continue
        avg = tms / n
        rec = {"launches": n, "avg_ms": round(avg, 4), "share": round(tms / total_k, 4)}
        if name == "select":
            rec["fp64_tflops"] = round(2.0 * w.head_dim * nb * nb * w.heads * w.batch * steps_or_1(args) /
                                       (tms * 1e-3) / 1e12, 3)
            if fp64_peak:
                rec["fp64_peak_tflops"] = fp64_peak
                rec["frac"] = round(rec["fp64_tflops"] / fp64_peak, 4)
                rec["peak_kind"] = "fp64 dense, measured in this run (cuBLAS DGEMM 4096^3, best of 5)"
        if name in ("attn_fwd", "attn_fwd_taylor"):
            rec["tflops"] = round(flops_fwd / (avg * 1e-3) / 1e12, 2)
        elif name == "attn_bwd":
            rec["tflops"] = round(flops_bwd / (avg * 1e-3) / 1e12, 2)
        else:
            by = kernel_bytes(name, w, nb, pairs)
            if by:
                rec["gbs"] = round(by / (avg * 1e-3) / 1e9, 1)
        kernels[name] = rec
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    if "tflops" in kernels[dom]:
        peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        ach = kernels[dom]["tflops"]
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": round(ach / peak, 4), "peak_kind": f"bf16 dense sustained ({peak_src})",
                "traffic": traffic_for(dom, w)}
    else:
        peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        ach = kernels[dom].get("gbs", 0.0)
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "peak_kind": f"HBM copy ({peak_src})", "traffic": traffic_for(dom, w)}
    # one timer record per kernel launch, except the CSR/CSC scope (9 kernels)
    launches_per_step = sum(n * (9 if k == "csr_csc" else 1) for k, (t, n) in timing.items()) // max(args.steps, 1)
    result = {
        "metric": METRIC,
        "value": round(aggregate_value(flops_step, args.steps, world, ms), 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 3),
        "ms_per_layer": round(ms / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name,
                   "plan": (f"Hilbert order, fixed {args.hilbert}-token blocks" if args.hilbert else
                            "Prism zones (dynamic volume and shape)"),
                   "pass": ("forward with the Taylor term for unselected blocks" if args.taylor else
                            "forward" if args.fwd_only else "forward+backward"),
                   "taylor_pooled_pairs": tpairs if args.taylor else None,
                   "grid": [w.T, w.H, w.W], "tokens": w.N, "heads": w.heads,
                   "head_dim": w.head_dim, "top_k": w.top_k, "top_p": w.top_p, "max_frac": w.max_frac,
                   "n_blocks": nb, "selected_token_pairs": pairs, "flops_per_step": flops_step,
                   "l2": l2_note, "launch": launch, "parallelism": f"replicas x{world}"},
        "kernels": kernels,
        "kernels_note": ("per-kernel times from a second pass of the same steps with the plan's event timers "
                         f"on ({ms_split / args.steps:.3f} ms per step); the headline pass runs without them"),
        "roofline": roof,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "clocks": clk,
    }
    plan.close()
    return result


def measure_fp64_peak(dev):
    """Dense fp64 TFLOP/s of this GPU, measured: cuBLAS DGEMM 4096^3, best of 5
    (the denominator of the selection kernels' fp64 scoring)."""
    import torch
    n = 4096
    a = torch.randn(n, n, dtype=torch.float64, device=dev)
    b = torch.randn(n, n, dtype=torch.float64, device=dev)
    c = torch.empty(n, n, dtype=torch.float64, device=dev)
    torch.matmul(a, b, out=c)
    best = None
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.matmul(a, b, out=c)
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1)
        best = t if best is None else min(best, t)
    del a, b, c
    return round(2.0 * n ** 3 / (best * 1e-3) / 1e12, 2)


def traffic_for(kernel, w):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the current kernel source and for this workload at this size (a record
    lists the workloads whose launch of the kernel it covers)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        rec = d.get(kernel)
        if not rec:
            return None
        if w.name not in rec["workloads"] or w.heads != rec["heads"] or w.batch != rec["batch"]:
            return None
        import hashlib
        src = os.path.join(ROOT, "dynamic_block_sparse_zone_b200", "csrc", rec["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return rec["bytes_per_launch"] if h == rec["source_sha"] else None
    except Exception:
        return None


# --------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# --------------------------------------------------------------------------
def oracle_setup(w, dev, hilbert=0):
    import numpy as np
    import oracle
    from dynamic_block_sparse_zone_b200.synth import bf16_bits, make_inputs
    inp = make_inputs(w, seed=0, device=dev, with_grad_output=True)
    bits = [bf16_bits(x[0]) for x in (inp.Q, inp.K, inp.V, inp.dO)]
    a = inp.a[0].cpu().numpy()
    del inp
    t0 = time.time()
    if hilbert:
        pl = oracle.plan_hilbert(bits[0], bits[1], bits[2], w.T, w.H, w.W, w.heads, w.head_dim, hilbert, w.top_k,
                                 float(np.float32(w.top_p)), float(np.float32(w.max_frac)), with_select=False)
    else:
        pl = oracle.plan(bits[0], bits[1], bits[2], a, w.T, w.H, w.W, w.heads, w.head_dim, w.top_k,
                         float(np.float32(w.top_p)), float(np.float32(w.max_frac)), with_select=False)
    head = [0]
    cnt, cols, diag = oracle.select(pl.Qbar[head], pl.Kbar[head], w.top_k, float(np.float32(w.top_p)),
                                    float(np.float32(w.max_frac)))
    pl.cnt, pl.cols, pl.diag = cnt, cols, diag
    pl.heads = 1
    hb = [np.ascontiguousarray(x[:, head, :]) for x in bits]
    plan_s = time.time() - t0
    return pl, hb, plan_s


def oracle_sample(pl, hb, w, rows, seed, taylor=False):
    """fwd + dQ of `rows` query tokens of one head (taylor: the forward with the
    Taylor term alone); returns (seconds, flops)."""
    import numpy as np
    import oracle
    rs = np.random.default_rng(seed)
    req_t = rs.integers(0, w.N, size=rows).astype(np.int32)
    req_h = np.zeros(rows, np.int32)
    off = pl.blk_off()
    sizes = np.diff(off)
    tok2blk = np.empty(w.N, np.int64)
    for j in range(pl.nb):
        tok2blk[pl.perm[off[j]:off[j + 1]]] = j
    keys = 0
    for t in req_t:
        i = tok2blk[t]
        keys += int(sizes[pl.cols[0, i, :pl.cnt[0, i]]].sum())
    if taylor:
        pooled = int(sum(pl.nb - pl.cnt[0, tok2blk[t]] for t in req_t))
        t0 = time.time()
        oracle.attn_fwd_taylor_rows(pl, hb[0], hb[1], hb[2], req_h, req_t)
        return time.time() - t0, 4.0 * w.head_dim * (keys + pooled)
    t0 = time.time()
    oracle.attn_fwd_rows(pl, hb[0], hb[1], hb[2], req_h, req_t)
    oracle.attn_bwd_dq_rows(pl, hb[0], hb[1], hb[2], hb[3], req_h, req_t)
    dt = time.time() - t0
    # forward 4*D per pair; dQ needs S, dP and dQ: 6*D per pair
    return dt, 10.0 * w.head_dim * keys


def cpu_baseline(w, dev, rows, taylor=False, hilbert=0):
    import oracle
    pl, hb, plan_s = oracle_setup(w, dev, hilbert)
    dt, fl = oracle_sample(pl, hb, w, rows, 123, taylor)
    what = "forward with the Taylor term" if taylor else "forward + dQ"
    return {"value": round(fl / dt / 1e12, 8), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"fp64 oracle {what} of {rows} random query tokens of head 0 on the same "
                      f"workload ({dt:.1f} s); oracle plan with 1-head selection took {plan_s:.1f} s, not counted"}


def run_reference(args, dev):
    import oracle
    from dynamic_block_sparse_zone_b200.synth import WORKLOADS
    w = workload_of(args)
    pl, hb, plan_s = oracle_setup(w, dev, args.hilbert)
    rows = args.ref_rows
    for s in range(args.warmup):
        oracle_sample(pl, hb, w, rows, 1000 + s)
    tot_t, tot_f = 0.0, 0.0
    for s in range(args.steps):
        dt, fl = oracle_sample(pl, hb, w, rows, s)
        tot_t += dt
        tot_f += fl
    val = tot_f / tot_t / 1e12
    sample = (f"fp64 oracle forward + dQ of {rows} random query tokens of head 0 per step; "
              f"oracle plan (1-head selection) {plan_s:.1f} s outside the timed steps")
    return {"impl": "reference", "metric": METRIC, "value": round(val, 8), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name},
            "cpu_baseline": {"value": round(val, 8), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(val, 8), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="latent2k_train_24x96x160")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--fwd-only", action="store_true", help="step = plan + forward (forward-only workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp64-peak", action="store_true", help="skip the fp64 DGEMM peak measurement")
    ap.add_argument("--graph", action="store_true", help="time replays of the step captured in a CUDA graph")
    ap.add_argument("--hilbert", type=int, default=0, choices=[0, 64, 128, 256],
                    help="Hilbert-order plan with fixed blocks of this many tokens (the DFSAttn-style baseline)")
    ap.add_argument("--taylor", action="store_true",
                    help="forward with the zeroth-order Taylor term for the unselected blocks (implies --fwd-only)")
    ap.add_argument("--heads", type=int, default=0, help="override the workload's head count (profiling)")
    ap.add_argument("--cpu-rows", type=int, default=6000)
    ap.add_argument("--ref-rows", type=int, default=1500)
    args = ap.parse_args()
    if args.taylor:
        args.fwd_only = True
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    import torch
    if args.impl == "reference":
        if rank == 0:
            dev = "cuda" if torch.cuda.is_available() else "cpu"
            print(json.dumps(run_reference(args, dev)), flush=True)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    res = run_ours(args, rank, world, dev)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            torch.cuda.empty_cache()
            from dynamic_block_sparse_zone_b200.synth import WORKLOADS
            res["cpu_baseline"] = cpu_baseline(workload_of(args), dev, args.cpu_rows, args.taylor, args.hilbert)
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
