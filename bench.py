#!/usr/bin/env python
"""MuSe forward benchmark: tokens/s per head on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl muse|reference]
                    [--workload acausal_n8k_bf16|causal_n16k_bf16|...]

A step is one whole forward pass (both K-means, summaries, refinement; plus the
diagonal blocks and merge on the causal workload) over one batch of seeded
synthetic inputs already resident in HBM.  Steps are replayed from a CUDA graph,
timed one by one with CUDA events on the launching stream, with a 256 MiB write
between steps to flush L2.  value = B*H*N*ranks / (mean step time), taking the
max over ranks.  ``e2e`` repeats the measurement through the public API with the
inputs copied from pinned host memory and the output copied back inside the
timed region.  The default run (acausal N = 8k) also measures the metric's second
headline size, the causal N = 16k workload, under the key ``second_headline``
(``--no-second`` skips it).  ``--impl reference`` times the float64 oracle on the
host cores, one (b,h) problem per step (extrapolated from timed parts where the
problem is too large; the line says how).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from clustered_softmax_attention_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MuSe fwd tokens/s per head at N=8k/16k on 1 B200; % roofline; rel sq err"
DEFAULT_WORKLOAD = "acausal_n8k_bf16"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # 148 SMs x 128 FP32 lanes x FMA x max clock


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="muse", choices=["muse", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-second", action="store_true",
                    help="skip the second headline workload (causal N = 16k) of the default run")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--block", type=int, default=0,
                    help="causal/retrieval block size S (default: the workload's); "
                         "N/2 gives the single-level decomposition")
    ap.add_argument("--clusters", type=int, default=0,
                    help="Cq = Ck override (default: the workload's)")
    ap.add_argument("--iters", type=int, default=0,
                    help="K-means rounds override (default: the workload's)")
    ap.add_argument("--monopole", action="store_true",
                    help="acausal: the monopole-only ablation (dipole term dropped)")
    ap.add_argument("--partial-dipole", action="store_true",
                    help="acausal: the partially specialised dipole (untilted covariances)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the first H (b,h) problems of the workload only (B = 1; the same "
                         "draws as the full workload's first problems), e.g. for a small profile")
    ap.add_argument("--refine-form", default="auto", choices=["auto", "summary", "pair"],
                    help="acausal: the form of the full method's refinement (auto: the "
                         "library's cost rule)")
    return ap.parse_args()


def workload_of(args):
    """The named workload, with the block size overridden if --block is given."""
    w = WORKLOADS[args.workload]
    if args.block:
        if w.mode == "acausal":
            raise SystemExit("--block applies to the causal and retrieval workloads")
        if args.block <= 0 or w.N % args.block:
            raise SystemExit(f"--block must divide N={w.N}")
        w = dataclasses.replace(w, block=args.block)
    if args.clusters:
        if not 1 <= args.clusters <= w.N:
            raise SystemExit(f"--clusters must be in [1, N={w.N}]")
        w = dataclasses.replace(w, Cq=args.clusters, Ck=args.clusters)
    if args.iters:
        w = dataclasses.replace(w, iters=args.iters)
    if args.heads:
        if not 1 <= args.heads <= w.B * w.H:
            raise SystemExit(f"--heads must be in [1, B*H={w.B * w.H}]")
        w = dataclasses.replace(w, B=1, H=args.heads)
    if (args.monopole or args.partial_dipole) and w.mode != "acausal":
        raise SystemExit("--monopole and --partial-dipole apply to the acausal workloads")
    if args.monopole and args.partial_dipole:
        raise SystemExit("--monopole and --partial-dipole exclude each other")
    if args.refine_form != "auto" and (w.mode != "acausal" or args.monopole or args.partial_dipole):
        raise SystemExit("--refine-form applies to the full method on the acausal workloads")
    return w


def refine_form_of(w, requested="auto"):
    """The form in which the library evaluates the full method's refinement of workload
    w ("summary" or "pair"), as the library itself decides it (muse_refine_form)."""
    from clustered_softmax_attention_b200 import muse as m
    if w.mode != "acausal":
        return "pair"
    d = m.MuseDims(w.B, w.H, w.N, w.D, w.Dv, m.MUSE_BF16 if w.dtype == "bf16" else m.MUSE_F32,
                   w.scale)
    flags = {"auto": 0, "summary": m.MUSE_FLAG_REFINE_SUMMARY, "pair": m.MUSE_FLAG_REFINE_PAIR}[requested]
    form = m.lib().muse_refine_form(d, w.Cq, w.Ck, flags)
    if form < 0:
        raise ValueError(f"muse_refine_form refused {w.name}")
    return "summary" if form == 1 else "pair"


def dist_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = ["clustered_softmax_attention_b200/csrc/refine_tc.cu",
                  "clustered_softmax_attention_b200/csrc/tc_ptx.cuh"]


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the refinement kernel from the committed ncu summary of
    this workload, if it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"refine_tc_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def algorithmic_flops(w):
    """Flops of the refinement contraction per launch (all problems).

    Per problem the tilted dipole contraction costs 2*Cq*N*D*Dv and the refinement
    2*N*Ck*D*Dv (acausal); the kernel evaluates the same contraction as
    sum over query/key pairs, 2*nq*nk*(D+Dv), equal to it when Cq*D*Dv*... matches:
    we count the smaller of the two per instance (the work the method needs).
    """
    def inst(nq, nk, cq, ck, D, Dv):
        s_form = 2.0 * cq * nk * D * Dv + 2.0 * nq * ck * D * Dv
        n_form = 2.0 * nq * nk * (D + Dv)
        return min(s_form, n_form)
    P = w.B * w.H
    if w.mode == "acausal":
        return P * inst(w.N, w.N, w.Cq, w.Ck, w.D, w.Dv)
    if w.mode == "retrieval":
        # the remainder over every query's causal prefix: the method's count over the
        # prefix (as in the acausal case) or the pair form over the causal pairs
        s_form = 2.0 * w.Cq * w.N * w.D * w.Dv + 2.0 * w.N * w.Ck * w.D * w.Dv
        n_form = 2.0 * (w.N * w.N / 2.0) * (w.D + w.Dv)
        return P * min(s_form, n_form)
    if w.mode == "causal":
        tot = 0.0
        s = w.block
        while s < w.N:
            r = 1
            while r * s < w.N:
                nq = min((r + 1) * s, w.N) - r * s
                tot += inst(nq, s, min(w.Cq, nq), min(w.Ck, s), w.D, w.Dv)
                r += 2
            s *= 2
        return P * tot
    raise ValueError(w.mode)


def summary_form_ablation(w):
    """Whether the library evaluates the monopole / partial-dipole ablations of this
    workload in summary form (bfloat16, Dv = 64; D = 64 with Ck <= 256, D = 128 with
    Ck <= 128)."""
    return w.dtype == "bf16" and w.Dv == 64 and ((w.D == 64 and w.Ck <= 256) or (w.D == 128 and w.Ck <= 128))


def summary_output_flops(w, partial):
    """Flops of the summary-form output kernel per launch (tensor cores): 2 N Ck D for the
    projections u, 2 N Ck Dv for sum_j p_j mu_v,ij, plus 2 N D Dv for s Cbar_i qt with
    the partial dipole."""
    per = 2.0 * w.N * w.Ck * (w.D + w.Dv) + (2.0 * w.N * w.D * w.Dv if partial else 0.0)
    return w.B * w.H * per


def retrieval_flops(w):
    """Algorithmic flops of one retrieval step (all problems): K-means of queries and keys,
    the tilted summaries and the refinement over the whole causal prefix counted as in
    the acausal case (2 Cq N D Dv + 2 N Ck D Dv), the exact diagonal (S N (D + Dv)) and
    the retrieved runs (about S / Ck keys per (cluster, block) pair, k1 k2 pairs)."""
    per = (2 * w.iters * 2.0 * w.N * w.Cq * w.D
           + 2.0 * w.Cq * w.N * w.D * w.Dv + 2.0 * w.N * w.Ck * w.D * w.Dv
           + float(w.block) * w.N * (w.D + w.Dv)
           + 2.0 * w.N * w.k1 * w.k2 * (w.block / w.Ck) * (w.D + w.Dv))
    return w.B * w.H * per


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.sel = device_index

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                   "-lms", "50"]
            if self.sel is not None:
                cmd += ["-i", str(self.sel)]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def nvsmi_index(local_rank):
    import torch
    try:
        p = torch.cuda.get_device_properties(local_rank)
        bus = getattr(p, "pci_bus_id", None)
        dom = getattr(p, "pci_domain_id", None)
        devid = getattr(p, "pci_device_id", None)
        if bus is not None and dom is not None and devid is not None:
            return f"{dom:08X}:{bus:02X}:{devid:02X}.0"
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v for v in vis.split(",") if v.strip().isdigit()]
    return ids[local_rank] if local_rank < len(ids) else local_rank


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


RETRIEVAL_SAMPLE_ROWS = 64  # the retrieval oracle costs seconds per query row at N = 32k
LARGE_SAMPLE_ROWS = 16      # acausal problems whose dipoles would not fit in 1 GiB of host memory


def oracle_sample(w, head=0):
    """The float64 oracle on one head of the workload: (seconds, tokens, note).

    Workloads the oracle finishes in seconds run whole (note None).  Two are too large
    and are extrapolated to the whole problem from timed parts (the note says how):
      * retrieval: both K-means and the block selection run whole; RETRIEVAL_SAMPLE_ROWS
        evenly spaced query rows are computed, and their time is scaled by the number of
        (query cluster, query block) groups of the problem over the sampled rows' groups
        (each group builds its own remainder summaries, which dominate the per-row work);
      * acausal problems whose dense C_ij would exceed 1 GiB: both K-means run whole;
        the summaries are built for the query clusters of LARGE_SAMPLE_ROWS evenly spaced
        rows and scaled by Cq over that count; the refinement of the sampled rows is
        scaled by N over the rows."""
    from oracle import muse_oracle as mo
    Q, K, V = make_inputs(w, heads=[head])
    Q, K, V = Q[0, 0], K[0, 0], V[0, 0]
    t0 = time.perf_counter()
    if w.mode == "acausal" and w.Cq * w.Ck * w.D * w.Dv * 8 > (1 << 30):
        rows = np.linspace(0, w.N - 1, LARGE_SAMPLE_ROWS).astype(np.int64)
        ql, qc = mo.kmeans(Q, w.Cq, w.iters)
        kl, _ = mo.kmeans(K, w.Ck, w.iters)
        t_km = time.perf_counter() - t0
        used = np.unique(ql[rows])
        t1 = time.perf_counter()
        lz, mk, mv, cv = mo.tilted_summaries(qc[used], K, V, kl, w.Ck, w.scale)
        t_sum = time.perf_counter() - t1
        remap = -np.ones(w.Cq, np.int64)
        remap[used] = np.arange(used.size)
        t2 = time.perf_counter()
        mo.refine(Q, remap[ql], qc[used], lz, mk, mv, cv, w.scale, rows=rows)
        t_ref = time.perf_counter() - t2
        secs = t_km + t_sum * w.Cq / used.size + t_ref * w.N / rows.size
        note = (f"extrapolated: both K-means whole ({t_km:.1f} s), summaries of {used.size} of "
                f"{w.Cq} query clusters ({t_sum:.1f} s) scaled x{w.Cq / used.size:.1f}, "
                f"refinement of {rows.size} rows ({t_ref:.2f} s) scaled x{w.N / rows.size:.0f}")
        return secs, w.N, note
    if w.mode == "acausal":
        mo.muse_acausal(Q, K, V, w.Cq, w.Ck, w.iters, w.scale)
        return time.perf_counter() - t0, w.N, None
    if w.mode == "causal":
        mo.muse_causal(Q, K, V, w.block, w.Cq, w.Ck, w.iters, w.scale)
        return time.perf_counter() - t0, w.N, None
    if w.mode == "retrieval":
        rows = np.linspace(0, w.N - 1, RETRIEVAL_SAMPLE_ROWS).astype(np.int64)
        ql, qc = mo.kmeans(Q, w.Cq, w.iters)
        kl, _ = mo.kmeans(K, w.Ck, w.iters)
        t_km = time.perf_counter() - t0
        t1 = time.perf_counter()
        qbar = mo.cluster_means(Q, ql, w.Cq)
        sel = mo.retrieval_select(mo.block_logZ(qbar, K, kl, w.Ck, w.block, w.scale), w.k1, w.k2)
        t_sel = time.perf_counter() - t1
        t2 = time.perf_counter()
        mo.muse_retrieval(Q, K, V, w.block, w.Cq, w.Ck, w.iters, w.k1, w.k2, w.scale,
                          q_labels=ql, k_labels=kl, selection=sel, rows=rows)
        t_rows = time.perf_counter() - t2
        blk = np.arange(w.N) // w.block
        g_all = len(set(zip(ql.tolist(), blk.tolist())))
        g_smp = len(set(zip(ql[rows].tolist(), blk[rows].tolist())))
        secs = t_km + t_sel + t_rows * g_all / g_smp
        note = (f"extrapolated: both K-means whole ({t_km:.1f} s), block selection whole "
                f"({t_sel:.1f} s), {rows.size} evenly spaced query rows in {g_smp} (query "
                f"cluster, block) groups ({t_rows:.1f} s) scaled to the problem's {g_all} groups")
        return secs, w.N, note
    raise ValueError(w.mode)


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = workload_of(args)
    for _ in range(args.warmup):
        oracle_sample(w)
    secs = []
    note = None
    for k in range(args.steps):
        s, n, note = oracle_sample(w, head=k % w.problems)
        secs.append(s)
    mean = sum(secs) / len(secs)
    value = n / mean
    cores = cpu_threads()
    sample = f"one (b,h) problem of {w.name} per step (N={w.N} tokens), float64 numpy oracle"
    if note:
        sample += f"; {note} (last step)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, graph=False),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, graph):
    c = {"workload": w.name, "mode": w.mode, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "Dv": w.Dv,
         "Cq": w.Cq, "Ck": w.Ck, "iters": w.iters, "scale": w.scale,
         "l2": "flushed between timed steps (256 MiB write)", "cuda_graph": graph,
         "parallelism": "replicas (every rank runs the whole workload; no collective)"}
    if w.mode != "acausal":
        c["block"] = w.block
    if w.mode == "retrieval":
        c.update(k1=w.k1, k2=w.k2)
    return c


SECOND_HEADLINE = "causal_n16k_bf16"   # the metric's other headline size (N = 16k, causal)


def measure(args, w, steps, warmup, world, rank, local_rank, cpu_baseline):
    """Time `steps` whole forward passes of workload w on this rank; the JSON fields of
    the measurement (rank 0: with the sampled RSE and, if asked, the CPU baseline)."""
    import torch
    from clustered_softmax_attention_b200 import muse as m
    dev = torch.device("cuda", local_rank)
    Qn, Kn, Vn = make_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Qh = torch.from_numpy(Qn).to(tdt).pin_memory()
    Kh = torch.from_numpy(Kn).to(tdt).pin_memory()
    Vh = torch.from_numpy(Vn).to(tdt).pin_memory()
    Qd, Kd, Vd = (x.to(dev) for x in (Qh, Kh, Vh))
    Od = torch.empty(w.B, w.H, w.N, w.Dv, dtype=tdt, device=dev)
    Oh = torch.empty_like(Od, device="cpu").pin_memory()
    d = m.dims(Qd, Vd, w.scale)
    monopole = args.monopole and w.mode == "acausal"
    partial = args.partial_dipole and w.mode == "acausal"
    if w.mode == "acausal":
        ws = m.workspace("muse_forward_ex", d, w.Cq, w.Ck)
        flags = (m.MUSE_FLAG_MONOPOLE if monopole else 0) | \
            (m.MUSE_FLAG_PARTIAL_DIPOLE if partial else 0) | \
            {"auto": 0, "summary": m.MUSE_FLAG_REFINE_SUMMARY,
             "pair": m.MUSE_FLAG_REFINE_PAIR}[args.refine_form]

        def step(Q=Qd, K=Kd, V=Vd, O=Od):
            m.muse_forward_ex(Q, K, V, w.Cq, w.Ck, w.iters, w.scale, flags=flags, out=O, ws=ws)
    elif w.mode == "causal":
        ws = m.workspace("muse_causal_blocks", d, w.Cq, w.Ck, w.block)

        def step(Q=Qd, K=Kd, V=Vd, O=Od):
            m.muse_causal_blocks(Q, K, V, w.block, w.Cq, w.Ck, w.iters, w.scale, out=O, ws=ws)
    elif w.mode == "retrieval":
        ws = m.workspace("muse_retrieve_exact", d, w.Cq, w.Ck, w.block, w.k1, w.k2)

        def step(Q=Qd, K=Kd, V=Vd, O=Od):
            m.muse_retrieve_exact(Q, K, V, w.block, w.Cq, w.Ck, w.iters, w.k1, w.k2, w.scale,
                                  out=O, ws=ws)
    else:
        raise SystemExit(f"workload {w.name} has an unknown mode")

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    kev0, kev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kev0.record(stream)   # creates the underlying cudaEvent_t
    kev1.record(stream)
    m.lib().muse_set_profile_events(ctypes_ptr(kev0), ctypes_ptr(kev1))

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    n0 = m.lib().muse_launch_counter()
    step()
    torch.cuda.synchronize()
    launches_per_step = int(m.lib().muse_launch_counter() - n0)
    assert m.muse_last_device_status() == 0

    graph = None
    if not args.no_graph:
        try:
            s = torch.cuda.Stream()
            s.wait_stream(stream)
            with torch.cuda.stream(s):
                step()
            stream.wait_stream(s)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            torch.cuda.synchronize()
            for _ in range(2):
                graph.replay()
            torch.cuda.synchronize()
        except Exception as e:  # capture refused: time eager launches instead
            print(f"cuda graph capture failed ({e}); timing eager launches", file=sys.stderr)
            graph = None

    def run_step():
        if graph is not None:
            graph.replay()
        else:
            step()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(nvsmi_index(local_rank))
    clocks.start()
    time.sleep(0.3)
    step_ms, kern_ms = [], []
    for k in range(steps):
        flush.zero_()
        ev[k][0].record(stream)
        run_step()
        ev[k][1].record(stream)
        torch.cuda.synchronize()
        step_ms.append(ev[k][0].elapsed_time(ev[k][1]))
        kern_ms.append(kev0.elapsed_time(kev1))
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    mean_ms = max_over_ranks(sum(step_ms), dev) / steps
    tokens = w.B * w.H * w.N
    value = world * tokens / (mean_ms / 1e3)
    assert m.muse_last_device_status() == 0

    # end to end through the public API: pinned host inputs -> device -> output -> host
    m.lib().muse_set_profile_events(None, None)
    e2e_ms = []
    for k in range(max(2, steps // 2)):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        Qd.copy_(Qh, non_blocking=True)
        Kd.copy_(Kh, non_blocking=True)
        Vd.copy_(Vh, non_blocking=True)
        step()
        Oh.copy_(Od, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    e2e_value = world * tokens / (max_over_ranks(sum(e2e_ms) / len(e2e_ms), dev) / 1e3)
    h2d = sum(x.numel() * x.element_size() for x in (Qh, Kh, Vh))
    d2h = Oh.numel() * Oh.element_size()

    # roofline of the dominant kernel (the refinement; on the retrieval workload its
    # retrieval mode, the remainder), timed live above
    peaks, peak_src = load_peaks()
    kmean = sum(kern_ms) / len(kern_ms)
    summary_form = (monopole or partial) and summary_form_ablation(w)
    if summary_form:
        # the ablations in summary form: the output kernel's products (u = qt . mu_k,
        # sum_j p_j mu_v,ij, plus s Cbar_i qt for the partial dipole) on the tensor cores
        flops = summary_output_flops(w, partial)
        peak, bound, unit = float(peaks["bf16_tflops"]), "tensor", "TFLOP/s"
        kname = "summary-form output (monopole" + (" + covariance)" if partial else ")")
    else:
        flops = algorithmic_flops(w)
        if w.dtype == "bf16":
            peak, bound, unit = float(peaks["bf16_tflops"]), "tensor", "TFLOP/s"
        else:
            peak, bound, unit = FP32_SIMT_TFLOPS, "alu", "TFLOP/s"
        kname = "refinement (retrieval remainder)" if w.mode == "retrieval" else "refinement"
        if w.mode == "acausal" and not (monopole or partial):
            form = refine_form_of(w, args.refine_form)
            kname += f" ({form} form)"
    achieved = flops / (kmean / 1e3) / 1e12
    roof = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak,
            "traffic": None if summary_form or "summary form" in kname else recorded_traffic(w.name),
            "kernel": kname, "kernel_ms": kmean, "flops_per_launch": flops,
            "peak_source": f"{peak_src} bf16_tflops (burst)" if bound == "tensor"
            else "derived: 148 SM x 128 FP32 lanes x 2 x 1965 MHz"}
    if w.mode == "retrieval":
        roof["step_flops"] = retrieval_flops(w)
    out = None
    if rank == 0:
        try:
            from oracle import muse_oracle as mo
            rng = np.random.default_rng(0)
            rows = rng.choice(w.N, 64, replace=False)
            On = Od[0, 0].float().cpu().numpy().astype(np.float64)
            E = mo.exact_attention(Qn[0, 0], Kn[0, 0], Vn[0, 0], w.scale, rows=rows,
                                   causal=(w.mode != "acausal"))
            rse = float(((On[rows] - E[rows]) ** 2).sum() / (E[rows] ** 2).sum())
        except Exception:
            rse = None
        cpu = None
        if cpu_baseline:
            secs, n, note = oracle_sample(w)
            what = f"one (b,h) problem of {w.name} (N={w.N} tokens)"
            if note:
                what += f"; {note}"
            cpu = {"value": n / secs, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                   "sample": f"{what}, float64 numpy oracle, {secs:.1f} s"}
        out = {
            "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": warmup,
            "ms_per_step": mean_ms, "dtype": w.dtype,
            "config": dict(config_of(w, graph is not None),
                           **({"monopole": True} if monopole else {}),
                           **({"partial_dipole": True} if partial else {})),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * steps,
            "clocks": clk, "rse_vs_exact_sampled": rse,
            "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms),
        }
    del graph
    return out


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def main():
    args = parse()
    rank, local_rank, world = dist_info()
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl" if args.impl == "muse" else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    if args.impl == "reference":
        run_reference(args, rank, world)
        if world > 1:
            dist.destroy_process_group()
        return

    torch.cuda.set_device(local_rank)
    w = workload_of(args)
    res = measure(args, w, args.steps, args.warmup, world, rank, local_rank,
                  cpu_baseline=(world == 1 and not args.no_cpu_baseline))
    # the metric names two headline sizes: the default run also measures the causal 16k
    # workload (every rank, same collective steps), reported under its own key
    second = None
    if args.workload == DEFAULT_WORKLOAD and not args.no_second and not (
            args.block or args.clusters or args.iters or args.heads or args.monopole or
            args.partial_dipole):
        second = measure(args, WORKLOADS[SECOND_HEADLINE], max(10, args.steps // 4), args.warmup,
                         world, rank, local_rank, cpu_baseline=False)
    if rank == 0:
        line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": res["dtype"], "data": "synthetic (seeded Gaussian-mixture Q/K, normal V)"}
        line.update({k: v for k, v in res.items() if k not in line})
        if second is not None:
            line["second_headline"] = dict(second, workload=SECOND_HEADLINE)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def ctypes_ptr(ev):
    import ctypes
    return ctypes.c_void_p(ev.cuda_event)


if __name__ == "__main__":
    main()
