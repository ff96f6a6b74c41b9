#!/usr/bin/env python
"""Benchmark of the factorized sparse attention hot path on B200.

One step = one forward + backward pass (recomputation backward) over one
batch of seeded synthetic inputs of the named workload. Prints ONE JSON line
(rank 0). Metric: useful TFLOP/s of fwd+bwd, counting 14 * d * nnz flops per
step (forward 4 d nnz, backward 10 d nnz including the recomputed S), with
nnz the live (query, key) pairs of the pattern.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference] [--no-extra]

--impl reference times the CPU oracle (the plain fp64 restatement the tests
check against) on a bounded sample of the same workload, on the host cores.
For N > 1 (torchrun), every rank runs its own batch of the workload on its
own GPU (weak scaling, no data-path collective); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

HEADLINE = "fixed-merged-T12288"
METRIC = "sparse attn fwd+bwd useful TFLOP/s and % of B200 bf16 tensor-core peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default=HEADLINE, choices=list(synth.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def nnz_of(layout, w):
    """Total live pairs over all B*H heads of the workload."""
    nhc, _ = layout.counts()
    if nhc == 1:
        return w.B * w.H * layout.nnz(0)
    return w.B * (((w.H + 1) // 2) * layout.nnz(0) + (w.H // 2) * layout.nnz(1))


def bwd_bytes(w):
    """Algorithmic HBM bytes of the backward attention kernel: read Q, K, V, dO
    (bf16) and LSE, D (fp32); write dQ, dK, dV (bf16)."""
    rows = w.B * w.H * w.T
    return rows * w.d * 2 * 7 + rows * 4 * 2


def fwd_bytes(w):
    rows = w.B * w.H * w.T
    return rows * w.d * 2 * 4 + rows * 4


def step_min_bytes(w):
    """Fewest HBM bytes a fwd + bwd step can move: the forward reads Q, K, V and
    writes O and LSE; the backward reads Q, K, V, O, dO and LSE and writes dQ,
    dK, dV."""
    rows = w.B * w.H * w.T
    e = 2 if w.dtype == "bf16" else 4
    return rows * w.d * e * 4 + rows * 4 + rows * w.d * e * 8 + rows * 4


def step_roofline(w, flops, ms, peaks):
    """The step's useful TFLOP/s against its roofline: the smaller of the
    measured tensor peak and (useful flops / minimum bytes) x measured HBM
    bandwidth."""
    b = step_min_bytes(w)
    roof = min(peaks["bf16_tflops"], flops / b * peaks["hbm_gbs"] * 1e9 / 1e12)
    achieved = flops / (ms * 1e-3) / 1e12
    return {"useful_tflops": achieved, "roofline_tflops": roof, "frac": achieved / roof,
            "min_bytes": b, "flop_per_byte": flops / b,
            "bound": "hbm" if roof < peaks["bf16_tflops"] else "tensor"}


def kernel_roofline(w, nnz, ms_bwd, peaks, peak_src):
    """Roofline of the dominant kernel (the backward attention kernel): its
    algorithmic bytes or flops per launch over its CUDA-event duration, against
    the measured peak of the resource that bounds it (HBM below the ridge,
    the bf16 tensor pipe above)."""
    bwd_flops = 10.0 * w.d * nnz
    bwd_b = bwd_bytes(w)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if bwd_flops / bwd_b < ridge:
        achieved = bwd_b / (ms_bwd * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = bwd_flops / (ms_bwd * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic("bwd_tc.cu", w.name)
    roof["kernel"] = "bwd_tc_kernel"
    roof["peak_source"] = f"{peak_src} (burst)"
    roof["algorithmic_bytes"] = bwd_b
    roof["algorithmic_flops"] = bwd_flops
    roof["ms_per_launch"] = ms_bwd
    return roof


def workload_config(w, world):
    """The `config` object of a bench line (both arms use the same one)."""
    return {"workload": w.name, "pattern": w.kind, "heads": w.mode, "B_per_gpu": w.B,
            "global_batch": w.B * world, "H": w.H, "T": w.T, "d": w.d, "l": w.l, "c": w.c,
            "parallelism": f"dp{world} (independent heads per GPU)",
            "l2": "flushed between timed steps (256 MB write)",
            "launch": "timed step = one CUDA-graph replay of the fwd + bwd calls"}


def max_over_ranks(x, device):
    """The largest of a float over all ranks (the slowest rank's time decides a
    multi-GPU number); the value itself when there is one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world, flops_per_rank, ms):
    """Throughput of the whole job: every rank's work over the slowest time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def source_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel_file, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    src = os.path.join(ROOT, "factorized_sparse_self_b200", "csrc", kernel_file)
    try:
        h = source_hash(src)
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 4 and parts[0] == kernel_file and parts[1] == workload \
                        and parts[3] == h:
                    return float(parts[2])
    except OSError:
        pass
    return None


# ---- clocks sampled during the timed region -----------------------------------

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4, "sync_boost": 0x10,
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2,
    }

    def __init__(self, device_index):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(device_index)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---- our implementation -----------------------------------------------------------

def capture_graph(fn):
    """CUDA graph of one call of fn (which must neither allocate nor synchronise)."""
    import torch
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            fn()
    torch.cuda.current_stream().wait_stream(cap)
    return graph


def run_ours(args):
    import torch
    import torch.distributed as dist

    import factorized_sparse_self_b200 as st

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = synth.WORKLOADS[args.workload]
    dt_code = st.ST_BF16 if w.dtype == "bf16" else st.ST_F32
    q, k, v, do = synth.draw(w.B, w.H, w.T, w.d, w.dtype, w.std, seed=rank)
    dev = torch.device("cuda", local)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    L = st.st_pattern_layout(w.kind, w.mode, w.T, w.l, w.c)
    nnz = nnz_of(L, w)
    flops = 14.0 * w.d * nnz
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd)
    ws = torch.empty(st.st_sparse_attn_bwd_workspace(L, dt_code, w.B, w.H, w.T, w.d),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        st.st_sparse_attn_fwd(L, qd, kd, vd, o=o, lse=lse)
        st.st_sparse_attn_bwd(L, qd, kd, vd, o, lse, dod, workspace=ws, dq=dq, dk=dk, dv=dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if st.st_last_device_status() != st.ST_OK:
        raise RuntimeError("device status error during warm-up")
    # The timed step is one replay of a CUDA graph holding the forward and
    # backward calls (they never allocate or synchronise), so the number is
    # the device's and not the Python launcher's. The end-to-end figure below
    # goes through the eager API.
    graph = capture_graph(step)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    times, kf, kb = [], [], []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            flush.zero_()  # evict L2 between timed steps (outside the events)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    if st.st_last_device_status() != st.ST_OK:
        raise RuntimeError("device status error in the timed region")
    # per-kernel times for the roofline: eager steps with the library's own
    # events around the attention kernels, on the stream they run on
    st.st_kernel_timing(True)
    kp, kn = [], []
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda._sleep(400000)  # the host queues the whole step before the GPU reaches it
        step()
        torch.cuda.synchronize()
        kf.append(st.st_kernel_elapsed_ms(0))
        kb.append(st.st_kernel_elapsed_ms(1))
        if dt_code != st.ST_F32:
            kp.append(st.st_kernel_elapsed_ms(2))
            kn.append(st.st_kernel_elapsed_ms(3))
    st.st_kernel_timing(False)
    del graph
    total_ms = max_over_ranks(sum(times), dev)
    ms_step = total_ms / args.steps
    value = whole_job_tflops(world, flops, ms_step)

    # ---- end to end through the public API, host buffers ------------------------
    hq, hk, hv, hdo = (x.pin_memory() for x in (q, k, v, do))
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    hdq, hdk, hdv = (torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(3))
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hdo))
    d2h = sum(x.numel() * x.element_size() for x in (ho, hl, hdq, hdk, hdv))

    # The step goes through the public API in chunks of G heads of one batch
    # entry (the head-range calls; about eight chunks per step), rotating over
    # four streams with a backward workspace each, so that the uploads of
    # later chunks and the downloads of earlier ones overlap the compute of
    # the current one (host-device copies run in both directions at once).
    n_streams = 4
    target = max(1, (w.H * w.B) // 8)
    G = max(g for g in range(1, w.H + 1) if w.H % g == 0 and g <= target)
    chunks = [(b, h0) for b in range(w.B) for h0 in range(0, w.H, G)]
    streams = [torch.cuda.Stream(device=dev) for _ in range(n_streams)]
    ws_b = [torch.empty(st.st_sparse_attn_bwd_workspace(L, dt_code, 1, w.H, w.T, w.d),
                        dtype=torch.uint8, device=dev) for _ in streams]

    def e2e_step():
        start = torch.cuda.Event()
        start.record(stream)
        for n, (b, h0) in enumerate(chunks):
            si = n % len(streams)
            sb = streams[si]
            sb.wait_event(start)
            with torch.cuda.stream(sb):
                sl = slice(b, b + 1)
                hs = slice(h0, h0 + G)
                for hsrc, ddst in ((hq, qd), (hk, kd), (hv, vd), (hdo, dod)):
                    ddst[sl, hs].copy_(hsrc[sl, hs], non_blocking=True)
                st.st_sparse_attn_fwd(L, qd[sl], kd[sl], vd[sl], o=o[sl], lse=lse[sl], stream=sb,
                                      heads=(h0, G))
                st.st_sparse_attn_bwd(L, qd[sl], kd[sl], vd[sl], o[sl], lse[sl], dod[sl],
                                      workspace=ws_b[si], dq=dq[sl], dk=dk[sl], dv=dv[sl],
                                      stream=sb, heads=(h0, G))
                for dsrc, hdst in ((o, ho), (lse, hl), (dq, hdq), (dk, hdk), (dv, hdv)):
                    hdst[sl, hs].copy_(dsrc[sl, hs], non_blocking=True)
        for sb in streams:
            done = torch.cuda.Event()
            done.record(sb)
            stream.wait_event(done)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 10))
    et = []
    for _ in range(e2e_steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        e1.synchronize()
        et.append(e0.elapsed_time(e1))
    if st.st_last_device_status() != st.ST_OK:
        raise RuntimeError("device status error in the end-to-end steps")
    e2e_ms = max_over_ranks(sum(et) / len(et), dev)
    e2e_value = whole_job_tflops(world, flops, e2e_ms)

    # ---- roofline of the dominant kernel (the backward attention kernel) ------
    peaks, peak_src = load_peaks()
    ms_f = statistics.mean(kf)
    ms_b = statistics.mean(kb)
    roof = kernel_roofline(w, nnz, ms_b, peaks, peak_src)

    fl, bl = L.launches(dt_code)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0, std) Q, K, V; N(0,1) dO)",
        "config": workload_config(w, world),
        "pct_of_peak": value / peaks["bf16_tflops"],
        "pct_of_spec_peak": value / 2250.0,
        "ms_fwd_kernel": ms_f,
        "ms_bwd_kernel": ms_b,
        "ms_bwd_prologue": statistics.mean(kp) if kp else None,
        "ms_bwd_epilogue": statistics.mean(kn) if kn else None,
        "nnz": nnz,
        "useful_flops_per_step": flops,
        # the same step counted without the backward's recomputation of S
        "useful_flops_no_recompute_per_step": 12.0 * w.d * nnz,
        "value_no_recompute": whole_job_tflops(world, 12.0 * w.d * nnz, ms_step),
        "step_roofline": step_roofline(w, flops, ms_step, peaks),
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "how": f"pinned host buffers; per chunk of {G} heads of one batch entry: "
                       "upload, forward, backward, download through the public API (head-"
                       f"range calls), {len(chunks)} chunks rotating over {n_streams} streams"},
        "gpu_launches": args.steps * (fl + bl),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(w)
        # the same kernels on the full causal set of the same shape
        line["dense_causal"] = dense_comparator(st, w, ms_step)
    if rank == 0 and not args.no_extra and world == 1:
        line["workloads"] = extra_workloads(st, w.name)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def time_workload(st, w, steps=5, warmup=2, kind=None):
    import torch
    kind = kind or w.kind
    dt_code = st.ST_BF16 if w.dtype == "bf16" else st.ST_F32
    q, k, v, do = (x.cuda() for x in synth.draw(w.B, w.H, w.T, w.d, w.dtype, w.std))
    L = st.st_pattern_layout(kind, w.mode, w.T, w.l, w.c)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(st.st_sparse_attn_bwd_workspace(L, dt_code, w.B, w.H, w.T, w.d),
                     dtype=torch.uint8, device="cuda")
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    def step():
        st.st_sparse_attn_fwd(L, q, k, v, o=o, lse=lse)
        st.st_sparse_attn_bwd(L, q, k, v, o, lse, do, workspace=ws, dq=dq, dk=dk, dv=dv)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = capture_graph(step)
    tf, tb, tot = [], [], []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        e1.synchronize()
        tot.append(e0.elapsed_time(e1))
    del graph
    st.st_kernel_timing(True)
    tp, tn = [], []
    for _ in range(steps):
        flush.zero_()
        torch.cuda._sleep(400000)  # the host queues the whole step before the GPU reaches it
        step()
        torch.cuda.synchronize()
        tf.append(st.st_kernel_elapsed_ms(0))
        tb.append(st.st_kernel_elapsed_ms(1))
        tp.append(st.st_kernel_elapsed_ms(2))
        tn.append(st.st_kernel_elapsed_ms(3))
    st.st_kernel_timing(False)
    assert st.st_last_device_status() == st.ST_OK
    nnz = nnz_of(L, w)
    ms = statistics.mean(tot)
    peaks, peak_src = load_peaks()
    flops = 14.0 * w.d * nnz
    return {"ms_step": ms, "ms_fwd_kernel": statistics.mean(tf),
            "ms_bwd_kernel": statistics.mean(tb), "ms_bwd_prologue": statistics.mean(tp),
            "ms_bwd_epilogue": statistics.mean(tn), "nnz": nnz,
            "useful_tflops": flops / (ms * 1e-3) / 1e12,
            "pct_of_peak": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "step_roofline": step_roofline(w, flops, ms, peaks),
            "roofline": kernel_roofline(w, nnz, statistics.mean(tb), peaks, peak_src),
            "fwd_tflops": 4.0 * w.d * nnz / (statistics.mean(tf) * 1e-3) / 1e12,
            "bwd_kernel_tflops": 10.0 * w.d * nnz / (statistics.mean(tb) * 1e-3) / 1e12}


def dense_comparator(st, w, sparse_ms):
    """The same kernels on the full causal set of the workload's shape: its
    time per fwd + bwd step, useful TFLOP/s over its own (causal) pairs, and
    how much faster the sparse step is."""
    steps, warmup = (3, 1) if w.T >= 32768 else (5, 2)
    r = time_workload(st, w, steps=steps, warmup=warmup, kind="dense")
    return {"ms_step": r["ms_step"], "useful_tflops": r["useful_tflops"],
            "ms_fwd_kernel": r["ms_fwd_kernel"], "ms_bwd_kernel": r["ms_bwd_kernel"],
            "nnz": r["nnz"], "sparse_speedup": r["ms_step"] / sparse_ms}


def extra_workloads(st, skip):
    out = {}
    for name in synth.ORDER:
        w = synth.WORKLOADS[name]
        if name == skip or w.dtype != "bf16":
            continue
        r = time_workload(st, w)
        r["dense_causal"] = dense_comparator(st, w, r["ms_step"])
        r["cpu_baseline"] = cpu_baseline(w, budget_s=6.0)
        out[name] = r
    return out


# ---- the oracle as CPU baseline / reference arm -------------------------------------

def oracle_sample(w, budget_s=15.0):
    """Heads of the workload for a bounded oracle run: whole head pairs (even
    and odd heads in split mode), as many as fit the time budget."""
    import oracle
    q, k, v, do = synth.draw(w.B, w.H, w.T, w.d, w.dtype, w.std)
    f = synth.as_f32
    qf, kf, vf, dof = f(q), f(k), f(v), f(do)
    BH = w.B * w.H
    qf, kf, vf, dof = (x.reshape(1, BH, w.T, w.d) for x in (qf, kf, vf, dof))
    threads = len(os.sched_getaffinity(0))

    def run(nh):
        """Seconds of one fwd + bwd over nh heads (the forward alone in run.fwd_s)."""
        args = [x[:, :nh].copy() for x in (qf, kf, vf, dof)]
        t0 = time.perf_counter()
        oracle.forward(w.kind, w.mode, args[0], args[1], args[2], w.l, w.c, threads=threads)
        run.fwd_s = time.perf_counter() - t0
        oracle.backward(w.kind, w.mode, args[0], args[1], args[2], args[3], w.l, w.c,
                        threads=threads)
        return time.perf_counter() - t0

    t2 = run(2)
    nh = 2
    while nh * 2 <= BH and t2 * (nh * 2) / 2 <= budget_s:
        nh *= 2
    nnz = sum(oracle.nnz(w.kind, w.mode, w.T, w.l, w.c, h % w.H) for h in range(nh))
    return run, nh, nnz, threads, t2


def cpu_baseline(w, budget_s=15.0):
    run, nh, nnz, threads, _ = oracle_sample(w, budget_s=budget_s)
    t = run(nh)
    tf = run.fwd_s
    return {"value": 14.0 * w.d * nnz / t / 1e12, "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{nh} of {w.B * w.H} heads of {w.name}, full T, fwd + bwd, fp64 C++ "
                      f"oracle, {t:.2f} s",
            "fwd_value": 4.0 * w.d * nnz / tf / 1e12, "fwd_s": tf, "fwd_bwd_s": t}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    run, nh, nnz, threads, _ = oracle_sample(w, budget_s=budget)
    for _ in range(args.warmup):
        run(nh)
    ts = [run(nh) for _ in range(args.steps)]
    ms = 1000.0 * sum(ts) / len(ts)
    value = 14.0 * w.d * nnz / (ms * 1e-3) / 1e12
    sample = f"{nh} of {w.B * w.H} heads of {w.name}, full T, fwd + bwd per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
