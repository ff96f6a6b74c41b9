"""Times the library's forward and backward on one pattern shape (no oracle).

  python -m factorized_sparse_self_b200.kernel_bench --kind dense --mode merged \
      --B 1 --H 8 --T 16384 --l 1 --c 1 --iters 5 --warmup 2

Prints one JSON line with per-call CUDA-event times of the forward attention
launches, of the backward attention kernel and of the whole forward + backward
call pair (ms_step), of the backward's prologue and epilogue kernels (16-bit
inputs), and the useful TFLOP/s (4 d nnz forward, 10 d nnz backward).
--flush writes 256 MB between iterations so that every call starts with a
cold L2. Inputs are the seeded synthetic ones
(bf16, std 0.5; dO ~ N(0, 1)).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kind", default="fixed", choices=["strided", "fixed", "dense"])
    ap.add_argument("--mode", default="merged", choices=["split", "merged"])
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=8)
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--d", type=int, default=64)
    ap.add_argument("--l", type=int, default=128)
    ap.add_argument("--c", type=int, default=8)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f16", "f32"])
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--flush", action="store_true")
    a = ap.parse_args()

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch

    import factorized_sparse_self_b200 as st
    import synth

    q, k, v, do = (x.cuda() for x in synth.draw(a.B, a.H, a.T, a.d, a.dtype, 0.5))
    L = st.st_pattern_layout(a.kind, a.mode, a.T, a.l, a.c)
    nhc, _ = L.counts()
    if nhc == 1:
        nnz = a.B * a.H * L.nnz(0)
    else:
        nnz = a.B * (((a.H + 1) // 2) * L.nnz(0) + (a.H // 2) * L.nnz(1))
    o = torch.empty_like(q)
    lse = torch.empty((a.B, a.H, a.T), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    code = {"bf16": st.ST_BF16, "f16": st.ST_F16, "f32": st.ST_F32}[a.dtype]
    ws = torch.empty(st.st_sparse_attn_bwd_workspace(L, code, a.B, a.H, a.T, a.d),
                     dtype=torch.uint8, device="cuda")

    def run():
        st.st_sparse_attn_fwd(L, q, k, v, o=o, lse=lse)
        if not a.fwd_only:
            st.st_sparse_attn_bwd(L, q, k, v, o, lse, do, workspace=ws, dq=dq, dk=dk, dv=dv)

    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda") if a.flush else None
    st.st_kernel_timing(True)
    tf, tb, ts, tp, te = [], [], [], [], []
    for _ in range(a.iters):
        if flush is not None:
            flush.zero_()
        torch.cuda._sleep(400000)  # the host queues the calls before the GPU reaches them
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
        tf.append(st.st_kernel_elapsed_ms(0))
        if not a.fwd_only:
            tb.append(st.st_kernel_elapsed_ms(1))
            if code != st.ST_F32:
                tp.append(st.st_kernel_elapsed_ms(2))
                te.append(st.st_kernel_elapsed_ms(3))
    st.st_kernel_timing(False)
    status = st.st_last_device_status()
    if status != st.ST_OK:
        raise SystemExit(f"device status {status}")
    res = {"kind": a.kind, "mode": a.mode, "B": a.B, "H": a.H, "T": a.T, "d": a.d, "l": a.l,
           "c": a.c, "nnz": nnz, "ms_step": statistics.mean(ts), "ms_fwd": statistics.mean(tf),
           "fwd_tflops": 4.0 * a.d * nnz / (statistics.mean(tf) * 1e-3) / 1e12}
    if tb:
        res["ms_bwd_kernel"] = statistics.mean(tb)
        res["bwd_kernel_tflops"] = 10.0 * a.d * nnz / (statistics.mean(tb) * 1e-3) / 1e12
    if tp:
        res["ms_bwd_prologue"] = statistics.mean(tp)
        res["ms_bwd_epilogue"] = statistics.mean(te)
    res["flush"] = bool(a.flush)
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
