"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import factorized_sparse_self_b200 as st
import synth

# Tolerances: fp32 max-abs 1e-4; bf16 max-abs 2e-2 and relative L2 1e-2 per
# output tensor, the oracle being fed the bf16-rounded inputs. fp16 runs the
# same kernels with every 16-bit rounding (P, dS and the outputs) eight times
# finer (unit roundoff 2^-11 against 2^-8), so its bounds are the bf16 ones
# divided by 5 (a margin of 8/5 over the scaled bf16 bounds).
TOL = {"f32": {"abs": 1e-4, "rel": None}, "bf16": {"abs": 2e-2, "rel": 1e-2},
       "f16": {"abs": 4e-3, "rel": 2e-3}}


def rel_l2(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = np.linalg.norm(y)
    return float(np.linalg.norm(x - y) / den) if den > 0 else float(np.linalg.norm(x - y))


def compare(name, got, ref, dtype, extra=""):
    """Asserts the tolerance; returns (max_abs, rel_l2)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values {extra}"
    ma = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rl = rel_l2(got, ref)
    t = TOL[dtype]
    assert ma <= t["abs"], f"{name}: max-abs {ma:.3g} > {t['abs']} (rel-L2 {rl:.3g}) {extra}"
    if t["rel"] is not None:
        assert rl <= t["rel"], f"{name}: rel-L2 {rl:.3g} > {t['rel']} (max-abs {ma:.3g}) {extra}"
    return ma, rl


def compare_lse(got, ref, dtype, extra=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    ninf_ref = np.isneginf(ref)
    np.testing.assert_array_equal(np.isneginf(got), ninf_ref, err_msg="LSE -inf rows " + extra)
    fin = ~ninf_ref
    return compare("LSE", got[fin], ref[fin], dtype, extra)


def device_inputs(B, H, T, d, dtype, std, seed=0):
    q, k, v, do = synth.draw(B, H, T, d, dtype, std, seed)
    return (q, k, v, do), tuple(x.cuda() for x in (q, k, v, do))


def run_library(layout, qd, kd, vd, dod, backward=True, forward=None):
    """Forward (or the given (o, lse)) and backward through the C ABI."""
    o, lse = forward if forward is not None else st.st_sparse_attn_fwd(layout, qd, kd, vd)
    grads = None
    if backward:
        grads = st.st_sparse_attn_bwd(layout, qd, kd, vd, o, lse, dod)
    torch.cuda.synchronize()
    assert st.st_last_device_status() == st.ST_OK
    return o, lse, grads


def f32(x):
    return synth.as_f32(x)
