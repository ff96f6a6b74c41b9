"""GPU parity of the fp16 variant (the same tensor-core kernels with fp16
operands, P and dS rounded to fp16, fp32 accumulation) against the oracle fed
the fp16-rounded inputs."""
import pytest
import torch

import factorized_sparse_self_b200 as st
from gpu_util import compare, compare_lse, device_inputs, f32, run_library

pytestmark = pytest.mark.gpu

# kind, mode, B, H, T, l, c, std
CASES = [
    ("fixed", "split", 1, 4, 1024, 64, 8, 64 ** -0.25),
    ("fixed", "merged", 1, 2, 1536, 128, 8, 0.5),
    ("strided", "split", 1, 4, 1536, 192, 1, 0.5),
    ("strided", "merged", 1, 2, 2048, 256, 1, 0.5),
    ("dense", "merged", 1, 2, 640, 1, 1, 0.5),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c[:7])))
def test_fp16_parity_small(orc, case):
    kind, mode, B, H, T, l, c, std = case
    d = 64
    (q, k, v, do), (qd, kd, vd, dod) = device_inputs(B, H, T, d, "f16", std, seed=0)
    assert qd.dtype == torch.float16
    L = st.st_pattern_layout(kind, mode, T, l, c)
    o, lse, (dq, dk, dv) = run_library(L, qd, kd, vd, dod)
    assert o.dtype == torch.float16 and dq.dtype == torch.float16
    ro, rlse = orc.forward(kind, mode, f32(q), f32(k), f32(v), l, c)
    rdq, rdk, rdv = orc.backward(kind, mode, f32(q), f32(k), f32(v), f32(do), l, c)
    tag = str(case)
    compare("O", f32(o.cpu()), ro, "f16", tag)
    compare_lse(lse.cpu().numpy(), rlse, "f16", tag)
    compare("dQ", f32(dq.cpu()), rdq, "f16", tag)
    compare("dK", f32(dk.cpu()), rdk, "f16", tag)
    compare("dV", f32(dv.cpu()), rdv, "f16", tag)


@pytest.mark.parametrize("case", [
    ("fixed", "split", 4, 8, 4096, 64, 8, 64 ** -0.25),
    ("fixed", "merged", 2, 8, 12288, 128, 8, 0.5),
    ("strided", "split", 4, 16, 12288, 192, 1, 0.5),
    ("strided", "merged", 1, 8, 65536, 256, 1, 0.5),
], ids=["fixed-split-T4096", "fixed-merged-T12288", "strided-split-T12288",
        "strided-merged-T65536"])
def test_fp16_full_size(orc, case):
    """The benchmark's four 16-bit shapes in fp16: every element of O, LSE, dQ,
    dK and dV against the oracle fed the fp16-rounded inputs."""
    kind, mode, B, H, T, l, c, std = case
    d = 64
    (q, k, v, do), (qd, kd, vd, dod) = device_inputs(B, H, T, d, "f16", std, seed=0)
    L = st.st_pattern_layout(kind, mode, T, l, c)
    o, lse, (dq, dk, dv) = run_library(L, qd, kd, vd, dod)
    qf, kf, vf, dof = f32(q), f32(k), f32(v), f32(do)
    del q, k, v, do
    tag = str(case)
    ro, rlse = orc.forward(kind, mode, qf, kf, vf, l, c)
    compare("O", f32(o.cpu()), ro, "f16", tag)
    compare_lse(lse.cpu().numpy(), rlse, "f16", tag)
    del ro, rlse
    rdq, rdk, rdv = orc.backward(kind, mode, qf, kf, vf, dof, l, c)
    compare("dQ", f32(dq.cpu()), rdq, "f16", tag)
    compare("dK", f32(dk.cpu()), rdk, "f16", tag)
    compare("dV", f32(dv.cpu()), rdv, "f16", tag)
