"""GPU parity of the fp16 variant (the same tensor-core kernels with fp16
operands, P and dS rounded to fp16, fp32 accumulation) against the oracle fed
the fp16-rounded inputs."""
import numpy as np
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


def test_fp16_headline_shape_sampled(orc):
    """The headline workload's shape in fp16, sampled rows."""
    B, H, T, d, l, c = 4, 8, 4096, 64, 64, 8
    (q, k, v, do), (qd, kd, vd, dod) = device_inputs(B, H, T, d, "f16", 64 ** -0.25, seed=0)
    L = st.st_pattern_layout("fixed", "split", T, l, c)
    o, lse, (dq, dk, dv) = run_library(L, qd, kd, vd, dod)
    rng = np.random.default_rng(5)
    n = 16
    bh = rng.integers(0, B * H, n)
    rows = np.concatenate([rng.integers(0, T, n - 3), [T - 1, l - 1, l]])
    qf, kf, vf, dof = f32(q), f32(k), f32(v), f32(do)
    ro, rlse = orc.forward_rows("fixed", "split", qf, kf, vf, l, c, bh, rows)
    compare("O rows", f32(o.cpu()).reshape(B * H, T, d)[bh, rows], ro, "f16")
    compare_lse(lse.cpu().numpy().reshape(B * H, T)[bh, rows], rlse, "f16")
    rdq = orc.backward_query_rows("fixed", "split", qf, kf, vf, dof, l, c, bh, rows)
    compare("dQ rows", f32(dq.cpu()).reshape(B * H, T, d)[bh, rows], rdq, "f16")
    kb, kr = bh[:4], np.array([l - 1, 0, T // 2, T - 1])
    rdk, rdv = orc.backward_key_rows("fixed", "split", qf, kf, vf, dof, l, c, kb, kr)
    compare("dK rows", f32(dk.cpu()).reshape(B * H, T, d)[kb, kr], rdk, "f16")
    compare("dV rows", f32(dv.cpu()).reshape(B * H, T, d)[kb, kr], rdv, "f16")
