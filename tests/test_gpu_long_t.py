"""Very long sequences: strided merged attention at T = 2^20 with l = 2^10
(= sqrt T, the pages' choice of stride for the O(T sqrt T) cost; they report
sequences of a million samples), checked on sampled rows against the oracle,
which computes those rows one by one."""
import numpy as np
import pytest
import torch

import factorized_sparse_self_b200 as st
from gpu_util import compare, compare_lse, device_inputs, f32, run_library

pytestmark = pytest.mark.gpu


def test_strided_merged_one_million_positions(orc):
    B, H, T, d, l = 1, 2, 1 << 20, 64, 1 << 10
    (q, k, v, do), (qd, kd, vd, dod) = device_inputs(B, H, T, d, "bf16", 0.5, seed=0)
    L = st.st_pattern_layout("strided", "merged", T, l, 1)
    o, lse, (dq, dk, dv) = run_library(L, qd, kd, vd, dod)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(3)
    n = 16
    bh = rng.integers(0, B * H, n)
    rows = np.concatenate([rng.integers(0, T, n - 4), [0, l, T - l - 1, T - 1]])
    qf, kf, vf, dof = f32(q), f32(k), f32(v), f32(do)
    ro, rlse = orc.forward_rows("strided", "merged", qf, kf, vf, l, 1, bh, rows)
    compare("O rows", f32(o.cpu()).reshape(B * H, T, d)[bh, rows], ro, "bf16")
    compare_lse(lse.cpu().numpy().reshape(B * H, T)[bh, rows], rlse, "bf16")
    rdq = orc.backward_query_rows("strided", "merged", qf, kf, vf, dof, l, 1, bh, rows)
    compare("dQ rows", f32(dq.cpu()).reshape(B * H, T, d)[bh, rows], rdq, "bf16")
    kb, kr = bh[:4], np.array([0, l - 1, T // 2, T - 1])
    rdk, rdv = orc.backward_key_rows("strided", "merged", qf, kf, vf, dof, l, 1, kb, kr)
    compare("dK rows", f32(dk.cpu()).reshape(B * H, T, d)[kb, kr], rdk, "bf16")
    compare("dV rows", f32(dv.cpu()).reshape(B * H, T, d)[kb, kr], rdv, "bf16")
