"""GPU parity for the head-range calls: strided and fixed patterns on
disjoint heads of one set of tensors ("Sparse Transformer", llm-arch-kb,
section 2, "How the two patterns are combined"), against the oracle run on
the full tensors with each pattern and sliced by head (so split layouts keep
the parity of the global head index). Rows of heads outside a call's range
must keep their previous contents."""
import numpy as np
import pytest
import torch

import factorized_sparse_self_b200 as st
from gpu_util import compare, compare_lse, device_inputs, f32

pytestmark = pytest.mark.gpu

SENTINEL = 7.0

# (first pattern, second pattern), heads of the first, B, H, T, d, dtype, std
CASES = [
    ((("strided", "split", 32, 1), ("fixed", "split", 64, 8)), 2, 2, 4, 1024, 64, "bf16", 0.5),
    ((("strided", "merged", 128, 1), ("fixed", "merged", 128, 8)), 2, 1, 4, 1536, 64, "bf16",
     0.5),
    ((("fixed", "split", 64, 8), ("strided", "split", 16, 1)), 2, 1, 6, 768, 64, "bf16", 0.5),
    ((("strided", "split", 16, 1), ("fixed", "merged", 32, 4)), 2, 2, 4, 256, 32, "f32", 1.0),
]


def _filled(shape, dtype, device):
    return torch.full(shape, SENTINEL, dtype=dtype, device=device)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0][0][0]}-{c[0][1][0]}-H{c[3]}-{c[6]}")
def test_mixed_pattern_heads(orc, case):
    (pa, pb), first, B, H, T, d, dtype, std = case
    ranges = [(0, first), (first, H - first)]
    (q, k, v, do), (qd, kd, vd, dod) = device_inputs(B, H, T, d, dtype, std, seed=0)
    o = _filled(qd.shape, qd.dtype, qd.device)
    lse = _filled((B, H, T), torch.float32, qd.device)
    dq, dk, dv = (_filled(qd.shape, qd.dtype, qd.device) for _ in range(3))
    layouts = [st.st_pattern_layout(kind, mode, T, l, c) for kind, mode, l, c in (pa, pb)]
    for n, (L, rng) in enumerate(zip(layouts, ranges)):
        st.st_sparse_attn_fwd(L, qd, kd, vd, o=o, lse=lse, heads=rng)
        st.st_sparse_attn_bwd(L, qd, kd, vd, o, lse, dod, dq=dq, dk=dk, dv=dv, heads=rng)
        torch.cuda.synchronize()
        assert st.st_last_device_status() == st.ST_OK
        if n == 0:  # the second range is still untouched
            h0, hn = ranges[1]
            for t in (o, dq, dk, dv, lse):
                assert torch.all(t[:, h0:h0 + hn] == SENTINEL)
    for (kind, mode, l, c), (h0, hn) in zip((pa, pb), ranges):
        ro, rlse = orc.forward(kind, mode, f32(q), f32(k), f32(v), l, c)
        rdq, rdk, rdv = orc.backward(kind, mode, f32(q), f32(k), f32(v), f32(do), l, c)
        sl = slice(h0, h0 + hn)
        tag = f"{kind}-{mode} heads {h0}..{h0 + hn - 1}"
        compare("O", f32(o.cpu())[:, sl], ro[:, sl], dtype, tag)
        compare_lse(lse.cpu().numpy()[:, sl], rlse[:, sl], dtype, tag)
        compare("dQ", f32(dq.cpu())[:, sl], rdq[:, sl], dtype, tag)
        compare("dK", f32(dk.cpu())[:, sl], rdk[:, sl], dtype, tag)
        compare("dV", f32(dv.cpu())[:, sl], rdv[:, sl], dtype, tag)


def test_odd_head_range_keeps_global_parity(orc):
    """A split layout on heads 1..2: head 1 (odd) takes A2, head 2 (even) A1."""
    B, H, T, d = 1, 4, 512, 64
    (q, k, v, do), (qd, kd, vd, dod) = device_inputs(B, H, T, d, "bf16", 0.5, seed=0)
    L = st.st_pattern_layout("fixed", "split", T, 64, 8)
    o = _filled(qd.shape, qd.dtype, qd.device)
    lse = _filled((B, H, T), torch.float32, qd.device)
    dq, dk, dv = (_filled(qd.shape, qd.dtype, qd.device) for _ in range(3))
    st.st_sparse_attn_fwd(L, qd, kd, vd, o=o, lse=lse, heads=(1, 2))
    st.st_sparse_attn_bwd(L, qd, kd, vd, o, lse, dod, dq=dq, dk=dk, dv=dv, heads=(1, 2))
    torch.cuda.synchronize()
    assert st.st_last_device_status() == st.ST_OK
    for t in (o, lse, dq, dk, dv):
        assert torch.all(t[:, 0] == SENTINEL) and torch.all(t[:, 3] == SENTINEL)
    ro, rlse = orc.forward("fixed", "split", f32(q), f32(k), f32(v), 64, 8)
    rdq, rdk, rdv = orc.backward("fixed", "split", f32(q), f32(k), f32(v), f32(do), 64, 8)
    sl = slice(1, 3)
    compare("O", f32(o.cpu())[:, sl], ro[:, sl], "bf16")
    compare_lse(lse.cpu().numpy()[:, sl], rlse[:, sl], "bf16")
    compare("dQ", f32(dq.cpu())[:, sl], rdq[:, sl], "bf16")
    compare("dK", f32(dk.cpu())[:, sl], rdk[:, sl], "bf16")
    compare("dV", f32(dv.cpu())[:, sl], rdv[:, sl], "bf16")


def test_bad_head_ranges_rejected():
    B, H, T, d = 1, 4, 256, 64
    _, (qd, kd, vd, dod) = device_inputs(B, H, T, d, "bf16", 0.5, seed=0)
    L = st.st_pattern_layout("fixed", "split", T, 64, 8)
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=qd.device)
    for rng in ((0, 0), (3, 2), (-1, 2), (4, 1)):
        with pytest.raises(st.StatusError) as e:
            st.st_sparse_attn_fwd(L, qd, kd, vd, o=o, lse=lse, heads=rng)
        assert e.value.code == st.ST_ERR_INVALID
