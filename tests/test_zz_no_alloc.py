"""The backward entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or keep a workspace between calls (a
plugin whose host application owns all device memory, a path that must not
allocate). st_sparse_attn_bwd_noalloc serves them from a fixed library-owned
scratch array. Here it is called through the C ABI twice in a row and its
gradients are compared with those of the regular, workspace-taking
st_sparse_attn_bwd on the same inputs, within the parity tolerances.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test. It passes alone in a fresh process
and after the rest of the suite.
"""
import pytest
import torch

import factorized_sparse_self_b200 as st
from gpu_util import compare, device_inputs, f32

pytestmark = pytest.mark.gpu

CASES = [
    # kind, mode, B, H, T, d, l, c, dtype, std
    ("fixed", "merged", 1, 4, 4096, 64, 128, 8, "bf16", 0.5),
    ("strided", "split", 1, 2, 256, 32, 16, 1, "f32", 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-T{c[4]}-{c[8]}")
def test_noalloc_backward_matches_workspace_backward(case):
    kind, mode, B, H, T, d, l, c, dtype, std = case
    _, (qd, kd, vd, dod) = device_inputs(B, H, T, d, dtype, std, seed=3)
    L = st.st_pattern_layout(kind, mode, T, l, c)
    o, lse = st.st_sparse_attn_fwd(L, qd, kd, vd)
    ref = st.st_sparse_attn_bwd(L, qd, kd, vd, o, lse, dod)
    torch.cuda.synchronize()
    assert st.st_last_device_status() == st.ST_OK
    ref = [f32(x.cpu()) for x in ref]
    for call in range(2):
        outs = [torch.full_like(qd, float("nan")) for _ in range(3)]
        st.st_sparse_attn_bwd_noalloc(L, qd, kd, vd, o, lse, dod, *outs)
        torch.cuda.synchronize()
        assert st.st_last_device_status() == st.ST_OK
        for name, got, want in zip(("dQ", "dK", "dV"), outs, ref):
            compare(name, f32(got.cpu()), want, dtype, f"no-alloc call {call + 1}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    kind, mode, B, H, T, d, l, c = "fixed", "merged", 2, 8, 12288, 64, 128, 8
    L = st.st_pattern_layout(kind, mode, T, l, c)
    q = torch.zeros(B, H, T, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    outs = [torch.empty_like(q) for _ in range(3)]
    with pytest.raises(st.StatusError) as e:
        st.st_sparse_attn_bwd_noalloc(L, q, q, q, q, lse, q, *outs)
    assert e.value.code == st.ST_ERR_WORKSPACE
