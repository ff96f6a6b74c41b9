"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad calls before touching the GPU (no compute call runs here)."""
import ctypes
import os
import re

import pytest

import factorized_sparse_self_b200 as st

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include",
                      "sparse_transformer_attn.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(st_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported_and_bound():
    names = declared_symbols()
    assert len(names) >= 14
    L = st.lib()
    for n in names:
        assert hasattr(L, n), n
        assert n in st.SIGNATURES, n


def test_status_strings_and_version():
    assert st.status_string(st.ST_OK) == "ok"
    assert "timed out" in st.status_string(st.ST_ERR_DEVICE_TIMEOUT)
    assert st.st_version().count(".") == 2


def test_host_only_layout_is_rejected_by_fwd():
    L = st.st_pattern_layout_host("fixed", "split", 256, 16, 4)
    dummy = ctypes.c_void_p(16)
    code = st.lib().st_sparse_attn_fwd(L.handle, st.ST_BF16, 1, 2, 256, 64, 0.0, dummy, dummy,
                                       dummy, dummy, dummy, None)
    assert code == st.ST_ERR_INVALID
    n = ctypes.c_size_t()
    assert st.lib().st_sparse_attn_bwd_workspace(L.handle, st.ST_BF16, 1, 2, 256, 64,
                                                 ctypes.byref(n)) == st.ST_OK
    # D, 3 fp32 accumulators, the work counter (256 bytes) and 1024 per-block
    # maxima of |dout| (4096 bytes)
    assert n.value == 2 * 256 * 4 + 3 * 2 * 256 * 64 * 4 + 256 + 4096
    assert st.lib().st_sparse_attn_bwd_workspace(L.handle, st.ST_BF16, 1, 2, 128, 64,
                                                 ctypes.byref(n)) == st.ST_ERR_INVALID


def test_null_arguments():
    assert st.lib().st_pattern_layout_host(None, None) == st.ST_ERR_INVALID
    assert st.lib().st_layout_counts(None, None, None) == st.ST_ERR_INVALID
    st.lib().st_layout_destroy(None)


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="CPU-only check")
def test_device_layout_without_gpu_reports_cuda_error():
    with pytest.raises(st.StatusError) as e:
        st.Layout("fixed", "split", 256, 16, 4, host_only=False, stream=type("S", (), {"cuda_stream": 0})())
    assert e.value.code == st.ST_ERR_CUDA
