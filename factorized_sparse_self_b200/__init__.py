"""Python binding of libsparse_transformer_attn.so (factorized sparse attention, B200).

Argument marshalling only: every step of the forward and backward pass runs
in the library's CUDA kernels. PyTorch supplies device memory and the current
stream. The names mirror the C ABI in include/sparse_transformer_attn.h.
There is no fallback: if the shared library is missing the import of any
entry point raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsparse_transformer_attn.so")

ST_OK, ST_ERR_INVALID, ST_ERR_UNSUPPORTED, ST_ERR_CUDA, ST_ERR_DEVICE_TIMEOUT, ST_ERR_WORKSPACE = range(6)
ST_STRIDED, ST_FIXED, ST_DENSE_CAUSAL = 0, 1, 2
ST_HEADS_SPLIT, ST_HEADS_MERGED = 0, 1
ST_F32, ST_BF16, ST_F16 = 0, 1, 2
KINDS = {"strided": ST_STRIDED, "fixed": ST_FIXED, "dense": ST_DENSE_CAUSAL}
MODES = {"split": ST_HEADS_SPLIT, "merged": ST_HEADS_MERGED}
VIEWS = {0: "natural", 1: "summary", 2: "class"}
RULES = {0: "causal", 1: "band", 2: "block", 3: "stride", 4: "stride_far", 5: "summary",
         6: "summary_earlier"}

# Every symbol the header declares, with its ctypes signature.
_i32, _i64, _u64, _P = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
SIGNATURES = {
    "st_pattern_layout": (ctypes.c_int, [_P, _P, _P]),
    "st_pattern_layout_host": (ctypes.c_int, [_P, _P]),
    "st_layout_destroy": (None, [_P]),
    "st_layout_counts": (ctypes.c_int, [_P, _P, _P]),
    "st_layout_segment_info": (ctypes.c_int, [_P, _i32, _i32, _P, _P, _P]),
    "st_layout_export": (ctypes.c_int, [_P, _i32, _i32, _i32, _P, _P, _P, _P, _P]),
    "st_layout_rows": (ctypes.c_int, [_P, _i32, _i32, _P, _P]),
    "st_layout_nnz": (ctypes.c_int, [_P, _i32, _P]),
    "st_sparse_attn_fwd": (ctypes.c_int, [_P, ctypes.c_int, _i32, _i32, _i32, _i32,
                                          ctypes.c_float, _P, _P, _P, _P, _P, _P]),
    "st_sparse_attn_bwd_workspace": (ctypes.c_int, [_P, ctypes.c_int, _i32, _i32, _i32, _i32,
                                                    _P]),
    "st_sparse_attn_bwd": (ctypes.c_int, [_P, ctypes.c_int, _i32, _i32, _i32, _i32,
                                          ctypes.c_float, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                          _P, ctypes.c_size_t, _P]),
    "st_sparse_attn_fwd_heads": (ctypes.c_int, [_P, ctypes.c_int, _i32, _i32, _i32, _i32, _i32,
                                                _i32, ctypes.c_float, _P, _P, _P, _P, _P, _P]),
    "st_sparse_attn_bwd_heads": (ctypes.c_int, [_P, ctypes.c_int, _i32, _i32, _i32, _i32, _i32,
                                                _i32, ctypes.c_float, _P, _P, _P, _P, _P, _P, _P,
                                                _P, _P, _P, ctypes.c_size_t, _P]),
    "st_sparse_attn_bwd_noalloc": (ctypes.c_int, [_P, ctypes.c_int, _i32, _i32, _i32, _i32,
                                                  ctypes.c_float, _P, _P, _P, _P, _P, _P, _P, _P,
                                                  _P, _P]),
    "st_last_device_status": (ctypes.c_int, [_P]),
    "st_set_wait_limit": (ctypes.c_int, [_u64, _i32]),
    "st_layout_launches": (ctypes.c_int, [_P, ctypes.c_int, _P, _P]),
    "st_kernel_timing": (ctypes.c_int, [_i32]),
    "st_kernel_elapsed_ms": (ctypes.c_int, [_i32, _P]),
    "st_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "st_version": (ctypes.c_char_p, []),
}


class _Desc(ctypes.Structure):
    _fields_ = [("kind", _i32), ("head_mode", _i32), ("T", _i32), ("l", _i32), ("c", _i32)]


class StatusError(RuntimeError):
    def __init__(self, code, where):
        self.code = int(code)
        msg = status_string(code) if _lib is not None else str(code)
        super().__init__(f"{where}: status {code} ({msg})")


_lib = None


def lib():
    """The loaded shared library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m factorized_sparse_self_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(code) -> str:
    return lib().st_status_string(int(code)).decode()


def _check(code, where):
    if code != ST_OK:
        raise StatusError(code, where)


def _stream_ptr(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class Layout:
    """Owner of one st_layout (host copy, and the device copy unless host_only)."""

    def __init__(self, kind, mode, T, l, c=1, host_only=False, stream=None):
        self.kind = KINDS[kind] if isinstance(kind, str) else int(kind)
        self.mode = MODES[mode] if isinstance(mode, str) else int(mode)
        self.T, self.l, self.c = int(T), int(l), int(c)
        d = _Desc(self.kind, self.mode, self.T, self.l, self.c)
        h = ctypes.c_void_p()
        if host_only:
            _check(lib().st_pattern_layout_host(ctypes.byref(d), ctypes.byref(h)),
                   "st_pattern_layout_host")
        else:
            _check(lib().st_pattern_layout(ctypes.byref(d), ctypes.byref(h), _stream_ptr(stream)),
                   "st_pattern_layout")
        self.handle = h
        self.host_only = host_only

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value and _lib is not None:
            _lib.st_layout_destroy(h)
            self.handle = None

    def counts(self):
        a, b = _i32(), _i32()
        _check(lib().st_layout_counts(self.handle, ctypes.byref(a), ctypes.byref(b)),
               "st_layout_counts")
        return a.value, b.value

    def segment_info(self, hc, seg):
        qv, kv, r = _i32(), _i32(), _i32()
        _check(lib().st_layout_segment_info(self.handle, hc, seg, ctypes.byref(qv),
                                            ctypes.byref(kv), ctypes.byref(r)),
               "st_layout_segment_info")
        return qv.value, kv.value, r.value

    def nnz(self, hc):
        n = _i64()
        _check(lib().st_layout_nnz(self.handle, hc, ctypes.byref(n)), "st_layout_nnz")
        return n.value

    def launches(self, dtype):
        """(forward, backward) kernel launches per call for this dtype code."""
        f, b = _i32(), _i32()
        _check(lib().st_layout_launches(self.handle, dtype, ctypes.byref(f), ctypes.byref(b)),
               "st_layout_launches")
        return f.value, b.value

    # row lists of st_layout_rows
    ROWS_Q_ACC, ROWS_K_ACC, ROWS_Q_ZERO, ROWS_K_ZERO = 0, 1, 2, 3

    def rows(self, hc, which):
        """Natural rows of head class hc in row list `which` (st_layout_rows)."""
        n = _i64(0)
        _check(lib().st_layout_rows(self.handle, hc, which, None, ctypes.byref(n)),
               "st_layout_rows")
        out = np.zeros(max(n.value, 1), dtype=np.int32)
        n2 = _i64(out.size)
        _check(lib().st_layout_rows(self.handle, hc, which, out.ctypes.data_as(_P),
                                    ctypes.byref(n2)), "st_layout_rows")
        return out[:n.value]

    def export(self, hc, seg, transpose=False):
        """(ptr, idx, flags, live) numpy arrays of one segment (seg = -1: natural tiling)."""
        sizes = (_i64 * 2)(0, 0)
        code = lib().st_layout_export(self.handle, hc, seg, int(transpose), None, None, None,
                                      None, sizes)
        _check(code, "st_layout_export")
        ptr = np.zeros(sizes[0], dtype=np.int32)
        idx = np.zeros(max(sizes[1], 1), dtype=np.int32)
        flags = np.zeros(max(sizes[1], 1), dtype=np.uint8)
        live = np.zeros(max(sizes[1], 1), dtype=np.int32)
        sizes2 = (_i64 * 2)(sizes[0], max(sizes[1], 1))
        _check(lib().st_layout_export(self.handle, hc, seg, int(transpose),
                                      ptr.ctypes.data_as(_P), idx.ctypes.data_as(_P),
                                      flags.ctypes.data_as(_P), live.ctypes.data_as(_P), sizes2),
               "st_layout_export")
        n = sizes[1]
        return ptr, idx[:n], flags[:n], live[:n]


def st_pattern_layout(kind, mode, T, l, c=1, stream=None) -> Layout:
    return Layout(kind, mode, T, l, c, host_only=False, stream=stream)


def st_pattern_layout_host(kind, mode, T, l, c=1) -> Layout:
    return Layout(kind, mode, T, l, c, host_only=True)


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return ST_F32
    if t.dtype == torch.bfloat16:
        return ST_BF16
    if t.dtype == torch.float16:
        return ST_F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t, name, like=None):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if like is not None and (t.dtype != like.dtype or t.shape != like.shape):
        raise ValueError(f"{name} must match q in dtype and shape")
    return ctypes.c_void_p(t.data_ptr())


def st_sparse_attn_fwd(layout: Layout, q, k, v, scale=None, o=None, lse=None, stream=None,
                       heads=None):
    """O [B,H,T,d] (dtype of q) and LSE [B,H,T] float32 for all heads, or for
    heads = (begin, count) only (st_sparse_attn_fwd_heads; other heads' rows
    of o and lse are left as they are)."""
    import torch
    B, H, T, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    args = [_need(x, n, q) for x, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"))]
    sc = float(scale) if scale else 0.0
    if heads is None:
        code = lib().st_sparse_attn_fwd(layout.handle, _dtype_code(q), B, H, T, d, sc, args[0],
                                        args[1], args[2], args[3], _need(lse, "lse"),
                                        _stream_ptr(stream))
        _check(code, "st_sparse_attn_fwd")
    else:
        code = lib().st_sparse_attn_fwd_heads(layout.handle, _dtype_code(q), B, H, heads[0],
                                              heads[1], T, d, sc, args[0], args[1], args[2],
                                              args[3], _need(lse, "lse"), _stream_ptr(stream))
        _check(code, "st_sparse_attn_fwd_heads")
    return o, lse


def st_sparse_attn_bwd_workspace(layout: Layout, dtype, B, H, T, d) -> int:
    n = ctypes.c_size_t()
    code = lib().st_sparse_attn_bwd_workspace(layout.handle, dtype, B, H, T, d, ctypes.byref(n))
    _check(code, "st_sparse_attn_bwd_workspace")
    return n.value


def st_sparse_attn_bwd(layout: Layout, q, k, v, o, lse, dout, scale=None, workspace=None,
                       dq=None, dk=None, dv=None, stream=None, heads=None):
    """dQ, dK, dV (dtype of q), with P recomputed from LSE; for heads =
    (begin, count) only when given (st_sparse_attn_bwd_heads)."""
    import torch
    B, H, T, d = q.shape
    if workspace is None:
        nb = st_sparse_attn_bwd_workspace(layout, _dtype_code(q), B, H, T, d)
        workspace = torch.empty(nb, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    ptrs = [_need(x, n, q) for x, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"),
                                        (dq, "dq"), (dk, "dk"), (dv, "dv"))]
    sc = float(scale) if scale else 0.0
    ws = ctypes.c_void_p(workspace.data_ptr())
    if heads is None:
        code = lib().st_sparse_attn_bwd(layout.handle, _dtype_code(q), B, H, T, d, sc, ptrs[0],
                                        ptrs[1], ptrs[2], ptrs[3], _need(lse, "lse"), ptrs[4],
                                        ptrs[5], ptrs[6], ptrs[7], ws, workspace.numel(),
                                        _stream_ptr(stream))
        _check(code, "st_sparse_attn_bwd")
    else:
        code = lib().st_sparse_attn_bwd_heads(layout.handle, _dtype_code(q), B, H, heads[0],
                                              heads[1], T, d, sc, ptrs[0], ptrs[1], ptrs[2],
                                              ptrs[3], _need(lse, "lse"), ptrs[4], ptrs[5],
                                              ptrs[6], ptrs[7], ws, workspace.numel(),
                                              _stream_ptr(stream))
        _check(code, "st_sparse_attn_bwd_heads")
    return dq, dk, dv


def st_sparse_attn_bwd_noalloc(layout: Layout, q, k, v, o, lse, dout, dq, dk, dv, scale=None,
                               stream=None):
    """Backward for callers that cannot allocate device memory: same result as
    st_sparse_attn_bwd, with the scratch in a fixed 64 MiB library-owned
    device array instead of a caller workspace. The caller passes every output
    buffer; nothing is allocated here or in the library. Calls whose GPU work
    overlaps share that array and race, so serialise them."""
    B, H, T, d = q.shape
    ptrs = [_need(x, n, q) for x, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"),
                                        (dq, "dq"), (dk, "dk"), (dv, "dv"))]
    code = lib().st_sparse_attn_bwd_noalloc(layout.handle, _dtype_code(q), B, H, T, d,
                                            float(scale) if scale else 0.0, ptrs[0], ptrs[1],
                                            ptrs[2], ptrs[3], _need(lse, "lse"), ptrs[4], ptrs[5],
                                            ptrs[6], ptrs[7], _stream_ptr(stream))
    _check(code, "st_sparse_attn_bwd_noalloc")
    return dq, dk, dv


def st_last_device_status(stream=None) -> int:
    return int(lib().st_last_device_status(_stream_ptr(stream)))


def st_set_wait_limit(ns: int, force_timeout: bool = False) -> None:
    _check(lib().st_set_wait_limit(int(ns), int(bool(force_timeout))), "st_set_wait_limit")


def st_kernel_timing(enable: bool) -> None:
    _check(lib().st_kernel_timing(int(bool(enable))), "st_kernel_timing")


def st_kernel_elapsed_ms(kernel: int) -> float:
    ms = ctypes.c_float()
    _check(lib().st_kernel_elapsed_ms(int(kernel), ctypes.byref(ms)), "st_kernel_elapsed_ms")
    return ms.value


def st_version() -> str:
    return lib().st_version().decode()
