"""Second, numpy-only restatement of the oracle, for tiny sizes (T <= 512).

TEST INFRASTRUCTURE, like the rest of ``oracle/``. Where ``oracle.cpp``
enumerates each index set constructively (window, stride walk, block and
summary loops), this module tests membership of every pair (i, j) against the
set definitions and runs the attention as dense float64 numpy algebra over
the resulting boolean mask. The two must agree; each is also pinned
independently by tests/test_oracle_pins.py.

Set definitions (positions 0-indexed, j <= i everywhere):
  strided A1: max(0, i-l) <= j            (local window, "Sparse Transformer",
                                           llm-arch-kb section 2, Pattern A)
  strided A2: (i - j) mod l == 0          (every l-th key back, same place)
  fixed A1:   floor(j/l) == floor(i/l)    (own block, section 2, Pattern B)
  fixed A2:   j mod l >= l - c            (last c positions of each block)
  split heads: even h -> A1, odd h -> A2; merged: A1 or A2.
"""
from __future__ import annotations

import numpy as np


def member(kind: str, mode: str, l: int, c: int, h: int, i: int, j: int) -> bool:
    if j > i or j < 0:
        return False
    if kind == "dense":
        return True
    if kind == "strided":
        a1 = j >= max(0, i - l)
        a2 = (i - j) % l == 0
    else:
        a1 = (j // l) == (i // l)
        a2 = (j % l) >= l - c
    if mode == "merged":
        return a1 or a2
    return a1 if h % 2 == 0 else a2


def mask(kind: str, mode: str, T: int, l: int, c: int, h: int) -> np.ndarray:
    """Boolean [T, T] mask, entry (i, j) true when j is in S_{h,i}."""
    m = np.zeros((T, T), dtype=bool)
    for i in range(T):
        for j in range(i + 1):
            m[i, j] = member(kind, mode, l, c, h, i, j)
    return m


def forward(kind, mode, q, k, v, l, c, scale=None):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, T, d = q.shape
    scale = scale if scale else 1.0 / np.sqrt(d)
    o = np.zeros((B, H, T, d))
    lse = np.zeros((B, H, T))
    for b in range(B):
        for h in range(H):
            m = mask(kind, mode, T, l, c, h)
            s = scale * q[b, h] @ k[b, h].T
            s = np.where(m, s, -np.inf)
            mx = s.max(axis=1)
            empty = ~m.any(axis=1)
            mx = np.where(empty, 0.0, mx)
            e = np.where(m, np.exp(s - mx[:, None]), 0.0)
            z = e.sum(axis=1)
            p = e / np.where(empty, 1.0, z)[:, None]
            o[b, h] = p @ v[b, h]
            lse[b, h] = np.where(empty, -np.inf, mx + np.log(np.where(empty, 1.0, z)))
    return o, lse


def backward(kind, mode, q, k, v, dout, l, c, scale=None):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, H, T, d = q.shape
    scale = scale if scale else 1.0 / np.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(q)
    dv = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            m = mask(kind, mode, T, l, c, h)
            s = scale * q[b, h] @ k[b, h].T
            s = np.where(m, s, -np.inf)
            empty = ~m.any(axis=1)
            mx = np.where(empty, 0.0, s.max(axis=1))
            e = np.where(m, np.exp(s - mx[:, None]), 0.0)
            z = np.where(empty, 1.0, e.sum(axis=1))
            p = e / z[:, None]
            dp = dout[b, h] @ v[b, h].T
            D = (p * dp).sum(axis=1)
            ds = p * (dp - D[:, None])
            dq[b, h] = scale * ds @ k[b, h]
            dk[b, h] = scale * ds.T @ q[b, h]
            dv[b, h] = p.T @ dout[b, h]
    return dq, dk, dv
