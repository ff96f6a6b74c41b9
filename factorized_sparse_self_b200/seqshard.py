"""Sequence sharding of strided attention across ranks (one long sequence).

A head's sequence of T positions is cut into N contiguous chunks of n = T / N
positions, one per rank, for sequences too long for one device. The strided
set of query i ("Sparse Transformer", llm-arch-kb, section 2, "Pattern A -
strided": the local window plus every l-th earlier key) splits into two
parts that need different data on a rank:

* the band  max(0, i-l) <= j <= i: the rank's own rows plus a halo, the last
  l rows of K and V of the previous rank (point-to-point exchange);
* the stride keys j = i - m*l: in residue-class order (position p*l + r is row
  p of class r) every class is a dense causal problem of length T / l, so an
  all-to-all regroups the rows by class, rank k taking classes
  [k*l/N, (k+1)*l/N) of every chunk; a class row p attends rows p' <= p - s,
  s = 2 for merged heads (keys i - l and i are in the band already) and
  s = 0 for the A2 heads of split heads.

Forward: halo exchange, band attention over [halo, own] keys, all-to-all into
class order, class attention, all-to-all back, and a log-sum-exp merge of the
two partial results (O, LSE) of every row. Backward (with the attention
recomputed from the merged LSE, milestone page "The idea"): the band and
class gradients of the same merged O, LSE; the halo rows' dK, dV go back to
the previous rank, the class-order gradients go back by the inverse
all-to-all, and the parts are summed.

The exchanges use torch.distributed (NCCL between GPUs, gloo on CPU). The
attention and the combining arithmetic are not here: they come from an `ops`
object (see `ShardOps`), so this module holds only the partition and the data
movement. Requirements: n % l == 0 (chunks hold whole l-blocks), l % N == 0
(classes split evenly) and, for N > 1, n >= l (the halo comes from one rank).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


class ShardOps:
    """The arithmetic the sharded driver needs, on tensors of one rank.

    band_fwd(q, k, v, l) -> (o, lse)          q, k, v [B, H, T, d]; row i attends
                                              keys max(0, i-l) .. i of the same T rows
    band_bwd(q, k, v, o, lse, do, l) -> (dq, dk, dv)   with P = exp(s - lse), D = do . o
    causal_fwd(q, k, v) -> (o, lse)           row i attends 0 .. i
    causal_bwd(q, k, v, o, lse, do) -> (dq, dk, dv)
    merge(o1, lse1, o2, lse2) -> (o, lse)     log-sum-exp merge of two partial results
    add(a, b) -> a + b                        gradient partial sums
    """


@dataclass(frozen=True)
class Plan:
    T: int
    l: int
    world: int
    rank: int
    mode: str = "merged"   # "merged": band + stride beyond it; "band"; "stride"

    def __post_init__(self):
        n, l, N = self.T // self.world, self.l, self.world
        if self.T % N or n % l or l % N or (N > 1 and n < l):
            raise ValueError(f"cannot shard T={self.T}, l={l} over {N} ranks")
        if self.mode not in ("merged", "band", "stride"):
            raise ValueError(f"unknown mode {self.mode}")

    @property
    def n(self):
        return self.T // self.world

    @property
    def classes(self):
        return self.l // self.world

    @property
    def shift(self):
        return 2 if self.mode == "merged" else 0

    def rows(self):
        """Natural positions of this rank's chunk."""
        return range(self.rank * self.n, (self.rank + 1) * self.n)


# ---- data movement -------------------------------------------------------------

def halo_from_previous(plan: Plan, *xs, group=None):
    """The last l rows of each x [B, H, n, d] of rank r - 1, received on rank r
    (rank 0 gets None); point-to-point."""
    if plan.world == 1:
        return [None for _ in xs]
    ops, out = [], []
    for x in xs:
        if plan.rank + 1 < plan.world:
            ops.append(dist.P2POp(dist.isend, x[:, :, -plan.l:].contiguous(), plan.rank + 1,
                                  group))
        if plan.rank > 0:
            buf = torch.empty_like(x[:, :, :plan.l])
            ops.append(dist.P2POp(dist.irecv, buf, plan.rank - 1, group))
            out.append(buf)
        else:
            out.append(None)
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    return out


def halo_to_previous(plan: Plan, *gs, group=None):
    """Sends the gradients g [B, H, l, d] of the halo rows back to rank r - 1;
    returns what rank r receives from rank r + 1 for its own last l rows (None
    on the last rank)."""
    if plan.world == 1:
        return [None for _ in gs]
    ops, out = [], []
    for g in gs:
        if plan.rank > 0:
            ops.append(dist.P2POp(dist.isend, g.contiguous(), plan.rank - 1, group))
        if plan.rank + 1 < plan.world:
            buf = torch.empty_like(g)
            ops.append(dist.P2POp(dist.irecv, buf, plan.rank + 1, group))
            out.append(buf)
        else:
            out.append(None)
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    return out


def to_class_order(plan: Plan, x, group=None):
    """[B, H, n, *e] in position order (this rank's chunk) -> [B, H, C, P, *e]:
    the classes C = l / N this rank owns, every row p = 0 .. T/l - 1 of them."""
    N, l, n, C = plan.world, plan.l, plan.n, plan.classes
    B, H = x.shape[:2]
    e = x.shape[3:]
    y = x.reshape(B, H, n // l, N, C, *e)          # (p_local, destination rank, class)
    y = y.movedim(3, 0).movedim(3, 4).contiguous()  # [N, B, H, C, p_local, *e]
    if N > 1:
        out = torch.empty_like(y)
        dist.all_to_all_single(out, y, group=group)
        y = out                                     # [source rank, B, H, C, p_local, *e]
    return y.movedim(0, 3).reshape(B, H, C, N * (n // l), *e)


def from_class_order(plan: Plan, y, group=None):
    """Inverse of to_class_order: [B, H, C, P, *e] -> [B, H, n, *e]."""
    N, l, n, C = plan.world, plan.l, plan.n, plan.classes
    B, H = y.shape[:2]
    e = y.shape[4:]
    z = y.reshape(B, H, C, N, n // l, *e).movedim(3, 0).contiguous()  # [dest, B, H, C, p_local]
    if N > 1:
        out = torch.empty_like(z)
        dist.all_to_all_single(out, z, group=group)
        z = out                                                       # [source, B, H, C, p_local]
    # (source rank k, class c) is class k*C + c of the chunk: position
    # p_local * l + k * C + c
    z = z.permute(1, 2, 4, 0, 3, *range(5, z.dim()))   # [B, H, p_local, N, C, *e]
    return z.reshape(B, H, n, *e)


# ---- the two parts of the set --------------------------------------------------

def _with_halo(plan: Plan, own, halo, fill=0.0):
    """[halo, own] along the rows; zero (or `fill`) rows stand for the halo of
    tensors that only the own rows have."""
    if halo is None:
        halo = torch.full_like(own[:, :, :plan.l], fill)
    return torch.cat([halo, own], dim=2)


def _class_rows(plan: Plan, x, keys: bool):
    """Class-order [B, H, C, P, *e] -> the causal problem of the stride part,
    [B, H*C, P - s, *e]: query rows p >= s against key rows p' <= p - s, i.e.
    queries shifted down by s."""
    B, H, C, P = x.shape[:4]
    y = x.reshape(B, H * C, P, *x.shape[4:])
    s = plan.shift
    return (y[:, :, :P - s] if keys else y[:, :, s:]).contiguous()


def _class_back(plan: Plan, y, shape, keys: bool, fill=0.0):
    """Inverse of _class_rows: rows the shifted problem does not cover get
    `fill` (queries p < s have an empty stride part; keys p' > P-1-s are never
    attended by it)."""
    B, H, C, P = shape[:4]
    s = plan.shift
    out = torch.full((B, H * C, P, *y.shape[3:]), fill, dtype=y.dtype, device=y.device)
    if keys:
        out[:, :, :P - s] = y
    else:
        out[:, :, s:] = y
    return out.reshape(B, H, C, P, *y.shape[3:])


# ---- forward and backward --------------------------------------------------------

def sharded_forward(plan: Plan, q, k, v, ops, group=None):
    """This rank's chunk q, k, v [B, H, n, d] -> o [B, H, n, d], lse [B, H, n]
    (natural log) of strided attention over the whole sequence."""
    parts = []
    if plan.mode in ("merged", "band"):
        kh, vh = halo_from_previous(plan, k, v, group=group)
        if kh is None:
            parts.append(ops.band_fwd(q, k, v, plan.l))
        else:
            ob, lb = ops.band_fwd(_with_halo(plan, q, None), _with_halo(plan, k, kh),
                                  _with_halo(plan, v, vh), plan.l)
            parts.append((ob[:, :, plan.l:], lb[:, :, plan.l:]))
    if plan.mode in ("merged", "stride"):
        qc, kc, vc = (to_class_order(plan, x, group) for x in (q, k, v))
        oc, lc = ops.causal_fwd(_class_rows(plan, qc, False), _class_rows(plan, kc, True),
                                _class_rows(plan, vc, True))
        oc = _class_back(plan, oc, qc.shape, keys=False)
        lc = _class_back(plan, lc, qc.shape[:4], keys=False, fill=float("-inf"))
        parts.append((from_class_order(plan, oc, group), from_class_order(plan, lc, group)))
    o, lse = parts[0]
    for o2, l2 in parts[1:]:
        o, lse = ops.merge(o, lse, o2, l2)
    return o, lse


def sharded_backward(plan: Plan, q, k, v, o, lse, do, ops, group=None):
    """Gradients dq, dk, dv [B, H, n, d] of this rank's chunk, from the merged
    o, lse of sharded_forward and the upstream gradient do."""
    l = plan.l
    grads = []
    if plan.mode in ("merged", "band"):
        kh, vh = halo_from_previous(plan, k, v, group=group)
        if kh is None:
            dq, dk, dv = ops.band_bwd(q, k, v, o, lse, do, l)
            gk = torch.zeros_like(k[:, :, :l])
            gv = torch.zeros_like(v[:, :, :l])
        else:
            # the halo rows' own queries take no part: zero q, o, do and lse
            dq, dk, dv = ops.band_bwd(_with_halo(plan, q, None), _with_halo(plan, k, kh),
                                      _with_halo(plan, v, vh), _with_halo(plan, o, None),
                                      _with_halo(plan, lse.unsqueeze(-1), None).squeeze(-1),
                                      _with_halo(plan, do, None), l)
            gk, gv = dk[:, :, :l], dv[:, :, :l]
            dq, dk, dv = dq[:, :, l:], dk[:, :, l:], dv[:, :, l:]
        # keys of the halo belong to the previous rank: their gradients go back
        rk, rv = halo_to_previous(plan, gk, gv, group=group)
        if rk is not None:
            dk = torch.cat([dk[:, :, :-l], ops.add(dk[:, :, -l:], rk)], dim=2)
            dv = torch.cat([dv[:, :, :-l], ops.add(dv[:, :, -l:], rv)], dim=2)
        grads.append((dq, dk, dv))
    if plan.mode in ("merged", "stride"):
        qc, kc, vc, oc, dc = (to_class_order(plan, x, group) for x in (q, k, v, o, do))
        lc = to_class_order(plan, lse, group)
        dqc, dkc, dvc = ops.causal_bwd(
            _class_rows(plan, qc, False), _class_rows(plan, kc, True),
            _class_rows(plan, vc, True), _class_rows(plan, oc, False),
            _class_rows(plan, lc, False), _class_rows(plan, dc, False))
        dqc = _class_back(plan, dqc, qc.shape, keys=False)
        dkc = _class_back(plan, dkc, kc.shape, keys=True)
        dvc = _class_back(plan, dvc, vc.shape, keys=True)
        grads.append(tuple(from_class_order(plan, x, group) for x in (dqc, dkc, dvc)))
    dq, dk, dv = grads[0]
    for g in grads[1:]:
        dq, dk, dv = ops.add(dq, g[0]), ops.add(dk, g[1]), ops.add(dv, g[2])
    return dq, dk, dv
