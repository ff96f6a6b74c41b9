"""Sequence sharding of strided attention (one long sequence over ranks), on
the CPU with two and four gloo ranks (one process each).

factorized_sparse_self_b200/seqshard.py moves the data: the band halo from
the previous rank and the all-to-all into residue-class order. The attention
arithmetic it calls is injected; here it is dense float64 algebra over an
explicit mask, written out in this file. The merged result of all ranks must
equal the oracle's attention over the whole sequence."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch


class DenseOps:
    """Dense float64 masked attention and its backward with P recomputed from a
    given LSE (natural log) and D = do . o; for the sharding test only."""

    @staticmethod
    def _mask(T, l):
        i = torch.arange(T)[:, None]
        j = torch.arange(T)[None, :]
        return (j <= i) & (j >= i - l) if l is not None else (j <= i)

    @staticmethod
    def _scores(q, k, M):
        s = q @ k.transpose(-1, -2) / np.sqrt(q.shape[-1])
        return s.masked_fill(~M, float("-inf"))

    def _fwd(self, q, k, v, l):
        s = self._scores(q, k, self._mask(q.shape[2], l))
        lse = torch.logsumexp(s, dim=-1)
        p = torch.exp(s - lse[..., None].masked_fill(torch.isinf(lse[..., None]), 0.0))
        return p @ v, lse

    def _bwd(self, q, k, v, o, lse, do, l):
        M = self._mask(q.shape[2], l)
        s = self._scores(q, k, M)
        p = torch.where(M, torch.exp(s - lse[..., None]), torch.zeros_like(s))
        D = (do * o).sum(-1, keepdim=True)
        ds = p * (do @ v.transpose(-1, -2) - D)
        sc = 1.0 / np.sqrt(q.shape[-1])
        return ds @ k * sc, ds.transpose(-1, -2) @ q * sc, p.transpose(-1, -2) @ do

    def band_fwd(self, q, k, v, l):
        return self._fwd(q, k, v, l)

    def band_bwd(self, q, k, v, o, lse, do, l):
        return self._bwd(q, k, v, o, lse, do, l)

    def causal_fwd(self, q, k, v):
        return self._fwd(q, k, v, None)

    def causal_bwd(self, q, k, v, o, lse, do):
        return self._bwd(q, k, v, o, lse, do, None)

    @staticmethod
    def merge(o1, l1, o2, l2):
        L = torch.logaddexp(l1, l2)
        fin = torch.isfinite(L)
        w1 = torch.where(fin, torch.exp(l1 - L.where(fin, torch.zeros_like(L))), 0.0)
        w2 = torch.where(fin, torch.exp(l2 - L.where(fin, torch.zeros_like(L))), 0.0)
        return w1[..., None] * o1 + w2[..., None] * o2, L

    @staticmethod
    def add(a, b):
        return a + b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, H, T, d, seed=0):
    import synth
    return [torch.from_numpy(synth.as_f32(x)).double() for x in synth.draw(B, H, T, d, "f32", 1.0, seed)]


def _rank_main(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from factorized_sparse_self_b200 import seqshard as ss
    B, H, T, d, l, mode = case
    q, k, v, do = _inputs(B, H, T, d)
    res = {}
    try:
        plan = ss.Plan(T, l, world, rank, mode)
        rows = slice(rank * plan.n, (rank + 1) * plan.n)
        mine = [x[:, :, rows].contiguous() for x in (q, k, v, do)]
        # data movement alone: class order holds exactly this rank's classes
        qc = ss.to_class_order(plan, mine[0])
        cls = range(rank * plan.classes, (rank + 1) * plan.classes)
        want = torch.stack([q[:, :, r::l] for r in cls], dim=2)
        res["class_order"] = bool(torch.equal(qc, want))
        res["round_trip"] = bool(torch.equal(ss.from_class_order(plan, qc), mine[0]))
        (kh,) = ss.halo_from_previous(plan, mine[1])
        res["halo"] = (kh is None) if rank == 0 else bool(
            torch.equal(kh, k[:, :, rank * plan.n - l:rank * plan.n]))
        ops = DenseOps()
        o, lse = ss.sharded_forward(plan, mine[0], mine[1], mine[2], ops)
        dq, dk, dv = ss.sharded_backward(plan, mine[0], mine[1], mine[2], o, lse, mine[3], ops)
        res["out"] = [x.numpy() for x in (o, lse, dq, dk, dv)]
    finally:
        out.put((rank, res))
        dist.barrier()
        dist.destroy_process_group()


def _run(world, case):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, out))
             for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = dict(out.get(timeout=300) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0] * world
    return [got[r] for r in range(world)]


CASES = [
    # B, H, T, d, l, world, oracle (kind, mode), heads
    ((1, 2, 512, 16, 32, "merged"), 2, "merged"),
    ((1, 2, 512, 16, 32, "merged"), 4, "merged"),
    ((1, 1, 384, 8, 48, "band"), 2, "split-even"),
    ((2, 1, 512, 8, 16, "stride"), 4, "split-odd"),
]


@pytest.mark.parametrize("case,world,ref", CASES,
                         ids=[f"{c[0][5]}-T{c[0][2]}-l{c[0][4]}-N{c[1]}" for c in CASES])
def test_sharded_strided_attention_matches_the_oracle(orc, case, world, ref):
    B, H, T, d, l, mode = case
    res = _run(world, case)
    for r in res:
        assert r["class_order"] and r["round_trip"] and r["halo"]
    got = [np.concatenate([r["out"][x] for r in res], axis=2) for x in range(5)]
    q, k, v, do = (x.numpy() for x in _inputs(B, H, T, d))
    if ref == "merged":
        kind_mode, sel = ("strided", "merged"), slice(None)
        args = (q, k, v, do)
    else:
        # split heads: head 0 of the oracle's pair of heads is an A1 (band) head,
        # head 1 an A2 (stride) head; the case's single head plays one of them
        h = 0 if ref == "split-even" else 1
        pad = [np.concatenate([x, x], axis=1) for x in (q, k, v, do)]
        kind_mode, sel = ("strided", "split"), slice(h, h + 1)
        args = tuple(pad)
    ro, rl = orc.forward(*kind_mode, args[0], args[1], args[2], l, 1)
    rdq, rdk, rdv = orc.backward(*kind_mode, *args, l, 1)
    for name, g, r in zip(("O", "LSE", "dQ", "dK", "dV"), got, (ro, rl, rdq, rdk, rdv)):
        np.testing.assert_allclose(g, r[:, sel], rtol=0, atol=1e-9, err_msg=name)


def test_plans_that_cannot_be_sharded_are_refused():
    from factorized_sparse_self_b200 import seqshard as ss
    for T, l, N in ((500, 32, 2), (512, 48, 2), (512, 32, 3), (256, 256, 2)):
        with pytest.raises(ValueError):
            ss.Plan(T, l, N, 0)
    assert ss.Plan(512, 32, 4, 3).rows() == range(384, 512)
