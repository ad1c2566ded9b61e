"""Host side of the boundary on real ranks (sp_region_b200.ranks), run as two
gloo ranks on the CPU.

The library calls are replaced by a stand-in that moves data the way the
kernels do: rank r reads its rows of every rank's partial buffer and pushes
its result rows into every rank's gathered buffer (forward) and every rank's
dY buffer (backward).  The buffers are shared
host tensors, standing in for peer-mapped GPU memory.  Rank 1 is made slow at
each step, so a missing rendezvous would show up as a wrong value on rank 0.
Failures are made on the host, as the failure-detection tests require: a
rank that raises, and a rank that never arrives."""
import os
import socket
import sys
import time
import types

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N, H, WORLD = 8, 4, 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _Ops:
    """Stand-in for the library: the same reads and pushes on host tensors."""

    def __init__(self, rank, raise_in_forward=False):
        self.rank, self.raise_in_forward = rank, raise_in_forward

    def forward(self, cfg, partials, bias, residual, gamma, beta, residual_out,
                gathered, mask, mean, rstd, stream):
        if self.raise_in_forward:
            raise ValueError("planted failure in the forward")
        r0, r1 = cfg.row_begin, cfg.row_end
        y = sum(p[r0:r1] for p in partials) + residual
        if self.rank == 1:
            time.sleep(0.3)          # pushes late
        residual_out.copy_(y)
        for g in gathered:
            g[r0:r1] = y

    def backward(self, cfg, dparts, drnext, residual_out, gamma, mask, mean, rstd,
                 dres, dY, dgamma, dbeta, dbias, workspace, stream):
        r0, r1 = cfg.row_begin, cfg.row_end
        dz = sum(d[r0:r1] for d in dparts)
        if self.rank == 1:
            time.sleep(0.3)
        dres.copy_(dz)
        for d in dY:                 # pushed into every rank's dY
            d[r0:r1] = dz
        dgamma.fill_(self.rank + 1.0)
        dbeta.fill_(10.0 * (self.rank + 1))

    def synchronize(self, stream):
        pass


def _worker(rank, port, scenario, bufs, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from sp_region_b200.ranks import RankFailure, SPBoundary
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}",
                            rank=rank, world_size=WORLD)
    try:
        cfg = types.SimpleNamespace(s=N, b=1, h=H, t=WORLD, row_begin=0, row_end=0)
        timeout = 1.0 if scenario == "absent" else 20.0
        ops = _Ops(rank, raise_in_forward=(scenario == "raise" and rank == 1))
        sb = SPBoundary(timeout_s=timeout, ops=ops)
        assert sb.row_range(N) == (rank * N // WORLD, (rank + 1) * N // WORLD)
        if scenario == "absent" and rank == 1:
            q.put((rank, "stayed away"))
            time.sleep(3.0)          # never arrives; leaves after rank 0 gave up
            return
        # this rank's partial sum (rank 1 writes late)
        if rank == 1:
            time.sleep(0.3)
        bufs["partials"][rank].fill_(rank + 1.0)
        residual = torch.zeros(N // WORLD, H)
        rout = torch.empty(N // WORLD, H)
        t0 = time.monotonic()
        try:
            sb.forward(cfg, bufs["partials"], None, residual, None, None, rout,
                       bufs["gathered"])
        except RankFailure as e:
            q.put((rank, "RankFailure", e.missing, dict(e.reasons),
                   time.monotonic() - t0))
            return
        except ValueError as e:
            q.put((rank, "ValueError", str(e)))
            return
        gathered_ok = bool((bufs["gathered"][rank] == 3.0).all())
        bufs["dparts"][rank].fill_(10.0 * (rank + 1))
        dY = bufs["dY"][rank]
        dres = torch.empty(N // WORLD, H)
        dg, db = torch.empty(H), torch.empty(H)
        sb.backward(cfg, bufs["dparts"], None, rout, None, None, None, None, dres,
                    bufs["dY"], dg, db, None, None)
        # the store keeps only each rank's key of the latest rendezvous
        rdv = sb.rdv
        old_keys = [rdv._key(q_, tag, rank) for q_, tag in
                    ((0, "forward inputs written"), (1, "forward outputs pushed"),
                     (2, "backward inputs written"))]
        kept = [k for k in old_keys if rdv.store.check([k])]
        q.put((rank, "ok", gathered_ok, bool((dY == 30.0).all()),
               dg.tolist(), db.tolist(), bool((dres == 30.0).all()), kept))
    finally:
        dist.destroy_process_group()


def _run(scenario):
    bufs = {k: [torch.zeros(N, H).share_memory_() for _ in range(WORLD)]
            for k in ("partials", "gathered", "dparts", "dY")}
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, port, scenario, bufs, q))
          for r in range(WORLD)]
    for p in ps:
        p.start()
    out = {}
    try:
        for _ in range(WORLD):
            item = q.get(timeout=120)
            out[item[0]] = item[1:]
    finally:
        for p in ps:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return out


def test_two_ranks_order_the_pushes_and_sum_parameter_gradients():
    out = _run("ok")
    for r in range(WORLD):
        kind, gathered_ok, dy_ok, dg, db, dres_ok, kept = out[r]
        assert kind == "ok"
        assert kept == [], "keys of earlier rendezvous left in the store"
        assert gathered_ok, "gathered read before the peer's rows landed"
        assert dy_ok and dres_ok
        assert dg == [3.0] * H and db == [30.0] * H


def test_a_rank_that_raises_is_reported_to_the_others():
    out = _run("raise")
    assert out[1][0] == "ValueError"
    kind, missing, reasons, waited = out[0]
    assert kind == "RankFailure" and missing == [1]
    assert "planted failure" in reasons[1]
    assert waited < 10.0          # reported, not run out


def test_a_rank_that_never_arrives_is_named_after_the_deadline():
    out = _run("absent")
    assert out[1][0] == "stayed away"
    kind, missing, reasons, waited = out[0]
    assert kind == "RankFailure" and missing == [1] and reasons == {}
    assert 0.9 < waited < 10.0
