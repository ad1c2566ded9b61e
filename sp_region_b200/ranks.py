"""The SP boundary over real ranks: one process per GPU.

Rank r of t owns the token rows [r*N/t, (r+1)*N/t).  Its forward is one fused
library call on that row range: the kernel reads rank r's rows of every rank's
partial-sum buffer (the peers' through peer-mapped memory; that read is the
reduce-scatter) and pushes its normalised rows into every rank's gathered
buffer (the all-gather) -- "Sequence Parallelism math", section "The
collective substitution".  The backward is the same with the upstream
gradients: it reads its rows of every rank's gradient partials and pushes
its rows of dY (the all-gather of the dropout gradient, the reduce-scatter's
backward) into every rank's dY buffer.  Last, the replicated parameters'
gradients (gamma, beta and the bias live on every rank) are summed over the
ranks.

The kernels never wait on another rank.  Ordering between ranks is kept on
the host: every rank's inputs are written before any rank's kernel reads
them, and every push has landed before any rank reads its gathered buffer.
Each of those points is a rendezvous through the process group's store with
a deadline.  A rank that raised reports it there, and one that exited or never
arrived is named once the deadline passes, so the others get a RankFailure
instead of waiting for good.
"""
from __future__ import annotations

import copy
import time
from typing import List, Optional, Sequence

import torch
import torch.distributed as dist


class RankFailure(RuntimeError):
    """Another rank did not reach a rendezvous: it failed or is missing."""

    def __init__(self, where: str, missing: Sequence[int], reasons: dict):
        self.where = where
        self.missing = list(missing)
        self.reasons = dict(reasons)
        detail = "; ".join(f"rank {r}: {m}" for r, m in sorted(self.reasons.items()))
        super().__init__(f"{where}: ranks {self.missing} did not arrive"
                         + (f" ({detail})" if detail else ""))


class Rendezvous:
    """All ranks meet at a named point through a key-value store.

    arrive(tag) publishes this rank's arrival and waits, at most timeout_s,
    for every rank's.  fail(exc) publishes this rank's failure, so that the
    others stop waiting at once.  Every call uses fresh keys (a per-instance
    sequence number), so points can repeat.  Once every rank has arrived at a
    point, every rank is done waiting at the one before, so each rank then
    deletes its own key of that earlier point: the store stays small over a
    long run."""

    def __init__(self, store, rank: int, world: int, timeout_s: float = 30.0,
                 prefix: str = "sp_boundary", poll_s: float = 0.005):
        self.store, self.rank, self.world = store, rank, world
        self.timeout_s, self.prefix, self.poll_s = timeout_s, prefix, poll_s
        self.seq = 0
        self._last_key = None

    def _key(self, seq: int, tag: str, r: int) -> str:
        return f"{self.prefix}/{seq}/{tag}/{r}"

    def _failures(self) -> dict:
        keys = [f"{self.prefix}/failed/{r}" for r in range(self.world)]
        out = {}
        for r, k in enumerate(keys):
            if r != self.rank and self.store.check([k]):
                out[r] = self.store.get(k).decode(errors="replace")
        return out

    def arrive(self, tag: str) -> None:
        seq, self.seq = self.seq, self.seq + 1
        self.store.set(self._key(seq, tag, self.rank), "1")
        want = [self._key(seq, tag, r) for r in range(self.world)]
        deadline = time.monotonic() + self.timeout_s
        while True:
            missing = [r for r, k in enumerate(want) if not self.store.check([k])]
            if not missing:
                if self._last_key is not None:
                    self.store.delete_key(self._last_key)
                self._last_key = want[self.rank]
                return
            failed = self._failures()
            if failed or time.monotonic() > deadline:
                raise RankFailure(f"{tag} (rendezvous {seq})", missing, failed)
            time.sleep(self.poll_s)

    def fail(self, exc: BaseException) -> None:
        self.store.set(f"{self.prefix}/failed/{self.rank}",
                       f"{type(exc).__name__}: {exc}")


class LibraryOps:
    """The CUDA library calls of one rank (the default operations)."""

    def forward(self, cfg, partials, bias, residual, gamma, beta, residual_out,
                gathered, mask, mean, rstd, stream):
        from sp_region_b200 import sp_rs_bias_dropout_add_norm_fwd
        sp_rs_bias_dropout_add_norm_fwd(cfg, partials, bias, residual, gamma, beta,
                                        residual_out, gathered, mask, mean, rstd,
                                        stream=stream)

    def backward(self, cfg, dparts, drnext, residual_out, gamma, mask, mean, rstd,
                 dres, dY, dgamma, dbeta, dbias, workspace, stream):
        from sp_region_b200 import sp_rs_norm_dropout_bwd_ag
        sp_rs_norm_dropout_bwd_ag(cfg, dparts, drnext, residual_out, gamma, mask, mean,
                                  rstd, dres, dY, dgamma, dbeta, dbias, workspace,
                                  stream=stream)

    def synchronize(self, stream):
        (stream or torch.cuda.current_stream()).synchronize()


def peer_buffers(tensor: torch.Tensor, group=None) -> List[torch.Tensor]:
    """The world's copies of a buffer, in rank order, for a tensor allocated
    with torch's symmetric memory (torch.distributed._symmetric_memory.empty):
    this rank's own tensor and every peer's mapped into this process.  The
    kernels read and write peers' buffers through these addresses with plain
    loads, stores and bulk copies from one source to one destination."""
    import torch.distributed._symmetric_memory as symm_mem
    h = symm_mem.rendezvous(tensor, group or dist.group.WORLD)
    return [tensor if r == h.rank else
            h.get_buffer(r, tuple(tensor.shape), tensor.dtype)
            for r in range(h.world_size)]


class SPBoundary:
    """One rank's side of the boundary on t = world ranks."""

    def __init__(self, group=None, timeout_s: float = 30.0, ops=None, store=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.ops = ops or LibraryOps()
        if store is None:
            store = dist.distributed_c10d._get_default_store()
        self.rdv = Rendezvous(store, self.rank, self.world, timeout_s)

    def row_range(self, n_rows: int):
        per = n_rows // self.world
        return self.rank * per, (self.rank + 1) * per

    def _cfg(self, cfg):
        if cfg.t != self.world:
            raise ValueError(f"cfg.t = {cfg.t}, but the group has {self.world} ranks")
        c = (type(cfg).from_buffer_copy(cfg) if hasattr(type(cfg), "from_buffer_copy")
             else copy.copy(cfg))
        c.row_begin, c.row_end = self.row_range(cfg.s * cfg.b)
        return c

    def _inputs_written(self, tag, stream):
        # this rank's inputs (produced on its stream) are complete, and so
        # are every other rank's
        try:
            self.ops.synchronize(stream)
        except BaseException as e:
            self.rdv.fail(e)
            raise
        self.rdv.arrive(tag)

    def _run(self, tag, fn, stream):
        try:
            fn()
            self.ops.synchronize(stream)   # this rank's pushes have completed
        except BaseException as e:
            self.rdv.fail(e)
            raise
        self.rdv.arrive(tag)               # ... and every other rank's

    def forward(self, cfg, partials, bias, residual, gamma, beta, residual_out,
                gathered, mask=None, mean=None, rstd=None, stream=None):
        """partials, gathered: the world's buffers in rank order (peer_buffers).
        residual, residual_out, mask, mean, rstd: this rank's shard."""
        if len(partials) != self.world or len(gathered) != self.world:
            raise ValueError("one partial and one gathered buffer per rank")
        c = self._cfg(cfg)
        self._inputs_written("forward inputs written", stream)
        self._run("forward outputs pushed",
                  lambda: self.ops.forward(c, partials, bias, residual, gamma, beta,
                                           residual_out, gathered, mask, mean, rstd,
                                           stream), stream)

    def backward(self, cfg, dparts, drnext, residual_out, gamma, mask, mean, rstd,
                 dres, dY, dgamma, dbeta, dbias, workspace, stream=None):
        """dparts, dY: the world's gradient partials and dY buffers in rank
        order (peer_buffers); every rank's dY is complete on return.  The rest
        are this rank's shard.  dgamma / dbeta / dbias come back summed over
        the ranks."""
        if len(dparts) != self.world or len(dY) != self.world:
            raise ValueError("one gradient partial and one dY buffer per rank")
        c = self._cfg(cfg)
        self._inputs_written("backward inputs written", stream)
        # each rank pushes its dY rows into every rank's dY; once all have
        # arrived, every copy is complete
        self._run("backward outputs pushed",
                  lambda: self.ops.backward(c, dparts, drnext, residual_out, gamma,
                                            mask, mean, rstd, dres, dY, dgamma, dbeta,
                                            dbias, workspace, stream),
                  stream)
        # gamma, beta and bias are replicated: sum their gradients over ranks
        for g in (dgamma, dbeta, dbias):
            if g is not None:
                dist.all_reduce(g, group=self.group)
