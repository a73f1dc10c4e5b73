"""Owner-sharded Muon across data-parallel ranks.

Newton-Schulz needs each whole matrix on one device, while data parallelism
keeps a full gradient on every rank ("3.9 Optimizers: SGD, Adam, Adafactor,
Lion, Muon & Shampoo", Wiring the hybrid recipe: a distributed Muon gathers
each matrix's gradient before it can iterate; ZeRO-1 shards optimizer state
across data-parallel ranks).  Here every hidden matrix has one owner rank:

  1. each owner's matrices' gradients are summed onto the owner (one
     reduce per owner over a flat bucket) and divided by the world size,
     i.e. the data-parallel mean gradient;
  2. the owner runs the Muon step on the matrices it owns, so momentum exists
     only on the owner (state sharded);
  3. each owner broadcasts its updated matrices to every rank.

With peer_params (every other rank's parameter tensors, addressable from
this GPU through peer access or symmetric memory), step 3 becomes part of
step 2: the owner's last Newton-Schulz epilogue stores each updated tile into
every rank's replica over NVLink (muon_step_replicated), and one barrier
orders the ranks after all owners' writes.  With peer_grads (every other
rank's gradient tensors, addressable likewise), step 1 becomes a barrier
(every rank's gradients are written) and a kernel on the owner that averages
its matrices' gradients from all ranks over NVLink (muon_reduce_mean).

AdamW parameters have their gradients all-reduced (mean) and are stepped on
every rank.  Owners are chosen by longest-processing-time over the executed
Newton-Schulz FLOPs of each matrix (3 m^2 n + m^3 for m <= n), so ranks get
similar work.

The per-rank compute is the CUDA library (MuonAdamW); `step_fn` can replace
it, which the CPU tests use to drive the same protocol on gloo ranks.
"""
from __future__ import annotations

import heapq
from typing import Callable, Dict, List, Optional, Sequence

import torch
import torch.distributed as dist


def ns_cost(rows: int, cols: int) -> float:
    m, n = min(rows, cols), max(rows, cols)
    return 3.0 * m * m * n + float(m) ** 3


def assign_owners(shapes: Sequence[Sequence[int]], world: int) -> List[int]:
    """Owner rank of each matrix: largest cost first onto the least-loaded rank
    (ties to the lower rank), deterministic on every rank."""
    order = sorted(range(len(shapes)), key=lambda i: (-ns_cost(*shapes[i]), i))
    heap = [(0.0, r) for r in range(world)]
    owners = [0] * len(shapes)
    for i in order:
        load, r = heapq.heappop(heap)
        owners[i] = r
        heapq.heappush(heap, (load + ns_cost(*shapes[i]), r))
    return owners


class DistributedMuonAdamW:
    """Data-parallel MuonAdamW with owner-sharded Muon matrices.

    muon_params / adamw_groups as for MuonAdamW (identical on every rank).
    step_fn(params, grads, momentum[, replicas]) -> None updates the owned
    params and momentum in place, and each replica list's tensors too when
    given (default: a MuonAdamW over the owned matrices, built with the
    keyword arguments given here).  peer_params: optional {rank: that rank's
    muon_params tensors in the same order} for every other rank, writable
    from this process (peer GPU memory); owners then write every rank's copy
    in their update and the broadcasts are skipped.  peer_grads: likewise
    every other rank's gradient tensors of muon_params (their .grad buffers,
    which must stay the same tensors across steps); owners then average
    their matrices' gradients from all ranks themselves instead of the
    per-owner reduces.  reduce_fn(dst, sources) replaces that average
    (default muon_reduce_mean).  The process group must be initialised
    unless world size is 1.
    """

    def __init__(self, muon_params: Sequence[torch.Tensor], adamw_groups: Sequence[Dict] = (),
                 process_group=None, step_fn: Optional[Callable] = None,
                 adamw_fn: Optional[Callable] = None,
                 peer_params: Optional[Dict[int, Sequence[torch.Tensor]]] = None,
                 peer_grads: Optional[Dict[int, Sequence[torch.Tensor]]] = None,
                 reduce_fn: Optional[Callable] = None, **muon_kwargs):
        self.group = process_group
        self.world = dist.get_world_size(process_group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(process_group) if dist.is_initialized() else 0
        self.muon_params = list(muon_params)
        self.owners = assign_owners([tuple(p.shape) for p in self.muon_params], self.world)
        self.owned = [i for i, o in enumerate(self.owners) if o == self.rank]
        self.adamw_groups = list(adamw_groups)
        self.step_fn = step_fn
        self.adamw_fn = adamw_fn
        self._local = None
        if step_fn is None:
            from .optimizer import MuonAdamW
            self._local = MuonAdamW([self.muon_params[i] for i in self.owned], self.adamw_groups,
                                    **muon_kwargs)
        self.momentum = {i: torch.zeros_like(self.muon_params[i]) for i in self.owned} \
            if step_fn is not None else None
        self.peer_params = None
        if peer_params is not None:
            others = sorted(r for r in range(self.world) if r != self.rank)
            if sorted(peer_params) != others:
                raise ValueError(f"peer_params must hold exactly the other ranks {others}")
            for r in others:
                if len(peer_params[r]) != len(self.muon_params) or any(
                        tuple(a.shape) != tuple(b.shape) for a, b in zip(peer_params[r], self.muon_params)):
                    raise ValueError(f"peer_params[{r}] does not match muon_params")
            self.peer_params = {r: list(peer_params[r]) for r in others}
        self.peer_grads = None
        if peer_grads is not None:
            others = sorted(r for r in range(self.world) if r != self.rank)
            if sorted(peer_grads) != others:
                raise ValueError(f"peer_grads must hold exactly the other ranks {others}")
            for r in others:
                if len(peer_grads[r]) != len(self.muon_params) or any(
                        tuple(a.shape) != tuple(b.shape) for a, b in zip(peer_grads[r], self.muon_params)):
                    raise ValueError(f"peer_grads[{r}] does not match muon_params")
            self.peer_grads = {r: list(peer_grads[r]) for r in others}
        self.reduce_fn = reduce_fn

    def _bucket(self, tensors: List[torch.Tensor]) -> torch.Tensor:
        return torch.cat([t.reshape(-1) for t in tensors]) if tensors else torch.empty(0)

    def _unbucket(self, flat: torch.Tensor, tensors: List[torch.Tensor]) -> None:
        off = 0
        for t in tensors:
            n = t.numel()
            t.copy_(flat[off:off + n].view_as(t))
            off += n

    def _owner_mean_from_peers(self) -> None:
        """Every rank's gradients are written (barrier); then each owner
        averages its matrices' gradients over all ranks, in rank order, into
        its own .grad tensors."""
        if self.world > 1:
            dist.barrier(group=self.group)
        own = self.owned
        if not own:
            return
        dst = [self.muon_params[i].grad for i in own]
        sources = [dst if r == self.rank else [self.peer_grads[r][i] for i in own]
                   for r in range(self.world)]
        if self.reduce_fn is not None:
            self.reduce_fn(dst, sources)
        else:
            from . import api
            api.muon_reduce_mean(dst, sources)

    @torch.no_grad()
    def step(self) -> None:
        # 1. mean gradient of each matrix onto its owner
        if self.peer_grads is not None:
            self._owner_mean_from_peers()
        else:
            for r in range(self.world):
                idx = [i for i, o in enumerate(self.owners) if o == r]
                if not idx:
                    continue
                grads = [self.muon_params[i].grad for i in idx]
                if self.world > 1:
                    flat = self._bucket(grads)
                    dist.reduce(flat, dst=r, op=dist.ReduceOp.SUM, group=self.group)
                    if r == self.rank:
                        flat.div_(self.world)
                        self._unbucket(flat, grads)
        # AdamW gradients: all-reduce mean
        adam_params = [p for g in self.adamw_groups for p in g["params"]]
        if adam_params and self.world > 1:
            flat = self._bucket([p.grad for p in adam_params])
            dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=self.group)
            flat.div_(self.world)
            self._unbucket(flat, [p.grad for p in adam_params])
        # 2. owners step their matrices (and every rank its AdamW params); with
        #    peer_params they write every other rank's copy as well
        replicas = None
        if self.peer_params is not None:
            replicas = [[self.peer_params[r][i] for i in self.owned] for r in sorted(self.peer_params)]
        if self.step_fn is not None:
            own = self.owned
            if own:
                args = ([self.muon_params[i] for i in own], [self.muon_params[i].grad for i in own],
                        [self.momentum[i] for i in own])
                if replicas is not None:
                    self.step_fn(*args, replicas)
                else:
                    self.step_fn(*args)
            if self.adamw_fn is not None and adam_params:
                self.adamw_fn(self.adamw_groups)
        else:
            self._local.step(replicas=replicas)
        if self.peer_params is not None:
            # 3. every owner's writes into this rank's replica are done
            if self.world > 1:
                dist.barrier(group=self.group)
            return
        # 3. owners broadcast their updated matrices
        if self.world > 1:
            for r in range(self.world):
                idx = [i for i, o in enumerate(self.owners) if o == r]
                if not idx:
                    continue
                ps = [self.muon_params[i] for i in idx]
                flat = self._bucket(ps)
                dist.broadcast(flat, src=r, group=self.group)
                if r != self.rank:
                    self._unbucket(flat, ps)
