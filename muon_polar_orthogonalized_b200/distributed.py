"""Owner-sharded Muon and ZeRO-1 AdamW across data-parallel ranks.

Newton-Schulz needs each whole matrix on one device, while data parallelism
keeps a full gradient on every rank ("3.9 Optimizers: SGD, Adam, Adafactor,
Lion, Muon & Shampoo", Wiring the hybrid recipe: a distributed Muon gathers
each matrix's gradient before it can iterate; ZeRO-1 shards optimizer state
across data-parallel ranks).

Layout, fixed at construction and the same on every rank (FlatLayout):
  * Muon: every hidden matrix has one owner rank, chosen by longest-
    processing-time over its executed Newton-Schulz FLOPs (3 m^2 n + m^3 for
    m <= n), so ranks get similar work.  The flat Muon buffers hold `world`
    regions of one length; region r holds the matrices rank r owns, in index
    order, each starting on a 64-element boundary.
  * AdamW: the tensors, each starting on a 64-element boundary, are laid end
    to end in one flat buffer cut into `world` equal slices.  Rank r owns
    slice r -- the pieces of the tensors that fall into it -- and keeps
    exp_avg / exp_avg_sq for those pieces only.
  Every parameter's data is a view of a flat parameter buffer and every
  gradient a view of a flat gradient buffer, so the collectives move the
  buffers themselves, with no packing or unpacking.

Per step, for each of the two buffers:
  1. one reduce_scatter (sum) of the gradient buffer: rank r receives
     region (slice) r summed over the ranks and divides it by the world size,
     the data-parallel mean gradient of what it owns;
  2. rank r steps what it owns: the Muon step on its matrices (momentum lives
     only there), AdamW on its slice;
  3. one all_gather of the parameter buffer, in place: every rank receives
     every region (slice).

Peer buffers (every other rank's flat buffers, addressable from this GPU
through peer access or symmetric memory) replace the collectives by this
library's own kernels over NVLink: with peer_grads, step 1 is a barrier
(every rank's gradients are written) and a kernel on each rank that averages
its region (slice) over every rank's gradient buffer (muon_reduce_mean);
with peer_params, the owner's last Newton-Schulz epilogue stores every
updated tile into every rank's parameter buffer as well
(muon_step_replicated), the AdamW slice is copied to every rank, and one
barrier orders the ranks after all writes.

The per-rank compute is the CUDA library (MuonAdamW); step_fn / adamw_fn can
replace it, which the CPU tests use to drive the same protocol on gloo ranks.
"""
from __future__ import annotations

import heapq
import math
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

ALIGN = 64   # elements: every tensor starts 256-byte aligned in fp32, 128-byte in bf16


def _align(n: int) -> int:
    return (n + ALIGN - 1) // ALIGN * ALIGN


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


class FlatLayout:
    """Where every tensor lives in the flat buffers (identical on every rank).

    muon_offset[i]: first element of Muon matrix i in the flat Muon buffers
    (region owners[i]); muon_region: elements per region.  adamw_offset[t]:
    first element of AdamW tensor t in the flat AdamW buffers; adamw_slice:
    elements per rank's slice."""

    def __init__(self, muon_shapes: Sequence[Sequence[int]], adamw_numels: Sequence[int], world: int):
        self.world = world
        self.muon_shapes = [tuple(s) for s in muon_shapes]
        self.owners = assign_owners(self.muon_shapes, world)
        used = [0] * world
        local = []
        for i, shp in enumerate(self.muon_shapes):
            r = self.owners[i]
            local.append(used[r])
            used[r] += _align(math.prod(shp))
        self.muon_region = _align(max(used + [0]))
        self.muon_offset = [self.owners[i] * self.muon_region + local[i] for i in range(len(local))]
        self.adamw_numels = [int(n) for n in adamw_numels]
        self.adamw_offset, total = [], 0
        for n in self.adamw_numels:
            self.adamw_offset.append(total)
            total += _align(n)
        self.adamw_slice = _align(-(-total // world)) if total else 0

    @property
    def muon_total(self) -> int:
        return self.world * self.muon_region

    @property
    def adamw_total(self) -> int:
        return self.world * self.adamw_slice

    def owned_matrices(self, rank: int) -> List[int]:
        return [i for i, o in enumerate(self.owners) if o == rank]

    def owned_pieces(self, rank: int) -> List[Tuple[int, int, int]]:
        """(tensor, first element within the tensor, length) of every piece of
        an AdamW tensor inside rank's slice."""
        lo, hi = rank * self.adamw_slice, (rank + 1) * self.adamw_slice
        out = []
        for t, (off, n) in enumerate(zip(self.adamw_offset, self.adamw_numels)):
            a, b = max(lo, off), min(hi, off + n)
            if a < b:
                out.append((t, a - off, b - a))
        return out


class DistributedMuonAdamW:
    """Data-parallel MuonAdamW: owner-sharded Muon, ZeRO-1 AdamW.

    muon_params: 2-D tensors; adamw_groups: dicts as for MuonAdamW (params,
    lr, betas, eps, weight_decay); both identical in shape and order on every
    rank.  At construction every parameter's data moves into the flat
    parameter buffers (p.data becomes a view; values kept).  Gradients live in
    the flat gradient buffers (grad_dtype / adamw_grad_dtype, default the
    parameter dtype): muon_grads[i] and adamw_grads[g][j] are the views the
    training loop writes, and each parameter's .grad is set to its view when
    the dtypes agree.  buffers: optional pre-allocated flat buffers
    {"muon_params", "muon_grads", "adamw_params", "adamw_grads"} of the
    layout's sizes (e.g. in peer-accessible memory).  peer_params /
    peer_grads: {rank: (muon buffer, adamw buffer)} of every other rank's
    parameter / gradient buffers, writable / readable from this process;
    reduce_fn(dst, sources) replaces muon_reduce_mean on the peer-gradient
    path.  step_fn(params, grads, momentum[, replicas]) and adamw_fn(pieces,
    step) replace the CUDA library: pieces is one dict per AdamW group with
    params, grads, exp_avg, exp_avg_sq (the owned pieces) and the group's
    hyperparameters.  The process group must be initialised unless world
    size is 1.
    """

    def __init__(self, muon_params: Sequence[torch.Tensor], adamw_groups: Sequence[Dict] = (),
                 process_group=None, grad_dtype: Optional[torch.dtype] = None,
                 adamw_grad_dtype: Optional[torch.dtype] = None,
                 buffers: Optional[Dict[str, torch.Tensor]] = None,
                 step_fn: Optional[Callable] = None, adamw_fn: Optional[Callable] = None,
                 peer_params: Optional[Dict[int, Sequence[torch.Tensor]]] = None,
                 peer_grads: Optional[Dict[int, Sequence[torch.Tensor]]] = None,
                 reduce_fn: Optional[Callable] = None, **muon_kwargs):
        self.group = process_group
        self.world = dist.get_world_size(process_group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(process_group) if dist.is_initialized() else 0
        self.muon_params = list(muon_params)
        self.adamw_groups = [dict(g) for g in adamw_groups]
        adam_params = [p for g in self.adamw_groups for p in g["params"]]
        self.layout = L = FlatLayout([tuple(p.shape) for p in self.muon_params],
                                     [p.numel() for p in adam_params], self.world)
        self.owners = L.owners
        self.owned = L.owned_matrices(self.rank)
        dev = (self.muon_params or adam_params or [torch.empty(0)])[0].device
        pdt = (self.muon_params or adam_params or [torch.empty(0)])[0].dtype
        mg_dt = grad_dtype or pdt
        ag_dt = adamw_grad_dtype or (adam_params[0].dtype if adam_params else pdt)
        b = dict(buffers or {})
        want = {"muon_params": (L.muon_total, pdt), "muon_grads": (L.muon_total, mg_dt),
                "adamw_params": (L.adamw_total, adam_params[0].dtype if adam_params else pdt),
                "adamw_grads": (L.adamw_total, ag_dt)}
        for k, (n, dt) in want.items():
            if k not in b:
                b[k] = torch.zeros(n, dtype=dt, device=dev)
            elif b[k].numel() != n or b[k].dtype != dt or not b[k].is_contiguous():
                raise ValueError(f"buffers[{k!r}] must be a contiguous {dt} tensor of {n} elements")
        self.buf = b
        # parameters and gradients become views of the flat buffers
        self.muon_grads: List[torch.Tensor] = []
        for i, p in enumerate(self.muon_params):
            o, n = L.muon_offset[i], p.numel()
            v = b["muon_params"][o:o + n].view(p.shape)
            v.copy_(p.detach())
            p.data = v
            g = b["muon_grads"][o:o + n].view(p.shape)
            self.muon_grads.append(g)
            if g.dtype == p.dtype:
                p.grad = g
        self.adamw_grads: List[List[torch.Tensor]] = []
        t = 0
        for grp in self.adamw_groups:
            gl = []
            for p in grp["params"]:
                o, n = L.adamw_offset[t], p.numel()
                v = b["adamw_params"][o:o + n].view(p.shape)
                v.copy_(p.detach())
                p.data = v
                g = b["adamw_grads"][o:o + n].view(p.shape)
                gl.append(g)
                if g.dtype == p.dtype:
                    p.grad = g
                t += 1
            self.adamw_grads.append(gl)
        # what this rank owns: its region / slice of each buffer
        r = self.rank
        self._mreg = slice(r * L.muon_region, (r + 1) * L.muon_region)
        self._areg = slice(r * L.adamw_slice, (r + 1) * L.adamw_slice)
        if self.world > 1:
            self.own_muon_grad = torch.zeros(L.muon_region, dtype=mg_dt, device=dev)
            self.own_adamw_grad = torch.zeros(L.adamw_slice, dtype=ag_dt, device=dev)
        else:
            self.own_muon_grad = b["muon_grads"][self._mreg]
            self.own_adamw_grad = b["adamw_grads"][self._areg]
        base = r * L.muon_region
        self._own_p = [b["muon_params"][L.muon_offset[i]:L.muon_offset[i] + self.muon_params[i].numel()]
                       .view(self.muon_params[i].shape) for i in self.owned]
        self._own_g = [self.own_muon_grad[L.muon_offset[i] - base:L.muon_offset[i] - base +
                                          self.muon_params[i].numel()].view(self.muon_params[i].shape)
                       for i in self.owned]
        # owned AdamW pieces, grouped as the AdamW groups are
        group_of = [gi for gi, grp in enumerate(self.adamw_groups) for _ in grp["params"]]
        abase = r * L.adamw_slice
        self._pieces: List[Dict] = []
        for gi, grp in enumerate(self.adamw_groups):
            ps, gs = [], []
            for (ti, start, n) in L.owned_pieces(r):
                if group_of[ti] != gi:
                    continue
                o = L.adamw_offset[ti] + start
                ps.append(b["adamw_params"][o:o + n])
                gs.append(self.own_adamw_grad[o - abase:o - abase + n])
            self._pieces.append(dict(params=ps, grads=gs, lr=grp.get("lr", 3e-4),
                                     betas=grp.get("betas", (0.9, 0.95)), eps=grp.get("eps", 1e-8),
                                     weight_decay=grp.get("weight_decay", 0.0)))
        # peers
        others = sorted(q for q in range(self.world) if q != r)
        self.peer_params = self._check_peers(peer_params, others, "peer_params", ("muon_params", "adamw_params"))
        self.peer_grads = self._check_peers(peer_grads, others, "peer_grads", ("muon_grads", "adamw_grads"))
        self.reduce_fn = reduce_fn
        # per-rank compute
        self.step_fn, self.adamw_fn = step_fn, adamw_fn
        self._local = None
        self.momentum = None
        self.step_count = 0
        if step_fn is None:
            from .optimizer import MuonAdamW
            self._local = MuonAdamW(self._own_p, [dict(params=pc["params"], lr=pc["lr"], betas=pc["betas"],
                                                       eps=pc["eps"], weight_decay=pc["weight_decay"])
                                                  for pc in self._pieces], **muon_kwargs)
        else:
            self.momentum = {i: torch.zeros_like(p) for i, p in zip(self.owned, self._own_p)}
            for pc in self._pieces:
                pc["exp_avg"] = [torch.zeros_like(p) for p in pc["params"]]
                pc["exp_avg_sq"] = [torch.zeros_like(p) for p in pc["params"]]

    def _check_peers(self, peers, others, what, keys):
        if peers is None:
            return None
        if sorted(peers) != others:
            raise ValueError(f"{what} must hold exactly the other ranks {others}")
        out = {}
        for q in others:
            mb, ab = peers[q]
            for buf, k in ((mb, keys[0]), (ab, keys[1])):
                mine = self.buf[k]
                if buf.numel() != mine.numel() or buf.dtype != mine.dtype:
                    raise ValueError(f"{what}[{q}] does not match this rank's {k} buffer")
            out[q] = (mb, ab)
        return out

    @staticmethod
    def buffer_numels(muon_shapes, adamw_numels, world: int) -> Dict[str, int]:
        """Element counts of the four flat buffers for pre-allocation."""
        L = FlatLayout(muon_shapes, adamw_numels, world)
        return {"muon_params": L.muon_total, "muon_grads": L.muon_total,
                "adamw_params": L.adamw_total, "adamw_grads": L.adamw_total}

    def _mean_grads(self) -> None:
        """Step 1: the mean gradient of this rank's region and slice."""
        if self.world == 1:
            return
        if self.peer_grads is not None:
            dist.barrier(group=self.group)
            srcs_m, srcs_a = [], []
            for q in range(self.world):
                mb, ab = (self.buf["muon_grads"], self.buf["adamw_grads"]) if q == self.rank \
                    else self.peer_grads[q]
                srcs_m.append([mb[self._mreg]])
                srcs_a.append([ab[self._areg]])
            fn = self.reduce_fn
            if fn is None:
                from . import api
                fn = api.muon_reduce_mean
            if self.layout.muon_region:
                fn([self.own_muon_grad], srcs_m)
            if self.layout.adamw_slice:
                fn([self.own_adamw_grad], srcs_a)
            return
        dist.reduce_scatter_tensor(self.own_muon_grad, self.buf["muon_grads"], op=dist.ReduceOp.SUM,
                                   group=self.group)
        dist.reduce_scatter_tensor(self.own_adamw_grad, self.buf["adamw_grads"], op=dist.ReduceOp.SUM,
                                   group=self.group)
        self.own_muon_grad.div_(self.world)
        self.own_adamw_grad.div_(self.world)

    def _gather_params(self) -> None:
        """Step 3: every rank receives every region and slice."""
        if self.world == 1:
            return
        if self.peer_params is not None:
            # the owners' Muon step wrote every rank's copy of its matrices
            # (replicas); the AdamW slice is copied here
            for q, (mb, ab) in self.peer_params.items():
                ab[self._areg].copy_(self.buf["adamw_params"][self._areg])
            dist.barrier(group=self.group)
            return
        dist.all_gather_into_tensor(self.buf["muon_params"], self.buf["muon_params"][self._mreg],
                                    group=self.group)
        dist.all_gather_into_tensor(self.buf["adamw_params"], self.buf["adamw_params"][self._areg],
                                    group=self.group)

    @torch.no_grad()
    def step(self, stream=None) -> None:
        self.step_count += 1
        self._mean_grads()
        replicas = None
        if self.peer_params is not None:
            L = self.layout
            replicas = [[self.peer_params[q][0][L.muon_offset[i]:L.muon_offset[i] + self.muon_params[i].numel()]
                         .view(self.muon_params[i].shape) for i in self.owned] for q in sorted(self.peer_params)]
        if self.step_fn is not None:
            if self.owned:
                args = (self._own_p, self._own_g, [self.momentum[i] for i in self.owned])
                if replicas is not None:
                    self.step_fn(*args, replicas)
                else:
                    self.step_fn(*args)
            if self.adamw_fn is not None and any(pc["params"] for pc in self._pieces):
                self.adamw_fn(self._pieces, self.step_count)
        else:
            self._local.step(stream=stream, replicas=replicas, muon_grads=self._own_g,
                             adamw_grads=[pc["grads"] for pc in self._pieces])
        self._gather_params()
