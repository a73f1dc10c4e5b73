"""MuonAdamW: the hybrid optimizer over two disjoint parameter sets.

Hidden 2-D weight matrices go to Muon; embeddings, the LM head, norm gains
and biases go to AdamW ("Chapter 4: The MuonAdamW Optimizer", Parameter
Dispatch; "3.9 Optimizers", Wiring the hybrid recipe).  The caller decides
the split.  This class only owns the state tensors (momentum, exp_avg,
exp_avg_sq, the step count), groups matrices by shape, and calls the C ABI;
all arithmetic runs in the CUDA library.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import torch

from . import _native as N
from . import api

DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)


class MuonAdamW:
    def __init__(self, muon_params: Sequence[torch.Tensor], adamw_groups: Sequence[Dict] = (),
                 lr: float = 0.02, momentum: float = 0.95, weight_decay: float = 0.01,
                 ns_steps: int = 5, coeffs=DEFAULT_COEFFS, nesterov: bool = True,
                 cautious: bool = True, lr_scale_fn=None, fp32_debug: bool = False,
                 fused_update: bool = True, normuon: bool = False, row_equilibrate: bool = False,
                 workspace_bytes: Optional[int] = None):
        """muon_params: fp32 2-D CUDA tensors.  adamw_groups: dicts with keys
        params, lr, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.  lr_scale_fn:
        optional (rows, cols) -> float learning-rate multiplier per shape.
        normuon: row-normalise the orthogonalised update (NorMuon).
        row_equilibrate: row-equilibrate the momentum-smoothed matrix before
        the orthogonalisation (MuonEq)."""
        self.lr, self.beta, self.wd = lr, momentum, weight_decay
        self.ns_steps, self.coeffs = ns_steps, coeffs
        self.flags = ((N.MUON_NESTEROV if nesterov else 0) | (N.MUON_CAUTIOUS_WD if cautious else 0)
                      | (N.MUON_FP32_DEBUG if fp32_debug else 0)
                      | (0 if fused_update else N.MUON_UNFUSED_UPDATE)
                      | (N.MUON_NORMUON if normuon else 0)
                      | (N.MUON_ROW_EQUILIBRATE if row_equilibrate else 0))
        # shape groups: matrices with equal (rows, cols) are contiguous in the pointer arrays
        muon_params = list(muon_params)
        order: Dict[tuple, List[int]] = {}
        for k, p in enumerate(muon_params):
            if p.dim() != 2 or p.dtype != torch.float32 or not p.is_cuda or not p.is_contiguous():
                raise ValueError("Muon parameters must be contiguous fp32 2-D CUDA tensors")
            order.setdefault(tuple(p.shape), []).append(k)
        self.muon_params: List[torch.Tensor] = []
        self._order: List[int] = []   # internal position -> position in muon_params as given
        self._shapes = []
        for (r, c), ks in order.items():
            self._shapes.append((r, c, len(ks), len(self.muon_params),
                                 float(lr_scale_fn(r, c)) if lr_scale_fn else 1.0))
            self.muon_params.extend(muon_params[k] for k in ks)
            self._order.extend(ks)
        self.momentum = [torch.zeros_like(p) for p in self.muon_params]
        self.adamw_groups = []
        for g in adamw_groups:
            ps = list(g["params"])
            self.adamw_groups.append(dict(
                params=ps, lr=g.get("lr", 3e-4), betas=g.get("betas", (0.9, 0.95)),
                eps=g.get("eps", 1e-8), weight_decay=g.get("weight_decay", 0.0),
                exp_avg=[torch.zeros_like(p) for p in ps],
                exp_avg_sq=[torch.zeros_like(p) for p in ps]))
        self.step_count = 0
        ws_need = api.muon_workspace_size(self._groups([torch.float32] * len(self._shapes)), self.flags) \
            if self.muon_params else 0
        nbytes = ws_need if workspace_bytes is None else max(int(workspace_bytes), 0)
        dev = self.muon_params[0].device if self.muon_params else torch.device("cuda")
        self.workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)

    def _groups(self, grad_dtypes):
        """Group descriptors, one gradient dtype per shape group."""
        return [(r, c, n, first, N.MUON_BF16 if dt == torch.bfloat16 else N.MUON_F32, ls)
                for (r, c, n, first, ls), dt in zip(self._shapes, grad_dtypes)]

    def _grad_dtypes(self, grads):
        """The gradient dtype of each shape group (fp32 or bf16, uniform within a group)."""
        out = []
        for (r, c, n, first, _) in self._shapes:
            dts = {grads[k].dtype for k in range(first, first + n)}
            if len(dts) != 1 or not dts <= {torch.float32, torch.bfloat16}:
                raise ValueError(f"the grads of the {r}x{c} Muon matrices must all be fp32 or all bf16")
            out.append(dts.pop())
        return out

    @torch.no_grad()
    def step(self, stream=None, replicas: Optional[Sequence[Sequence[torch.Tensor]]] = None,
             muon_grads: Optional[Sequence[torch.Tensor]] = None,
             adamw_grads: Optional[Sequence[Sequence[torch.Tensor]]] = None) -> None:
        """One MuonAdamW step.  replicas: optional copies of the Muon
        parameters (replicas[r][k] is copy r of the k-th tensor given at
        construction, e.g. another data-parallel rank's replica in peer
        memory); each receives the updated values (muon_step_replicated).
        muon_grads / adamw_grads: the gradients to use instead of each
        parameter's .grad (muon_grads[k] for the k-th Muon tensor given at
        construction, adamw_grads[g][j] for tensor j of AdamW group g)."""
        self.step_count += 1
        if self.muon_params:
            if muon_grads is not None:
                if len(muon_grads) != len(self.muon_params):
                    raise ValueError("muon_grads must hold one gradient per Muon parameter")
                grads = [muon_grads[k] for k in self._order]
            else:
                grads = [p.grad for p in self.muon_params]
            if any(g is None for g in grads):
                raise ValueError("every Muon parameter needs a .grad")
            gd = self._grad_dtypes(grads)
            if replicas:
                reps = [[rep[k] for k in self._order] for rep in replicas]
                api.muon_step_replicated(self.muon_params, grads, self.momentum, self._groups(gd), self.lr,
                                         self.beta, self.wd, self.ns_steps, self.coeffs, self.flags,
                                         self.workspace, reps, stream=stream)
            else:
                api.muon_step(self.muon_params, grads, self.momentum, self._groups(gd), self.lr,
                              self.beta, self.wd, self.ns_steps, self.coeffs, self.flags,
                              self.workspace, stream=stream)
        specs = []
        if adamw_grads is not None and len(adamw_grads) != len(self.adamw_groups):
            raise ValueError("adamw_grads must hold one list per AdamW group")
        for gi, g in enumerate(self.adamw_groups):
            grads = list(adamw_grads[gi]) if adamw_grads is not None else [p.grad for p in g["params"]]
            if any(x is None for x in grads):
                raise ValueError("every AdamW parameter needs a .grad")
            specs.append(api.AdamWSpec(g["params"], grads, g["exp_avg"], g["exp_avg_sq"], g["lr"],
                                       g["betas"][0], g["betas"][1], g["eps"], g["weight_decay"]))
        if specs:
            api.adamw_step(specs, self.step_count, stream=stream)

    def state_dict(self) -> dict:
        """Step count and optimizer state; "momentum" follows the order in
        which the Muon parameters were given, not the internal grouping."""
        mom: List[Optional[torch.Tensor]] = [None] * len(self.momentum)
        for k, pos in enumerate(self._order):
            mom[pos] = self.momentum[k].clone()
        return {"step": self.step_count,
                "momentum": mom,
                "exp_avg": [[t.clone() for t in g["exp_avg"]] for g in self.adamw_groups],
                "exp_avg_sq": [[t.clone() for t in g["exp_avg_sq"]] for g in self.adamw_groups]}

    def load_state_dict(self, sd: dict) -> None:
        """Restore a state_dict of an optimizer over parameters of the same
        shapes, given in the same order; nothing is changed if it does not fit."""
        def fits(dst: List[torch.Tensor], src, what: str) -> None:
            if len(src) != len(dst) or any(tuple(a.shape) != tuple(b.shape) for a, b in zip(dst, src)):
                raise ValueError(f"state_dict: {what} does not match this optimizer's parameters")
        mom_internal = [sd["momentum"][pos] for pos in self._order] \
            if len(sd["momentum"]) == len(self.momentum) else sd["momentum"]
        fits(self.momentum, mom_internal, "momentum")
        if len(sd["exp_avg"]) != len(self.adamw_groups) or len(sd["exp_avg_sq"]) != len(self.adamw_groups):
            raise ValueError("state_dict: AdamW group count does not match")
        for g, ea, es in zip(self.adamw_groups, sd["exp_avg"], sd["exp_avg_sq"]):
            fits(g["exp_avg"], ea, "exp_avg")
            fits(g["exp_avg_sq"], es, "exp_avg_sq")
        self.step_count = int(sd["step"])
        for dst, src in zip(self.momentum, mom_internal):
            dst.copy_(src)
        for g, ea, es in zip(self.adamw_groups, sd["exp_avg"], sd["exp_avg_sq"]):
            for dst, src in zip(g["exp_avg"], ea):
                dst.copy_(src)
            for dst, src in zip(g["exp_avg_sq"], es):
                dst.copy_(src)
