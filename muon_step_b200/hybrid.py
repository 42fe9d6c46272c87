"""Muon for the hidden matrices, AdamW for the rest: one optimizer object.

[V4-breakdown] "Muon 优化器完全拆解…", section "为什么嵌入层、输出头、bias、
RMSNorm 还在用 AdamW": embeddings, the prediction head, biases, gates and the
RMSNorm weights stay on AdamW; every other module is updated by Muon. Section
"更新尺度：让 Muon 借用 AdamW 的超参": with the shape rescale the two groups share
the learning rate and the weight decay.

Both groups run in the library's kernels: one Muon plan (MuonPlan) and one
AdamW plan (AdamWPlan), executed on the same stream. Plans record pointers, so
gradients should stay in place between steps (accumulate into .grad, zero it
with ``zero_grad()`` here); if a parameter's or a gradient's storage is
replaced, the next step rebuilds the plans.
"""

from __future__ import annotations

from typing import Iterable, Optional, Sequence, Tuple

import torch

from . import AdamWPlan, MuonPlan

DEFAULT_ADAMW_NAMES = ("embed", "head")


def route(named_shapes: Iterable[Tuple[str, Sequence[int]]],
          adamw_names: Sequence[str] = DEFAULT_ADAMW_NAMES):
    """Split parameter names between Muon and AdamW.

    A parameter goes to Muon when it has exactly two dimensions and its name
    contains none of ``adamw_names`` (case-insensitive; by default the
    embedding and prediction-head tables). Vectors and scalars (biases, gates,
    norm weights), tensors of three or more dimensions and the named tables go
    to AdamW. Returns (muon_names, adamw_names), each in input order.
    """
    tags = tuple(t.lower() for t in adamw_names)
    muon, adamw = [], []
    for name, shape in named_shapes:
        if len(tuple(shape)) == 2 and not any(t in name.lower() for t in tags):
            muon.append(name)
        else:
            adamw.append(name)
    return muon, adamw


def route_module(model, adamw_names: Sequence[str] = ()):
    """Split a module's parameters between Muon and AdamW by what they are.

    AdamW: the weights of embedding tables (torch.nn.Embedding); a linear
    layer's weight that is the same tensor as an embedding's (a tied
    prediction head) or whose output width is an embedding's vocabulary size
    (an untied head); every parameter that is not 2-D; and names containing
    any of ``adamw_names`` (case-insensitive). Muon: every other 2-D
    parameter. Names follow ``model.named_parameters()`` (a tied tensor is
    listed once, under its first name). Returns (muon_names, adamw_names).
    """
    import torch.nn as nn

    tables = [m for m in model.modules() if isinstance(m, nn.Embedding)]
    table_ids = {id(m.weight) for m in tables}
    vocab = {m.num_embeddings for m in tables}
    head_ids = set()
    for m in model.modules():
        if isinstance(m, nn.Linear) and (id(m.weight) in table_ids or m.out_features in vocab):
            head_ids.add(id(m.weight))
    tags = tuple(t.lower() for t in adamw_names)
    muon, adamw = [], []
    for name, p in model.named_parameters():
        to_adamw = (p.dim() != 2 or id(p) in table_ids or id(p) in head_ids
                    or any(t in name.lower() for t in tags))
        (adamw if to_adamw else muon).append(name)
    return muon, adamw


class HybridOptimizer:
    """Muon + AdamW over a model's named parameters (float32 CUDA tensors).

    Muon matrices must be contiguous 2-D; AdamW tensors contiguous. The Muon
    momentum and the AdamW moments are owned here (zeros at the start).
    """

    def __init__(self, named_params: Iterable[Tuple[str, torch.Tensor]], lr=0.02, momentum=0.95,
                 weight_decay=0.1, gamma=0.2, nesterov=True, betas=(0.9, 0.999), eps=1e-8,
                 precision="bf16", schedule=None, scale_mode="shape",
                 adamw_names: Sequence[str] = DEFAULT_ADAMW_NAMES,
                 muon_names: Optional[Sequence[str]] = None):
        params = list(named_params)
        if not params:
            raise ValueError("no parameters")
        by_name = dict(params)
        if muon_names is None:
            muon_names, adamw_names_ = route(((n, p.shape) for n, p in params), adamw_names)
        else:
            chosen = set(muon_names)
            unknown = chosen - set(by_name)
            if unknown:
                raise ValueError(f"unknown parameter names: {sorted(unknown)}")
            bad = [n for n in chosen if by_name[n].dim() != 2]
            if bad:
                raise ValueError(f"Muon parameters must be 2-D: {sorted(bad)}")
            muon_names = [n for n, _ in params if n in chosen]
            adamw_names_ = [n for n, _ in params if n not in chosen]
        self.muon_params = [(n, by_name[n]) for n in muon_names]
        self.adamw_params = [(n, by_name[n]) for n in adamw_names_]
        self.hyper = dict(lr=lr, momentum=momentum, weight_decay=weight_decay, gamma=gamma,
                          nesterov=nesterov, betas=tuple(betas), eps=eps)
        self.precision, self.schedule, self.scale_mode = precision, schedule, scale_mode
        self.momentum_buffers = {n: torch.zeros_like(p) for n, p in self.muon_params}
        self.exp_avg = {n: torch.zeros_like(p) for n, p in self.adamw_params}
        self.exp_avg_sq = {n: torch.zeros_like(p) for n, p in self.adamw_params}
        self.step_count = 0
        self._ptrs = None
        self._muon = self._adamw = None
        self._muon_ws = self._adamw_ws = None
        self._diag: Optional[torch.Tensor] = None

    @classmethod
    def from_module(cls, model, adamw_names: Sequence[str] = (), **kw):
        """A HybridOptimizer over ``model``'s parameters, split by
        ``route_module`` (embedding tables and prediction heads on AdamW)."""
        muon, _ = route_module(model, adamw_names)
        return cls(model.named_parameters(), muon_names=muon, **kw)

    # ------------------------------------------------------------------ plans
    def _current_ptrs(self):
        """The parameter and gradient addresses the plans were built on."""
        ptrs = []
        for n, p in self.muon_params + self.adamw_params:
            if p.grad is None:
                raise RuntimeError(f"parameter {n!r} has no gradient")
            ptrs.append((p.data_ptr(), p.grad.data_ptr()))
        return tuple(ptrs)

    def _build(self):
        if self.muon_params:
            self._muon = MuonPlan([(p, p.grad, self.momentum_buffers[n]) for n, p in self.muon_params],
                                  precision=self.precision, schedule=self.schedule,
                                  scale_mode=self.scale_mode)
            need = self._muon.workspace_bytes
            if self._muon_ws is None or self._muon_ws.numel() < need:
                self._muon_ws = self._muon.alloc_workspace()
            if self._diag is not None:
                self._muon.set_diagnostics(self._diag)
        if self.adamw_params:
            self._adamw = AdamWPlan([(p, p.grad, self.exp_avg[n], self.exp_avg_sq[n])
                                     for n, p in self.adamw_params])
            need = self._adamw.workspace_bytes
            if self._adamw_ws is None or self._adamw_ws.numel() < need:
                self._adamw_ws = self._adamw.alloc_workspace()

    def enable_diagnostics(self, on: bool = True) -> Optional[torch.Tensor]:
        """Per Muon matrix, (||N||_F, RMS of the update) after every step, as a
        (count, 2) float32 CUDA tensor in the order of ``muon_params``."""
        if on and self.muon_params:
            dev = self.muon_params[0][1].device
            self._diag = torch.zeros((len(self.muon_params), 2), dtype=torch.float32, device=dev)
        else:
            self._diag = None
        if self._muon is not None:
            self._muon.set_diagnostics(self._diag)
        return self._diag

    # ------------------------------------------------------------------ step
    def step(self, stream=None):
        """One step of both groups on `stream` (default: the current stream)."""
        ptrs = self._current_ptrs()
        if ptrs != self._ptrs:
            self._build()
            self._ptrs = ptrs
        self.step_count += 1
        h = self.hyper
        if self._muon is not None:
            self._muon.execute(self._muon_ws, lr=h["lr"], momentum=h["momentum"],
                               weight_decay=h["weight_decay"], gamma=h["gamma"],
                               nesterov=h["nesterov"], stream=stream)
        if self._adamw is not None:
            self._adamw.execute(self._adamw_ws, lr=h["lr"], betas=h["betas"], eps=h["eps"],
                                weight_decay=h["weight_decay"], step=self.step_count, stream=stream)

    def zero_grad(self):
        """Zero the gradients in place (their pointers stay those the plans hold)."""
        for _, p in self.muon_params + self.adamw_params:
            if p.grad is not None:
                p.grad.zero_()
