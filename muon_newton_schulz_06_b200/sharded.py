"""Matrix-sharded Muon across ranks (one process per GPU, torch.distributed).

Every matrix of a Muon step is independent, so N ranks can split the matrices,
orthogonalise only their own, and exchange the updated weights: the only exchange step
is one all-gather of the new weights.  Momentum buffers exist only on the owning rank.

Layout: all parameters live in one flat buffer of world_size equal chunks; chunk r
holds, contiguously, the matrices rank r owns (each at a 128-element-aligned offset),
and every parameter tensor is a view into it.  A rank's step updates its own chunk in
place (C-ABI muon_step), then ``all_gather_into_tensor(flat, flat[chunk r])`` (NCCL,
in place) brings every rank the other chunks.  No copies before or after.

The pages' own 8-GPU run keeps the optimizer replicated (plain DDP); this class is the
sharded alternative.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from .cost import ns_flops

_ALIGN = 128  # elements; keeps every view 256-byte aligned for bf16


def partition_lpt(shapes: Sequence[Tuple[int, int]], world: int, ns_steps: int = 5) -> List[int]:
    """Owner rank of each matrix: longest-processing-time-first greedy on the
    algorithmic Newton-Schulz flops (ties broken by matrix index, then rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = [ns_flops([sh], ns_steps)["algorithmic"] for sh in shapes]
    order = sorted(range(len(shapes)), key=lambda i: (-cost[i], i))
    load = [0] * world
    owner = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += cost[i]
    return owner


def _round_up(v: int, a: int) -> int:
    return (v + a - 1) // a * a


class ShardedMuon:
    """Muon over matrices split across the ranks of ``group``.

    ``params``: the same list of 2-D tensors (same shapes and values) on every rank.
    Their data is moved into the flat buffer; ``self.params[i]`` are the views to use
    from then on (the model's parameters should be re-pointed at them, e.g. with
    ``p.data = view``).  ``step_fn`` (tests only) replaces the C-ABI call with a
    function ``f(params, grads, moms, **kw)`` working on the owned matrices.
    """

    def __init__(self, params: Sequence[torch.Tensor], group=None, device=None,
                 step_fn: Optional[Callable] = None, handle=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        shapes = [tuple(p.shape) for p in params]
        if any(len(s) != 2 for s in shapes):
            raise ValueError("Muon matrices must be 2-D")
        dtypes = {p.dtype for p in params}
        if len(dtypes) != 1:
            raise ValueError("all matrices must share one dtype for the flat buffer")
        self.dtype = dtypes.pop()
        self.device = torch.device(device) if device is not None else params[0].device
        self.owner = partition_lpt(shapes, self.world)
        # offsets inside each owner's chunk
        local_off = [0] * len(params)
        used = [0] * self.world
        for i, (r, c) in enumerate(shapes):
            o = self.owner[i]
            local_off[i] = used[o]
            used[o] = _round_up(used[o] + r * c, _ALIGN)
        self.chunk = max(max(used), _ALIGN)
        self.flat = torch.zeros(self.world * self.chunk, dtype=self.dtype, device=self.device)
        self.params: List[torch.Tensor] = []
        for i, (p, (r, c)) in enumerate(zip(params, shapes)):
            start = self.owner[i] * self.chunk + local_off[i]
            view = self.flat[start:start + r * c].view(r, c)
            view.copy_(p.detach())
            self.params.append(view)
        self.mine = [i for i in range(len(params)) if self.owner[i] == self.rank]
        self.moms = {i: torch.zeros(shapes[i], dtype=torch.float32, device=self.device) for i in self.mine}
        self._step_fn = step_fn
        self._handle = handle
        self._own_handle = handle is None

    def owned(self) -> List[int]:
        return list(self.mine)

    def _local_step(self, grads, **kw):
        P = [self.params[i] for i in self.mine]
        G = [grads[i] for i in self.mine]
        M = [self.moms[i] for i in self.mine]
        if not P:
            return
        if self._step_fn is not None:
            self._step_fn(P, G, M, **kw)
            return
        from . import muon_init, muon_step
        if self._handle is None:
            self._handle = muon_init(self.device.index if self.device.index is not None else 0)
        muon_step(self._handle, P, G, M, **kw)

    def step(self, grads: Sequence[torch.Tensor], **kw) -> None:
        """One Muon step.  ``grads`` is indexed like ``params``; only the owned entries
        are read (the others may be None).  Keyword arguments go to muon_step."""
        self._local_step(grads, **kw)
        if self.world > 1:
            mine = self.flat[self.rank * self.chunk:(self.rank + 1) * self.chunk]
            dist.all_gather_into_tensor(self.flat, mine, group=self.group)

    def close(self):
        if self._handle is not None and self._own_handle:
            from . import muon_destroy
            muon_destroy(self._handle)
            self._handle = None
