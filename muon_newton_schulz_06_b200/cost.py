"""Algorithmic work of one Muon step (host-side bookkeeping for the benchmark).

Per matrix with s = min(rows, cols), L = max(rows, cols) and one Newton-Schulz step:
  Gram    s x s from an s x L operand, one triangle:   L * s * (s + 1)   flops
  Poly    s x s from an s x s operand, one triangle:   s * s * (s + 1)   flops
  Update  s x L from s x s times s x L:                2 * L * s * s     flops
The dense equivalent (both triangles) is 4*L*s^2 + 2*s^3 per step.

Elementwise passes, bytes per element: momentum/norm reads G and M, writes M and U;
apply reads O and W and writes W.
"""
from __future__ import annotations

from typing import Iterable, Tuple

_BYTES = {"bf16": 2, "fp32": 4}


def ns_flops(shapes: Iterable[Tuple[int, int]], ns_steps: int = 5) -> dict:
    gram = poly = update = dense = 0
    for r, c in shapes:
        s, L = min(r, c), max(r, c)
        gram += L * s * (s + 1)
        poly += s * s * (s + 1)
        update += 2 * L * s * s
        dense += 4 * L * s * s + 2 * s ** 3
    k = ns_steps
    return {"gram": gram * k, "poly": poly * k, "update": update * k,
            "algorithmic": (gram + poly + update) * k, "dense_equivalent": dense * k,
            "per_launch": {"gram": gram, "poly": poly, "update": update}}


def elementwise_bytes(shapes: Iterable[Tuple[int, int]], param="bf16", grad="bf16", work="bf16") -> dict:
    numel = sum(r * c for r, c in shapes)
    pb, gb, wb = _BYTES[param], _BYTES[grad], _BYTES[work]
    return {"momentum_norm": numel * (gb + 4 + 4 + wb), "apply": numel * (wb + 2 * pb), "numel": numel}


def contiguous_chunks(shapes, n_chunks: int, ns_steps: int = 5):
    """Cut the matrix list into at most n_chunks contiguous, non-empty runs of about
    equal algorithmic Newton-Schulz work; returns [(begin, end), ...] covering all of it.
    Cut c goes at the matrix boundary whose running sum is closest to c/n_chunks of the
    total (keeping every run non-empty)."""
    shapes = list(shapes)
    n = len(shapes)
    if n == 0:
        return []
    n_chunks = max(1, min(int(n_chunks), n))
    work = [ns_flops([sh], ns_steps)["algorithmic"] for sh in shapes]
    prefix = [0]
    for w in work:
        prefix.append(prefix[-1] + w)
    total = float(prefix[-1])
    cuts = [0]
    for c in range(1, n_chunks):
        target = total * c / n_chunks
        lo = cuts[-1] + 1                      # at least one matrix in the run before
        hi = n - (n_chunks - c)                # at least one matrix for each later run
        best = min(range(lo, hi + 1), key=lambda i: (abs(prefix[i] - target), i))
        cuts.append(best)
    cuts.append(n)
    return [(cuts[i], cuts[i + 1]) for i in range(n_chunks)]
