"""Seeded synthetic inputs for the Muon step: matrix shapes of the pages' models and
gradients / momentum buffers / weights drawn from fixed distributions.

This module holds no arithmetic of the method itself (no momentum, no
normalisation, no Newton-Schulz, no update).  Both the CUDA path's tests and the
oracle's tests draw their inputs from here, so that the two sides see the same
numbers.

Shapes (rows = out_features, cols = in_features):

* ``tiny``   : 128x64, 64x128, 96x96, 256x32; fp32; G ~ N(0,1); M = 0; W = 0.
* ``d8``     : depth-8 GPT, d_model 512, MLP 2048 (autoresearch-like), 48 matrices.
* ``d12``    : depth-12 GPT, d_model 768, MLP 3072 (nanochat-like), 72 matrices.
* ``d24``    : depth-24 GPT, d_model 1536, MLP 6144, 144 matrices, heavy-tailed
               gradient spectrum (singular values proportional to 1/i).
* ``llama3p8b``: 28 layers, d_model 3072, GQA 24 q / 8 kv heads of 128, relu^2 MLP
               12288, 168 matrices (the 3.8B model of the "little-lm on 8xB200"
               write-up, hackernews.jp story 49637435, parameter table: 28 decoder
               layers hold 2,818.7M parameters).

Gradient recipe for the GPT/Llama sets (a reading of "N(0, sigma) with sigma
log-uniform in [1e-4, 1e-2] plus a rank-4 spike of 10x magnitude"):
G = sigma*Z + sum_{j<4} 10*sigma*(sqrt(r)+sqrt(c)) u_j v_j^T with orthonormal u, v
(each spike's singular value is 10x the spectral edge of the noise).  The
heavy-tailed set uses G = U diag(1/i) V^T (Haar U, V) rescaled to
||G||_F = sigma*sqrt(r*c).  M ~ N(0, sigma) float32, W ~ N(0, 0.02).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

CONFIG_NAMES = ("tiny", "d8", "d12", "d24", "llama3p8b")


@dataclass(frozen=True)
class MatrixSpec:
    name: str
    rows: int
    cols: int


def _gpt_layer(d: int, hidden: int) -> List[MatrixSpec]:
    return [MatrixSpec("wq", d, d), MatrixSpec("wk", d, d), MatrixSpec("wv", d, d),
            MatrixSpec("wo", d, d), MatrixSpec("w_fc", hidden, d),
            MatrixSpec("w_proj", d, hidden)]


def config_shapes(config: int | str, layers: Optional[Sequence[int]] = None) -> List[MatrixSpec]:
    """Matrix shapes of one configuration, in layer order.  ``layers`` keeps only
    the listed layer indices (all layers by default)."""
    cid = config if isinstance(config, int) else CONFIG_NAMES.index(config)
    if cid == 0:
        return [MatrixSpec("m0", 128, 64), MatrixSpec("m1", 64, 128),
                MatrixSpec("m2", 96, 96), MatrixSpec("m3", 256, 32)]
    if cid == 1:
        depth, per = 8, _gpt_layer(512, 2048)
    elif cid == 2:
        depth, per = 12, _gpt_layer(768, 3072)
    elif cid == 3:
        depth, per = 24, _gpt_layer(1536, 6144)
    elif cid == 4:
        depth = 28
        per = [MatrixSpec("wq", 3072, 3072), MatrixSpec("wk", 1024, 3072),
               MatrixSpec("wv", 1024, 3072), MatrixSpec("wo", 3072, 3072),
               MatrixSpec("w_fc", 12288, 3072), MatrixSpec("w_proj", 3072, 12288)]
    else:
        raise ValueError(f"unknown config {config!r}")
    keep = range(depth) if layers is None else layers
    return [MatrixSpec(f"l{li}.{m.name}", m.rows, m.cols) for li in keep for m in per]


def base_seed(config: int) -> int:
    return 1000 + int(config)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _orthonormal(rows: int, k: int, gen, device) -> torch.Tensor:
    z = torch.randn(rows, k, generator=gen, device=device, dtype=torch.float32)
    q, _ = torch.linalg.qr(z)
    return q


def make_gradient(config: int, spec: MatrixSpec, index: int, device="cpu") -> tuple:
    """(G float32, M float32, W float32, sigma) for one matrix of a GPT/Llama set or
    the tiny set.  Draws are keyed by (config, index) only."""
    device = torch.device(device)
    gen = _gen(device, base_seed(config) * 1000 + index)
    r, c = spec.rows, spec.cols
    if config == 0:
        g = torch.randn(r, c, generator=gen, device=device, dtype=torch.float32)
        z = torch.zeros(r, c, device=device, dtype=torch.float32)
        return g, z, z.clone(), 1.0
    u01 = torch.rand((), generator=gen, device=device, dtype=torch.float64).item()
    sigma = 10.0 ** (-4.0 + 2.0 * u01)
    if config == 3:
        s = min(r, c)
        uu = _orthonormal(r, s, gen, device)
        vv = _orthonormal(c, s, gen, device)
        sv = 1.0 / torch.arange(1, s + 1, device=device, dtype=torch.float32)
        g = (uu * sv) @ vv.T
        g = g * (sigma * math.sqrt(r * c) / torch.linalg.vector_norm(g))
    else:
        g = sigma * torch.randn(r, c, generator=gen, device=device, dtype=torch.float32)
        uu = _orthonormal(r, 4, gen, device)
        vv = _orthonormal(c, 4, gen, device)
        g = g + (10.0 * sigma * (math.sqrt(r) + math.sqrt(c))) * (uu @ vv.T)
    m = sigma * torch.randn(r, c, generator=gen, device=device, dtype=torch.float32)
    w = 0.02 * torch.randn(r, c, generator=gen, device=device, dtype=torch.float32)
    return g, m, w, sigma


def make_matrix_set(config: int, device="cpu", layers: Optional[Sequence[int]] = None,
                    indices: Optional[Sequence[int]] = None):
    """All inputs of one configuration.

    Returns a dict with ``specs`` and lists ``W`` (param dtype), ``G`` (grad
    dtype), ``M`` (float32).  Config 0 is float32 throughout, the others bf16
    params and grads.  ``layers`` or ``indices`` select a subset; the draws of a
    kept matrix do not depend on which others are kept.
    """
    specs_all = config_shapes(config)
    if layers is not None:
        per = len(config_shapes(config, layers=[0]))
        idx = [li * per + j for li in layers for j in range(per)]
    elif indices is not None:
        idx = list(indices)
    else:
        idx = list(range(len(specs_all)))
    dt = torch.float32 if config == 0 else torch.bfloat16
    out = {"specs": [], "W": [], "G": [], "M": [], "sigma": [], "index": idx}
    for i in idx:
        spec = specs_all[i]
        g, m, w, sigma = make_gradient(config, spec, i, device)
        out["specs"].append(spec)
        out["G"].append(g.to(dt).contiguous())
        out["M"].append(m.contiguous())
        out["W"].append(w.to(dt).contiguous())
        out["sigma"].append(sigma)
    return out


def random_matrix(rows: int, cols: int, seed: int, device="cpu", dtype=torch.float32):
    """Plain N(0,1) matrix from a seeded generator (edge-case tests)."""
    gen = _gen(torch.device(device), seed)
    return torch.randn(rows, cols, generator=gen, device=device, dtype=torch.float32).to(dtype)
