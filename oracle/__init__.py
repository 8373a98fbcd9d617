"""Plain CPU oracle for the Muon optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its
Python binding) imports, links or runs this package; only the tests, the smoke
check and the CPU baseline of the benchmark do.  It shares no code with the CUDA
path.

Sources (cited by page title and passage):

* "karpathy/autoresearch train.py, read line by line" (web3.cnoyu.systems, post
  71151920174080), the paragraph on the MuonAdamW optimizer: Muon takes the
  gradient of each 2-D weight, applies Nesterov momentum, and runs five
  Newton-Schulz steps that approximate the orthogonal factor U of the polar
  decomposition G = U S; tall matrices (more rows than columns) use A = X^T X and
  X <- aX + X(bA + cA^2), wide ones A = X X^T and X <- aX + (bA + cA^2)X, with
  hard-coded per-step coefficients ("Polar Express").  The momentum buffer has the
  parameter's shape.
* The benchmark spec of this library adds what the page leaves open: Frobenius
  normalisation with eps before the iteration, the update W -= lr*sqrt(max(1,r/c))*O,
  and the quintic triple (3.4445, -4.7750, 2.0315) as the default for every step.

Readings where the page is silent are listed in the module docstrings of
``oracle.muon``.
"""
from .muon import (  # noqa: F401
    QUINTIC,
    CUBIC,
    nesterov_momentum_f32,
    frobenius_normalise,
    newton_schulz,
    update_scale,
    muon_step_matrix,
    muon_step,
    cautious_mask,
    normuon_rescale,
)
