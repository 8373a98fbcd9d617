"""Muon optimizer step, written out plainly in NumPy (float64, plus float32 where the
momentum buffer's own precision is the definition).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product path.  It shares no code with
the CUDA library.

The method, as the autoresearch ``train.py`` review (web3.cnoyu.systems post
71151920174080, MuonAdamW paragraph) describes it, for one 2-D weight W with
gradient G and momentum buffer M:

1. Nesterov momentum on the gradient.
2. Frobenius normalisation of the result (added by the benchmark spec; the page
   is silent).
3. Five Newton-Schulz steps with a per-step coefficient triple (a, b, c):
   tall (rows > cols):  A = X^T X,  X <- a X + X (b A + c A^2)
   otherwise (wide):    A = X X^T,  X <- a X + (b A + c A^2) X
4. W <- W - lr * sqrt(max(1, rows/cols)) * O with O the last X (task statement).

Readings taken where the page is silent or open (each is also listed in the
design notes of the library):

* Nesterov form: the PyTorch-SGD form M <- mu*M + G, U = G + mu*M (new M); with
  nesterov off, U = M.  The buffer is float32 and each product and sum is rounded
  on its own (no fused multiply-add), which is what the bit-exact buffer check
  compares against.
* Normalisation: X0 = U / (||U||_F + eps), eps added to the norm, not its square.
* A square matrix takes the wide rule (the page calls "tall" only rows > cols);
  both rules agree in exact arithmetic.
* The per-step coefficient table is an input; the page says the values are
  precomputed ("Polar Express") but prints none.  ``QUINTIC`` repeated five times
  is the default.
* Weight decay is optional (default off): W -= lr*wd*W on every entry, or only where
  the update and the parameter agree in sign (cautious decay; the page gives the mask
  (g x parameter) >= 0, read with g = O, the update that is applied).
* The interpolation form of the momentum (M <- mu*M + (1-mu)*G) is an option next to
  the default SGD form.
* NorMuon is optional (see ``normuon_rescale`` for its readings).
"""
from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

# Quintic triple used for every Newton-Schulz step unless a table is passed.
QUINTIC = (3.4445, -4.7750, 2.0315)
# Cubic triple of the classical Newton-Schulz polar iteration X <- 1.5X - 0.5 X X^T X;
# it converges to the polar factor and is used by the pins, not by the method.
CUBIC = (1.5, -0.5, 0.0)


def nesterov_momentum_f32(grad, momentum, mu: float, nesterov: bool = True, lerp: bool = False):
    """Momentum step on the float32 buffer (autoresearch review, MuonAdamW paragraph:
    Muon applies Nesterov momentum to the gradient; the buffer has the parameter's
    shape).

    Returns (M_new float32, U float64).  SGD form (default): M_new = fl32(fl32(mu*M) + G),
    U = G + mu*M_new for Nesterov, else M_new.  Interpolation ("lerp") form:
    M_new = fl32(fl32(mu*M) + fl32((1-mu)*G)), U = (1-mu)*G + mu*M_new for Nesterov, else
    M_new, with 1-mu rounded to float32 once.  NumPy float32 arithmetic rounds every
    product and sum separately; U is evaluated in float64 from the float32 values.
    """
    g32 = np.asarray(grad, dtype=np.float32)
    m32 = np.asarray(momentum, dtype=np.float32)
    mu32 = np.float32(mu)
    prod = np.multiply(mu32, m32, dtype=np.float32)
    if lerp:
        omu = np.float32(np.float32(1.0) - mu32)
        m_new = np.add(prod, np.multiply(omu, g32, dtype=np.float32), dtype=np.float32)
        if nesterov:
            u = np.float64(omu) * g32.astype(np.float64) + np.float64(mu32) * m_new.astype(np.float64)
        else:
            u = m_new.astype(np.float64)
        return m_new, u
    m_new = np.add(prod, g32, dtype=np.float32)
    if nesterov:
        u = g32.astype(np.float64) + np.float64(mu32) * m_new.astype(np.float64)
    else:
        u = m_new.astype(np.float64)
    return m_new, u


def frobenius_normalise(u, eps: float):
    """X0 = U / (||U||_F + eps), float64 (normalisation before the iteration, as the
    task statement fixes it)."""
    u = np.asarray(u, dtype=np.float64)
    norm = math.sqrt(float(np.sum(u * u)))
    return u / (norm + eps)


def newton_schulz(x0, coeffs: Sequence[Sequence[float]]):
    """Newton-Schulz steps in float64, one per row (a, b, c) of ``coeffs``
    (autoresearch review, MuonAdamW paragraph: tall rule A = X^T X,
    X <- aX + X(bA + cA^2); wide rule A = X X^T, X <- aX + (bA + cA^2)X).
    Rows > cols is tall; everything else takes the wide rule."""
    x = np.array(x0, dtype=np.float64, copy=True)
    if x.ndim != 2:
        raise ValueError("newton_schulz expects a 2-D matrix")
    tall = x.shape[0] > x.shape[1]
    for row in coeffs:
        a, b, c = (float(v) for v in row)
        if tall:
            gram = x.T @ x
            poly = b * gram + c * (gram @ gram)
            x = a * x + x @ poly
        else:
            gram = x @ x.T
            poly = b * gram + c * (gram @ gram)
            x = a * x + poly @ x
    return x


def update_scale(rows: int, cols: int) -> float:
    """sqrt(max(1, rows/cols)), the shape factor of the applied update (task
    statement; the page gives none)."""
    return math.sqrt(max(1.0, rows / cols))


def cautious_mask(o, w):
    """Cautious weight decay (autoresearch review, MuonAdamW paragraph): only entries whose
    update and parameter agree in sign decay, mask = (O * W) >= 0 (zeros included)."""
    return (np.asarray(o, dtype=np.float64) * np.asarray(w, dtype=np.float64)) >= 0


def normuon_rescale(o, v, beta2: float, eps: float):
    """NorMuon (autoresearch review, MuonAdamW paragraph): after orthogonalisation, a
    second-moment estimate per row -- or per column, by aspect ratio -- kept as an EMA
    and used to give every output dimension its own step size.

    Readings: the statistics run over the longer dimension, one per index of the
    shorter one (rows of a wide matrix, columns of a tall one); v <- beta2*v +
    (1-beta2)*mean(O^2); O' = O / (sqrt(v) + eps); O' is rescaled to the Frobenius norm
    of O, which keeps the step size's meaning and makes a bias correction of v
    unnecessary (it would scale every row alike).  Returns (O'' float64, v_new float64).
    """
    o = np.asarray(o, dtype=np.float64)
    rows, cols = o.shape
    per_row = rows <= cols
    q = np.mean(o * o, axis=1 if per_row else 0)
    v_new = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * q
    f = 1.0 / (np.sqrt(v_new) + eps)
    o1 = o * (f[:, None] if per_row else f[None, :])
    n0, n1 = math.sqrt(float(np.sum(o * o))), math.sqrt(float(np.sum(o1 * o1)))
    o2 = o1 * (n0 / n1) if n1 > 0 else o1
    return o2, v_new


def muon_step_matrix(w, grad, momentum, *, lr: float, mu: float, nesterov: bool = True,
                     coeffs: Sequence[Sequence[float]] | None = None, eps: float = 1e-7,
                     lerp: bool = False, weight_decay: float = 0.0, cautious: bool = False,
                     normuon_state=None, normuon_beta2: float = 0.95, normuon_eps: float = 1e-8):
    """One Muon step for one matrix.

    Returns (W_new float64, M_new float32, O float64).  W_new is the exact
    W - lr*scale*O - lr*weight_decay*mask*W with mask = 1 everywhere, or the cautious
    mask when ``cautious``; rounding to the parameter's dtype is the caller's concern.
    With ``normuon_state`` (the previous second-moment vector), O is replaced by its
    NorMuon rescaling and the function returns (W_new, M_new, O'', v_new).
    """
    if coeffs is None:
        coeffs = [QUINTIC] * 5
    w64 = np.asarray(w, dtype=np.float64)
    rows, cols = w64.shape
    m_new, u = nesterov_momentum_f32(grad, momentum, mu, nesterov, lerp=lerp)
    x0 = frobenius_normalise(u, eps)
    o = newton_schulz(x0, coeffs)
    v_new = None
    if normuon_state is not None:
        o, v_new = normuon_rescale(o, normuon_state, normuon_beta2, normuon_eps)
    w_new = w64 - lr * update_scale(rows, cols) * o
    if weight_decay:
        mask = cautious_mask(o, w64) if cautious else np.ones_like(w64, dtype=bool)
        w_new = w_new - lr * weight_decay * np.where(mask, w64, 0.0)
    if v_new is not None:
        return w_new, m_new, o, v_new
    return w_new, m_new, o


def muon_step(params: Iterable, grads: Iterable, moms: Iterable, **kw):
    """Muon step over a list of matrices, one after another (no grouping)."""
    out = []
    for w, g, m in zip(params, grads, moms):
        out.append(muon_step_matrix(w, g, m, **kw))
    return out
