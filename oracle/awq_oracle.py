"""Plain, slow, fp64 CPU oracle for the AWQ scale search.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py`` import this module.  It shares no code
with the CUDA library, and the library never imports it.

What it follows (dingiv.github.io "量化" page, section AWQ):

* the salient input channels are the ones with large activations, measured
  per channel as the mean activation magnitude ``s_X``;
* equivalent transform: the weights of input channel ``k`` are multiplied by
  ``s_k`` before quantization and the activations divided by ``s_k``, so the
  layer computes ``Q(W diag(s)) diag(s)^-1 X``;
* ``s = s_X ** alpha`` with a single exponent ``alpha`` in ``[0, 1]`` chosen by
  a 20-point grid search: ``alpha* = argmin_alpha L(s_X ** alpha)``;
* 4-bit weights (AWQ is INT4 weight-only on the page).

Readings of points the page leaves open (each also listed in the design
notes):

* ``L`` is the layer's output error on the calibration tokens,
  ``||W X - Q(W diag(s)) diag(s)^-1 X||_F^2``, the objective of the GPTQ
  section.  It is evaluated as ``1/2 sum_r dW_r H dW_r^T`` with
  ``H = 2 X X^T`` (equal by algebra; pinned against the direct form);
* the grid is the 20 points ``alpha_a = a / 19``, ``a = 0..19``, both ends
  included;
* ``Q`` is the GPTQ oracle's asymmetric min-max quantizer, per group of
  ``group`` input channels (per output row when ``group`` is 0), applied to
  the scaled weights once (no error feedback);
* a channel with ``s_X = 0`` (no activation at all) keeps ``s = 1``;
* ties go to the smallest ``alpha``.

``dtype`` is the precision of the integer decisions, as in the GPTQ
oracle: float64 here, float32 when matching a float32 implementation (then
``s`` and ``W diag(s)`` are also rounded to float32 before quantization).
"""
from __future__ import annotations

import numpy as np

from . import gptq_oracle as G

F64 = np.float64


def channel_scale(x_tokens) -> np.ndarray:
    """``s_X[k]``: the mean of ``|x[t][k]|`` over the tokens ``t`` (fp64)."""
    x = np.asarray(x_tokens, dtype=F64)
    return np.mean(np.abs(x), axis=0)


def alpha_grid(n_grid: int = 20) -> np.ndarray:
    """``alpha_a = a / (n_grid - 1)`` for ``a = 0 .. n_grid - 1``."""
    return np.arange(n_grid, dtype=F64) / F64(n_grid - 1)


def scales_for(sx, alpha: float, dtype=F64) -> np.ndarray:
    """``s = s_X ** alpha`` (fp64), ``s = 1`` where ``s_X = 0``; rounded to
    ``dtype``."""
    sx = np.asarray(sx, dtype=F64)
    s = np.where(sx > 0, np.power(np.where(sx > 0, sx, 1.0), F64(alpha)), 1.0)
    return s.astype(dtype)


def quantize_scaled(w, s, bits: int = 4, group: int = 128, dtype=F64) -> dict:
    """Quantize ``W diag(s)`` with the min-max quantizer; ``w_hat`` is the
    effective weight ``Q(W diag(s)) diag(s)^-1`` (fp64)."""
    w = np.asarray(w, dtype=F64)
    s = np.asarray(s, dtype=dtype)
    ws = (w.astype(dtype) * s[None, :]).astype(dtype)
    r = G.rtn(ws, bits=bits, group=group, sym=False, dtype=dtype)
    r["w_scaled"] = ws.astype(F64)
    r["w_hat"] = r["w_hat"] / s.astype(F64)[None, :]
    return r


def search(w, h, sx, bits: int = 4, group: int = 128, n_grid: int = 20, dtype=F64) -> dict:
    """The grid search: the loss of every ``alpha`` and the quantization at
    the best one (``codes``, ``scales``, ``zeros`` of ``W diag(s*)``, and
    ``s*``)."""
    alphas = alpha_grid(n_grid)
    losses = np.zeros(n_grid)
    for a, alpha in enumerate(alphas):
        s = scales_for(sx, alpha, dtype)
        r = quantize_scaled(w, s, bits, group, dtype)
        losses[a] = G.layer_loss_hessian(w, r["w_hat"], h)
    best = int(np.argmin(losses))  # the first minimum: ties go to the smaller alpha
    s = scales_for(sx, alphas[best], dtype)
    r = quantize_scaled(w, s, bits, group, dtype)
    return dict(alphas=alphas, losses=losses, best=best, s=s.astype(F64), codes=r["codes"],
                scales=r["scales"], zeros=r["zeros"], w_hat=r["w_hat"])
