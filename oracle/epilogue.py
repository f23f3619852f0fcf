"""float64 oracle of the GLA layer's output epilogue.

TEST INFRASTRUCTURE ONLY (never imported by the product path).

"Gated Linear Attention Transformers with Hardware-Efficient Training", the GLA
layer around the recurrence: every head's output o_t (d_v values) is normalised
by a LayerNorm over its d_v channels, the heads are concatenated, and the result
is multiplied elementwise by a Swish output gate r_t (Swish(x) = x sigmoid(x))
before the output projection (which is outside this epilogue).  Readings: the
LayerNorm has one affine weight w and bias b of size d_v shared by every head,
epsilon 1e-5, biased variance; r_t arrives in o's [B,H,T,d_v] layout.

    y = (w (.) (o - mean(o)) / sqrt(var(o) + eps) + b) (.) r sigmoid(r)

The backward is the chain rule written out for these two elementwise maps and
the normalisation, in float64.
"""
from __future__ import annotations

import numpy as np


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def fwd(o, r, w=None, b=None, eps=1e-5):
    """y [..., V] from o, r [..., V]; w, b [V] (None: ones / zeros)."""
    o = np.asarray(o, np.float64)
    r = np.asarray(r, np.float64)
    V = o.shape[-1]
    w = np.ones(V) if w is None else np.asarray(w, np.float64)
    b = np.zeros(V) if b is None else np.asarray(b, np.float64)
    mu = o.mean(axis=-1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=-1, keepdims=True)
    xhat = (o - mu) / np.sqrt(var + eps)
    n = xhat * w + b
    return n * (r * _sigmoid(r))


def bwd(o, r, dy, w=None, b=None, eps=1e-5):
    """(do, dr, dw, db) for y = fwd(o, r, w, b, eps) and upstream dy."""
    o = np.asarray(o, np.float64)
    r = np.asarray(r, np.float64)
    dy = np.asarray(dy, np.float64)
    V = o.shape[-1]
    w = np.ones(V) if w is None else np.asarray(w, np.float64)
    b = np.zeros(V) if b is None else np.asarray(b, np.float64)
    mu = o.mean(axis=-1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (o - mu) * rstd
    n = xhat * w + b
    sg = _sigmoid(r)
    g = r * sg
    dn = dy * g
    dr = dy * n * (sg * (1.0 + r * (1.0 - sg)))       # d/dr of r sigmoid(r)
    dxhat = dn * w
    do = rstd * (dxhat - dxhat.mean(axis=-1, keepdims=True) - xhat * (dxhat * xhat).mean(axis=-1, keepdims=True))
    red = tuple(range(o.ndim - 1))
    dw = (dn * xhat).sum(axis=red)
    db = dn.sum(axis=red)
    return do, dr, dw, db
