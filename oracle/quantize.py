"""Per-vector quantiser: norm, rotation, Lloyd-Max codes, QJL residual bits.

Oracle module (test infrastructure only).

Steps follow the two-stage description on the wis-web.com llama.cpp-fork post
(PolarQuant paragraph: rotate, keep a radius, code the direction against a law
known in advance; QJL paragraph: one bit per projection of the residual, no
stored quantisation constants), with these readings:

* the "radius" is the L2 norm n = ||x||, stored in fp16;
* the direction y = R x / n is coded coordinate by coordinate with the fixed
  b-bit codebook (no per-block scale);
* keys only: residual u = y - c[code] in the rotated unit domain, its scaled
  norm gamma = n ||u|| (fp16), and sign bits s_r = [ (S u)_r >= 0 ] for the m
  rows of the seeded Gaussian sketch S. Because R is orthogonal, S R^T is
  again i.i.d. Gaussian, so sketching u (rotated domain) has the same law as
  sketching the residual k - k_hat in the original domain;
* the zero vector gets y = 0 (codes by the tie rule) and n = gamma = 0.
"""

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .codebook import encode
from .hadamard import rotate


@dataclass
class Quantized:
    norm: np.ndarray            # exact float64 norms
    norm16: np.ndarray          # stored fp16 norms (as float64)
    y: np.ndarray               # rotated unit vectors
    codes: np.ndarray           # int64 codes, ascending-centroid index
    residual: Optional[np.ndarray] = None   # u = y - c[code]            (keys)
    gamma: Optional[np.ndarray] = None      # n ||u||                    (keys)
    gamma16: Optional[np.ndarray] = None    # stored fp16 gamma          (keys)
    projection: Optional[np.ndarray] = None  # z = S u                   (keys)
    sign_bits: Optional[np.ndarray] = None   # [z >= 0] as 0/1 int64     (keys)


def quantize(x, signs, centroids, thresholds, sketch=None) -> Quantized:
    """Quantise vectors x[..., d]; pass ``sketch`` (m x d) for keys."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    n = np.sqrt(np.sum(x * x, axis=-1))
    safe = np.where(n > 0, n, 1.0)
    y = rotate(x, signs) / safe[..., None]
    y = np.where((n > 0)[..., None], y, 0.0)
    codes = encode(y, thresholds)
    out = Quantized(norm=n, norm16=n.astype(np.float16).astype(np.float64), y=y, codes=codes)
    if sketch is not None:
        u = y - np.asarray(centroids)[codes]
        gamma = n * np.sqrt(np.sum(u * u, axis=-1))
        z = u @ np.asarray(sketch, dtype=np.float64).T
        out.residual = u
        out.gamma = gamma
        out.gamma16 = gamma.astype(np.float16).astype(np.float64)
        out.projection = z
        out.sign_bits = (z >= 0).astype(np.int64)
    assert d == y.shape[-1]
    return out
