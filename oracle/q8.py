"""Asymmetric cache: q8_0 keys, TurboQuant values.

Oracle module (test infrastructure only).

The wis-web.com llama.cpp-fork post (first finding) reports that values can be
compressed to 2 bits at no measurable cost as long as the keys stay in q8_0,
and that the asymmetric configuration (K in q8_0, V in turbo3) recovers models
where symmetric compression fails. The pages name q8_0 without defining it; the
reading (llama.cpp's block format) is: each key vector is cut into blocks of 32
consecutive coordinates; a block stores d = max|x| / 127 as fp16 and the values
q_i = rint(x_i / d) as int8 (0 for an all-zero block); the key is d16 * q. No
rotation and no QJL bits for such keys. Values are quantized exactly as in
quantize.py.

Decode: l_t = scale * sum_b d16_tb <q_b, k8_tb> with the raw query q (blocks b
of 32 coordinates), then the usual softmax and value sum.
"""

from dataclasses import dataclass

import numpy as np

BLOCK = 32


@dataclass
class Q8:
    values: np.ndarray      # int64 in [-127, 127], [..., d]
    scales16: np.ndarray    # stored fp16 scales (as float64), [..., d / 32]
    ratio: np.ndarray       # x / d before rounding (for the rounding-boundary test), [..., d]


def quantize_q8(x) -> Q8:
    """q8_0 blocks of x[..., d] (d a multiple of 32)."""
    x = np.asarray(x, dtype=np.float64)
    blk = x.reshape(x.shape[:-1] + (x.shape[-1] // BLOCK, BLOCK))
    amax = np.max(np.abs(blk), axis=-1)
    d = amax / 127.0
    safe = np.where(d > 0, d, 1.0)
    ratio = np.where((d > 0)[..., None], blk / safe[..., None], 0.0)
    q = np.rint(ratio).astype(np.int64)
    return Q8(values=q.reshape(x.shape), scales16=d.astype(np.float16).astype(np.float64),
              ratio=ratio.reshape(x.shape))


def dequantize_q8(values, scales16):
    v = np.asarray(values, dtype=np.float64)
    blk = v.reshape(v.shape[:-1] + (v.shape[-1] // BLOCK, BLOCK))
    return (blk * np.asarray(scales16, dtype=np.float64)[..., None]).reshape(v.shape)


def logits_q8(q, values, scales16, scale):
    """Logits of T q8_0 keys for one raw query q[d]: values [T, d], scales16 [T, d / 32]."""
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    T, d = v.shape
    part = np.einsum("tbi,bi->tb", v.reshape(T, d // BLOCK, BLOCK), q.reshape(d // BLOCK, BLOCK))
    return scale * np.sum(np.asarray(scales16, dtype=np.float64) * part, axis=1)
