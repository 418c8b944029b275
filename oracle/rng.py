"""Seeded random tables of the method: sign vectors D and the Gaussian sketch S.

Oracle module (test infrastructure only).

The pages fix only that the rotation signs and the QJL projection are random
and seeded ("data-oblivious", snilld.dk "Hvad papiret haevder"; QJL paragraph of
the wis-web.com llama.cpp-fork post). The generator is a reading: SplitMix64
(Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014), used counter-style, with the Box-Muller transform (1958) for
normal deviates. The CUDA library implements the same published definitions
independently.
"""

import numpy as np

GOLDEN_GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB


def splitmix64(seed: int, n: int) -> np.ndarray:
    """First ``n`` outputs of SplitMix64 started from state ``seed``.

    Output j is the 64-bit finaliser applied to ``seed + (j + 1) * gamma``
    (mod 2**64): the state is advanced by the golden gamma before each output.
    """
    j = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed % (1 << 64)) + j * np.uint64(GOLDEN_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MIX2)
        z = z ^ (z >> np.uint64(31))
    return z


def sign_vector(seed: int, d: int) -> np.ndarray:
    """Random +-1 diagonal D (float64): entry i is -1 iff the top bit of output i is set."""
    top = splitmix64(seed, d) >> np.uint64(63)
    return np.where(top == 0, 1.0, -1.0)


def uniform53(words: np.ndarray) -> np.ndarray:
    """Top 53 bits of each 64-bit word as a double in [0, 1)."""
    return (words >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def gaussian_sketch(seed: int, m: int, d: int) -> np.ndarray:
    """QJL projection S (m x d), entries N(0,1) rounded to fp16, returned as float64.

    Entry k = r*d + c uses outputs 2k and 2k+1: u1 = (top53 + 1) * 2**-53 in (0, 1],
    u2 = top53 * 2**-53 in [0, 1), value = sqrt(-2 ln u1) * cos(2 pi u2)
    (the cosine branch of Box-Muller). The fp16 rounding (round to nearest even)
    is part of the definition: the fp16 value IS the sketch entry everywhere.
    """
    w = splitmix64(seed, 2 * m * d)
    u1 = uniform53(w[0::2]) + 2.0 ** -53
    u2 = uniform53(w[1::2])
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return z.astype(np.float16).astype(np.float64).reshape(m, d)
