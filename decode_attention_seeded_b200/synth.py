"""Seeded synthetic workloads (inputs only; none of the method's arithmetic).

Shared by the tests, ``bench.py`` and the oracle-driven checks. Everything is
drawn with NumPy's PCG64 from a per-workload seed, so both the CUDA path and the
float64 oracle see identical inputs.

Workloads (head_dim 128, QJL rows m = 128, 16-token pages), shaped like the
pages' examples (Llama-3.1-8B, Llama-70B, Command-R+ 104B class GQA decode):

* ``tiny``      1 KV / 1 query head, 1024 tokens, fp32 K/V i.i.d. N(0,1) with 4
                outlier channels x20, keys 3-bit + QJL, values 3-bit.
* ``llama8b``   batch 1, 32 q / 8 KV heads, 32768 cached tokens, bf16 K/V
                N(0,1) x per-(head, channel) lognormal(0,1) scale x 10 on
                round(2% * 128) = 3 outlier channels; keys 3-bit, values 2-bit;
                decode steps append one token each.
* ``batched``   16 sequences, 32 q / 8 KV heads, lengths uniform in
                [2048, 8192], data as ``llama8b``; keys 4-bit, values 4-bit.
* ``llama70b``  batch 1, 64 q / 8 KV heads, 131072 tokens, lognormal scales,
                no outliers; keys 3-bit, values 2-bit.
* ``cmdr104b``  batch 4, 96 q / 8 KV heads, 131072 tokens each, N(0,1) with
                round(1% * 128) = 1 outlier channel x20; keys 4-bit, values 2-bit.

Queries are N(0,1). Physical pages are a random permutation of the pool.
"""

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

HEAD_DIM = 128
QJL_ROWS = 128
PAGE_SIZE = 16


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    context: int                 # cached tokens per sequence (max for ragged)
    key_bits: int
    value_bits: int
    dtype: str                   # "fp32" or "bf16" K/V inputs
    lognormal: bool
    outlier_frac: float          # fraction of channels that are outliers
    outlier_count: int           # explicit count (overrides the fraction when > 0)
    outlier_scale: float
    ragged: Optional[tuple] = None   # (lo, hi) inclusive context lengths
    n_layers: int = 1
    decode_steps: int = 1
    notes: List[str] = field(default_factory=list)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 1, 1, 1024, 3, 3, "fp32", False, 0.0, 4, 20.0),
    "llama8b": Workload("llama8b", 1, 1, 32, 8, 32768, 3, 2, "bf16", True, 0.02, 0, 10.0,
                        n_layers=32, decode_steps=128),
    "batched": Workload("batched", 2, 16, 32, 8, 8192, 4, 4, "bf16", True, 0.02, 0, 10.0,
                        ragged=(2048, 8192)),
    "llama70b": Workload("llama70b", 3, 1, 64, 8, 131072, 3, 2, "bf16", True, 0.0, 0, 1.0,
                         decode_steps=32),
    "cmdr104b": Workload("cmdr104b", 4, 4, 96, 8, 131072, 4, 2, "bf16", False, 0.01, 0, 20.0),
    # the llama8b cache with q8_0 keys and 3-bit TurboQuant values (the asymmetric setting)
    "llama8b_q8k": Workload("llama8b_q8k", 1, 1, 32, 8, 32768, 8, 3, "bf16", True, 0.02, 0, 10.0,
                            n_layers=32, decode_steps=128),
}


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((a >> np.uint32(16)) & np.uint32(1))
    r = ((a + bias) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32)


class Generator:
    """Deterministic inputs of one workload: channel scales are fixed per seed."""

    def __init__(self, wl: Workload, layer: int = 0):
        self.wl = wl
        self.layer = layer
        root = np.random.default_rng([wl.seed, layer, 0x7A11])
        d, h = HEAD_DIM, wl.n_kv_heads
        n_out = wl.outlier_count if wl.outlier_count > 0 else int(round(wl.outlier_frac * d))
        self.scales = {}
        for which in ("k", "v"):
            s = np.exp(root.standard_normal((h, d))) if wl.lognormal else np.ones((h, d))
            for hh in range(h):
                ch = root.choice(d, size=n_out, replace=False) if n_out else []
                s[hh, ch] *= wl.outlier_scale
            self.scales[which] = s
        self._seed_root = root.integers(0, 2 ** 62, size=8)

    def method_seeds(self):
        """(seed_k, seed_v, seed_s) for the rotation signs and the sketch."""
        return tuple(int(x) for x in self._seed_root[:3])

    def _cast(self, x: np.ndarray) -> np.ndarray:
        x = x.astype(np.float32)
        return round_to_bf16(x) if self.wl.dtype == "bf16" else x

    def kv(self, which: str, start: int, count: int, stream: int = 0) -> np.ndarray:
        """Tokens [start, start+count) of K or V for one sequence: [count, n_kv, d] float32."""
        wl = self.wl
        rng = np.random.default_rng([wl.seed, self.layer, 1 if which == "k" else 2, stream, start, count])
        x = rng.standard_normal((count, wl.n_kv_heads, HEAD_DIM)) * self.scales[which][None]
        return self._cast(x)

    def queries(self, step: int = 0) -> np.ndarray:
        wl = self.wl
        rng = np.random.default_rng([wl.seed, self.layer, 3, step])
        return self._cast(rng.standard_normal((wl.batch, wl.n_q_heads, HEAD_DIM)))

    def seq_lens(self) -> np.ndarray:
        wl = self.wl
        if wl.ragged is None:
            return np.full(wl.batch, wl.context, dtype=np.int64)
        rng = np.random.default_rng([wl.seed, 4])
        return rng.integers(wl.ragged[0], wl.ragged[1] + 1, size=wl.batch).astype(np.int64)

    def page_pool(self, pages_per_seq: np.ndarray, extra: int = 0):
        """Randomly permuted physical pages; returns (block_tables [B, max_pages], n_pages)."""
        total = int(np.sum(pages_per_seq)) + extra
        rng = np.random.default_rng([self.wl.seed, 5, self.layer])
        perm = rng.permutation(total).astype(np.int32)
        maxp = int(np.max(pages_per_seq))
        bt = np.zeros((len(pages_per_seq), maxp), dtype=np.int32)
        o = 0
        for b, n in enumerate(pages_per_seq):
            bt[b, :n] = perm[o:o + n]
            o += n
        return bt, total


def slots_for(block_table: np.ndarray, start: int, count: int) -> np.ndarray:
    """Slot ids (physical_page * 16 + offset) of logical tokens [start, start+count)."""
    pos = np.arange(start, start + count)
    return (block_table[pos // PAGE_SIZE].astype(np.int64) * PAGE_SIZE + pos % PAGE_SIZE)
