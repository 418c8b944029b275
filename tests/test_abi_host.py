"""CPU tests of the C-ABI library: it loads, exports every declared symbol, and
its host-side tables equal the oracle's bit for bit (no GPU needed)."""
import os
import re

import numpy as np
import pytest

from decode_attention_seeded_b200 import binding
from oracle import codebook as cb
from oracle import rng

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = binding.lib()
    names = declared_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert L.tq_version() >= 100
    assert L.tq_status_string(0) == b"ok"


@pytest.mark.parametrize("seed", [0, 1, 12345678901234567])
def test_sign_vector_matches_oracle(seed):
    host = binding.host_sign_vector(seed, 128).astype(np.float64)
    assert np.array_equal(host, rng.sign_vector(seed, 128))


@pytest.mark.parametrize("seed", [3, 2 ** 63 + 5])
def test_gaussian_sketch_matches_oracle_bitwise(seed):
    host = binding.host_gaussian_sketch(seed, 128, 128)
    ora = rng.gaussian_sketch(seed, 128, 128).astype(np.float16)
    assert np.array_equal(host.view(np.uint16), ora.view(np.uint16))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_matches_oracle_bitwise(bits):
    c, t = binding.host_codebook(bits, 128)
    book = cb.codebook(bits, 128)
    assert np.array_equal(c.astype(np.float64), book.centroids)
    assert np.array_equal(t.astype(np.float64), book.thresholds)


def test_host_rejects_bad_arguments():
    L = binding.lib()
    assert L.tq_host_sign_vector(1, 0, None) == 1
    assert L.tq_host_codebook(5, 128, None, None) == 1
    h = binding.ctypes.c_void_p()
    assert L.tq_create(binding.ctypes.byref(h), 64, 128, 16, 0) == 2      # unsupported head_dim
    assert L.tq_create(None, 128, 128, 16, 0) == 1
