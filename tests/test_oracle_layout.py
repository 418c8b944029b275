"""Pins of the page-block byte layout."""
import json
import os

import numpy as np
import pytest

from oracle import layout as lay

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = [(bk, bv) for bk in (2, 3, 4) for bv in (2, 3, 4)]


@pytest.mark.parametrize("bk,bv", BITS)
def test_every_bit_used_exactly_once(bk, bv):
    off = lay.section_offsets(bk, bv)
    used = np.concatenate([lay.k_bit_index(bk).ravel(), lay.sign_bit_index(bk).ravel(),
                           lay.v_bit_index(bk, bv).ravel()])
    assert used.size == len(np.unique(used))
    assert used.min() == 0 and used.max() == 8 * off["norm"] - 1
    assert used.size == 8 * off["norm"]


@pytest.mark.parametrize("bk,bv", BITS)
def test_pack_unpack_round_trip(bk, bv):
    rng = np.random.default_rng(bk * 10 + bv)
    blk = rng.integers(0, 256, size=lay.block_bytes(bk, bv), dtype=np.uint8)   # stale bytes
    kc = rng.integers(0, 2 ** bk, size=(16, 128))
    sb = rng.integers(0, 2, size=(16, 128))
    vc = rng.integers(0, 2 ** bv, size=(16, 128))
    nrm = rng.standard_normal((3, 16)).astype(np.float16).astype(np.float64)
    for t in rng.permutation(16):
        lay.write_token(blk, t, bk, bv, kc[t], sb[t], vc[t], nrm[0, t], nrm[1, t], nrm[2, t])
    got = lay.read_page(blk, bk, bv)
    for a, b in zip(got[:3], (kc, sb, vc)):
        assert np.array_equal(a, b)
    for a, b in zip(got[3:], nrm):
        assert np.array_equal(a, b)


def test_hand_derived_positions():
    ref = json.load(open(os.path.join(GOLDEN, "layout_positions.json")))
    for c in ref["cases"]:
        if c["field"] == "k":
            got = lay.k_bit_index(c["bk"])[c["token"], c["index"]]
        elif c["field"] == "sign":
            got = [lay.sign_bit_index(c["bk"])[c["token"], c["index"]]]
        else:
            got = lay.v_bit_index(c["bk"], c["bv"])[c["token"], c["index"]]
        assert list(map(int, got)) == c["bits"], c["derivation"]


def test_byte_accounting():
    # per (token, KV head): K = 16 b_k + 16 (sign bits) + 4 (two fp16 norms); V = 16 b_v + 2
    for bk, bv, per_token in [(3, 2, 102), (4, 4, 150), (4, 2, 118), (3, 3, 118)]:
        assert lay.block_bytes(bk, bv) == 16 * per_token
    # the 70B-class fp16 cache at 128K context (80 layers x 8 KV heads) exceeds 40 GB
    fp16_bytes = 80 * 8 * 128 * 2 * 2 * 131072
    assert fp16_bytes > 40e9
    assert abs(512 / 102 - 5.02) < 0.01


def test_hand_derived_norm_and_scale_bytes():
    # Each case writes one token with distinctive fp16 fields into a zero block and
    # reads the two bytes at the hand-derived offset (not through norm_slot).
    ref = json.load(open(os.path.join(GOLDEN, "layout_positions.json")))
    vals = {"norm_k": 1.5, "gamma": 2.5, "norm_v": 3.5, "q8_norm_v": 3.5, "q8_scale": 0.75}
    for c in ref["byte_cases"]:
        bk, bv, tau = c["bk"], c["bv"], c["token"]
        blk = np.zeros(lay.block_bytes(bk, bv), dtype=np.uint8)
        if bk == 8:
            scales = [0.25, 0.5, 0.75, 1.0]
            lay.write_token_q8(blk, tau, bv, np.zeros(128, dtype=np.int64), scales, np.zeros(128, dtype=np.int64),
                               3.5)
        else:
            lay.write_token(blk, tau, bk, bv, np.zeros(128, dtype=np.int64), np.zeros(128, dtype=np.int64),
                            np.zeros(128, dtype=np.int64), 1.5, 2.5, 3.5)
        got = float(blk[c["byte"]:c["byte"] + 2].view(np.float16)[0])
        assert got == vals[c["field"]], c["derivation"]
        # and nothing else in the norm/scale sections holds that value's bytes
        want = np.array([vals[c["field"]]], dtype=np.float16).view(np.uint8)
        hits = [i for i in range(0, blk.size - 1, 2) if blk[i] == want[0] and blk[i + 1] == want[1]]
        assert hits == [c["byte"]], c["derivation"]
