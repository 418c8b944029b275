"""Pins of the oracle's q8_0 keys (asymmetric cache: q8_0 keys, TurboQuant values)."""
import numpy as np
import pytest

from oracle import codebook as cb
from oracle import decode as dec
from oracle import layout as lay
from oracle import q8
from oracle.hadamard import unrotate
from oracle.quantize import quantize
from oracle.rng import sign_vector

D = 128


def test_hand_worked_blocks():
    x = np.zeros(D)
    x[:6] = [127.0, -63.5, 0.4, -0.6, 2.5, -127.0]       # block 0: amax 127 -> d = 1
    x[64:66] = [1.27, 0.635]                              # block 2: d = 0.01, 0.635 / 0.01 = 63.5
    r = q8.quantize_q8(x)
    assert list(r.values[:6]) == [127, -64, 0, -1, 2, -127]   # rint: halves to even
    assert r.scales16[0] == 1.0
    assert r.scales16[1] == 0.0 and np.all(r.values[32:64] == 0)     # all-zero block
    assert r.values[64] == 127 and r.values[65] == 64
    assert r.scales16[2] == np.float64(np.float16(0.01))
    assert r.scales16[3] == 0.0


def test_error_bound_and_extremes():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((500, D)) * np.exp(rng.standard_normal(D))
    r = q8.quantize_q8(x)
    blk = x.reshape(500, 4, 32)
    d = np.max(np.abs(blk), axis=-1) / 127.0
    err = np.abs(blk - r.values.reshape(500, 4, 32) * r.scales16[..., None])
    lim = d[..., None] / 2 + 127 * np.abs(d - r.scales16)[..., None]
    assert np.all(err <= lim * (1 + 1e-12))
    # the largest coordinate of each block maps to +-127
    amax_pos = np.argmax(np.abs(blk), axis=-1)
    v = np.take_along_axis(r.values.reshape(500, 4, 32), amax_pos[..., None], axis=-1)[..., 0]
    assert np.all(np.abs(v) == 127)
    assert np.all(np.abs(r.values) <= 127)


def test_exactly_representable_keys_give_the_plain_dot_product():
    # keys equal to an fp16 scale times integers with max |n| = 127 are stored
    # exactly, so the logits are the plain scaled dot products
    rng = np.random.default_rng(4)
    n = rng.integers(-127, 128, size=(40, 4, 32))
    n[:, :, 0] = 127
    s = np.float16(rng.uniform(0.01, 2.0, size=(40, 4))).astype(np.float64)
    k = (n * s[..., None]).reshape(40, D)
    r = q8.quantize_q8(k)
    assert np.array_equal(r.values, n.reshape(40, D)) and np.array_equal(r.scales16, s)
    q = rng.standard_normal(D)
    got = q8.logits_q8(q, r.values, r.scales16, 0.25)
    np.testing.assert_allclose(got, 0.25 * (k @ q), rtol=1e-13)


def test_layout_covers_every_byte_and_round_trips():
    idx = lay.q8_byte_index()
    assert np.array_equal(np.sort(idx.ravel()), np.arange(2048))
    entries = sorted(lay.q8_scale_entry(t, kt) for t in range(16) for kt in range(4))
    assert entries == list(range(64))
    for bv in (2, 3, 4):
        off = lay.section_offsets(8, bv)
        vb = lay.v_bit_index(8, bv)
        assert vb.min() == 8 * off["v"] and vb.max() == 8 * off["norm"] - 1
        assert lay.block_bytes(8, bv) == 16 * (128 + 8 + 16 * bv + 2)
        rng = np.random.default_rng(bv)
        blk = rng.integers(0, 256, size=lay.block_bytes(8, bv), dtype=np.uint8)
        vals = rng.integers(-127, 128, size=(16, D))
        sc = rng.standard_normal((16, 4)).astype(np.float16).astype(np.float64)
        vc = rng.integers(0, 2 ** bv, size=(16, D))
        vn = np.abs(rng.standard_normal(16)).astype(np.float16).astype(np.float64)
        for t in rng.permutation(16):
            lay.write_token_q8(blk, t, bv, vals[t], sc[t], vc[t], vn[t])
        got = lay.read_page_q8(blk, bv)
        for a, b in zip(got, (vals, sc, vc, vn)):
            assert np.array_equal(a, b)


def test_hand_derived_q8_positions():
    # token 9, coordinate 77: g=1 th=1 kt=2 sub=0 t=3 q=1 -> lane 7 -> byte 64*7 + 32 + 16 + 0 + 1
    assert lay.q8_byte_index()[9, 77] == 497
    # its block scale: entry 8*1 + 4*1 + 2
    assert lay.q8_scale_entry(9, 2) == 14


def test_q8_paged_decode_is_attention_over_the_dequantised_keys():
    rng = np.random.default_rng(7)
    bv, L = 2, 70
    book = cb.codebook(bv)
    dv = sign_vector(21, D)
    k = rng.standard_normal((L, D)) * 3.0
    v = rng.standard_normal((L, D))
    kq = q8.quantize_q8(k)
    qv = quantize(v, dv, book.centroids, book.thresholds)
    pages = (L + 15) // 16
    perm = rng.permutation(pages)
    cache = np.zeros((pages, 1, lay.block_bytes(8, bv)), dtype=np.uint8)
    for t in range(L):
        lay.write_token_q8(cache[perm[t // 16], 0], t % 16, bv, kq.values[t], kq.scales16[t], qv.codes[t],
                           qv.norm16[t])
    tables = dict(signs_k=None, signs_v=dv, sketch=np.zeros((128, D)), centroids_k=None,
                  centroids_v=book.centroids, bk=8, bv=bv)
    qry = rng.standard_normal((1, 2, D))
    out = dec.decode_paged(cache, perm[None], [L], qry, tables)
    khat = q8.dequantize_q8(kq.values, kq.scales16)
    vhat = qv.norm16[:, None] * unrotate(book.centroids[qv.codes], dv)
    for h in range(2):
        lg = khat @ qry[0, h] / np.sqrt(D)
        w = np.exp(lg - lg.max())
        np.testing.assert_allclose(out[0, h], (w / w.sum()) @ vhat, rtol=1e-11, atol=1e-13)
