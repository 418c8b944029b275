"""Pins of the oracle's quantizer, QJL estimator and decode attention."""
import numpy as np
import pytest

from oracle import codebook as cb
from oracle import decode as dec
from oracle import layout as lay
from oracle.hadamard import rotate, unrotate
from oracle.quantize import quantize
from oracle.rng import gaussian_sketch, sign_vector

D = 128


def test_zero_vector():
    book = cb.codebook(3)
    s = gaussian_sketch(1, D, D)
    qz = quantize(np.zeros((1, D)), sign_vector(2, D), book.centroids, book.thresholds, s)
    assert qz.norm16[0] == 0 and qz.gamma16[0] == 0 and np.all(qz.y == 0)
    assert np.all(qz.codes == 3)          # y = 0 equals the middle threshold -> lower cell


def test_rotated_vector_unit_and_norm_exact():
    book = cb.codebook(2)
    x = np.random.default_rng(0).standard_normal((50, D)) * 7
    qz = quantize(x, sign_vector(2, D), book.centroids, book.thresholds)
    np.testing.assert_allclose(np.linalg.norm(qz.y, axis=1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(qz.norm, np.linalg.norm(x, axis=1), rtol=1e-15)
    assert np.array_equal(qz.norm16, qz.norm.astype(np.float16).astype(np.float64))


def test_main_term_rotated_route_equals_explicit_dequantisation():
    book = cb.codebook(3)
    dk = sign_vector(5, D)
    rng = np.random.default_rng(1)
    k = rng.standard_normal((40, D)) * np.exp(rng.standard_normal(D))
    q = rng.standard_normal(D)
    qz = quantize(k, dk, book.centroids, book.thresholds)
    khat = qz.norm[:, None] * unrotate(book.centroids[qz.codes], dk)    # n R^T c
    qt = rotate(q, dk)
    rotated = qz.norm * (book.centroids[qz.codes] @ qt)
    np.testing.assert_allclose(rotated, khat @ q, rtol=1e-12, atol=1e-12 * np.abs(khat @ q).max())


def test_qjl_estimator_unbiased_with_closed_form_variance():
    """Over independent sketches S: E[X] = <q~, n u>, Var[X] = (pi/2 |q~|^2 gamma^2 - <q~,n u>^2)/m."""
    d = m = 32
    book = cb.codebook(2, d)
    dk = sign_vector(3, d)
    rng = np.random.default_rng(2)
    k = rng.standard_normal((1, d))
    qt = rotate(rng.standard_normal(d), dk)
    qz0 = quantize(k, dk, book.centroids, book.thresholds)
    u = qz0.y[0] - book.centroids[qz0.codes[0]]
    target = qz0.norm[0] * (qt @ u)
    gamma = qz0.norm[0] * np.linalg.norm(u)
    n_seeds = 20000
    xs = np.empty(n_seeds)
    for i in range(n_seeds):
        s = gaussian_sketch(1000 + i, m, d)
        qz = quantize(k, dk, book.centroids, book.thresholds, s)
        p = s @ qt
        # the QJL term alone: zero key norm removes the main term; exact gamma is used
        xs[i] = dec.logits(qt, p, qz.codes, [0.0], [gamma], qz.sign_bits, book.centroids, 1.0, m)[0]
    var = (np.pi / 2 * (qt @ qt) * gamma ** 2 - target ** 2) / m
    assert abs(xs.mean() - target) < 5 * np.sqrt(var / n_seeds)
    # sample variance within a generous chi-square band (n large -> normal approx, 6 sigma)
    assert abs(xs.var() / var - 1) < 6 * np.sqrt(2.0 / n_seeds) + 0.02


def test_full_logit_unbiased_for_q_dot_k():
    d = m = 32
    book = cb.codebook(3, d)
    dk = sign_vector(4, d)
    rng = np.random.default_rng(3)
    k = rng.standard_normal((1, d)) * 3
    q = rng.standard_normal(d)
    qt = rotate(q, dk)
    vals = []
    for i in range(8000):
        s = gaussian_sketch(50_000 + i, m, d)
        qz = quantize(k, dk, book.centroids, book.thresholds, s)
        vals.append(dec.logits(qt, s @ qt, qz.codes, qz.norm, qz.gamma, qz.sign_bits,
                               book.centroids, 1.0, m)[0])
    vals = np.array(vals)
    assert abs(vals.mean() - q @ k[0]) < 5 * vals.std() / np.sqrt(len(vals))


def _identity_tables(y):
    """Code tables that reproduce y exactly: code (t, i) indexes a table of all values."""
    flat = y.ravel()
    return flat, np.arange(flat.size).reshape(y.shape)


def test_bypassed_quantisation_is_textbook_attention():
    rng = np.random.default_rng(4)
    T = 37
    k = rng.standard_normal((T, D)) * 2
    v = rng.standard_normal((T, D))
    q = rng.standard_normal(D)
    dk, dv = sign_vector(1, D), sign_vector(2, D)
    nk, nv = np.linalg.norm(k, axis=1), np.linalg.norm(v, axis=1)
    tk, ck = _identity_tables(rotate(k, dk) / nk[:, None])
    tv, cv = _identity_tables(rotate(v, dv) / nv[:, None])
    qt = rotate(q, dk)
    lg = dec.logits(qt, np.zeros(D), ck, nk, np.zeros(T), np.zeros((T, D)), tk, 1 / np.sqrt(D), D)
    o = dec.attend(lg, cv, nv, tv, dv)
    s = k @ q / np.sqrt(D)
    w = np.exp(s - s.max())
    w /= w.sum()
    np.testing.assert_allclose(o, w @ v, rtol=0, atol=1e-12)


def test_single_token_returns_its_value_and_identical_keys_average():
    book = cb.codebook(2)
    dv = sign_vector(8, D)
    rng = np.random.default_rng(5)
    v = rng.standard_normal((4, D))
    qv = quantize(v, dv, book.centroids, book.thresholds)
    vhat = qv.norm16[:, None] * unrotate(book.centroids[qv.codes], dv)
    o1 = dec.attend(np.array([3.7]), qv.codes[:1], qv.norm16[:1], book.centroids, dv)
    np.testing.assert_allclose(o1, vhat[0], atol=1e-13)
    o4 = dec.attend(np.full(4, -2.5), qv.codes, qv.norm16, book.centroids, dv)
    np.testing.assert_allclose(o4, vhat.mean(axis=0), atol=1e-13)
    assert np.all(dec.attend(np.zeros(0), qv.codes[:0], qv.norm16[:0], book.centroids, dv) == 0)


def _build_cache(bk, bv, seq_lens, n_kv, seed, perm_seed):
    books = cb.codebook(bk), cb.codebook(bv)
    tables = dict(signs_k=sign_vector(seed, D), signs_v=sign_vector(seed + 1, D),
                  sketch=gaussian_sketch(seed + 2, D, D), centroids_k=books[0].centroids,
                  centroids_v=books[1].centroids, bk=bk, bv=bv)
    pages = [(L + 15) // 16 for L in seq_lens]
    total = sum(pages)
    perm = np.random.default_rng(perm_seed).permutation(total)
    bt = np.zeros((len(seq_lens), max(pages)), dtype=np.int64)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    cache = np.zeros((total, n_kv, lay.block_bytes(bk, bv)), dtype=np.uint8)
    rng = np.random.default_rng(seed)
    for b, L in enumerate(seq_lens):
        k = rng.standard_normal((L, n_kv, D))
        v = rng.standard_normal((L, n_kv, D))
        for h in range(n_kv):
            qk = quantize(k[:, h], tables["signs_k"], books[0].centroids, books[0].thresholds, tables["sketch"])
            qv = quantize(v[:, h], tables["signs_v"], books[1].centroids, books[1].thresholds)
            for t in range(L):
                blk = cache[bt[b, t // 16], h]
                lay.write_token(blk, t % 16, bk, bv, qk.codes[t], qk.sign_bits[t], qv.codes[t],
                                qk.norm16[t], qk.gamma16[t], qv.norm16[t])
    return cache, bt, tables


def test_page_permutation_invariance():
    seq = [40, 17]
    c1, bt1, tab = _build_cache(3, 2, seq, 2, 10, 0)
    q = np.random.default_rng(9).standard_normal((2, 4, D))
    out1 = dec.decode_paged(c1, bt1, seq, q, tab)
    # move every physical page to a new slot and rewrite the block tables accordingly
    perm = np.random.default_rng(77).permutation(c1.shape[0])
    c2 = np.empty_like(c1)
    c2[perm] = c1
    bt2 = perm[bt1]
    out2 = dec.decode_paged(c2, bt2, seq, q, tab)
    np.testing.assert_allclose(out1, out2, rtol=0, atol=0)
    assert np.all(np.isfinite(out1))


def test_paged_decode_equals_direct_decode():
    seq = [33]
    cache, bt, tab = _build_cache(4, 3, seq, 1, 20, 1)
    q = np.random.default_rng(3).standard_normal((1, 2, D))
    out = dec.decode_paged(cache, bt, seq, q, tab)
    kc, sb, vc, nk, gm, nv = dec.gather_sequence(cache, bt[0], 33, 0, 4, 3)
    for h in range(2):
        qt, p = dec.transform_query(q[0, h], tab["signs_k"], tab["sketch"])
        lg = dec.logits(qt, p, kc, nk, gm, sb, tab["centroids_k"], 1 / np.sqrt(D), D)
        np.testing.assert_allclose(out[0, h], dec.attend(lg, vc, nv, tab["centroids_v"], tab["signs_v"]))


def _sparse_case(seed, T=200, spread=3.0):
    book = cb.codebook(2)
    dv = sign_vector(seed, D)
    rng = np.random.default_rng(seed)
    qv = quantize(rng.standard_normal((T, D)), dv, book.centroids, book.thresholds)
    lg = rng.standard_normal(T) * spread
    return lg, qv, book, dv


def test_sparse_v_zero_threshold_is_dense_attention():
    lg, qv, book, dv = _sparse_case(11)
    dense = dec.attend(lg, qv.codes, qv.norm16, book.centroids, dv)
    assert np.array_equal(dec.attend(lg, qv.codes, qv.norm16, book.centroids, dv, 0.0), dense)
    assert dec.sparse_bound(lg, qv.codes, qv.norm16, book.centroids, 0.0) == 0.0


def test_sparse_v_threshold_one_keeps_only_the_largest_weight():
    # closed form: with tau = 1 only the argmax position adds its value, with its
    # softmax weight (the normalisation still covers every position)
    lg, qv, book, dv = _sparse_case(12)
    j = int(np.argmax(lg))
    p_max = 1.0 / np.sum(np.exp(lg - lg[j]))
    vhat_j = qv.norm16[j] * unrotate(book.centroids[qv.codes[j]], dv)
    got = dec.attend(lg, qv.codes, qv.norm16, book.centroids, dv, 1.0)
    np.testing.assert_allclose(got, p_max * vhat_j, rtol=1e-12, atol=1e-15)


def test_sparse_v_dropping_one_position_moves_the_output_by_its_contribution():
    # exactly one position below the threshold: the output changes by w_t ||v_t||
    # (the inverse rotation is orthogonal), which is what sparse_bound reports
    lg, qv, book, dv = _sparse_case(13, T=50, spread=0.5)
    lg[7] = lg.max() - 8.0                        # weight e^-8 of the largest; all others > e^-3
    tau = 1e-3
    w = np.exp(lg - lg.max())
    assert np.sum(w < tau) == 1
    dense = dec.attend(lg, qv.codes, qv.norm16, book.centroids, dv)
    sparse = dec.attend(lg, qv.codes, qv.norm16, book.centroids, dv, tau)
    bound = dec.sparse_bound(lg, qv.codes, qv.norm16, book.centroids, tau)
    vhat7 = qv.norm16[7] * unrotate(book.centroids[qv.codes[7]], dv)
    expect = (w[7] / w.sum()) * vhat7
    np.testing.assert_allclose(dense - sparse, expect, rtol=1e-9, atol=1e-9 * np.linalg.norm(expect))
    assert np.isclose(np.linalg.norm(dense - sparse), bound, rtol=1e-9)


@pytest.mark.parametrize("tau", [1e-6, 1e-3, 1e-1])
def test_sparse_v_change_is_within_the_dropped_mass(tau):
    lg, qv, book, dv = _sparse_case(14, T=400, spread=4.0)
    dense = dec.attend(lg, qv.codes, qv.norm16, book.centroids, dv)
    sparse = dec.attend(lg, qv.codes, qv.norm16, book.centroids, dv, tau)
    bound = dec.sparse_bound(lg, qv.codes, qv.norm16, book.centroids, tau)
    assert np.linalg.norm(dense - sparse) <= bound * (1 + 1e-12) + 1e-300
