"""Decode attention on the compressed cache: query transform, logits, softmax, value sum.

Oracle module (test infrastructure only).

The logit of cached token t is the QJL-corrected inner-product estimate
(wis-web.com llama.cpp-fork post, QJL paragraph: the 1-bit corrector removes
the residual bias), written in the rotated domain:

    q~ = R_K q,  p = S q~,
    l_t = scale * ( n_t <q~, c[code_t]> + gamma_t sqrt(pi/2)/m sum_r p_r (2 s_tr - 1) ).

Softmax with the maximum subtracted, then the value sum in the rotated domain,
a = sum_t w_t ||v_t|| c_v[code_v,t], and one inverse rotation o = R_V^T a.
Readings: scale = 1/sqrt(d) (the pages do not state one); values carry no QJL
bits; all stored quantities (fp16 norms, fp16 centroids) are used as stored; a
sequence with no cached tokens attends to nothing and returns 0. Query head h
reads KV head floor(h / g) with g = n_q_heads / n_kv_heads.

Sparse V (wis-web.com llama.cpp-fork post, third finding: decoding skips the V
positions with a low attention weight): with a threshold tau > 0, position t
contributes no value when its softmax weight is below tau times the largest
weight; the softmax denominator still covers every position. The pages give no
threshold; tau is a parameter and tau = 0 is dense attention.
"""

import numpy as np

from .hadamard import rotate, unrotate
from .layout import read_page, read_page_q8, PAGE
from .q8 import logits_q8


def transform_query(q, signs_k, sketch):
    """q~ = R_K q and p = S q~ (float64)."""
    qt = rotate(np.asarray(q, dtype=np.float64), signs_k)
    return qt, qt @ np.asarray(sketch, dtype=np.float64).T


def logits(qt, p, k_codes, k_norm, gamma, sign_bits, centroids_k, scale, m):
    """Estimated logits of T tokens for one query (qt, p: [d] / [m]; codes: [T, d])."""
    c = np.asarray(centroids_k, dtype=np.float64)[np.asarray(k_codes)]
    main = np.asarray(k_norm, dtype=np.float64) * (c @ qt)
    pm = (2.0 * np.asarray(sign_bits, dtype=np.float64) - 1.0) @ p
    qjl = np.asarray(gamma, dtype=np.float64) * np.sqrt(np.pi / 2.0) / m * pm
    return scale * (main + qjl)


def attend(lg, v_codes, v_norm, centroids_v, signs_v, sparse_tau=0.0):
    """Softmax over the logits and the de-rotated weighted value sum (float64, [d]).

    sparse_tau > 0: positions whose weight is below sparse_tau * max weight add no
    value (Sparse V); the normalisation is unchanged."""
    d = len(signs_v)
    if len(lg) == 0:
        return np.zeros(d)
    w = np.exp(lg - np.max(lg))                 # the largest weight is 1
    w = w / np.sum(w)
    if sparse_tau > 0.0:
        w = np.where(w >= sparse_tau * np.max(w), w, 0.0)
    cv = np.asarray(centroids_v, dtype=np.float64)[np.asarray(v_codes)]
    a = (w * np.asarray(v_norm, dtype=np.float64)) @ cv
    return unrotate(a, signs_v)


def sparse_bound(lg, v_codes, v_norm, centroids_v, sparse_tau):
    """Sum over the positions Sparse V drops of w_t ||v_t c_t||: an upper bound of the
    2-norm change of the output (the inverse rotation preserves norms)."""
    if len(lg) == 0 or sparse_tau <= 0.0:
        return 0.0
    w = np.exp(lg - np.max(lg))
    w = w / np.sum(w)
    drop = w < sparse_tau * np.max(w)
    cv = np.asarray(centroids_v, dtype=np.float64)[np.asarray(v_codes)]
    vn = np.asarray(v_norm, dtype=np.float64) * np.linalg.norm(cv, axis=1)
    return float(np.sum(w[drop] * vn[drop]))


def gather_sequence(cache, block_table, seq_len, kv_head, bk, bv):
    """Unpacked fields of the first seq_len tokens of one sequence and KV head."""
    n_pages = (seq_len + PAGE - 1) // PAGE
    parts = [read_page(cache[int(block_table[i]), kv_head], bk, bv) for i in range(n_pages)]
    if not parts:
        z = np.zeros((0, 128), dtype=np.int64)
        e = np.zeros(0)
        return z, z, z, e, e, e
    cat = [np.concatenate([pp[f] for pp in parts])[:seq_len] for f in range(6)]
    return tuple(cat)


def gather_sequence_q8(cache, block_table, seq_len, kv_head, bv):
    """q8_0-key cache: values [T, d], scales16 [T, 4], v_codes [T, d], v_norm [T]."""
    n_pages = (seq_len + PAGE - 1) // PAGE
    parts = [read_page_q8(cache[int(block_table[i]), kv_head], bv) for i in range(n_pages)]
    if not parts:
        z = np.zeros((0, 128), dtype=np.int64)
        return z, np.zeros((0, 4)), z, np.zeros(0)
    return tuple(np.concatenate([pp[f] for pp in parts])[:seq_len] for f in range(4))


def decode_paged(cache, block_tables, seq_lens, q, tables, scale=None, sparse_tau=0.0, bounds=None):
    """Reference decode over a paged cache.

    cache: uint8 [n_pages, n_kv, block_bytes]; block_tables: int [B, max_pages];
    seq_lens: int [B]; q: [B, Hq, d]; tables: dict with signs_k, signs_v, sketch,
    centroids_k, centroids_v, bk, bv (bk = 8: q8_0 keys). Returns out [B, Hq, d] float64. sparse_tau:
    Sparse V threshold (0: dense); bounds, if given ([B, Hq]), receives each head's
    sparse_bound.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    n_kv = cache.shape[1]
    g = Hq // n_kv
    m = tables["sketch"].shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((B, Hq, d))
    for b in range(B):
        for hk in range(n_kv):
            if tables["bk"] == 8:                  # q8_0 keys: raw query, block scales
                k8, sc, vc, nv = gather_sequence_q8(cache, block_tables[b], int(seq_lens[b]), hk, tables["bv"])
            else:
                kc, sb, vc, nk, gm, nv = gather_sequence(cache, block_tables[b], int(seq_lens[b]), hk,
                                                         tables["bk"], tables["bv"])
            for hh in range(g):
                h = hk * g + hh
                if tables["bk"] == 8:
                    lg = logits_q8(q[b, h], k8, sc, scale)
                else:
                    qt, p = transform_query(q[b, h], tables["signs_k"], tables["sketch"])
                    lg = logits(qt, p, kc, nk, gm, sb, tables["centroids_k"], scale, m)
                out[b, h] = attend(lg, vc, nv, tables["centroids_v"], tables["signs_v"], sparse_tau)
                if bounds is not None:
                    bounds[b, h] = sparse_bound(lg, vc, nv, tables["centroids_v"], sparse_tau)
    return out
