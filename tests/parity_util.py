"""Helpers shared by the GPU parity tests: build caches with the library and
with the oracle from the same seeded inputs, and compare field by field."""

import numpy as np

from oracle import codebook as cb
from oracle import layout as lay
from oracle import quantize as oq
from oracle import rng as orng

D = 128
NEAR = 1e-5          # coordinates / sketch rows this close to a decision boundary are excused


def oracle_tables(seeds, bk, bv):
    kb, vb = cb.codebook(bk), cb.codebook(bv)
    return dict(signs_k=orng.sign_vector(seeds[0], D), signs_v=orng.sign_vector(seeds[1], D),
                sketch=orng.gaussian_sketch(seeds[2], D, D), centroids_k=kb.centroids,
                centroids_v=vb.centroids, thresholds_k=kb.thresholds, thresholds_v=vb.thresholds,
                bk=bk, bv=bv)


def oracle_quantize(x_k, x_v, tab):
    """Oracle quantization of [T, d] key and value rows (float64 promotion)."""
    qk = oq.quantize(x_k, tab["signs_k"], tab["centroids_k"], tab["thresholds_k"], tab["sketch"])
    qv = oq.quantize(x_v, tab["signs_v"], tab["centroids_v"], tab["thresholds_v"])
    return qk, qv


def oracle_cache(k, v, block_tables, seq_lens, n_pages, tab):
    """Packed cache written by the oracle: k, v [B][T_b, n_kv, d] lists."""
    n_kv = k[0].shape[1]
    cache = np.zeros((n_pages, n_kv, lay.block_bytes(tab["bk"], tab["bv"])), dtype=np.uint8)
    for b, L in enumerate(seq_lens):
        for h in range(n_kv):
            qk, qv = oracle_quantize(k[b][:L, h], v[b][:L, h], tab)
            for t in range(L):
                blk = cache[block_tables[b][t // 16], h]
                lay.write_token(blk, t % 16, tab["bk"], tab["bv"], qk.codes[t], qk.sign_bits[t], qv.codes[t],
                                qk.norm16[t], qk.gamma16[t], qv.norm16[t])
    return cache


def near_boundary(y, thresholds):
    return np.min(np.abs(y[..., None] - thresholds), axis=-1) < NEAR


def half_ulps_apart(a, b):
    """Distance in fp16 units in the last place between two fp16-valued arrays."""
    ia = np.asarray(a, dtype=np.float16).view(np.int16).astype(np.int64)
    ib = np.asarray(b, dtype=np.float16).view(np.int16).astype(np.int64)
    # map sign-magnitude to a monotone integer line
    ia = np.where(ia < 0, -(ia & 0x7FFF), ia)
    ib = np.where(ib < 0, -(ib & 0x7FFF), ib)
    return np.abs(ia - ib)


def compare_tokens(gpu_fields, qk, qv, tab):
    """Compare unpacked GPU fields of T tokens with the oracle's quantization.

    gpu_fields: (k_codes, sign_bits, v_codes, k_norm, gamma, v_norm) arrays [T, ...].
    Returns a dict of mismatch counts; 'bad_*' must be zero, 'excused_*' are the
    boundary cases the tolerance allows (reported, not hidden).
    """
    kc, sb, vc, nk, gm, nv = gpu_fields
    near_k = near_boundary(qk.y, tab["thresholds_k"])
    near_v = near_boundary(qv.y, tab["thresholds_v"])
    dk = kc != qk.codes
    dv = vc != qv.codes
    out = dict(bad_k_codes=int(np.sum(dk & ~near_k)), excused_k_codes=int(np.sum(dk & near_k)),
               bad_v_codes=int(np.sum(dv & ~near_v)), excused_v_codes=int(np.sum(dv & near_v)))
    # sign bits: only for vectors whose codes all agree; excuse rows with |z| < NEAR |u|
    same_codes = ~np.any(dk, axis=1)
    unorm = np.linalg.norm(qk.residual, axis=1)
    near_s = np.abs(qk.projection) < NEAR * unorm[:, None]
    ds = (sb != qk.sign_bits) & same_codes[:, None]
    out["bad_signs"] = int(np.sum(ds & ~near_s))
    out["excused_signs"] = int(np.sum(ds & near_s))
    out["bad_k_norm"] = int(np.sum(half_ulps_apart(nk, qk.norm16) > 1))
    out["bad_v_norm"] = int(np.sum(half_ulps_apart(nv, qv.norm16) > 1))
    g_ok = same_codes
    out["bad_gamma"] = int(np.sum(half_ulps_apart(gm[g_ok], qk.gamma16[g_ok]) > 1))
    out["ulp_norms"] = int(np.sum(half_ulps_apart(nk, qk.norm16) == 1) + np.sum(half_ulps_apart(nv, qv.norm16) == 1))
    return out


def unpack_tokens(cache, block_table, start, count, h, bk, bv):
    """Unpacked fields of logical tokens [start, start+count) of one sequence/head."""
    fields = [[] for _ in range(6)]
    for pos in range(start, start + count):
        pg = block_table[pos // 16]
        f = lay.read_page(cache[pg, h], bk, bv)
        for i in range(6):
            fields[i].append(f[i][pos % 16])
    return tuple(np.array(x) for x in fields)


def assert_outputs_close(got, want, rtol=1e-3):
    """Output tolerance, checked two ways for every (batch, head):

    per head    ||got - want||_2 <= rtol ||want||_2;
    per element |got_i - want_i| <= rtol max(|want_i|, ||want||_2 / sqrt(d)),
                i.e. relative to the element itself, floored at the head's rms
                element size, so one wrong lane or column cannot hide in the norm.
    Returns the worst per-head relative error."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.linalg.norm(got - want, axis=-1)
    ref = np.linalg.norm(want, axis=-1)
    worst = float(np.max(err / np.maximum(ref, 1e-30)))
    assert np.all(err <= rtol * ref + 1e-30), f"worst relative error {worst:.3e}"
    floor = ref[..., None] / np.sqrt(want.shape[-1])
    bound = rtol * np.maximum(np.abs(want), floor) + 1e-30
    ediff = np.abs(got - want)
    worst_e = float(np.max(ediff / bound)) * rtol
    assert np.all(ediff <= bound), f"worst element error {worst_e:.3e} (relative to max(|o_i|, rms))"
    return worst
