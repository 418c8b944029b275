"""Sparse V on the GPU against the oracle's definition.

The kernel skips the value of a position when its weight is below tau times the
largest weight its warp has seen so far, which never exceeds the largest weight
overall: it skips a subset of the positions the oracle's rule drops. So the GPU
output lies within B of both the oracle's sparse and dense outputs, where B (the
oracle's sparse_bound) is the summed contribution of the positions the rule
drops; plus the dense tolerance of 1e-3 relative.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding, synth  # noqa: E402
from oracle import decode as odec  # noqa: E402

from parity_util import oracle_cache, oracle_tables  # noqa: E402

DEV = "cuda:0"


def _case(seq_lens, n_kv, g, seed, peaked):
    bk, bv = 3, 2
    seeds = (500 + seed, 600 + seed, 700 + seed)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(seed)
    ks, vs = [], []
    for L in seq_lens:
        scale = np.exp(rng.standard_normal((n_kv, 128)))
        ks.append(synth.round_to_bf16(rng.standard_normal((L, n_kv, 128)) * scale).astype(np.float64))
        vs.append(synth.round_to_bf16(rng.standard_normal((L, n_kv, 128)) * scale).astype(np.float64))
    pages = [(L + 15) // 16 for L in seq_lens]
    perm = rng.permutation(sum(pages)).astype(np.int32)
    bt = np.zeros((len(seq_lens), max(pages)), dtype=np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    n_pages = sum(pages)
    cache_np = oracle_cache(ks, vs, bt, seq_lens, n_pages, tab)
    q = rng.standard_normal((len(seq_lens), n_kv * g, 128))
    if peaked:
        # each query points at a few keys of its KV head: attention concentrates there
        for b, L in enumerate(seq_lens):
            for h in range(n_kv * g):
                hk = h // g
                j = rng.choice(L, size=3, replace=False)
                kk = ks[b][j, hk]
                q[b, h] = 5.0 * np.sum(kk / np.linalg.norm(kk, axis=1, keepdims=True), axis=0)
    q = synth.round_to_bf16(q.astype(np.float32)).astype(np.float64)
    return tab, cache_np, bt, n_pages, q


def _gpu(tab_seeds_bits, cache_np, bt, n_pages, q, seq_lens, n_kv, tau):
    seeds, bk, bv = tab_seeds_bits
    ctx = binding.Context(bk, bv, seeds, device=0)
    ctx.set_sparse_v(tau)
    cache = torch.from_numpy(cache_np.reshape(-1)).to(DEV)
    max_len = max(seq_lens)
    ws = torch.zeros(ctx.decode_workspace_bytes(len(seq_lens), q.shape[1], n_kv, max_len), dtype=torch.uint8,
                     device=DEV)
    out = torch.full(q.shape, float("nan"), device=DEV)
    ctx.decode_attention(torch.from_numpy(q.astype(np.float32)).to(DEV).to(torch.bfloat16), cache, n_pages,
                         torch.from_numpy(bt).to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV), n_kv,
                         max_len, out, ws)
    assert ctx.device_error() == 0
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("peaked,tau", [(True, 1e-3), (True, 1e-6), (False, 1e-2)])
def test_sparse_v_within_the_dropped_mass(peaked, tau):
    seq_lens, n_kv, g, seed = [3000, 700], 2, 4, 3
    tab, cache_np, bt, n_pages, q = _case(seq_lens, n_kv, g, seed, peaked)
    key = ((500 + seed, 600 + seed, 700 + seed), 3, 2)
    got = _gpu(key, cache_np, bt, n_pages, q, seq_lens, n_kv, tau)
    bounds = np.zeros(q.shape[:2])
    sparse = odec.decode_paged(cache_np, bt, seq_lens, q, tab, sparse_tau=tau, bounds=bounds)
    dense = odec.decode_paged(cache_np, bt, seq_lens, q, tab)
    for ref in (sparse, dense):
        err = np.linalg.norm(got - ref, axis=-1)
        lim = bounds + 1e-3 * np.linalg.norm(ref, axis=-1)
        assert np.all(err <= lim), (np.max(err - lim), tau, peaked)
    frac = float(np.mean(bounds / np.maximum(np.linalg.norm(dense, axis=-1), 1e-30)))
    print(f"peaked={peaked} tau={tau}: mean dropped mass / |o| = {frac:.2e}")


def test_sparse_v_zero_is_the_dense_path_bit_for_bit():
    seq_lens, n_kv, g, seed = [1500, 260], 2, 4, 4
    tab, cache_np, bt, n_pages, q = _case(seq_lens, n_kv, g, seed, True)
    key = ((500 + seed, 600 + seed, 700 + seed), 3, 2)
    a = _gpu(key, cache_np, bt, n_pages, q, seq_lens, n_kv, 0.0)
    ctx = binding.Context(3, 2, key[0], device=0)
    with pytest.raises(binding.TQError):
        ctx.set_sparse_v(-1.0)
    cache = torch.from_numpy(cache_np.reshape(-1)).to(DEV)
    ws = torch.zeros(ctx.decode_workspace_bytes(2, q.shape[1], n_kv, max(seq_lens)), dtype=torch.uint8, device=DEV)
    out = torch.zeros(q.shape, device=DEV)
    ctx.decode_attention(torch.from_numpy(q.astype(np.float32)).to(DEV).to(torch.bfloat16), cache, n_pages,
                         torch.from_numpy(bt).to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV), n_kv,
                         max(seq_lens), out, ws)
    assert np.array_equal(a, out.cpu().numpy().astype(np.float64))
