"""tq_decode_logits (logits only) against the oracle's logits, through the C ABI.

Tolerance per logit (the relative error is undefined near a zero logit):
  |l_gpu - l_oracle| <= 1e-3 * max(|l|, scale * n_t * |q~| * |c_t|),
with n_t the stored key norm and c_t the token's centroid vector. Positions at or
beyond a sequence's length must be left untouched.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding, synth  # noqa: E402
from oracle import decode as odec  # noqa: E402

from parity_util import oracle_cache, oracle_tables  # noqa: E402

DEV = "cuda:0"
SENTINEL = 12345.0


def _case(bk, bv, seq_lens, n_kv, g, seed, qdtype):
    seeds = (800 + seed, 900 + seed, 1000 + seed)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(seed)
    ks, vs = [], []
    for L in seq_lens:
        scale = np.exp(rng.standard_normal((n_kv, 128)))
        ks.append(synth.round_to_bf16(rng.standard_normal((max(L, 1), n_kv, 128)) * scale).astype(np.float64))
        vs.append(synth.round_to_bf16(rng.standard_normal((max(L, 1), n_kv, 128)) * scale).astype(np.float64))
    pages = [max((L + 15) // 16, 1) for L in seq_lens]
    perm = rng.permutation(sum(pages)).astype(np.int32)
    bt = np.zeros((len(seq_lens), max(pages)), dtype=np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    cache_np = oracle_cache(ks, vs, bt, seq_lens, sum(pages), tab)
    q = rng.standard_normal((len(seq_lens), n_kv * g, 128)).astype(np.float32)
    if qdtype == "bf16":
        q = synth.round_to_bf16(q)
    ctx = binding.Context(bk, bv, seeds, device=0)
    max_len = max(max(seq_lens), 1)
    stride = max_len + 5
    logits = torch.full((len(seq_lens), n_kv * g, stride), SENTINEL, device=DEV)
    tq = torch.from_numpy(q).to(DEV)
    ctx.decode_logits(tq.to(torch.bfloat16) if qdtype == "bf16" else tq, torch.from_numpy(cache_np.reshape(-1)).to(DEV),
                      sum(pages), torch.from_numpy(bt).to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                      n_kv, max_len, logits)
    assert ctx.device_error() == 0
    return tab, cache_np, bt, q.astype(np.float64), logits.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("bk,bv,g,qdtype", [(3, 2, 4, "bf16"), (4, 4, 8, "bf16"), (2, 3, 12, "fp32"), (4, 2, 1, "bf16")])
def test_logits_match_oracle(bk, bv, g, qdtype):
    seq_lens, n_kv = [1000, 37, 0], 2
    tab, cache_np, bt, q, got = _case(bk, bv, seq_lens, n_kv, g, seed=bk * 7 + bv + g, qdtype=qdtype)
    scale = 1.0 / np.sqrt(128)
    worst = 0.0
    for b, L in enumerate(seq_lens):
        assert np.all(got[b, :, L:] == SENTINEL)
        if L == 0:
            continue
        for hk in range(n_kv):
            kc, sb, vc, nk, gm, nv = odec.gather_sequence(cache_np, bt[b], L, hk, bk, bv)
            cnorm = np.linalg.norm(tab["centroids_k"][kc], axis=1)
            for hh in range(g):
                h = hk * g + hh
                qt, p = odec.transform_query(q[b, h], tab["signs_k"], tab["sketch"])
                want = odec.logits(qt, p, kc, nk, gm, sb, tab["centroids_k"], scale, 128)
                ref = np.maximum(np.abs(want), scale * nk * np.linalg.norm(qt) * cnorm)
                err = np.abs(got[b, h, :L] - want)
                assert np.all(err <= 1e-3 * ref), float(np.max(err / ref))
                worst = max(worst, float(np.max(err / ref)))
    print("worst scaled logit error", worst)
