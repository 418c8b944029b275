"""Decode with many (sequence, KV head) pairs, ragged and empty sequences, against the oracle.

More pairs than SMs, and 32 pairs (one uniform chunk count would leave 20 of 148 SMs
idle), through tq_decode_attention, tq_decode_step and tq_decode_logits. With four
query heads per KV head these run the uniform split (several waves of chunks); with
8 or 12 they run the balanced split (equal shares of all pages, one CTA per share).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding, synth  # noqa: E402
from oracle import decode as odec  # noqa: E402

from parity_util import assert_outputs_close, oracle_cache, oracle_tables  # noqa: E402

DEV = "cuda:0"


def _case(seq_lens, n_kv, g, seed, bk=3, bv=2, extra_steps=0):
    seeds = (300 + seed, 400 + seed, 500 + seed)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(seed)
    ks, vs = [], []
    for L in seq_lens:
        scale = np.exp(rng.standard_normal((n_kv, 128)))
        n = max(L + extra_steps, 1)
        ks.append(synth.round_to_bf16(rng.standard_normal((n, n_kv, 128)) * scale).astype(np.float64))
        vs.append(synth.round_to_bf16(rng.standard_normal((n, n_kv, 128)) * scale).astype(np.float64))
    pages = [max((L + extra_steps + 15) // 16, 1) for L in seq_lens]
    perm = rng.permutation(sum(pages)).astype(np.int32)
    bt = np.zeros((len(seq_lens), max(pages)), dtype=np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    cache_np = oracle_cache(ks, vs, bt, seq_lens, sum(pages), tab)
    q = synth.round_to_bf16(rng.standard_normal((len(seq_lens), n_kv * g, 128)).astype(np.float32))
    ctx = binding.Context(bk, bv, seeds, device=0)
    return tab, ks, vs, cache_np, bt, sum(pages), q, ctx


def _lens(rng, n, hi, zeros):
    lens = rng.integers(1, hi, size=n)
    lens[rng.choice(n, size=zeros, replace=False)] = 0
    return [int(x) for x in lens]


@pytest.mark.parametrize("n_seq,n_kv,g,hi,zeros,bk,bv", [(20, 8, 4, 300, 3, 3, 2), (8, 4, 4, 2500, 1, 3, 2),
                                                         (40, 4, 12, 120, 5, 3, 2), (8, 4, 8, 2500, 1, 3, 2),
                                                         (20, 8, 8, 300, 3, 3, 2), (40, 4, 12, 120, 5, 4, 2),
                                                         (20, 8, 8, 300, 3, 4, 4)])
def test_balanced_decode_matches_oracle(n_seq, n_kv, g, hi, zeros, bk, bv):
    seq_lens = _lens(np.random.default_rng(n_seq + hi), n_seq, hi, zeros)
    tab, _, _, cache_np, bt, n_pages, q, ctx = _case(seq_lens, n_kv, g, seed=n_seq, bk=bk, bv=bv)
    max_len = max(seq_lens)
    ws = torch.zeros(ctx.decode_workspace_bytes(n_seq, n_kv * g, n_kv, max_len), dtype=torch.uint8, device=DEV)
    out = torch.full((n_seq, n_kv * g, 128), float("nan"), device=DEV)
    cache = torch.from_numpy(cache_np.reshape(-1)).to(DEV)
    args = (cache, n_pages, torch.from_numpy(bt).to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
            n_kv, max_len, out, ws)
    want = odec.decode_paged(cache_np, bt, seq_lens, q.astype(np.float64), tab)
    live = np.array(seq_lens) > 0
    for _ in range(2):                    # the second call checks that the counters were reset
        out.fill_(float("nan"))
        ctx.decode_attention(torch.from_numpy(q).to(DEV).to(torch.bfloat16), *args)
        assert ctx.device_error() == 0
        got = out.cpu().numpy().astype(np.float64)
        assert np.all(got[~live] == 0)
        print("worst rel err", assert_outputs_close(got[live], want[live]))


@pytest.mark.parametrize("g", [4, 8])
def test_balanced_decode_step_and_logits(g):
    rng = np.random.default_rng(7 + g)
    n_seq, n_kv = 20, 8
    seq_lens = _lens(rng, n_seq, 260, 2)
    steps = 2
    tab, ks, vs, cache_np, bt, n_pages, q, ctx = _case(seq_lens, n_kv, g, seed=11, extra_steps=steps)
    cache = torch.from_numpy(cache_np.reshape(-1)).to(DEV)
    btt = torch.from_numpy(bt).to(DEV)
    max_len = max(seq_lens) + steps
    ws = torch.zeros(ctx.decode_workspace_bytes(n_seq, n_kv * g, n_kv, max_len), dtype=torch.uint8, device=DEV)
    lens = list(seq_lens)
    for step in range(steps):
        lens = [L + 1 if L > 0 else 0 for L in lens]
        k_new = np.stack([ks[b][max(L - 1, 0)] for b, L in enumerate(lens)]).astype(np.float32)
        v_new = np.stack([vs[b][max(L - 1, 0)] for b, L in enumerate(lens)]).astype(np.float32)
        qs = synth.round_to_bf16(rng.standard_normal((n_seq, n_kv * g, 128)).astype(np.float32))
        out = torch.full((n_seq, n_kv * g, 128), float("nan"), device=DEV)
        ctx.decode_step(torch.from_numpy(k_new).to(DEV).to(torch.bfloat16),
                        torch.from_numpy(v_new).to(DEV).to(torch.bfloat16),
                        torch.from_numpy(qs).to(DEV).to(torch.bfloat16), cache, n_pages, btt,
                        torch.tensor(lens, dtype=torch.int32, device=DEV), n_kv, max_len, out, ws)
        assert ctx.device_error() == 0
        host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
        want = odec.decode_paged(host, bt, lens, qs.astype(np.float64), tab)
        got = out.cpu().numpy().astype(np.float64)
        live = np.array(lens) > 0
        assert np.all(got[~live] == 0)
        print("step", step, "worst rel err", assert_outputs_close(got[live], want[live]))
    # logits of the final cache
    stride = max_len + 3
    logits = torch.full((n_seq, n_kv * g, stride), 12345.0, device=DEV)
    ctx.decode_logits(torch.from_numpy(qs).to(DEV).to(torch.bfloat16), cache, n_pages, btt,
                      torch.tensor(lens, dtype=torch.int32, device=DEV), n_kv, max_len, logits)
    assert ctx.device_error() == 0
    got = logits.cpu().numpy().astype(np.float64)
    scale = 1.0 / np.sqrt(128)
    for b, L in enumerate(lens):
        assert np.all(got[b, :, L:] == 12345.0)
        for hk in range(n_kv):
            if L == 0:
                continue
            kc, sb, vc, nk, gm, nv = odec.gather_sequence(host, bt[b], L, hk, 3, 2)
            cnorm = np.linalg.norm(tab["centroids_k"][kc], axis=1)
            for hh in range(g):
                h = hk * g + hh
                qt, pp = odec.transform_query(qs[b, h].astype(np.float64), tab["signs_k"], tab["sketch"])
                want = odec.logits(qt, pp, kc, nk, gm, sb, tab["centroids_k"], scale, 128)
                ref = np.maximum(np.abs(want), scale * nk * np.linalg.norm(qt) * cnorm)
                assert np.all(np.abs(got[b, h, :L] - want) <= 1e-3 * ref)
