"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle.

Quantize: codes and sign bits bit-exact except within 1e-5 of a decision
boundary (counts reported), fp16 norms within one unit in the last place.
Decode: given identical codes (the cache the oracle itself packs), outputs
within 1e-3 relative error per head (2-norm).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding, synth  # noqa: E402
from oracle import decode as odec  # noqa: E402
from oracle import layout as lay  # noqa: E402

from parity_util import (assert_outputs_close, compare_tokens, oracle_cache, oracle_quantize,  # noqa: E402
                         oracle_tables, unpack_tokens)

DEV = "cuda:0"


def _ctx(bk, bv, seeds):
    return binding.Context(bk, bv, seeds, device=0)


def _pool(seq_lens, seed, extra=3):
    pages = [(L + 15) // 16 for L in seq_lens]
    total = int(sum(pages)) + extra
    perm = np.random.default_rng(seed).permutation(total).astype(np.int32)
    bt = np.zeros((len(seq_lens), max(1, max(pages))), dtype=np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    return bt, total


def _rand_kv(rng, L, n_kv, dtype, outliers=True):
    scale = np.exp(rng.standard_normal((n_kv, 128))) if outliers else np.ones((n_kv, 128))
    if outliers:
        scale[:, rng.choice(128, 3, replace=False)] *= 10
    k = rng.standard_normal((L, n_kv, 128)) * scale
    v = rng.standard_normal((L, n_kv, 128)) * scale[:, ::-1]
    k, v = k.astype(np.float32), v.astype(np.float32)
    if dtype == "bf16":
        k, v = synth.round_to_bf16(k), synth.round_to_bf16(v)
    elif dtype == "fp16":
        k, v = k.astype(np.float16).astype(np.float32), v.astype(np.float16).astype(np.float32)
    return k, v


def _t(x, dtype):
    tdt = {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}[dtype]
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(DEV).to(tdt)


# ----------------------------------------------------------------- quantize
@pytest.mark.parametrize("bk,bv,dtype,path", [(3, 3, "fp32", "prefill"), (3, 2, "bf16", "append"),
                                              (4, 4, "bf16", "prefill"), (2, 4, "fp16", "append"),
                                              (4, 2, "bf16", "append"), (2, 3, "bf16", "prefill"),
                                              (3, 4, "fp16", "prefill")])
def test_quantize_matches_oracle(bk, bv, dtype, path):
    seeds = (11 + bk, 22 + bv, 33)
    ctx = _ctx(bk, bv, seeds)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(bk * 7 + bv)
    L, n_kv = 301, 2                      # 18 full pages and a ragged tail
    k, v = _rand_kv(rng, L, n_kv, dtype)
    bt, n_pages = _pool([L], 5)
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    kt, vt = _t(k, dtype), _t(v, dtype)
    if path == "prefill":
        # two chunks: the second starts inside a page (merge path)
        btt = torch.from_numpy(bt[0]).to(DEV)
        ctx.quantize_prefill(kt[:150], vt[:150], btt, 0, cache, n_pages)
        ctx.quantize_prefill(kt[150:], vt[150:], btt, 150, cache, n_pages)
    else:
        slots = torch.from_numpy(synth.slots_for(bt[0], 0, L)[::-1].copy()).to(DEV)   # any order
        ctx.quantize_append(kt.flip(0), vt.flip(0), slots, cache, n_pages)
    assert ctx.device_error() == 0
    host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
    kf = k.astype(np.float64)
    vf = v.astype(np.float64)
    for h in range(n_kv):
        qk, qv = oracle_quantize(kf[:, h], vf[:, h], tab)
        fields = unpack_tokens(host, bt[0], 0, L, h, bk, bv)
        rep = compare_tokens(fields, qk, qv, tab)
        print(h, rep)
        assert all(v == 0 for key, v in rep.items() if key.startswith("bad")), rep
        assert rep["excused_k_codes"] + rep["excused_v_codes"] < 0.001 * L * 128


@pytest.mark.parametrize("bk,bv,dtype", [(3, 2, "bf16"), (4, 4, "fp16"), (2, 3, "bf16")])
def test_prefill_short_runs_match_oracle(bk, bv, dtype):
    """A context built by prefill calls of 1, 3, 12, 1, 33 and 150 tokens: runs that
    start and end inside a page, single tokens, runs spanning several pages, an odd
    number of KV heads. Every token is checked against the oracle's quantization."""
    seeds = (41 + bk, 42 + bv, 43)
    ctx = _ctx(bk, bv, seeds)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(bk * 11 + bv)
    runs = [1, 3, 12, 1, 33, 150]
    L, n_kv = sum(runs), 3
    k, v = _rand_kv(rng, L, n_kv, dtype)
    bt, n_pages = _pool([L], 7)
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    kt, vt = _t(k, dtype), _t(v, dtype)
    btt = torch.from_numpy(bt[0]).to(DEV)
    pos = 0
    for n in runs:
        ctx.quantize_prefill(kt[pos:pos + n].contiguous(), vt[pos:pos + n].contiguous(), btt, pos, cache, n_pages)
        pos += n
    assert ctx.device_error() == 0
    host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
    for h in range(n_kv):
        qk, qv = oracle_quantize(k[:, h].astype(np.float64), v[:, h].astype(np.float64), tab)
        rep = compare_tokens(unpack_tokens(host, bt[0], 0, L, h, bk, bv), qk, qv, tab)
        assert all(x == 0 for key, x in rep.items() if key.startswith("bad")), (h, rep)


def test_prefill_bad_page_sets_device_error_and_spares_the_rest():
    """A block-table entry outside the pool: that page is skipped with
    TQ_DEV_BAD_SLOT, every other page is written as usual."""
    bk, bv, n_kv = 3, 2, 2
    seeds = (51, 52, 53)
    ctx = _ctx(bk, bv, seeds)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(9)
    L = 64                                      # 4 pages
    k, v = _rand_kv(rng, L, n_kv, "bf16")
    bt, n_pages = _pool([L], 3)
    bad = bt[0].copy()
    bad[2] = n_pages + 5                        # third page out of range
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    ctx.quantize_prefill(_t(k, "bf16"), _t(v, "bf16"), torch.from_numpy(bad).to(DEV), 0, cache, n_pages)
    assert ctx.device_error() & binding.DEV_BAD_SLOT
    host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
    good_tokens = np.r_[0:32, 48:64]
    for h in range(n_kv):
        # the oracle quantizes each token on its own: quantize the kept tokens only
        qk, qv = oracle_quantize(k[good_tokens, h].astype(np.float64), v[good_tokens, h].astype(np.float64), tab)
        got = unpack_tokens(host, bt[0], 0, L, h, bk, bv)
        rep = compare_tokens(tuple(np.asarray(x)[good_tokens] for x in got), qk, qv, tab)
        assert all(x == 0 for key, x in rep.items() if key.startswith("bad")), (h, rep)


def test_quantize_bad_slot_sets_device_error():
    ctx = _ctx(3, 2, (1, 2, 3))
    n_pages = 2
    cache = torch.zeros(n_pages * ctx.page_bytes(1), dtype=torch.uint8, device=DEV)
    k = torch.randn(2, 1, 128, device=DEV)
    slots = torch.tensor([5, 10_000], dtype=torch.int64, device=DEV)
    ctx.quantize_append(k, k, slots, cache, n_pages)
    assert ctx.device_error() & binding.DEV_BAD_SLOT
    assert ctx.device_error() == 0          # cleared by the read


# ------------------------------------------------------------------- decode
def _decode_case(bk, bv, seq_lens, n_kv, g, qdtype="bf16", seed=0):
    seeds = (100 + seed, 200 + seed, 300 + seed)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(seed)
    ks, vs = [], []
    for L in seq_lens:
        k, v = _rand_kv(rng, max(L, 1), n_kv, "bf16")
        ks.append(k.astype(np.float64))
        vs.append(v.astype(np.float64))
    bt, n_pages = _pool(seq_lens, seed + 1)
    cache_np = oracle_cache(ks, vs, bt, seq_lens, n_pages, tab)
    q = rng.standard_normal((len(seq_lens), n_kv * g, 128)).astype(np.float32)
    if qdtype == "bf16":
        q = synth.round_to_bf16(q)
    want = odec.decode_paged(cache_np, bt, seq_lens, q.astype(np.float64), tab)
    ctx = _ctx(bk, bv, seeds)
    cache = torch.from_numpy(cache_np.reshape(-1)).to(DEV)
    max_len = max(max(seq_lens), 1)
    ws = torch.zeros(ctx.decode_workspace_bytes(len(seq_lens), n_kv * g, n_kv, max_len), dtype=torch.uint8,
                     device=DEV)
    out = torch.full((len(seq_lens), n_kv * g, 128), float("nan"), device=DEV)
    ctx.decode_attention(_t(q, qdtype), cache, n_pages, torch.from_numpy(bt).to(DEV),
                         torch.tensor(seq_lens, dtype=torch.int32, device=DEV), n_kv, max_len, out, ws)
    assert ctx.device_error() == 0
    return out.cpu().numpy().astype(np.float64), want


@pytest.mark.parametrize("bk,bv", [(3, 2), (3, 3), (4, 4), (4, 2), (2, 2), (2, 4), (3, 4), (4, 3), (2, 3)])
def test_decode_matches_oracle_all_bit_widths(bk, bv):
    got, want = _decode_case(bk, bv, [333, 17, 64], n_kv=2, g=4, seed=bk * 10 + bv)
    print("worst rel err", assert_outputs_close(got, want))


@pytest.mark.parametrize("g", [1, 4, 8, 12])
def test_decode_gqa_groups(g):
    got, want = _decode_case(3, 2, [200, 1, 16, 47], n_kv=2, g=g, seed=40 + g)
    print("worst rel err", assert_outputs_close(got, want))


@pytest.mark.parametrize("g,bv", [(8, 2), (12, 4), (8, 3)])
def test_decode_4bit_keys_head_groups(g, bv):
    """4-bit keys with two or three groups of 4 query heads: the key term on fp16
    tensor cores (centroid pairs from the byte table, q~ in fp16 high and low parts),
    the sign term on the int8 limbs, the lowest sketch limbs of two groups in one n-tile."""
    got, want = _decode_case(4, bv, [333, 17, 64], n_kv=2, g=g, seed=70 + g + bv)
    print("worst rel err", assert_outputs_close(got, want))


def test_decode_long_context_many_chunks():
    # spans many split-K chunks with a ragged final page
    got, want = _decode_case(3, 2, [4000, 2500], n_kv=1, g=4, seed=7)
    print("worst rel err", assert_outputs_close(got, want))


def test_decode_empty_sequence_returns_zeros():
    got, want = _decode_case(3, 2, [0, 33], n_kv=1, g=4, seed=9)
    assert np.all(got[0] == 0) and np.all(want[0] == 0)
    assert_outputs_close(got[1:], want[1:])


def test_decode_fp32_query_and_tiny_workload():
    """The tiny workload: 1 KV / 1 query head, 1024 fp32 tokens with 4 outlier channels x20, 3/3 bits."""
    wl = synth.WORKLOADS["tiny"]
    gen = synth.Generator(wl)
    seeds = gen.method_seeds()
    tab = oracle_tables(seeds, 3, 3)
    k = gen.kv("k", 0, 1024)
    v = gen.kv("v", 0, 1024)
    bt, n_pages = gen.page_pool(np.array([64]))
    ctx = _ctx(3, 3, seeds)
    cache = torch.zeros(n_pages * ctx.page_bytes(1), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    ctx.quantize_prefill(_t(k, "fp32"), _t(v, "fp32"), btt[0], 0, cache, n_pages)
    host = cache.cpu().numpy().reshape(n_pages, 1, -1)
    qk, qv = oracle_quantize(k[:, 0].astype(np.float64), v[:, 0].astype(np.float64), tab)
    rep = compare_tokens(unpack_tokens(host, bt[0], 0, 1024, 0, 3, 3), qk, qv, tab)
    print(rep)
    assert all(val == 0 for key, val in rep.items() if key.startswith("bad")), rep
    q = gen.queries()
    out = torch.zeros(1, 1, 128, device=DEV)
    ws = torch.zeros(ctx.decode_workspace_bytes(1, 1, 1, 1024), dtype=torch.uint8, device=DEV)
    ctx.decode_attention(_t(q, "fp32"), cache, n_pages, btt, torch.tensor([1024], dtype=torch.int32, device=DEV),
                         1, 1024, out, ws)
    want = odec.decode_paged(host, bt, [1024], q.astype(np.float64), tab)
    print("tiny worst rel err", assert_outputs_close(out.cpu().numpy().astype(np.float64), want))


def test_decode_bad_page_sets_device_error():
    ctx = _ctx(3, 2, (1, 2, 3))
    n_pages = 4
    cache = torch.zeros(n_pages * ctx.page_bytes(1), dtype=torch.uint8, device=DEV)
    bt = torch.tensor([[0, 99]], dtype=torch.int32, device=DEV)
    ws = torch.zeros(ctx.decode_workspace_bytes(1, 4, 1, 32), dtype=torch.uint8, device=DEV)
    out = torch.zeros(1, 4, 128, device=DEV)
    ctx.decode_attention(torch.randn(1, 4, 128, device=DEV), cache, n_pages, bt,
                         torch.tensor([32], dtype=torch.int32, device=DEV), 1, 32, out, ws)
    assert ctx.device_error() & binding.DEV_BAD_PAGE
    assert torch.isfinite(out).all()


def test_invalid_arguments_are_rejected_before_launch():
    ctx = _ctx(3, 2, (1, 2, 3))
    L = binding.lib()
    ws = torch.zeros(1024, dtype=torch.uint8, device=DEV)
    out = torch.zeros(1, 4, 128, device=DEV)
    q = torch.zeros(1, 4, 128, device=DEV)
    bt = torch.zeros(1, 1, dtype=torch.int32, device=DEV)
    sl = torch.ones(1, dtype=torch.int32, device=DEV)
    cache = torch.zeros(1 * ctx.page_bytes(1), dtype=torch.uint8, device=DEV)
    with pytest.raises(binding.TQError) as e:      # workspace too small
        ctx.decode_attention(q, cache, 1, bt, sl, 1, 16, out, ws[:8])
    assert e.value.code == 3
    with pytest.raises(binding.TQError) as e:      # 4 query heads over 3 KV heads
        ctx.decode_attention(q, cache, 1, bt, sl, 3, 16, out, ws)
    assert e.value.code == 1
    assert L.tq_init_codebooks(ctx._h, 5, 2, None) == 2


# ------------------------------------------------- append then decode (a step)
def test_decode_step_attends_the_appended_token():
    bk, bv, n_kv, g = 3, 2, 2, 4
    seeds = (5, 6, 7)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(3)
    L0 = 47
    k, v = _rand_kv(rng, L0 + 3, n_kv, "bf16")
    bt, n_pages = _pool([L0 + 3], 2)
    ctx = _ctx(bk, bv, seeds)
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    ctx.quantize_prefill(_t(k[:L0], "bf16"), _t(v[:L0], "bf16"), btt[0], 0, cache, n_pages)
    ws = torch.zeros(ctx.decode_workspace_bytes(1, n_kv * g, n_kv, L0 + 3), dtype=torch.uint8, device=DEV)
    for step in range(3):
        L = L0 + step + 1
        slots = torch.from_numpy(synth.slots_for(bt[0], L - 1, 1)).to(DEV)
        ctx.quantize_append(_t(k[L - 1:L], "bf16"), _t(v[L - 1:L], "bf16"), slots, cache, n_pages)
        q = synth.round_to_bf16(rng.standard_normal((1, n_kv * g, 128)).astype(np.float32))
        out = torch.zeros(1, n_kv * g, 128, device=DEV)
        ctx.decode_attention(_t(q, "bf16"), cache, n_pages, btt, torch.tensor([L], dtype=torch.int32, device=DEV),
                             n_kv, L0 + 3, out, ws)
        host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
        want = odec.decode_paged(host, bt, [L], q.astype(np.float64), tab)
        assert_outputs_close(out.cpu().numpy().astype(np.float64), want)
    assert ctx.device_error() == 0


def test_decode_step_api_matches_oracle():
    """tq_decode_step: append one token per sequence at seq_len - 1, then attend (batch 2)."""
    bk, bv, n_kv, g = 3, 2, 2, 4
    seeds = (8, 9, 10)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(11)
    L0 = [47, 16]                                   # appends cross a page boundary in both
    steps = 3
    kv = [_rand_kv(rng, L + steps, n_kv, "bf16") for L in L0]
    bt, n_pages = _pool([L + steps for L in L0], 4)
    ctx = _ctx(bk, bv, seeds)
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    for b, L in enumerate(L0):
        ctx.quantize_prefill(_t(kv[b][0][:L], "bf16"), _t(kv[b][1][:L], "bf16"), btt[b], 0, cache, n_pages)
    max_len = max(L0) + steps
    ws = torch.zeros(ctx.decode_workspace_bytes(2, n_kv * g, n_kv, max_len), dtype=torch.uint8, device=DEV)
    for step in range(steps):
        lens = [L + step + 1 for L in L0]
        k_new = np.stack([kv[b][0][lens[b] - 1] for b in range(2)])
        v_new = np.stack([kv[b][1][lens[b] - 1] for b in range(2)])
        q = synth.round_to_bf16(rng.standard_normal((2, n_kv * g, 128)).astype(np.float32))
        out = torch.full((2, n_kv * g, 128), float("nan"), device=DEV)
        ctx.decode_step(_t(k_new, "bf16"), _t(v_new, "bf16"), _t(q, "bf16"), cache, n_pages, btt,
                        torch.tensor(lens, dtype=torch.int32, device=DEV), n_kv, max_len, out, ws)
        host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
        # the appended token equals the oracle's quantization of it
        for b in range(2):
            for h in range(n_kv):
                qk, qv = oracle_quantize(k_new[b:b + 1, h].astype(np.float64), v_new[b:b + 1, h].astype(np.float64), tab)
                rep = compare_tokens(unpack_tokens(host, bt[b], lens[b] - 1, 1, h, bk, bv), qk, qv, tab)
                assert all(val == 0 for key, val in rep.items() if key.startswith("bad")), rep
        want = odec.decode_paged(host, bt, lens, q.astype(np.float64), tab)
        assert_outputs_close(out.cpu().numpy().astype(np.float64), want)
    assert ctx.device_error() == 0


@pytest.mark.parametrize("path", ["prefill", "append"])
def test_zero_vectors_and_zero_query(path):
    """Zero key / value rows quantize to norm 0 (and gamma 0) with no NaN, and a zero
    query head attends uniformly; both against the oracle from the GPU-written bytes."""
    bk, bv, n_kv, g, L = 3, 2, 2, 4, 53
    seeds = (61, 62, 63)
    tab = oracle_tables(seeds, bk, bv)
    rng = np.random.default_rng(17)
    k, v = _rand_kv(rng, L, n_kv, "bf16")
    k[[5, 17, 40]] = 0.0
    v[[9, 17]] = 0.0
    k[30, 1] = 0.0
    bt, n_pages = _pool([L], 23)
    ctx = _ctx(bk, bv, seeds)
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    if path == "prefill":
        ctx.quantize_prefill(_t(k, "bf16"), _t(v, "bf16"), btt[0], 0, cache, n_pages)
    else:
        slots = torch.from_numpy(synth.slots_for(bt[0], 0, L)).to(DEV)
        ctx.quantize_append(_t(k, "bf16"), _t(v, "bf16"), slots, cache, n_pages)
    host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
    for h in range(n_kv):
        qk, qv = oracle_quantize(k[:, h].astype(np.float64), v[:, h].astype(np.float64), tab)
        fields = unpack_tokens(host, bt[0], 0, L, h, bk, bv)
        rep = compare_tokens(fields, qk, qv, tab)
        assert all(val == 0 for key, val in rep.items() if key.startswith("bad")), rep
        zk = np.all(k[:, h] == 0, axis=1)
        assert np.all(fields[3][zk] == 0) and np.all(fields[4][zk] == 0)      # key norm, gamma
        assert np.all(fields[5][np.all(v[:, h] == 0, axis=1)] == 0)           # value norm
    q = synth.round_to_bf16(rng.standard_normal((1, n_kv * g, 128)).astype(np.float32))
    q[0, 2] = 0.0
    ws = torch.zeros(ctx.decode_workspace_bytes(1, n_kv * g, n_kv, L), dtype=torch.uint8, device=DEV)
    out = torch.full((1, n_kv * g, 128), float("nan"), device=DEV)
    ctx.decode_attention(_t(q, "bf16"), cache, n_pages, btt, torch.tensor([L], dtype=torch.int32, device=DEV),
                         n_kv, L, out, ws)
    assert ctx.device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    want = odec.decode_paged(host, bt, [L], q.astype(np.float64), tab)
    print("worst rel err", assert_outputs_close(got, want))
