"""Asymmetric cache (q8_0 keys, TurboQuant values) on the GPU against the oracle.

Quantize: int8 key values equal the oracle's except where x / d lies within 1e-5 of
a rounding boundary (a half-integer), fp16 scales and value norms within one unit in
the last place, value codes bit-exact outside the 1e-5 boundary band.
Decode and logits: given the bytes the GPU wrote, outputs within 1e-3 relative
error per head, logits within 1e-3 of max(|l|, scale * |q| * |k_hat|).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding, synth  # noqa: E402
from oracle import decode as odec  # noqa: E402
from oracle import layout as lay  # noqa: E402
from oracle import q8  # noqa: E402

from parity_util import (assert_outputs_close, half_ulps_apart, near_boundary, oracle_quantize,  # noqa: E402
                         oracle_tables)

DEV = "cuda:0"


def _rows(rng, L, n_kv, outliers=True):
    scale = np.exp(rng.standard_normal((n_kv, 128)))
    if outliers:
        scale[:, rng.choice(128, 3, replace=False)] *= 10
    k = synth.round_to_bf16(rng.standard_normal((L, n_kv, 128)) * scale).astype(np.float64)
    v = synth.round_to_bf16(rng.standard_normal((L, n_kv, 128)) * scale[:, ::-1]).astype(np.float64)
    return k, v


def _gpu_cache(bv, seeds, k, v, path, start=0):
    """Quantize [L, n_kv, 128] rows into a fresh cache at positions start.. with prefill or append."""
    L, n_kv = k.shape[0], k.shape[1]
    ctx = binding.Context(8, bv, seeds, device=0)
    pages = (start + L + 15) // 16
    bt = np.random.default_rng(1).permutation(pages + 1)[:pages].astype(np.int32)
    n_pages = pages + 1
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    kt = torch.from_numpy(k.astype(np.float32)).to(DEV).to(torch.bfloat16)
    vt = torch.from_numpy(v.astype(np.float32)).to(DEV).to(torch.bfloat16)
    if path == "prefill":
        ctx.quantize_prefill(kt, vt, torch.from_numpy(bt).to(DEV), start, cache, n_pages)
    else:
        slots = synth.slots_for(bt, start, L)
        ctx.quantize_append(kt, vt, torch.from_numpy(slots).to(DEV), cache, n_pages)
    assert ctx.device_error() == 0
    return ctx, cache.cpu().numpy().reshape(n_pages, n_kv, -1), bt, n_pages


@pytest.mark.parametrize("bv,path,start", [(2, "prefill", 0), (3, "prefill", 5), (4, "append", 0), (2, "append", 9)])
def test_q8_quantize_matches_oracle(bv, path, start):
    rng = np.random.default_rng(bv * 10 + start)
    seeds = (31, 32, 33)
    tab = oracle_tables(seeds, 2, bv)
    k, v = _rows(rng, 75, 2)
    _, cache, bt, _ = _gpu_cache(bv, seeds, k, v, path, start)
    bad = excused = 0
    for h in range(2):
        kq = q8.quantize_q8(k[:, h])
        _, qv = oracle_quantize(k[:, h], v[:, h], tab)
        for t in range(75):
            pos = start + t
            vals, sc, vc, vn = lay.read_page_q8(cache[bt[pos // 16], h], bv)
            tau = pos % 16
            near = np.abs(np.abs(kq.ratio[t]) % 1.0 - 0.5) < 1e-5
            dk = vals[tau] != kq.values[t]
            bad += int(np.sum(dk & ~near))
            excused += int(np.sum(dk & near))
            assert np.all(half_ulps_apart(sc[tau], kq.scales16[t]) <= 1)
            dv = vc[tau] != qv.codes[t]
            nb = near_boundary(qv.y[t], tab["thresholds_v"])
            bad += int(np.sum(dv & ~nb))
            assert half_ulps_apart(np.array([vn[tau]]), np.array([qv.norm16[t]]))[0] <= 1
    print(f"bv={bv} {path}: excused {excused}")
    assert bad == 0


# ------------------------------------------------------------------- decode
def _oracle_cache_q8(ks, vs, bt, seq_lens, n_pages, tab):
    """Cache written by the oracle alone: q8_0 keys, TurboQuant values."""
    n_kv = ks[0].shape[1]
    cache = np.zeros((n_pages, n_kv, lay.block_bytes(8, tab["bv"])), dtype=np.uint8)
    for b, L in enumerate(seq_lens):
        for h in range(n_kv):
            kq = q8.quantize_q8(ks[b][:L, h])
            _, qv = oracle_quantize(ks[b][:L, h], vs[b][:L, h], tab)
            for t in range(L):
                lay.write_token_q8(cache[bt[b][t // 16], h], t % 16, tab["bv"], kq.values[t], kq.scales16[t],
                                   qv.codes[t], qv.norm16[t])
    return cache


def _q8_case(bv, seq_lens, n_kv, g, seed):
    seeds = (40 + seed, 50 + seed, 60 + seed)
    tab = dict(oracle_tables(seeds, 2, bv), bk=8)
    rng = np.random.default_rng(seed)
    ks, vs = [], []
    for L in seq_lens:
        k, v = _rows(rng, max(L, 1), n_kv)
        ks.append(k)
        vs.append(v)
    pages = [max((L + 15) // 16, 1) for L in seq_lens]
    perm = rng.permutation(sum(pages)).astype(np.int32)
    bt = np.zeros((len(seq_lens), max(pages)), dtype=np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    cache_np = _oracle_cache_q8(ks, vs, bt, seq_lens, sum(pages), tab)
    q = synth.round_to_bf16(rng.standard_normal((len(seq_lens), n_kv * g, 128)).astype(np.float32))
    return seeds, tab, cache_np, bt, sum(pages), q


@pytest.mark.parametrize("bv,g,seq_lens", [(2, 4, [333, 17, 0, 64]), (3, 1, [700, 1]), (4, 8, [129, 250]),
                                           (3, 12, [200, 47]), (3, 4, [4000, 2500])])
def test_q8_decode_matches_oracle(bv, g, seq_lens):
    n_kv = 2
    seeds, tab, cache_np, bt, n_pages, q = _q8_case(bv, seq_lens, n_kv, g, seed=bv * 13 + g)
    want = odec.decode_paged(cache_np, bt, seq_lens, q.astype(np.float64), tab)
    ctx = binding.Context(8, bv, seeds, device=0)
    max_len = max(seq_lens)
    ws = torch.zeros(ctx.decode_workspace_bytes(len(seq_lens), n_kv * g, n_kv, max_len), dtype=torch.uint8,
                     device=DEV)
    out = torch.full(q.shape, float("nan"), device=DEV)
    ctx.decode_attention(torch.from_numpy(q).to(DEV).to(torch.bfloat16), torch.from_numpy(cache_np.reshape(-1)).to(DEV),
                         n_pages, torch.from_numpy(bt).to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                         n_kv, max_len, out, ws)
    assert ctx.device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    live = np.array(seq_lens) > 0
    assert np.all(got[~live] == 0)
    print("worst rel err", assert_outputs_close(got[live], want[live]))


@pytest.mark.parametrize("bv,g", [(3, 4), (2, 1)])
def test_q8_logits_match_oracle(bv, g):
    seq_lens, n_kv = [1000, 37, 0], 2
    seeds, tab, cache_np, bt, n_pages, q = _q8_case(bv, seq_lens, n_kv, g, seed=70 + bv + g)
    ctx = binding.Context(8, bv, seeds, device=0)
    stride = max(seq_lens) + 5
    sentinel = 12345.0
    logits = torch.full((len(seq_lens), n_kv * g, stride), sentinel, device=DEV)
    ctx.decode_logits(torch.from_numpy(q).to(DEV).to(torch.bfloat16), torch.from_numpy(cache_np.reshape(-1)).to(DEV),
                      n_pages, torch.from_numpy(bt).to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                      n_kv, max(seq_lens), logits)
    assert ctx.device_error() == 0
    got = logits.cpu().numpy().astype(np.float64)
    scale = 1.0 / np.sqrt(128)
    for b, L in enumerate(seq_lens):
        assert np.all(got[b, :, L:] == sentinel)
        if L == 0:
            continue
        for hk in range(n_kv):
            k8, sc, _, _ = odec.gather_sequence_q8(cache_np, bt[b], L, hk, bv)
            khat = q8.dequantize_q8(k8, sc)
            for hh in range(g):
                h = hk * g + hh
                qq = q[b, h].astype(np.float64)
                want = q8.logits_q8(qq, k8, sc, scale)
                ref = np.maximum(np.abs(want), scale * np.linalg.norm(qq) * np.linalg.norm(khat, axis=1))
                err = np.abs(got[b, h, :L] - want)
                assert np.all(err <= 1e-3 * ref), float(np.max(err / ref))


def test_q8_decode_step_appends_and_attends():
    """tq_decode_step with q8_0 keys: the appended token matches the oracle's quantization, then attend."""
    bv, n_kv, g, steps = 3, 2, 4, 3
    seeds = (81, 82, 83)
    tab = dict(oracle_tables(seeds, 2, bv), bk=8)
    rng = np.random.default_rng(12)
    L0 = [47, 16]
    kv = [_rows(rng, L + steps, n_kv) for L in L0]
    pages = [(L + steps + 15) // 16 for L in L0]
    perm = rng.permutation(sum(pages) + 2).astype(np.int32)
    bt = np.stack([perm[:pages[0]], np.resize(perm[pages[0]:pages[0] + pages[1]], pages[0])]).astype(np.int32)
    n_pages = sum(pages) + 2
    ctx = binding.Context(8, bv, seeds, device=0)
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)

    def bf(x):
        return torch.from_numpy(x.astype(np.float32)).to(DEV).to(torch.bfloat16)

    for b, L in enumerate(L0):
        ctx.quantize_prefill(bf(kv[b][0][:L]), bf(kv[b][1][:L]), btt[b], 0, cache, n_pages)
    max_len = max(L0) + steps
    ws = torch.zeros(ctx.decode_workspace_bytes(2, n_kv * g, n_kv, max_len), dtype=torch.uint8, device=DEV)
    for step in range(steps):
        lens = [L + step + 1 for L in L0]
        k_new = np.stack([kv[b][0][lens[b] - 1] for b in range(2)])
        v_new = np.stack([kv[b][1][lens[b] - 1] for b in range(2)])
        q = synth.round_to_bf16(rng.standard_normal((2, n_kv * g, 128)).astype(np.float32))
        out = torch.full((2, n_kv * g, 128), float("nan"), device=DEV)
        ctx.decode_step(bf(k_new), bf(v_new), bf(q), cache, n_pages, btt,
                        torch.tensor(lens, dtype=torch.int32, device=DEV), n_kv, max_len, out, ws)
        host = cache.cpu().numpy().reshape(n_pages, n_kv, -1)
        for b in range(2):
            pos = lens[b] - 1
            for h in range(n_kv):
                vals, sc, vc, vn = lay.read_page_q8(host[bt[b][pos // 16], h], bv)
                kq = q8.quantize_q8(k_new[b, h])
                near = np.abs(np.abs(kq.ratio) % 1.0 - 0.5) < 1e-5
                assert np.all((vals[pos % 16] == kq.values) | near)
                assert np.all(half_ulps_apart(sc[pos % 16], kq.scales16) <= 1)
                _, qv = oracle_quantize(k_new[b:b + 1, h], v_new[b:b + 1, h], tab)
                nb = near_boundary(qv.y[0], tab["thresholds_v"])
                assert np.all((vc[pos % 16] == qv.codes[0]) | nb)
        want = odec.decode_paged(host, bt, lens, q.astype(np.float64), tab)
        print("worst rel err", assert_outputs_close(out.cpu().numpy().astype(np.float64), want))
    assert ctx.device_error() == 0


def test_q8_full_size_sampled_parity():
    """Llama-8B 32K with q8_0 keys and 3-bit values, in the launch configuration bench.py times:
    prefill of the whole context, one decode step; sampled rows and one KV head's decode
    against the oracle."""
    wl = synth.WORKLOADS["llama8b_q8k"]
    gen = synth.Generator(wl)
    seeds = gen.method_seeds()
    tab = dict(oracle_tables(seeds, 2, wl.value_bits), bk=8)
    ctx = binding.Context(8, wl.value_bits, seeds, device=0)
    L = int(gen.seq_lens()[0])
    bt, n_pages = gen.page_pool(np.array([(L + 1 + 15) // 16]))
    n_kv = wl.n_kv_heads
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    tg = torch.Generator(device=DEV)
    tg.manual_seed(4242)
    sk = torch.from_numpy(gen.scales["k"]).float().to(DEV)
    sv = torch.from_numpy(gen.scales["v"]).float().to(DEV)
    k = (torch.randn((L, n_kv, 128), generator=tg, device=DEV) * sk).to(torch.bfloat16)
    v = (torch.randn((L, n_kv, 128), generator=tg, device=DEV) * sv).to(torch.bfloat16)
    ctx.quantize_prefill(k, v, btt[0], 0, cache, n_pages)
    k_new = (torch.randn((1, n_kv, 128), generator=tg, device=DEV) * sk).to(torch.bfloat16)
    v_new = (torch.randn((1, n_kv, 128), generator=tg, device=DEV) * sv).to(torch.bfloat16)
    q = torch.randn((1, wl.n_q_heads, 128), generator=tg, device=DEV).to(torch.bfloat16)
    ws = torch.zeros(ctx.decode_workspace_bytes(1, wl.n_q_heads, n_kv, L + 1), dtype=torch.uint8, device=DEV)
    out = torch.full((1, wl.n_q_heads, 128), float("nan"), device=DEV)
    ctx.decode_step(k_new, v_new, q, cache, n_pages, btt, torch.tensor([L + 1], dtype=torch.int32, device=DEV),
                    n_kv, L + 1, out, ws)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    cache3 = cache.view(n_pages, n_kv, ctx.block_bytes)
    rng = np.random.default_rng(5)
    pos = np.append(rng.choice(L, size=200, replace=False), L)
    heads = rng.integers(0, n_kv, size=len(pos))
    kn, vn_ = k.float().cpu().numpy(), v.float().cpu().numpy()
    knew, vnew = k_new.float().cpu().numpy()[0], v_new.float().cpu().numpy()[0]
    bad = 0
    for p, h in zip(pos, heads):
        kr = (knew[h] if p == L else kn[p, h]).astype(np.float64)
        vr = (vnew[h] if p == L else vn_[p, h]).astype(np.float64)
        vals, sc, vc, vnorm = lay.read_page_q8(cache3[int(bt[0, p // 16]), int(h)].cpu().numpy(), wl.value_bits)
        kq = q8.quantize_q8(kr)
        near = np.abs(np.abs(kq.ratio) % 1.0 - 0.5) < 1e-5
        bad += int(np.sum((vals[p % 16] != kq.values) & ~near))
        assert np.all(half_ulps_apart(sc[p % 16], kq.scales16) <= 1)
        _, qv = oracle_quantize(kr[None], vr[None], tab)
        bad += int(np.sum((vc[p % 16] != qv.codes[0]) & ~near_boundary(qv.y[0], tab["thresholds_v"])))
        assert half_ulps_apart(np.array([vnorm[p % 16]]), np.array([qv.norm16[0]]))[0] <= 1
    assert bad == 0
    g = wl.group
    h = int(rng.integers(0, n_kv))
    pg = bt[0, :(L + 1 + 15) // 16]
    sub = cache3[torch.from_numpy(pg.astype(np.int64)).to(DEV), h].cpu().numpy()[:, None, :]
    qn = q.float().cpu().numpy().astype(np.float64)
    want = odec.decode_paged(sub, np.arange(len(pg))[None], [L + 1], qn[:, h * g:(h + 1) * g], tab)
    got = out.cpu().numpy().astype(np.float64)[:, h * g:(h + 1) * g]
    print("q8 full size: decode worst rel err", assert_outputs_close(got, want))


@pytest.mark.parametrize("path", ["prefill", "append"])
def test_q8_zero_blocks(path):
    """All-zero 32-coordinate key blocks store scale 0 and values 0; a zero key row and
    zero value rows decode without NaN; decode matches the oracle on the GPU-written bytes."""
    bv, n_kv, g, L = 3, 2, 4, 41
    seeds = (91, 92, 93)
    tab = dict(oracle_tables(seeds, 2, bv), bk=8)
    rng = np.random.default_rng(44)
    k, v = _rows(rng, L, n_kv)
    k[3, 0, 32:64] = 0.0
    k[7, 1, 96:] = 0.0
    k[11] = 0.0
    v[[11, 20]] = 0.0
    ctx, cache, bt, n_pages = _gpu_cache(bv, seeds, k, v, path)
    for t in range(L):
        for h in range(n_kv):
            vals, sc, vc, vn = lay.read_page_q8(cache[bt[t // 16], h], bv)
            kq = q8.quantize_q8(k[t, h])
            zero = np.all(k[t, h].reshape(4, 32) == 0, axis=1)
            assert np.all(sc[t % 16][zero] == 0) and np.all(vals[t % 16].reshape(4, 32)[zero] == 0)
            near = np.abs(np.abs(kq.ratio) % 1.0 - 0.5) < 1e-5
            assert np.all((vals[t % 16] == kq.values) | near)
            if np.all(v[t, h] == 0):
                assert vn[t % 16] == 0
    q = synth.round_to_bf16(rng.standard_normal((1, n_kv * g, 128)).astype(np.float32))
    ws = torch.zeros(ctx.decode_workspace_bytes(1, n_kv * g, n_kv, L), dtype=torch.uint8, device=DEV)
    out = torch.full((1, n_kv * g, 128), float("nan"), device=DEV)
    dc = torch.from_numpy(cache.reshape(-1)).to(DEV)
    ctx.decode_attention(torch.from_numpy(q).to(DEV).to(torch.bfloat16), dc, n_pages, torch.from_numpy(bt[None]).to(DEV),
                         torch.tensor([L], dtype=torch.int32, device=DEV), n_kv, L, out, ws)
    assert ctx.device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    want = odec.decode_paged(cache, bt[None], [L], q.astype(np.float64), tab)
    print("worst rel err", assert_outputs_close(got, want))
