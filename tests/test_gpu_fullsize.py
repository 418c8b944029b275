"""Parity at the benchmark workloads' full sizes, on sampled outputs.

For each workload (Llama-8B 32K, batched ragged 16 x [2K, 8K], Llama-70B 128K,
Command-R+ 4 x 128K), in the launch configuration bench.py times:
  1. quantize-prefill of every sequence's full context on the GPU;
  2. one tq_decode_step (append one token per sequence, then attend).
Quantize parity: a seeded sample of at least 4096 (sequence, token, KV head)
rows unpacked from the GPU cache against the oracle's quantization of the same
input rows (codes and sign bits bit-exact outside the 1e-5 boundary band, fp16
norms within one unit in the last place). The appended tokens are checked the
same way.
Decode parity: for at least 4 (sequence, KV head) pairs, the oracle decodes from
the bytes the GPU wrote (identical codes) over the whole context including the
appended token; outputs within the element-wise and per-head bounds of
parity_util.assert_outputs_close.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding, synth  # noqa: E402
from oracle import decode as odec  # noqa: E402
from oracle import layout as lay  # noqa: E402

from parity_util import assert_outputs_close, compare_tokens, oracle_quantize, oracle_tables  # noqa: E402

DEV = "cuda:0"
N_QUANT = 4096          # sampled (sequence, token, KV head) rows per workload
N_DECODE = 4            # (sequence, KV head) pairs decoded by the oracle over the full context


def _bf16_rows(x):
    return x.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name", ["llama8b", "batched", "llama70b", "cmdr104b"])
def test_full_size_sampled_parity(name):
    wl = synth.WORKLOADS[name]
    gen = synth.Generator(wl)
    seeds = gen.method_seeds()
    tab = oracle_tables(seeds, wl.key_bits, wl.value_bits)
    ctx = binding.Context(wl.key_bits, wl.value_bits, seeds, device=0)
    lens = gen.seq_lens().astype(np.int64)                     # cached tokens before the step
    pages = (lens + 1 + 15) // 16                               # room for the appended token
    bt, n_pages = gen.page_pool(pages)
    n_kv, bb = wl.n_kv_heads, ctx.block_bytes
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    tg = torch.Generator(device=DEV)
    tg.manual_seed(1000 + wl.seed)
    sk = torch.from_numpy(gen.scales["k"]).float().to(DEV)
    sv = torch.from_numpy(gen.scales["v"]).float().to(DEV)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    rng = np.random.default_rng(77 + wl.seed)
    samples = []                                                # (b, pos, head, k_row, v_row)
    for b, L in enumerate(lens):
        k = (torch.randn((int(L), n_kv, 128), generator=tg, device=DEV) * sk).to(dt)
        v = (torch.randn((int(L), n_kv, 128), generator=tg, device=DEV) * sv).to(dt)
        ctx.quantize_prefill(k, v, btt[b], 0, cache, n_pages)
        pos = rng.choice(int(L), size=min(int(L), -(-N_QUANT // len(lens)) + 16), replace=False)
        heads = rng.integers(0, n_kv, size=len(pos))
        kr = _bf16_rows(k[torch.from_numpy(pos).to(DEV), torch.from_numpy(heads).to(DEV)])
        vr = _bf16_rows(v[torch.from_numpy(pos).to(DEV), torch.from_numpy(heads).to(DEV)])
        samples += [(b, int(p), int(h), kr[i], vr[i]) for i, (p, h) in enumerate(zip(pos, heads))]
        del k, v
    # one decode step in the bench's launch configuration
    k_new = (torch.randn((wl.batch, n_kv, 128), generator=tg, device=DEV) * sk).to(dt)
    v_new = (torch.randn((wl.batch, n_kv, 128), generator=tg, device=DEV) * sv).to(dt)
    q = torch.randn((wl.batch, wl.n_q_heads, 128), generator=tg, device=DEV).to(dt)
    new_lens = torch.from_numpy(lens + 1).to(torch.int32).to(DEV)
    max_len = int(lens.max()) + 1
    ws = torch.zeros(ctx.decode_workspace_bytes(wl.batch, wl.n_q_heads, n_kv, max_len), dtype=torch.uint8,
                     device=DEV)
    out = torch.full((wl.batch, wl.n_q_heads, 128), float("nan"), device=DEV)
    ctx.decode_step(k_new, v_new, q, cache, n_pages, btt, new_lens, n_kv, max_len, out, ws)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    assert torch.isfinite(out).all()
    cache3 = cache.view(n_pages, n_kv, bb)

    # quantize parity on the sampled rows and on every appended token
    for b in range(wl.batch):
        for h in range(n_kv):
            samples.append((b, int(lens[b]), h, _bf16_rows(k_new[b, h]), _bf16_rows(v_new[b, h])))
    assert len(samples) >= N_QUANT
    # unpack every sampled row, one read per (page, KV head) block
    by_block = {}
    for i, (b, p, h, kr, vr) in enumerate(samples):
        by_block.setdefault((int(bt[b, p // 16]), h), []).append(i)
    fields = [[None] * len(samples) for _ in range(6)]
    for (pg, h), idx in by_block.items():
        f = lay.read_page(cache3[pg, h].cpu().numpy(), wl.key_bits, wl.value_bits)
        for i in idx:
            tau = samples[i][1] % 16
            for j in range(6):
                fields[j][i] = f[j][tau]
    xk = [smp[3] for smp in samples]
    xv = [smp[4] for smp in samples]
    qk, qv = oracle_quantize(np.array(xk), np.array(xv), tab)
    res = compare_tokens(tuple(np.array(x) for x in fields), qk, qv, tab)
    print(name, res)
    assert all(v == 0 for key, v in res.items() if key.startswith("bad")), res

    # decode parity for sampled (sequence, KV head) pairs, from the GPU-written bytes
    qn = q.float().cpu().numpy().astype(np.float64)
    g = wl.n_q_heads // n_kv
    got_all = out.cpu().numpy().astype(np.float64)
    pairs = [(b, h) for b in range(wl.batch) for h in range(n_kv)]
    order = [pairs[int(i)] for i in rng.permutation(len(pairs))]
    last = [pr for pr in order if pr[0] == wl.batch - 1][:1]        # the last sequence is always checked
    checks = last + [pr for pr in order if pr not in last][:N_DECODE - len(last)]
    assert len(set(checks)) >= N_DECODE
    for b, h in checks:
        L = int(lens[b]) + 1
        pg = bt[b, :(L + 15) // 16]
        sub = cache3[torch.from_numpy(pg.astype(np.int64)).to(DEV), h].cpu().numpy()[:, None, :]
        want = odec.decode_paged(sub, np.arange(len(pg))[None], [L], qn[b:b + 1, h * g:(h + 1) * g], tab)
        got = got_all[b:b + 1, h * g:(h + 1) * g]
        print(name, "decode", b, h, "worst rel err", assert_outputs_close(got, want))
