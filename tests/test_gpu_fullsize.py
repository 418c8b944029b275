"""Parity at the benchmark workloads' full sizes, on sampled outputs.

For each workload (Llama-8B 32K, batched ragged 16 x [2K, 8K], Llama-70B 128K,
Command-R+ 4 x 128K), in the launch configuration bench.py times:
  1. quantize-prefill of every sequence's full context on the GPU;
  2. one tq_decode_step (append one token per sequence, then attend).
Quantize parity: a seeded sample of (sequence, token, KV head) rows unpacked from
the GPU cache against the oracle's quantization of the same input rows
(codes and sign bits bit-exact outside the 1e-5 boundary band, fp16 norms within
one unit in the last place). The appended tokens are checked the same way.
Decode parity: for sampled (sequence, KV head) pairs, the oracle decodes from the
bytes the GPU wrote (identical codes) over the whole context including the
appended token; outputs within 1e-3 relative error per head.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding, synth  # noqa: E402
from oracle import decode as odec  # noqa: E402

from parity_util import (assert_outputs_close, compare_tokens, oracle_quantize, oracle_tables,  # noqa: E402
                         unpack_tokens)

DEV = "cuda:0"


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
        pos = rng.choice(int(L), size=min(int(L), 256 // len(lens) + 16), replace=False)
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
    rows = {}
    for (b, p, h, kr, vr) in samples:
        pg = int(bt[b, p // 16])
        rows.setdefault((pg, h), None)
    blocks = {key: cache3[key[0], key[1]].cpu().numpy() for key in rows}
    fields = [[] for _ in range(6)]
    xk, xv = [], []
    for (b, p, h, kr, vr) in samples:
        blk = blocks[(int(bt[b, p // 16]), h)]
        f = unpack_tokens(blk[None, None], np.array([0]), p % 16, 1, 0, wl.key_bits, wl.value_bits)
        for i in range(6):
            fields[i].append(f[i][0])
        xk.append(kr)
        xv.append(vr)
    qk, qv = oracle_quantize(np.array(xk), np.array(xv), tab)
    res = compare_tokens(tuple(np.array(x) for x in fields), qk, qv, tab)
    print(name, res)
    assert all(v == 0 for key, v in res.items() if key.startswith("bad")), res

    # decode parity for sampled (sequence, KV head) pairs, from the GPU-written bytes
    qn = q.float().cpu().numpy().astype(np.float64)
    g = wl.n_q_heads // n_kv
    got_all = out.cpu().numpy().astype(np.float64)
    checks = [(0, int(rng.integers(0, n_kv)))]
    if wl.batch > 1:
        checks.append((wl.batch - 1, int(rng.integers(0, n_kv))))
    for b, h in checks:
        L = int(lens[b]) + 1
        pg = bt[b, :(L + 15) // 16]
        sub = cache3[torch.from_numpy(pg.astype(np.int64)).to(DEV), h].cpu().numpy()[:, None, :]
        want = odec.decode_paged(sub, np.arange(len(pg))[None], [L], qn[b:b + 1, h * g:(h + 1) * g], tab)
        got = got_all[b:b + 1, h * g:(h + 1) * g]
        print(name, "decode", b, h, "worst rel err", assert_outputs_close(got, want))
