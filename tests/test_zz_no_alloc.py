"""tq_decode_attention_noalloc against tq_decode_attention, through the C ABI.

The no-alloc entry point runs the same decode kernel with the library's fixed
per-device scratch in place of a caller workspace. Pages are handed to the
warps of a thread block at run time, so the order of the floating-point sums
can change from run to run: the two entry points are compared within a tight
relative tolerance (and both against the oracle at the decode tolerance), on
several consecutive calls, so that a completion counter left non-zero by one
call (which would merge the wrong records in the next) shows up as a large
error. Two shapes are covered: a small uniform split and a ragged batch that
takes the balanced split, where one thread block serves several (sequence, KV
head) pairs. This file is named so that pytest collects it last; it passes
alone as well.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding  # noqa: E402
from oracle import decode as odec  # noqa: E402

from parity_util import assert_outputs_close, oracle_tables  # noqa: E402

DEV = "cuda:0"
SCRATCH_BYTES = 4 << 20          # the fixed scratch declared in include/tq.h
SEEDS = (11, 22, 33)


def _cache_with_prefill(ctx, seq_lens, n_kv, seed):
    """Quantize random bf16 K/V of each sequence into a randomly permuted page pool."""
    pages = [(L + 15) // 16 for L in seq_lens]
    n_pages = sum(pages) + 2
    perm = np.random.default_rng(seed).permutation(n_pages).astype(np.int32)
    bt = np.zeros((len(seq_lens), max(pages)), dtype=np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    for b, L in enumerate(seq_lens):
        scale = torch.exp(torch.randn((n_kv, 128), generator=g, device=DEV))
        k = (torch.randn((L, n_kv, 128), generator=g, device=DEV) * scale).to(torch.bfloat16)
        v = (torch.randn((L, n_kv, 128), generator=g, device=DEV) * scale).to(torch.bfloat16)
        ctx.quantize_prefill(k, v, btt[b], 0, cache, n_pages)
    return cache, n_pages, bt, btt


@pytest.mark.parametrize("seq_lens,n_kv,group,calls", [
    ([3000, 17, 1234], 4, 4, 3),                                   # uniform split
    (list(np.random.default_rng(3).integers(2048, 8193, size=16)), 8, 4, 3),   # balanced split
])
def test_noalloc_matches_workspace_entry_point_and_oracle(seq_lens, n_kv, group, calls):
    seq_lens = [int(x) for x in seq_lens]
    bk, bv = 3, 2
    ctx = binding.Context(bk, bv, SEEDS, device=0)
    cache, n_pages, bt, btt = _cache_with_prefill(ctx, seq_lens, n_kv, seed=5)
    lens = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    max_len = max(seq_lens)
    batch, n_q = len(seq_lens), n_kv * group
    need = ctx.decode_workspace_bytes(batch, n_q, n_kv, max_len)
    assert 0 < need <= SCRATCH_BYTES
    if batch == 16:
        # the balanced split keeps one record per share (one per SM) plus one per pair,
        # 4 heads x 132 floats each; the uniform split would keep one per pair here
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        assert need >= (sms + batch * n_kv) * 4 * 132 * 4
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    tab = oracle_tables(SEEDS, bk, bv)
    host = cache.view(n_pages, n_kv, -1).cpu().numpy()
    g = torch.Generator(device=DEV)
    g.manual_seed(9)
    for call in range(calls):
        q = torch.randn((batch, n_q, 128), generator=g, device=DEV).to(torch.bfloat16)
        want = torch.full((batch, n_q, 128), float("nan"), device=DEV)
        got = torch.full_like(want, float("nan"))
        ctx.decode_attention(q, cache, n_pages, btt, lens, n_kv, max_len, want, ws)
        ctx.decode_attention_noalloc(q, cache, n_pages, btt, lens, n_kv, max_len, got)
        torch.cuda.synchronize()
        assert ctx.device_error() == 0
        assert torch.isfinite(want).all() and torch.isfinite(got).all()
        w, o = want.cpu().numpy().astype(np.float64), got.cpu().numpy().astype(np.float64)
        # the two entry points: same kernel, sums in a possibly different order
        assert_outputs_close(o, w, rtol=1e-5)
        # both against the oracle, on two sequences
        for b in (0, batch - 1):
            ref = odec.decode_paged(host, bt[b:b + 1], [seq_lens[b]], q[b:b + 1].float().cpu().numpy(), tab)
            assert_outputs_close(o[b:b + 1], ref)
            assert_outputs_close(w[b:b + 1], ref)


def test_noalloc_refuses_calls_larger_than_its_scratch():
    # 64 sequences x 8 KV heads x 16 query heads per KV head need more than 4 MiB of
    # split-K records; the call must return TQ_ERR_WORKSPACE and enqueue nothing.
    batch, n_kv, n_q, max_len = 64, 8, 128, 16
    ctx = binding.Context(3, 2, SEEDS, device=0)
    assert ctx.decode_workspace_bytes(batch, n_q, n_kv, max_len) > SCRATCH_BYTES
    q = torch.zeros((batch, n_q, 128), dtype=torch.bfloat16, device=DEV)
    out = torch.full((batch, n_q, 128), 7.0, device=DEV)
    cache = torch.zeros(ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.zeros((batch, 1), dtype=torch.int32, device=DEV)
    lens = torch.zeros(batch, dtype=torch.int32, device=DEV)
    with pytest.raises(binding.TQError) as e:
        ctx.decode_attention_noalloc(q, cache, 1, btt, lens, n_kv, max_len, out)
    assert e.value.code == 3            # TQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())     # nothing ran
