"""tq_decode_attention_noalloc against tq_decode_attention, through the C ABI.

The no-alloc entry point runs the same decode kernel with the library's fixed
per-device scratch in place of a caller workspace, so its outputs must equal
those of the workspace entry point bit for bit, on consecutive calls (the
scratch's completion counters must come back to zero after each call). This
file is named so that pytest collects it last; it passes alone as well.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding  # noqa: E402

DEV = "cuda:0"
SCRATCH_BYTES = 4 << 20          # the fixed scratch declared in include/tq.h


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
    return cache, n_pages, btt


def test_noalloc_equals_workspace_entry_point_on_consecutive_calls():
    seq_lens, n_kv, group = [3000, 17, 1234], 4, 4
    ctx = binding.Context(3, 2, (11, 22, 33), device=0)
    cache, n_pages, btt = _cache_with_prefill(ctx, seq_lens, n_kv, seed=5)
    lens = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    max_len = max(seq_lens)
    need = ctx.decode_workspace_bytes(len(seq_lens), n_kv * group, n_kv, max_len)
    assert 0 < need <= SCRATCH_BYTES
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(9)
    for call in range(2):
        q = torch.randn((len(seq_lens), n_kv * group, 128), generator=g, device=DEV).to(torch.bfloat16)
        want = torch.full((len(seq_lens), n_kv * group, 128), float("nan"), device=DEV)
        got = torch.full_like(want, float("nan"))
        ctx.decode_attention(q, cache, n_pages, btt, lens, n_kv, max_len, want, ws)
        ctx.decode_attention_noalloc(q, cache, n_pages, btt, lens, n_kv, max_len, got)
        torch.cuda.synchronize()
        assert ctx.device_error() == 0
        assert torch.isfinite(want).all()
        assert torch.equal(got, want), f"call {call}: max |diff| {(got - want).abs().max().item()}"


def test_noalloc_refuses_calls_larger_than_its_scratch():
    # 64 sequences x 8 KV heads x 16 query heads per KV head need more than 4 MiB of
    # split-K records; the call must return TQ_ERR_WORKSPACE and enqueue nothing.
    batch, n_kv, n_q, max_len = 64, 8, 128, 16
    ctx = binding.Context(3, 2, (11, 22, 33), device=0)
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
