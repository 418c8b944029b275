"""Device-side error paths of the decode kernel, exercised without any fault.

* TQ_DEV_TIMEOUT: the TQ_TEST_WAIT_RUNS_OUT test hook makes warp 0 of thread
  block 0 wait, with a short limit, on a barrier that nothing completes. The
  wait runs out, the error bit is recorded, the warp lets its copies in flight
  land and the call finishes with finite outputs (missing that warp's pages).
  The next call without the hook must match the oracle again -- for the
  no-alloc entry point this also shows that a call which recorded a device
  error leaves the fixed scratch's completion counters at zero.
* TQ_DEV_BAD_LENGTH: a seq_lens entry above max_seq_len (or negative) is
  recorded and clamped; the block table is sized so that even an unclamped read
  would stay inside it.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from decode_attention_seeded_b200 import binding  # noqa: E402
from oracle import decode as odec  # noqa: E402

from parity_util import assert_outputs_close, oracle_tables  # noqa: E402

DEV = "cuda:0"
SEEDS = (5, 6, 7)


def _setup(seq_lens, n_kv, bk=3, bv=2, table_pages=None):
    ctx = binding.Context(bk, bv, SEEDS, device=0)
    pages = [(L + 15) // 16 for L in seq_lens]
    width = table_pages or max(pages)
    n_pages = len(seq_lens) * width
    perm = np.random.default_rng(1).permutation(n_pages).astype(np.int32)
    bt = perm.reshape(len(seq_lens), width)
    cache = torch.zeros(n_pages * ctx.page_bytes(n_kv), dtype=torch.uint8, device=DEV)
    btt = torch.from_numpy(bt).to(DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(2)
    for b in range(len(seq_lens)):
        L = width * 16                                       # fill every page the table names
        k = torch.randn((L, n_kv, 128), generator=g, device=DEV).to(torch.bfloat16)
        v = torch.randn((L, n_kv, 128), generator=g, device=DEV).to(torch.bfloat16)
        ctx.quantize_prefill(k, v, btt[b], 0, cache, n_pages)
    return ctx, cache, n_pages, bt, btt


@pytest.mark.parametrize("noalloc", [False, True])
def test_wait_that_runs_out_is_reported_and_the_next_call_is_exact(noalloc):
    seq_lens, n_kv, group = [1500, 700], 2, 4
    ctx, cache, n_pages, bt, btt = _setup(seq_lens, n_kv)
    batch, n_q, max_len = len(seq_lens), n_kv * group, max(seq_lens)
    lens = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    ws = torch.zeros(ctx.decode_workspace_bytes(batch, n_q, n_kv, max_len), dtype=torch.uint8, device=DEV)
    q = torch.randn((batch, n_q, 128), device=DEV).to(torch.bfloat16)

    def run(out):
        if noalloc:
            ctx.decode_attention_noalloc(q, cache, n_pages, btt, lens, n_kv, max_len, out)
        else:
            ctx.decode_attention(q, cache, n_pages, btt, lens, n_kv, max_len, out, ws)

    ctx.set_test_flags(binding.TEST_WAIT_RUNS_OUT)
    out = torch.full((batch, n_q, 128), float("nan"), device=DEV)
    run(out)
    err = ctx.device_error()
    assert err & binding.DEV_TIMEOUT, hex(err)
    assert torch.isfinite(out).all()

    ctx.set_test_flags(0)
    out = torch.full((batch, n_q, 128), float("nan"), device=DEV)
    run(out)
    assert ctx.device_error() == 0
    tab = oracle_tables(SEEDS, 3, 2)
    host = cache.view(n_pages, n_kv, -1).cpu().numpy()
    want = odec.decode_paged(host, bt, seq_lens, q.float().cpu().numpy(), tab)
    assert_outputs_close(out.cpu().numpy().astype(np.float64), want)


def test_test_flags_reject_unknown_bits():
    ctx = binding.Context(3, 2, SEEDS, device=0)
    with pytest.raises(binding.TQError) as e:
        ctx.set_test_flags(0x80)
    assert e.value.code == 1


def test_bad_length_is_reported_and_clamped():
    n_kv, group, max_len = 2, 4, 600
    # the block table is wide enough for 1000 tokens, so even an unclamped read stays inside it
    ctx, cache, n_pages, bt, btt = _setup([1000, 1000], n_kv, table_pages=63)
    batch, n_q = 2, n_kv * group
    lens = torch.tensor([max_len + 37, -5], dtype=torch.int32, device=DEV)
    ws = torch.zeros(ctx.decode_workspace_bytes(batch, n_q, n_kv, max_len), dtype=torch.uint8, device=DEV)
    q = torch.randn((batch, n_q, 128), device=DEV).to(torch.bfloat16)
    out = torch.full((batch, n_q, 128), float("nan"), device=DEV)
    ctx.decode_attention(q, cache, n_pages, btt, lens, n_kv, max_len, out, ws)
    err = ctx.device_error()
    assert err & binding.DEV_BAD_LENGTH, hex(err)
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    # sequence 0 is clamped to max_seq_len, sequence 1 (negative) to an empty sequence
    tab = oracle_tables(SEEDS, 3, 2)
    host = cache.view(n_pages, n_kv, -1).cpu().numpy()
    want = odec.decode_paged(host, bt, [max_len, 0], q.float().cpu().numpy(), tab)
    assert_outputs_close(got, want)
    assert np.all(got[1] == 0.0)
    # the next call with valid lengths is clean
    lens = torch.tensor([max_len, 17], dtype=torch.int32, device=DEV)
    ctx.decode_attention(q, cache, n_pages, btt, lens, n_kv, max_len, out, ws)
    assert ctx.device_error() == 0
