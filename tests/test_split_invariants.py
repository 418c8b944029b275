"""Invariants of the balanced split-K partition (host-side restatement of its integer formulas).

The decode kernel's balanced split lays the (sequence, KV head) pairs' pages end to
end, each non-empty pair preceded by seg_w virtual pages, cuts that line into G equal
shares, and serves in share i one segment per pair the share overlaps. Segment
(share i, pair of ordinal o) writes record i + o. The final merge of a pair reads
records first .. first + n - 1, with first = (share of the pair's first page) + o and
n = its number of shares. This restates those formulas and checks, over random
ragged batches with empty sequences:
  - every real page of every pair is in exactly one segment;
  - record slots are unique, below shares + pairs, and consecutive per pair, matching
    first and n;
  - a segment never exceeds the host's bound on a share (its block-table window).
The GPU tests check the kernel itself against the oracle on such batches.
"""
import numpy as np
import pytest

PAGE = 16


def plan(n_seq, n_kv, max_len, sm=148, n_hg=1, min_share=48):
    pairs = n_seq * n_kv
    max_pages = max(1, (max_len + PAGE - 1) // PAGE)
    seg_w = max(8, 36 // n_hg)
    share_bound = max(min_share, (pairs * (max_pages + seg_w) + sm - 1) // sm) + 2
    return dict(seg_w=seg_w, shares=sm, records=sm + pairs, window=share_bound, min_share=min_share)


def segments(lens, n_kv, max_len, P):
    B = len(lens)
    vl = []
    for L in lens:
        pg = (min(max(L, 0), max_len) + PAGE - 1) // PAGE
        vl.append(pg + P["seg_w"] if pg > 0 else 0)
    vs = np.concatenate([[0], np.cumsum(vl)]).astype(np.int64)            # virtual pages before b
    ne = np.concatenate([[0], np.cumsum([v > 0 for v in vl])]).astype(np.int64)   # non-empty before b
    n = n_kv * int(vs[B])
    if n == 0:
        return []
    g = min(P["shares"], max(1, (n + P["min_share"] - 1) // P["min_share"]))

    def pair_at(y):                         # sequence, head, ordinal, virtual length, first virtual page
        lo, hi = 0, B
        while hi - lo > 1:
            mid = (lo + hi) >> 1
            if n_kv * vs[mid] <= y:
                lo = mid
            else:
                hi = mid
        v = int(vs[lo + 1] - vs[lo])
        assert v > 0
        hk = (y - n_kv * int(vs[lo])) // v
        return lo, hk, n_kv * int(ne[lo]) + hk, v, n_kv * int(vs[lo]) + hk * v

    share_lo = lambda i: i * n // g
    share_of = lambda y: ((y + 1) * g + n - 1) // n - 1
    out = []
    for i in range(g):
        x, hi = share_lo(i), share_lo(i + 1)
        while x < hi:
            b, hk, o, v, vp = pair_at(x)
            r0 = vp + P["seg_w"]
            s0, s1 = max(x, r0), min(hi, vp + v)
            x = vp + v
            if s1 > s0:
                f, l = share_of(r0), share_of(r0 + (v - P["seg_w"]) - 1)
                out.append(dict(share=i, pair=b * n_kv + hk, p0=s0 - r0, len=s1 - s0, slot=i + o, first=f + o,
                                n=l - f + 1))
    return out


def _cases():
    rng = np.random.default_rng(0)
    cases = [([32772], 8, 32772), ([131072] * 4, 8, 131072), ([0, 0, 0], 8, 100), ([1] * 300, 8, 1),
             ([int(x) for x in np.random.default_rng(2).integers(2048, 8193, 16)], 8, 8192)]
    for _ in range(120):
        B = int(rng.integers(1, 40))
        n_kv = int(rng.choice([1, 2, 8]))
        max_len = int(rng.integers(1, 20000))
        lens = rng.integers(0, max_len + 1, size=B)
        if rng.random() < 0.3:
            lens[rng.random(B) < 0.3] = 0
        cases.append(([int(v) for v in lens], n_kv, max_len))
    return cases


@pytest.mark.parametrize("n_hg", [1, 3])
def test_balanced_split_covers_every_page_once_with_consecutive_records(n_hg):
    for lens, n_kv, max_len in _cases():
        P = plan(len(lens), n_kv, max_len, n_hg=n_hg)
        segs = segments(lens, n_kv, max_len, P)
        slots = [s["slot"] for s in segs]
        assert len(set(slots)) == len(slots) and all(0 <= x < P["records"] for x in slots)
        covered = set()
        for s in segs:
            assert 0 < s["len"] <= P["window"]
            for pg in range(s["p0"], s["p0"] + s["len"]):
                assert (s["pair"], pg) not in covered
                covered.add((s["pair"], pg))
        want = {(b * n_kv + hk, pg) for b, L in enumerate(lens) for hk in range(n_kv)
                for pg in range((min(max(L, 0), max_len) + PAGE - 1) // PAGE)}
        assert covered == want
        by_pair = {}
        for s in segs:
            by_pair.setdefault(s["pair"], []).append(s)
        for ss in by_pair.values():
            sl = sorted(s["slot"] for s in ss)
            assert sl == list(range(sl[0], sl[0] + len(sl)))
            assert all(s["first"] == sl[0] and s["n"] == len(sl) for s in ss)
