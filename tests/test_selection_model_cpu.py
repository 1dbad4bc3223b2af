"""The decode kernel's way of finding the cut and laying out the selected rows, restated in
Python, agrees with the oracle's sorted walk (ClusterKV explainer, section 3.3) on
adversarial cases.

The kernel does not sort all the clusters. Each CTA:
1. maps the fp32 scores monotonically onto 256 linear buckets between the smallest and the
   largest score of the clusters with tokens;
2. builds a histogram of cluster sizes per bucket and finds the bucket b* holding the cut
   (the first cluster, in descending (score, -index) order, whose inclusive size exceeds the
   remaining budget);
3. compacts the clusters with tokens in buckets >= b* (the candidates) and ranks each one
   among them by the key (orderable score, -index), with the tokens of the candidates before
   it (its prefix); the orderable score maps -0 and +0 to one key, so they tie like equal
   doubles. A candidate whose prefix plus size fits is whole at its rank; the one whose
   prefix fits and whose prefix plus size does not is the cut;
4. lays the whole clusters out in that rank (walk) order: selection position x maps to the
   whole cluster k with the largest prefix <= x, row offsets[c_k] + x - prefix_k (a binary
   search).

This model is checked against the oracle's `select` on stores whose scores are exactly the
chosen fp32 values (centroid c = s_c * e_0, query e_0): many ties, all-equal scores, a tiny
score range, and zero-size clusters. It is a check of the algorithm; the GPU parity tests
check the kernel.
"""
import numpy as np

import oracle

D = 128


def _orderable(x: np.float32) -> int:
    """Unsigned key with the order of the float; -0 and +0 give the same key (they tie)."""
    u = int((np.array([x], np.float32) + np.float32(0)).view(np.uint32)[0])
    return (~u) & 0xFFFFFFFF if u & 0x80000000 else u | 0x80000000


def bucket_cut(sc: np.ndarray, sz: np.ndarray, R: int):
    """Whole clusters in walk order (list of (cluster, prefix)), the cut cluster and W (tokens
    in whole clusters), or None if all fit."""
    sc = sc.astype(np.float32)
    if sz.sum() <= R:
        return None
    live = sz > 0
    keys = [_orderable(x) for x in sc[live]]
    mn = np.float32(sc[live][int(np.argmin(keys))])
    mx = np.float32(sc[live][int(np.argmax(keys))])
    span = np.float32(mx - mn)
    inv = np.float32(255.99) / span if span > 1e-30 else np.float32(0)
    b = np.clip(np.nan_to_num((sc - mn).astype(np.float32) * inv, nan=0.0), 0, 255).astype(np.int64)
    hist = np.zeros(256, np.int64)
    np.add.at(hist, b[live], sz[live])
    above, bstar = 0, 0
    for d in range(255, -1, -1):
        if above <= R < above + hist[d]:
            bstar = d
            break
        above += hist[d]
    cand = [c for c in range(len(sc)) if sz[c] > 0 and b[c] >= bstar]
    key = {c: (_orderable(sc[c]) << 32) | (0xFFFFFFFF - c) for c in range(len(sc))}
    whole, cuts = {}, []
    for c in cand:
        before = [j for j in cand if key[j] > key[c]]
        rank, pre = len(before), sum(int(sz[j]) for j in before)
        if pre + sz[c] <= R:
            whole[rank] = (c, pre)
        elif pre <= R:
            cuts.append((c, pre, rank))
    assert len(cuts) == 1
    cut, pre_cut, rank_cut = cuts[0]
    assert sorted(whole) == list(range(rank_cut))  # the whole clusters take ranks 0 .. cut - 1
    return [whole[k] for k in range(rank_cut)], cut, pre_cut


def layout_rows(offs: np.ndarray, whole: list, W: int) -> list:
    """Store rows of selection positions 0..W-1 of the whole clusters (walk order)."""
    pre = [p for _, p in whole] + [W]
    rows = []
    for x in range(W):
        k0, khi = 0, len(whole) - 1  # the last whole cluster with prefix <= x
        while k0 < khi:
            mid = (k0 + khi + 1) >> 1
            if pre[mid] <= x:
                k0 = mid
            else:
                khi = mid - 1
        c = whole[k0][0]
        assert pre[k0] <= x < pre[k0 + 1] and pre[k0 + 1] - pre[k0] == offs[c + 1] - offs[c]
        rows.append(int(offs[c] + x - pre[k0]))
    return rows


def _store(sc, sz):
    m = int(sz.sum())
    offs = np.concatenate([[0], np.cumsum(sz)]).astype(np.int32)
    mu = np.zeros((len(sc), D))
    mu[:, 0] = sc.astype(np.float64)
    kp = np.zeros((m, D), np.uint16)
    kp[:, 1] = 0x3F80  # 1.0: every token scores 0 on e_0, the partial fill is by id
    sink = np.zeros((16, D), np.uint16)
    return oracle.Store(sink, sink.copy(), kp, kp.copy(), np.arange(16, 16 + m, dtype=np.int32),
                        offs, mu)


def test_bucket_histogram_cut_equals_the_sorted_walk():
    rng = np.random.default_rng(0)
    qbar = np.zeros(D)
    qbar[0] = 1.0
    checked = 0
    for trial in range(800):
        C = int(rng.integers(1, 80))
        kind = trial % 4
        sc = rng.normal(0, 30, C).astype(np.float32)
        if kind == 1:
            sc = (np.round(sc / 10) * 10).astype(np.float32)       # many ties
        elif kind == 2:
            sc[:] = np.float32(5.0)                                  # all equal
        elif kind == 3:
            sc = (rng.normal(0, 1e-6, C) + 100).astype(np.float32)  # a tiny range
        sz = rng.integers(0, 60, C)
        if trial % 5 == 0:
            sz[rng.integers(0, C, max(1, C // 3))] = 0
        R = int(rng.integers(0, max(1, int(sz.sum()) + 10)))
        st = _store(sc, sz)
        sel = oracle.select_qbar(st, qbar, R + 16)
        got = bucket_cut(sc, sz, R)
        if got is None:
            assert sel.cut == -1
            continue
        whole, cut, W = got
        assert cut == sel.cut, (trial, cut, sel.cut)
        assert R - W == sel.r, (trial, R - W, sel.r)
        taken = {int(c) for c in np.searchsorted(st.offsets, sel.rows[sel.rows >= 0], side="right") - 1}
        assert {c for c, _ in whole} == taken - {cut}, trial
        # the whole clusters' rows, laid out in walk order, are the oracle's whole rows
        rows = layout_rows(st.offsets, whole, W)
        assert len(set(rows)) == W
        want = {int(r) for r in sel.rows[sel.rows >= 0]
                if not (st.offsets[cut] <= r < st.offsets[cut + 1])}
        assert set(rows) == want, trial
        checked += 1
    assert checked > 600
