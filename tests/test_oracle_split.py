"""Pins of the oracle's drift check and cluster split (ClusterKV explainer, section 3.2,
decode phase: a cluster whose mean intra-cluster distance passes a threshold is split).

Readings (the page gives no formula): a member's distance is its cosine distance to the
cluster centroid; the threshold is a parameter; a split is 2-cluster cosine K-means on the
cluster's own rows, whose halves take the cluster's place (indices c and c + 1, later
clusters shift up by one). The pins are closed forms of the drift, scipy's cosine
distance, exact recovery of two tight groups, and the layout invariants of the split.
"""
import math

import numpy as np
import pytest
from scipy.spatial import distance

import oracle
import synth_inputs as si

D = 128


def _store(rows_per_cluster, seed=0):
    """A store whose clusters hold the given rows (lists of float [128] arrays, exact in
    bf16), with raw-mean centroids and ids ascending in each cluster."""
    g = np.random.default_rng(seed)
    kp = [r for rows in rows_per_cluster for r in rows]
    m = len(kp)
    kp = si.to_bf16_bits(np.array(kp, np.float32).reshape(m, D)) if m else np.zeros((0, D), np.uint16)
    sizes = [len(r) for r in rows_per_cluster]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    mu = np.zeros((len(sizes), D))
    for c in range(len(sizes)):
        if sizes[c]:
            mu[c] = oracle.bf16_to_f64(kp[offsets[c]:offsets[c + 1]]).mean(axis=0)
    vp = si.to_bf16_bits(g.standard_normal((m, D)).astype(np.float32))
    sink = si.to_bf16_bits(g.standard_normal((16, D)).astype(np.float32))
    ids = np.arange(16, 16 + m, dtype=np.int32)
    return oracle.Store(sink, sink.copy(), kp, vp, ids, offsets, mu)


def _e(i, scale=1.0):
    v = np.zeros(D, np.float32)
    v[i] = scale
    return v


def test_drift_closed_forms():
    x = np.linspace(-1.0, 1.0, D).astype(np.float32)
    st = _store([
        [x, x, x],                            # identical members: drift 0
        [_e(0, 2.0), _e(4, 2.0)],             # orthogonal pair: mu = (1, 1), cos = 1/sqrt(2)
        [_e(3), -_e(3)],                      # antipodal pair: mu = 0, cosine counted as 0
        [],                                   # empty cluster: drift 0
        [_e(1), _e(2), _e(5)],                # orthonormal triple: cos = 1/sqrt(3)
        [x * 0.5, x, x * 4.0],                # one direction, three norms: drift 0
        [_e(7, 3.0)],                         # single member: drift 0
    ])
    d = oracle.cluster_drift(st)
    expect = [0.0, 1 - 1 / math.sqrt(2), 1.0, 0.0, 1 - 1 / math.sqrt(3), 0.0, 0.0]
    np.testing.assert_allclose(d, expect, rtol=0, atol=1e-14)


def test_drift_matches_scipy_cosine_distance():
    K, V = si.keys_values(4, 1, 700, 9)
    st, _ = oracle.prefill_unit(K, V, 7, oracle.stream_key(4, 1, 0), iters=4)
    d = oracle.cluster_drift(st)
    keys = oracle.bf16_to_f64(st.kp)
    for c in range(st.C):
        lo, hi = st.offsets[c], st.offsets[c + 1]
        ref = np.mean([distance.cosine(keys[j], st.mu[c]) for j in range(lo, hi)]) if hi > lo else 0.0
        assert abs(d[c] - ref) < 1e-12, (c, d[c], ref)


def test_drift_is_scale_and_order_invariant():
    K, V = si.keys_values(5, 2, 500, 6)
    st, _ = oracle.prefill_unit(K, V, 5, oracle.stream_key(5, 2, 0), iters=3)
    d = oracle.cluster_drift(st)
    # doubling every key is exact in bf16 and doubles the raw means
    k2 = si.to_bf16_bits(oracle.bf16_to_f64(st.kp) * 2.0)
    st2 = oracle.Store(st.sp_k, st.sp_v, k2, st.vp, st.ids, st.offsets, st.mu * 2.0)
    np.testing.assert_allclose(oracle.cluster_drift(st2), d, rtol=0, atol=1e-13)
    # reversing the rows inside every cluster
    perm = np.concatenate([np.arange(st.offsets[c + 1] - 1, st.offsets[c] - 1, -1)
                           for c in range(st.C)]).astype(np.int64)
    st3 = oracle.Store(st.sp_k, st.sp_v, st.kp[perm].copy(), st.vp[perm].copy(), st.ids[perm].copy(),
                       st.offsets, st.mu)
    np.testing.assert_allclose(oracle.cluster_drift(st3), d, rtol=0, atol=1e-13)


def _prefilled(seed=3, unit=2, n=900, C=6, n_centers=14):
    K, V = si.keys_values(seed, unit, n, n_centers)
    st, _ = oracle.prefill_unit(K, V, C, oracle.stream_key(seed, unit, 0), iters=5)
    return st, K, V


def test_threshold_above_every_drift_changes_nothing():
    st, _, _ = _prefilled()
    d = oracle.cluster_drift(st)
    new, flags = oracle.split_drifted(st, float(d.max()) + 1e-9, 3, 2, room=10)
    assert flags.sum() == 0
    for name in ("kp", "vp", "ids", "offsets", "mu"):
        np.testing.assert_array_equal(getattr(new, name), getattr(st, name))


def test_split_layout_means_and_renumbering():
    st, K, V = _prefilled()
    new, flags = oracle.split_drifted(st, -1.0, 3, 2, room=100)
    sizes = np.diff(st.offsets)
    np.testing.assert_array_equal(flags, (sizes >= 2).astype(np.int32))
    assert new.C == st.C + int(flags.sum()) and new.m == st.m
    keys = oracle.bf16_to_f64(new.kp)
    for c in range(st.C):
        c2 = c + int(flags[:c].sum())
        lo, hi = st.offsets[c], st.offsets[c + 1]
        assert new.offsets[c2] == lo
        if not flags[c]:
            assert new.offsets[c2 + 1] == hi
            np.testing.assert_array_equal(new.mu[c2], st.mu[c])
            np.testing.assert_array_equal(new.kp[lo:hi], st.kp[lo:hi])
            continue
        mid = new.offsets[c2 + 1]
        assert lo <= mid <= hi and new.offsets[c2 + 2] == hi
        parent, a, b = st.ids[lo:hi], new.ids[lo:mid], new.ids[mid:hi]
        # a stable partition: each child keeps the parent's order, together every member once
        np.testing.assert_array_equal(np.sort(np.concatenate([a, b])), np.sort(parent))
        pos = {int(t): i for i, t in enumerate(parent)}
        assert all(np.diff([pos[int(t)] for t in a]) > 0) and all(np.diff([pos[int(t)] for t in b]) > 0)
        # rows travel with their ids
        np.testing.assert_array_equal(new.kp[lo:hi], K[new.ids[lo:hi]])
        np.testing.assert_array_equal(new.vp[lo:hi], V[new.ids[lo:hi]])
        # children's centroids are the raw means of their rows
        for j, (s, e) in enumerate(((lo, mid), (mid, hi))):
            if e > s:
                np.testing.assert_allclose(new.mu[c2 + j], keys[s:e].mean(axis=0), rtol=0, atol=1e-12)
    assert new.offsets[-1] == st.m


def test_split_recovers_two_tight_groups():
    seed, unit, s = 11, 3, 40
    key = oracle.split_key(seed, unit, 0, 0)
    i0, i1 = oracle.init_indices(s, 2, key)
    g = np.random.default_rng(7)
    lab = g.integers(0, 2, s)
    lab[i0], lab[i1] = 0, 1          # one initial member in each group
    dA, dB = g.standard_normal(D), g.standard_normal(D)
    dA, dB = dA / np.linalg.norm(dA), dB / np.linalg.norm(dB)
    rows = [8.0 * ((dA if l == 0 else dB) + 1e-3 * g.standard_normal(D)) for l in lab]
    tight = [8.0 * (dA + 1e-3 * g.standard_normal(D)) for _ in range(10)]
    st = _store([rows, tight])
    d = oracle.cluster_drift(st)
    assert d[0] > 0.1 and d[1] < 1e-4
    new, flags = oracle.split_drifted(st, 0.01, seed, unit, room=4)
    np.testing.assert_array_equal(flags, [1, 0])
    A, B = np.flatnonzero(lab == 0), np.flatnonzero(lab == 1)
    np.testing.assert_array_equal(new.offsets, [0, len(A), s, s + 10])
    np.testing.assert_array_equal(new.ids[:s], st.ids[np.concatenate([A, B])])
    np.testing.assert_array_equal(new.mu[2], st.mu[1])
    assert oracle.cluster_drift(new)[:2].max() < 1e-4


def test_room_keeps_the_lowest_indices():
    st, _, _ = _prefilled()
    new, flags = oracle.split_drifted(st, -1.0, 3, 2, room=2)
    eligible = np.flatnonzero(np.diff(st.offsets) >= 2)
    np.testing.assert_array_equal(np.flatnonzero(flags), eligible[:2])
    assert new.C == st.C + 2
    new0, flags0 = oracle.split_drifted(st, -1.0, 3, 2, room=0)
    assert flags0.sum() == 0 and new0.C == st.C


def test_singletons_and_empty_clusters_never_split():
    g = np.random.default_rng(1)
    rows = [g.standard_normal(D).astype(np.float32) for _ in range(5)]
    st = _store([[rows[0]], [], rows])
    new, flags = oracle.split_drifted(st, -1.0, 0, 0, room=8)
    np.testing.assert_array_equal(flags, [0, 0, 1])
    assert new.C == 4
    np.testing.assert_array_equal(new.offsets[:3], [0, 1, 1])


def test_split_keeps_every_token_and_padding_keeps_selection():
    st, _, _ = _prefilled()
    new, flags = oracle.split_drifted(st, float(np.median(oracle.cluster_drift(st))), 3, 2, room=100)
    assert 0 < flags.sum() < st.C
    q = si.queries(3, 0, 0, 1, 4)[0]
    full = oracle.select(new, q, new.n_total)
    np.testing.assert_array_equal(np.sort(full.ids), np.arange(new.n_total))
    padded = oracle.pad_clusters(new, new.C + 5)
    assert padded.C == new.C + 5 and padded.offsets[-1] == new.m
    for budget in (16, 40, 200, 517, new.n_total):
        a, b = oracle.select(new, q, budget), oracle.select(padded, q, budget)
        np.testing.assert_array_equal(np.sort(a.ids), np.sort(b.ids))
        assert len(a.ids) == min(budget, new.n_total)


def test_split_keys_differ_per_cluster_and_window():
    keys = {oracle.split_key(5, u, w, c) for u in range(3) for w in range(3) for c in range(50)}
    assert len(keys) == 3 * 3 * 50
    assert oracle.split_key(5, 1, 2, 0) != oracle.stream_key(5, 1, 2)


@pytest.mark.parametrize("iters", [1, 10])
def test_split_children_match_two_cluster_kmeans_on_the_rows(iters):
    st, _, _ = _prefilled()
    new, flags = oracle.split_drifted(st, -1.0, 3, 2, room=100, iters=iters)
    c = int(np.flatnonzero(flags)[1])
    lo, hi = st.offsets[c], st.offsets[c + 1]
    init = oracle.init_indices(hi - lo, 2, oracle.split_key(3, 2, 0, c))
    mu, offs, perm, _ = oracle.kmeans(st.kp[lo:hi], 2, iters, init)
    c2 = c + int(flags[:c].sum())
    np.testing.assert_array_equal(new.offsets[c2:c2 + 3], lo + offs)
    np.testing.assert_array_equal(new.ids[lo:hi], st.ids[lo + perm])
    np.testing.assert_array_equal(new.mu[c2:c2 + 2], mu)


def test_split_then_window_keeps_the_store_consistent():
    seed, unit, n, n_centers = 8, 1, 1200, 10
    K, V = si.keys_values(seed, unit, n, n_centers)
    st, _ = oracle.prefill_unit(K, V, 10, oracle.stream_key(seed, unit, 0), iters=5)
    st, flags = oracle.split_drifted(st, float(np.median(oracle.cluster_drift(st))), seed, unit, room=10)
    C1 = st.C
    assert C1 == 10 + int(flags.sum())
    ka, va = si.appended_tokens(seed, unit, oracle.WINDOW, n_centers)
    for j in range(oracle.WINDOW):
        st = oracle.append(st, ka[j], va[j])
    new, _ = oracle.recluster(st, seed, unit)
    assert new.C == C1 + 4 and new.windows == 1
    np.testing.assert_array_equal(new.offsets[:C1 + 1], st.offsets)
    np.testing.assert_array_equal(np.sort(np.concatenate([np.arange(16), new.ids])), np.arange(new.n_total))
    for c in range(new.C):  # ids ascend inside every cluster, the decode's tie rule
        seg = new.ids[new.offsets[c]:new.offsets[c + 1]]
        assert np.all(np.diff(seg) > 0)
    q = si.queries(seed, 0, 0, 1, 4)[0]
    for budget in (100, 600, new.n_total):
        assert len(oracle.select(new, q, budget).ids) == min(budget, new.n_total)
    # a second split pass draws its inits from the new window number
    again, flags2 = oracle.split_drifted(new, -1.0, seed, unit, room=2)
    c = int(np.flatnonzero(flags2)[0])
    lo, hi = new.offsets[c], new.offsets[c + 1]
    init = oracle.init_indices(hi - lo, 2, oracle.split_key(seed, unit, 1, c))
    mu, offs, perm, _ = oracle.kmeans(new.kp[lo:hi], 2, oracle.ITERS, init)
    np.testing.assert_array_equal(again.ids[lo:hi], new.ids[lo + perm])
