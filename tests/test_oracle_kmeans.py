"""Pins of the oracle's cosine K-means (ClusterKV explainer, section 3.2 and section 4.1).

They check exhaustive argmax optimality and the tie rule, direction-not-magnitude
assignment, exact recovery of a noiseless mixture, the empty-cluster rule, stable
cluster-contiguous layout invariants, and convergence to a fixed point.
"""
import numpy as np

import oracle
import synth_inputs as si

D = 128


def _bf16(x):
    return oracle.bf16_from_f64(np.asarray(x, dtype=np.float64))


def _dots(keys, mu_hat):
    return oracle.bf16_to_f64(keys) @ oracle.bf16_to_f64(mu_hat).T


def test_assign_single_cluster_is_all_zero():
    k, _ = si.keys_values(5, 0, 300, 8)
    mh = oracle.normalize(oracle.bf16_to_f64(k[:1]))
    assert np.all(oracle.assign(k, mh) == 0)


def test_assign_is_exhaustive_argmax_with_lower_index_ties():
    rng = np.random.default_rng(3)
    for C in (2, 3, 17):
        keys = _bf16(rng.integers(-3, 4, size=(200, D)))
        mh = _bf16(rng.integers(-2, 3, size=(C, D)))
        mh[C - 1] = mh[0]   # an exact duplicate: every tie must go to cluster 0
        a = oracle.assign(keys, mh)
        dots = _dots(keys, mh)
        best = dots.max(axis=1)
        assert np.all(dots[np.arange(200), a] == best)
        first = np.array([np.flatnonzero(row == row.max())[0] for row in dots])
        np.testing.assert_array_equal(a, first)
        assert not np.any(a == C - 1)


def test_assign_depends_on_direction_not_magnitude():
    # Cluster A has a huge-norm centroid, B a tiny one. The probe key is closer in angle to B.
    # The cosine rule (via normalised mu_hat) sends it to B. Using the raw centroid would send
    # it to A.
    a = np.zeros(D); a[0] = 1.0
    b = np.zeros(D); b[1] = 1.0
    keys = _bf16(np.stack([100 * a, 100 * a, 100 * a, b, b, b, 0.5 * a + 0.8 * b]))
    init = np.array([0, 3], np.int32)
    mu, offsets, perm, assign = oracle.kmeans(keys, 2, 3, init)
    assert assign.tolist() == [0, 0, 0, 1, 1, 1, 1]
    # the raw-mean reading of the centroid is kept for scoring: |mu_A| ~ 100, |mu_B| ~ 1
    assert abs(np.linalg.norm(mu[0]) - 100.0) < 1.0


def test_noiseless_mixture_is_recovered_exactly():
    rng = np.random.default_rng(4)
    n_centers, per = 6, 25
    cen = rng.standard_normal((n_centers, D))
    cen /= np.linalg.norm(cen, axis=1, keepdims=True)
    labels = rng.permutation(np.repeat(np.arange(n_centers), per))
    keys = _bf16(8.0 * cen[labels])                        # sigma = 0: identical keys per center
    init = np.array([np.flatnonzero(labels == j)[0] for j in range(n_centers)], np.int32)
    mu, offsets, perm, assign = oracle.kmeans(keys, n_centers, 10, init)
    np.testing.assert_array_equal(assign, labels)
    np.testing.assert_array_equal(np.diff(offsets), np.full(n_centers, per))
    kf = oracle.bf16_to_f64(keys)
    for j in range(n_centers):
        np.testing.assert_array_equal(mu[j], kf[init[j]])   # mean of identical rows is the row


def test_update_layout_invariants_and_means():
    k, _ = si.keys_values(6, 2, 2000, 32)
    rng = np.random.default_rng(5)
    C = 40
    a = rng.integers(0, C - 1, size=k.shape[0]).astype(np.int32)  # cluster C-1 stays empty
    mu_prev = rng.standard_normal((C, D))
    mu, offsets, perm = oracle.update(k, a, C, mu_prev)
    sizes = np.diff(offsets)
    assert offsets[0] == 0 and offsets[-1] == k.shape[0] and sizes.sum() == k.shape[0]
    np.testing.assert_array_equal(np.sort(perm), np.arange(k.shape[0]))
    kf = oracle.bf16_to_f64(k)
    for c in range(C):
        seg = perm[offsets[c]:offsets[c + 1]]
        assert np.all(a[seg] == c)
        assert np.all(np.diff(seg) > 0)                    # stable: ascending key index
        if len(seg):
            np.testing.assert_allclose(mu[c], kf[seg].mean(axis=0), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(mu[C - 1], mu_prev[C - 1])  # empty keeps previous


def test_tiny_kmeans_reaches_a_fixed_point():
    rng = np.random.default_rng(6)
    cen = np.eye(3, D)
    labels = np.array([0, 0, 0, 1, 1, 1, 2, 2, 2, 2])
    keys = _bf16(4.0 * (cen[labels] + 0.05 * rng.standard_normal((10, D))))
    init = oracle.init_indices(10, 3, 11)
    mu, offsets, perm, assign = oracle.kmeans(keys, 3, 30, init)
    again = oracle.assign(keys, oracle.normalize(mu))
    np.testing.assert_array_equal(again, assign)
    # the partition is the generating one, up to a relabelling
    assert len({(labels[i], assign[i]) for i in range(10)}) == 3


def test_prefill_unit_store_invariants_tiny_config():
    n, C = 2048, 32
    K, V = si.keys_values(0, 0, n, 32)
    st, a = oracle.prefill_unit(K, V, C, oracle.stream_key(0, 0, 0))
    assert st.m == n - 16 and st.C == C and st.pending == 0
    np.testing.assert_array_equal(np.sort(st.ids), np.arange(16, n))
    np.testing.assert_array_equal(st.sp_k, K[:16])
    np.testing.assert_array_equal(st.kp, K[st.ids])
    np.testing.assert_array_equal(st.vp, V[st.ids])
    kf = oracle.bf16_to_f64(K)
    for c in range(C):
        ids = st.ids[st.offsets[c]:st.offsets[c + 1]]
        assert np.all(np.diff(ids) > 0)
        assert np.all(a[ids - 16] == c)
        if len(ids):
            np.testing.assert_allclose(st.mu[c], kf[ids].mean(axis=0), atol=1e-12)
    # the run starts from the seeded init: C distinct non-sink tokens
    init = oracle.init_indices(n - 16, C, oracle.stream_key(0, 0, 0))
    assert len(set(init.tolist())) == C


def test_assign_gap_closed_forms_and_brute_force():
    """The cosine gap that the GPU parity tests use to accept near-tie disagreements:
    (k . mu_hat_best - k . mu_hat_other) / |k|, zero for the argmax itself, positive for
    a worse cluster, infinite for an index outside [0, C)."""
    e = np.zeros((3, 128), np.float32)
    e[0, 0], e[1, 1], e[2, 0] = 1.0, 1.0, 2.0
    mu_hat = si.to_bf16_bits(e[:2])                 # unit vectors along dims 0 and 1
    keys = si.to_bf16_bits(np.stack([e[0], 3.0 * e[1], e[2]]))
    gap = oracle.assign_gap(keys, mu_hat, np.array([1, 0, 1], np.int32))
    np.testing.assert_allclose(gap, [1.0, 1.0, 1.0], rtol=0, atol=1e-15)
    gap0 = oracle.assign_gap(keys, mu_hat, oracle.assign(keys, mu_hat))
    np.testing.assert_array_equal(gap0, [0.0, 0.0, 0.0])
    assert np.isinf(oracle.assign_gap(keys[:1], mu_hat, np.array([5], np.int32))[0])
    # brute force on a random case, every (key, other cluster) pair
    K, _ = si.keys_values(6, 0, 300, 7)
    mu = oracle.bf16_to_f64(K[:9])
    mh = oracle.normalize(mu)
    k = oracle.bf16_to_f64(K)
    s = k @ oracle.bf16_to_f64(mh).T
    for c in range(9):
        other = np.full(300, c, np.int32)
        want = (s.max(axis=1) - s[:, c]) / np.linalg.norm(k, axis=1)
        got = oracle.assign_gap(K, mh, other)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
        assert np.all(got >= 0)
