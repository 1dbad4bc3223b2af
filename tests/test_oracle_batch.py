"""Pins of the oracle's batched entry points against its single-unit functions.

``orc_prefill_batch`` and ``orc_select_attend_batch`` run many independent units (OpenMP over
units) and are what the CPU baseline and the benchmark's reference arm time. Each unit's
arithmetic must be exactly the single-unit function's, so the batched results must equal,
bit for bit, per unit:

* ``orc_prefill_unit`` (ClusterKV explainer section 3.2, prefill clustering) for the batched
  prefill;
* ``orc_select`` followed by ``orc_attend`` (section 3.3's select_clusters, then section
  3.1's attention) for the batched decode.

The units carry distinct data (their own keys, values, queries and centroid counts per
cluster), pending tokens, and G = 4 query heads, so a mistake in any per-unit stride (the
sink/pending rows, the C + 1 offsets, the G x 128 queries, the outputs) lands on another
unit's data and changes a result.
"""
import numpy as np

import oracle
import synth_inputs as si

D = 128
N_SINK = 16


def _units(U, n, C_, seed, iters=3):
    stores, Ks, Vs, keys = [], [], [], []
    for u in range(U):
        K, V = si.keys_values(seed, u, n, C_ + u)  # distinct mixtures per unit
        key = oracle.stream_key(seed, u, 0)
        st, _ = oracle.prefill_unit(K, V, C_, key, iters=iters)
        stores.append(st)
        Ks.append(K)
        Vs.append(V)
        keys.append(key)
    return stores, np.stack(Ks), np.stack(Vs), np.array(keys, dtype=np.uint64)


def test_prefill_batch_equals_prefill_unit():
    U, n, C_, seed, iters = 3, 420, 7, 11, 3
    stores, K, V, keys = _units(U, n, C_, seed, iters)
    kp, vp, ids, offsets, mu, a = oracle.prefill_batch(K, V, C_, keys, iters=iters)
    for u, st in enumerate(stores):
        _, a_ref = oracle.prefill_unit(K[u], V[u], C_, int(keys[u]), iters=iters)
        assert np.array_equal(kp[u], st.kp)
        assert np.array_equal(vp[u], st.vp)
        assert np.array_equal(ids[u], st.ids)
        assert np.array_equal(offsets[u], st.offsets)
        assert np.array_equal(mu[u], st.mu)  # bit-equal float64
        assert np.array_equal(a[u], a_ref)
    # the units really differ, so a stride mistake cannot pass by reading equal data
    assert not np.array_equal(mu[0], mu[1]) and not np.array_equal(offsets[0], offsets[2])


def _with_pending(st, u, seed, pending):
    for j in range(pending):
        k, v = si.keys_values(seed + 100 + j, u, 1, 4)
        st = oracle.append(st, k, v)
    return st


def test_select_attend_batch_equals_select_then_attend():
    U, n, C_, seed, G, pending, budget = 3, 520, 9, 23, 4, 5, 160
    stores, _, _, _ = _units(U, n, C_, seed)
    stores = [_with_pending(st, u, seed, pending) for u, st in enumerate(stores)]
    q = si.queries(seed, 0, 0, 1, U * G)[0].reshape(U, G, D)
    assert q.shape == (U, G, D)
    out, sel, cnt = oracle.select_attend_batch(
        np.stack([s.sp_k for s in stores]), np.stack([s.sp_v for s in stores]),
        np.stack([s.kp for s in stores]), np.stack([s.vp for s in stores]),
        np.stack([s.ids for s in stores]), np.stack([s.offsets for s in stores]),
        np.stack([s.mu for s in stores]), q, budget)
    for u, st in enumerate(stores):
        o_ref, s_ref = oracle.select_and_attend(st, q[u], budget)
        assert cnt[u] == len(s_ref.ids) == min(budget, st.n_total)
        assert np.array_equal(sel[u, : cnt[u]], s_ref.ids)
        assert np.array_equal(out[u], o_ref)  # bit-equal float64
        # the pending tokens are selected (ids n_sink + m ... n_total - 1)
        assert set(range(N_SINK + st.m, st.n_total)) <= set(s_ref.ids.tolist())
    assert not np.array_equal(out[0], out[1]) and not np.array_equal(out[1], out[2])


def test_select_attend_batch_budget_covers_everything():
    # budget >= n: every token of every unit, each unit attending only its own rows
    U, n, C_, seed, G = 2, 200, 5, 31, 4
    stores, _, _, _ = _units(U, n, C_, seed)
    stores = [_with_pending(st, u, seed, 3) for u, st in enumerate(stores)]
    q = si.queries(seed, 0, 1, 1, U * G)[0].reshape(U, G, D)
    budget = n + 3
    out, sel, cnt = oracle.select_attend_batch(
        np.stack([s.sp_k for s in stores]), np.stack([s.sp_v for s in stores]),
        np.stack([s.kp for s in stores]), np.stack([s.vp for s in stores]),
        np.stack([s.ids for s in stores]), np.stack([s.offsets for s in stores]),
        np.stack([s.mu for s in stores]), q, budget)
    for u, st in enumerate(stores):
        assert cnt[u] == st.n_total
        assert sorted(sel[u, : cnt[u]].tolist()) == list(range(st.n_total))
        assert np.array_equal(out[u], oracle.select_and_attend(st, q[u], budget)[0])
