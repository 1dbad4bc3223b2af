"""Pins of the oracle's incremental clustering (ClusterKV explainer, section 3.2: a new
clustering every 320 generated tokens).

Reading: cosine K-means with 4 clusters runs on the 320 pending tokens alone, keyed by
(seed, unit, window number). Existing clusters stay unchanged. The pins are equality
with a prefill-style K-means on the same 320 rows and the store invariants.
"""
import numpy as np

import oracle
import synth_inputs as si


def _store_with_window(seed=2, unit=5, n=1200, C=12, n_centers=10):
    K, V = si.keys_values(seed, unit, n, n_centers)
    st, _ = oracle.prefill_unit(K, V, C, oracle.stream_key(seed, unit, 0), iters=5)
    ka, va = si.appended_tokens(seed, unit, oracle.WINDOW, n_centers)
    for j in range(oracle.WINDOW):
        st = oracle.append(st, ka[j], va[j])
    return st, ka, va


def test_window_equals_standalone_kmeans_on_its_rows():
    seed, unit = 2, 5
    st, ka, va = _store_with_window(seed, unit)
    new, a = oracle.recluster(st, seed, unit)
    key = oracle.stream_key(seed, unit, 1)
    init = oracle.init_indices(oracle.WINDOW, 4, key)
    mu, offs, perm, a2 = oracle.kmeans(ka, 4, oracle.ITERS, init)
    np.testing.assert_array_equal(a, a2)
    np.testing.assert_array_equal(new.mu[-4:], mu)
    np.testing.assert_array_equal(new.offsets[-5:], st.m + offs)
    np.testing.assert_array_equal(new.kp[st.m:], ka[perm])
    np.testing.assert_array_equal(new.vp[st.m:], va[perm])
    np.testing.assert_array_equal(new.ids[st.m:], 16 + st.m + perm)


def test_window_leaves_old_clusters_and_keeps_every_token_once():
    st, ka, va = _store_with_window()
    new, _ = oracle.recluster(st, 2, 5)
    assert new.C == st.C + 4 and new.m == st.m + 320 and new.pending == 0 and new.windows == 1
    np.testing.assert_array_equal(new.mu[: st.C], st.mu)
    np.testing.assert_array_equal(new.offsets[: st.C + 1], st.offsets)
    np.testing.assert_array_equal(new.kp[: st.m], st.kp)
    all_ids = np.concatenate([np.arange(16), new.ids])
    np.testing.assert_array_equal(np.sort(all_ids), np.arange(new.n_total))
    # the next window uses a different stream key
    assert oracle.stream_key(2, 5, 1) != oracle.stream_key(2, 5, 2)


def test_selection_after_window_counts_new_clusters():
    st, _, _ = _store_with_window()
    new, _ = oracle.recluster(st, 2, 5)
    q = si.queries(2, 0, 0, 1, 4)[0]
    sel = oracle.select(new, q, 400)
    assert len(sel.ids) == 400
    sel_all = oracle.select(new, q, new.n_total)
    assert sorted(sel_all.ids.tolist()) == list(range(new.n_total))
