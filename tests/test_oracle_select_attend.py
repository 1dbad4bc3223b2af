"""Pins of the oracle's selection (ClusterKV explainer section 3.3) and attention (section 3.1).

The pins are:
* a hand-worked example in ``golden/select_hand_example.json``;
* invariants: the selected count is min(budget, n); the whole-selected clusters
  outrank the cut cluster, which outranks the rest; the partial tokens outrank the
  cut cluster's other tokens; an exact prefix budget gives no partial;
* dense attention from ``torch.nn.functional.scaled_dot_product_attention`` (float64) when
  budget >= n;
* a single selected row gives that row's value;
* shifting all keys by a constant vector leaves the output unchanged;
* the Jensen bound of the centroid relation in section 3.1 and its O(sigma^2) tightness.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

D = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return oracle.bf16_from_f64(np.asarray(x, dtype=np.float64))


def _row(v2):
    r = np.zeros(D)
    r[: len(v2)] = v2
    return r


def _hand_store():
    ex = json.load(open(os.path.join(GOLDEN, "select_hand_example.json")))
    s = ex["store"]
    kp, ids, offs, mu = [], [], [0], []
    for cl in s["clusters"]:
        kp += [_row(k) for k in cl["keys"]]
        ids += cl["ids"]
        offs.append(offs[-1] + len(cl["ids"]))
        mu.append(_row(cl["mu"]))
    kp = _bf16(np.stack(kp))
    sp_k = _bf16(np.stack([_row(k) for k in s["sink_keys"] + s["pending_keys"]]))
    sp_v = _bf16(np.stack([_row(v) for v in s["sink_values"] + s["pending_values"]]))
    st = oracle.Store(sp_k, sp_v, kp, kp.copy(), np.array(ids, np.int32),
                      np.array(offs, np.int32), np.stack(mu), n_sink=s["n_sink"])
    q = _bf16(np.stack([_row(v) for v in ex["queries"]]))
    return ex, st, q


def test_hand_example_cases():
    ex, st, q = _hand_store()
    assert st.pending == 1 and st.m == 12
    for case in ex["cases"]:
        sel = oracle.select(st, q, case["budget"])
        assert sel.ids.tolist() == case["selected"], case
        assert (sel.cut, sel.r, sel.n_whole) == (case["cut"], case["r"], case["n_whole"]), case
    for case in ex["error_cases"]:
        with pytest.raises(ValueError):
            oracle.select(st, q, case["budget"])


def test_hand_example_attention_closed_form():
    ex, st, q = _hand_store()
    o, sel = oracle.select_and_attend(st, q, 3)
    a = 1.0 / math.sqrt(128.0)
    ea = math.exp(a)
    want0 = [(1 + ea) / (1 + 2 * ea), 2 * ea / (1 + 2 * ea)]
    want1 = [2 / (2 + ea), (ea + 1) / (2 + ea)]
    np.testing.assert_allclose(o[0, :2], want0, rtol=1e-14)
    np.testing.assert_allclose(o[1, :2], want1, rtol=1e-14)
    assert np.all(o[:, 2:] == 0.0)


def _random_store(seed=0, n=3000, C=40, n_centers=30, pending=5):
    K, V = si.keys_values(seed, 1, n, n_centers)
    st, _ = oracle.prefill_unit(K, V, C, oracle.stream_key(seed, 1, 0), iters=4)
    ka, va = si.appended_tokens(seed, 1, pending, n_centers)
    for j in range(pending):
        st = oracle.append(st, ka[j], va[j])
    return st


@pytest.mark.parametrize("budget", [21, 22, 64, 256, 1000, 2999, 3005, 3006, 5000])
def test_selection_invariants(budget):
    st = _random_store()
    q = si.queries(0, 0, 0, 1, 4)[0]
    sel = oracle.select(st, q, budget)
    n_total = st.n_total
    assert len(sel.ids) == min(budget, n_total)
    assert len(set(sel.ids.tolist())) == len(sel.ids)
    assert set(range(16)) | set(range(16 + st.m, n_total)) <= set(sel.ids.tolist())
    qbar = oracle.bf16_to_f64(q).sum(axis=0)
    scores = st.mu @ qbar
    np.testing.assert_allclose(sel.scores, scores, rtol=1e-12, atol=1e-9)
    chosen = set(sel.ids.tolist())
    whole = [c for c in range(st.C)
             if set(st.ids[st.offsets[c]:st.offsets[c + 1]].tolist()) <= chosen
             and st.offsets[c + 1] > st.offsets[c]]
    if sel.cut < 0:
        assert len(whole) == sum(1 for c in range(st.C) if st.offsets[c + 1] > st.offsets[c])
        return
    # rank order: every whole cluster outranks the cut, which outranks the untouched ones
    def key(c):
        return (-scores[c], c)
    untouched = [c for c in range(st.C) if c not in whole and c != sel.cut
                 and st.offsets[c + 1] > st.offsets[c]]
    assert all(key(c) < key(sel.cut) for c in whole)
    assert all(key(sel.cut) < key(c) for c in untouched)
    # partial tokens are the top-r of the cut cluster by qbar . k (ties -> lower id)
    lo, hi = st.offsets[sel.cut], st.offsets[sel.cut + 1]
    t = oracle.bf16_to_f64(st.kp[lo:hi]) @ qbar
    order = sorted(range(hi - lo), key=lambda j: (-t[j], st.ids[lo + j]))
    want = set(st.ids[lo + np.array(order[:sel.r], dtype=int)].tolist()) if sel.r else set()
    got = chosen & set(st.ids[lo:hi].tolist())
    assert got == want
    assert 0 <= sel.r < hi - lo


def test_exact_prefix_budget_takes_no_partial():
    st = _random_store()
    q = si.queries(0, 0, 0, 1, 4)[0]
    sel = oracle.select(st, q, 10_000)  # everything, to learn the visit order
    qbar = oracle.bf16_to_f64(q).sum(axis=0)
    order = sorted(range(st.C), key=lambda c: (-(st.mu[c] @ qbar), c))
    sizes = np.diff(st.offsets)
    for k in (1, 3, 7):
        budget = 16 + st.pending + int(sizes[order[:k]].sum())
        sel = oracle.select(st, q, budget)
        assert sel.r == 0 and sel.n_whole >= k and len(sel.ids) == budget


def test_full_budget_equals_dense_attention_from_torch():
    n = 1500
    K, V = si.keys_values(9, 3, n, 20)
    st, _ = oracle.prefill_unit(K, V, 24, oracle.stream_key(9, 3, 0), iters=3)
    q = si.queries(9, 0, 0, 1, 4)[0]
    o, sel = oracle.select_and_attend(st, q, n + 50)
    assert len(sel.ids) == n
    Kt = torch.from_numpy(oracle.bf16_to_f64(K))[None, None].expand(1, 4, n, D)
    Vt = torch.from_numpy(oracle.bf16_to_f64(V))[None, None].expand(1, 4, n, D)
    qt = torch.from_numpy(oracle.bf16_to_f64(q))[None, :, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[0, :, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.dense_attention(K, V, q), ref, rtol=0, atol=1e-12)


def test_single_row_gives_its_value():
    K, V = si.keys_values(1, 0, 200, 4)
    st, _ = oracle.prefill_unit(K, V, 4, 5, iters=2, n_sink=1)
    q = si.queries(1, 0, 0, 1, 4)[0]
    o, sel = oracle.select_and_attend(st, q, 1)
    assert sel.ids.tolist() == [0]
    np.testing.assert_array_equal(o, np.tile(oracle.bf16_to_f64(V[0]), (4, 1)))


def test_constant_key_shift_leaves_attention_unchanged():
    rng = np.random.default_rng(8)
    n = 400
    K = _bf16(rng.integers(-8, 9, size=(n, D)))
    V = _bf16(rng.standard_normal((n, D)))
    w = rng.integers(-4, 5, size=D)
    K2 = _bf16(oracle.bf16_to_f64(K) + w)   # small integers: exact in bf16
    q = _bf16(rng.integers(-1, 2, size=(4, D)) / 8.0)
    np.testing.assert_allclose(oracle.dense_attention(K2, V, q), oracle.dense_attention(K, V, q),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("sigma", [0.02, 0.04, 0.08])
def test_centroid_relation_jensen_and_tightness(sigma):
    # For a cluster with mean mu: sum_i exp(q.k_i) >= n exp(q.mu) (Jensen), and for tight
    # clusters the ratio is 1 + Var(q.k)/2 + O(sigma^3).
    rng = np.random.default_rng(10)
    c = rng.standard_normal(D)
    c /= np.linalg.norm(c)
    keys = _bf16(c + sigma * rng.standard_normal((400, D)))
    mu, _, _ = oracle.update(keys, np.zeros(400, np.int32), 1, np.zeros((1, D)))
    q = rng.standard_normal(D) / math.sqrt(D)
    t = oracle.bf16_to_f64(keys) @ q
    ratio = np.exp(t).sum() / (400 * math.exp(mu[0] @ q))
    assert ratio >= 1.0
    np.testing.assert_allclose(ratio - 1.0, 0.5 * t.var(), rtol=0.05)
