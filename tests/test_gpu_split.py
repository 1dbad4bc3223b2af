"""GPU parity of split_drifted_clusters against the oracle (ClusterKV explainer, section 3.2,
decode phase: a cluster whose mean intra-cluster distance passes a threshold is split).

Staged: the oracle splits the store the GPU exported just before the call (fp32 centroids),
so both sides start from identical inputs.
* drift: within 2e-5 of the oracle's fp64 value; the threshold is placed in a gap of the
  oracle's drift values, so the split decisions are compared exactly;
* every split cluster: the halves' sizes, row order and token ids exactly equal to the
  oracle's 2-means, except where the oracle's own trajectory passes a cosine near-tie
  (gap < 1e-4), in which case the GPU's halves must still be a stable partition whose
  centroids are the means of their rows; the halves' centroids within 1e-3;
* every other cluster: rows and centroid unchanged, at its shifted index; padding clusters
  empty with a zero centroid;
* decode on the split store matches the oracle;
* the layer's cluster count grows by exactly min(max_splits, room), with no read-back, so the
  call can be captured in a CUDA graph (checked by capturing one and replaying it).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_helpers import COS_GAP_TOL, MU_TOL, check_decode_unit, store_from_export, to_dev

pytestmark = pytest.mark.gpu

DRIFT_TOL = 2e-5


def _ctx(B, Hkv, n, C, n_centers, seed, max_clusters, G=4, window=320):
    import recallable_kv_cache_cosine_b200 as ckv
    K = np.empty((B, Hkv, n, 128), np.uint16)
    V = np.empty_like(K)
    for b in range(B):
        for h in range(Hkv):
            K[b, h], V[b, h] = si.keys_values(seed, si.unit_id(0, b, h, B, Hkv), n, n_centers)
    ctx = ckv.ClusterKV(1, B, Hkv, Hkv * G, capacity=n + 2 * window, max_clusters=max_clusters,
                        seed=seed, window=window)
    ctx.cluster_prefill(0, to_dev(K), to_dev(V), C)
    torch.cuda.synchronize()
    return ctx, K, V


def _split(ctx, layer, tau, max_splits, drift=None):
    """split_drifted_clusters with its per-unit split counts read back as a list."""
    U = ctx.cfg.batch * ctx.cfg.n_kv_heads
    cnt = torch.full((U,), -1, device="cuda", dtype=torch.int32)
    ctx.split_drifted_clusters(layer, tau, max_splits, drift, cnt)
    return cnt.tolist()


def _stores(ctx, B, Hkv, windows=0):
    return [store_from_export(ctx.export_unit(0, b, h), windows=windows)
            for b in range(B) for h in range(Hkv)]


def _threshold_in_gap(drifts, q=0.5):
    """A threshold between two neighbouring drift values near quantile q whose gap is wide
    enough that fp32 and fp64 drifts fall on the same side."""
    v = np.unique(np.concatenate(drifts))
    k0 = int(q * (len(v) - 1))
    for k in sorted(range(len(v) - 1), key=lambda k: abs(k - k0)):
        if v[k + 1] - v[k] > 10 * DRIFT_TOL:
            return float(0.5 * (v[k] + v[k + 1]))
    raise AssertionError("no gap in the drift values")


def _trajectory_min_gap(rows_u16, init, iters):
    """Smallest cosine gap between the two halves over the oracle's 2-means trajectory."""
    mu = oracle.bf16_to_f64(rows_u16[init])
    kn = np.linalg.norm(oracle.bf16_to_f64(rows_u16), axis=1)
    g = math.inf
    for _ in range(iters):
        mh = oracle.normalize(mu)
        s = oracle.bf16_to_f64(rows_u16) @ oracle.bf16_to_f64(mh).T
        g = min(g, float(np.min(np.abs(s[:, 0] - s[:, 1]) / np.maximum(kn, 1e-30))))
        a = oracle.assign(rows_u16, mh)
        mu, _, _ = oracle.update(rows_u16, a, 2, mu)
    return g


def _check_split_unit(pre, post, want, flags, seed, unit, iters, stats):
    """pre: GPU store before the split; post: GPU store after it (padded); want: the oracle's
    split of `pre` (padded to post.C)."""
    C = pre.C
    assert post.offsets[0] == 0
    n_split = int(flags.sum())
    for c in range(C):
        c2 = c + int(flags[:c].sum())
        lo, hi = pre.offsets[c], pre.offsets[c + 1]
        assert post.offsets[c2] == lo
        if not flags[c]:
            assert post.offsets[c2 + 1] == hi
            np.testing.assert_array_equal(post.mu[c2], pre.mu[c])
            np.testing.assert_array_equal(post.ids[lo:hi], pre.ids[lo:hi])
            np.testing.assert_array_equal(post.kp[lo:hi], pre.kp[lo:hi])
            continue
        stats["split"] = stats.get("split", 0) + 1
        same = (post.offsets[c2 + 1] == want.offsets[c2 + 1]
                and np.array_equal(post.ids[lo:hi], want.ids[lo:hi]))
        if same:
            np.testing.assert_array_equal(post.kp[lo:hi], want.kp[lo:hi])
            np.testing.assert_array_equal(post.vp[lo:hi], want.vp[lo:hi])
            err = float(np.abs(post.mu[c2:c2 + 2] - want.mu[c2:c2 + 2]).max())
            assert err <= MU_TOL, f"half centroids differ by {err}"
            continue
        stats["near_tie"] = stats.get("near_tie", 0) + 1
        init = oracle.init_indices(hi - lo, 2, oracle.split_key(seed, unit, pre.windows, c))
        gap = _trajectory_min_gap(pre.kp[lo:hi], init, iters)
        assert gap < COS_GAP_TOL, f"cluster {c}: halves differ without a near-tie (gap {gap})"
        mid = post.offsets[c2 + 1]
        assert lo <= mid <= hi
        pos = {int(t): i for i, t in enumerate(pre.ids[lo:hi])}
        for s_, e_ in ((lo, mid), (mid, hi)):
            order = [pos[int(t)] for t in post.ids[s_:e_]]
            assert all(np.diff(order) > 0)
        np.testing.assert_array_equal(np.sort(post.ids[lo:hi]), np.sort(pre.ids[lo:hi]))
        keys = oracle.bf16_to_f64(post.kp)
        for j, (s_, e_) in enumerate(((lo, mid), (mid, hi))):
            if e_ > s_:
                assert np.abs(post.mu[c2 + j] - keys[s_:e_].mean(axis=0)).max() <= MU_TOL
    # padding: empty clusters with a zero centroid
    for c2 in range(C + n_split, post.C):
        assert post.offsets[c2] == post.m and post.offsets[c2 + 1] == post.m
        assert not post.mu[c2].any()
    assert post.offsets[post.C] == post.m


def _decode_all(ctx, B, Hkv, G, budget, seed, windows, stats):
    q = np.stack([si.queries(seed, 0, b, 1, Hkv * G)[0] for b in range(B)])  # [B, Hq, 128]
    out = torch.empty(B, Hkv * G, 128, device="cuda", dtype=torch.float32)
    sel = torch.empty(B, Hkv, budget, device="cuda", dtype=torch.int32)
    cnt = torch.empty(B, Hkv, device="cuda", dtype=torch.int32)
    ctx.select_and_attend(0, to_dev(q), budget, out, sel, cnt)
    torch.cuda.synchronize()
    ctx.check_device_error()
    for b in range(B):
        for h in range(Hkv):
            st = store_from_export(ctx.export_unit(0, b, h), windows=windows)
            check_decode_unit(st, q[b, h * G:(h + 1) * G], budget, out[b, h * G:(h + 1) * G].cpu().numpy(),
                              sel[b, h].cpu().numpy(), int(cnt[b, h]), stats)


@pytest.mark.parametrize("B,Hkv,n,C,n_centers,q", [(1, 2, 3000, 12, 30, 0.5),
                                                   (2, 2, 4096, 40, 24, 0.3)])
def test_split_matches_oracle(B, Hkv, n, C, n_centers, q):
    seed, G, iters = 9, 4, 10
    U = B * Hkv
    ctx, _, _ = _ctx(B, Hkv, n, C, n_centers, seed, max_clusters=2 * C + 8)
    pre = _stores(ctx, B, Hkv)
    drifts = [oracle.cluster_drift(st) for st in pre]
    tau = _threshold_in_gap(drifts, q)
    drift_gpu = torch.full((U, C), -7.0, device="cuda", dtype=torch.float32)
    room = (2 * C + 8) - C
    splits = _split(ctx, 0, tau, room, drift_gpu)
    ctx.check_device_error()
    d = drift_gpu.cpu().numpy()
    for u in range(U):
        assert np.abs(d[u] - drifts[u]).max() <= DRIFT_TOL
    info = ctx.layer_info(0)
    assert info.C == C + room and info.m == n - 16
    post = _stores(ctx, B, Hkv)
    stats = {}
    for u in range(U):
        want, flags = oracle.split_drifted(pre[u], tau, seed, u, room=2 * C + 8 - C, iters=iters)
        assert splits[u] == int(flags.sum())
        want = oracle.pad_clusters(want, info.C)
        assert post[u].C == info.C
        _check_split_unit(pre[u], post[u], want, flags, seed, u, iters, stats)
    assert 0 < sum(splits) < U * C
    assert stats.get("near_tie", 0) <= max(1, stats["split"] // 10), stats
    _decode_all(ctx, B, Hkv, G, 512, seed, 0, {})


def test_split_large_clusters_through_global_memory():
    # 2 clusters of ~1500 rows: every segment is above the shared-memory staging size
    B, Hkv, n, C, seed, iters = 1, 2, 3000, 2, 4, 10
    ctx, _, _ = _ctx(B, Hkv, n, C, 8, seed, max_clusters=8)
    pre = _stores(ctx, B, Hkv)
    assert all(np.diff(st.offsets).max() > 384 for st in pre)
    splits = _split(ctx, 0, -math.inf, 6)
    ctx.check_device_error()
    assert splits == [2, 2] and ctx.layer_info(0).C == 8  # 2 + 6: two splits, two padding
    post = _stores(ctx, B, Hkv)
    stats = {}
    for u in range(B * Hkv):
        want, flags = oracle.split_drifted(pre[u], -math.inf, seed, u, room=6, iters=iters)
        _check_split_unit(pre[u], post[u], oracle.pad_clusters(want, 8), flags, seed, u, iters, stats)
    _decode_all(ctx, B, Hkv, 4, 700, seed, 0, {})


def test_split_room_cap_padding_and_no_op():
    B, Hkv, n, C, seed = 1, 2, 2048, 16, 3
    ctx, _, _ = _ctx(B, Hkv, n, C, 20, seed, max_clusters=C + 5)
    pre = _stores(ctx, B, Hkv)
    # +inf with max_splits 0 only measures: every byte of the store stays as it was
    assert _split(ctx, 0, math.inf, 0) == [0, 0]
    assert ctx.layer_info(0).C == C
    same = _stores(ctx, B, Hkv)
    for a, b in zip(pre, same):
        for name in ("kp", "vp", "ids", "offsets", "mu"):
            np.testing.assert_array_equal(getattr(a, name), getattr(b, name))
    # -inf: every cluster of 2+ rows qualifies; max_splits 3 keeps the lowest three
    splits = _split(ctx, 0, -math.inf, 3)
    assert splits == [3, 3] and ctx.layer_info(0).C == C + 3
    post = _stores(ctx, B, Hkv)
    stats = {}
    for u in range(2):
        want, flags = oracle.split_drifted(pre[u], -math.inf, seed, u, room=3)
        np.testing.assert_array_equal(np.flatnonzero(flags), np.flatnonzero(np.diff(pre[u].offsets) >= 2)[:3])
        _check_split_unit(pre[u], post[u], want, flags, seed, u, 10, stats)
    # +inf with max_splits 2: nothing splits, the count still grows by 2 (empty padding)
    assert _split(ctx, 0, math.inf, 2) == [0, 0]
    assert ctx.layer_info(0).C == C + 5
    padded = _stores(ctx, B, Hkv)
    for a, b in zip(post, padded):
        np.testing.assert_array_equal(b.offsets[: a.C + 1], a.offsets)
        np.testing.assert_array_equal(b.mu[: a.C], a.mu)
        assert np.all(b.offsets[a.C:] == b.m) and not b.mu[a.C:].any()
    # no room left: nothing splits and the count stays
    assert _split(ctx, 0, -math.inf, 4) == [0, 0]
    assert ctx.layer_info(0).C == C + 5
    ctx.check_device_error()
    _decode_all(ctx, B, Hkv, 4, 500, seed, 0, {})


def test_split_is_captured_in_a_cuda_graph():
    """The split needs no read-back, so it can be recorded in a CUDA graph with a decode step
    after it; one replay gives the oracle's split and decode."""
    B, Hkv, n, C, seed, G = 1, 2, 3000, 12, 8, 4
    ctx, _, _ = _ctx(B, Hkv, n, C, 30, seed, max_clusters=C + 16)
    ctx.split_drifted_clusters(0, math.inf, 0)  # first call: allocates the scratch
    torch.cuda.synchronize()
    pre = _stores(ctx, B, Hkv)
    tau = _threshold_in_gap([oracle.cluster_drift(st) for st in pre], 0.5)
    budget = 400
    q = np.stack([si.queries(seed, 0, b, 1, Hkv * G)[0] for b in range(B)])
    qd = to_dev(q)
    out = torch.empty(B, Hkv * G, 128, device="cuda", dtype=torch.float32)
    sel = torch.empty(B, Hkv, budget, device="cuda", dtype=torch.int32)
    cnt = torch.empty(B, Hkv, device="cuda", dtype=torch.int32)
    splits = torch.zeros(B * Hkv, device="cuda", dtype=torch.int32)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
        ctx.split_drifted_clusters(0, tau, 8, splits=splits, stream=s)
        ctx.select_and_attend(0, qd, budget, out, sel, cnt, stream=s)
    assert ctx.layer_info(0).C == C + 8  # the host count moved at capture
    g.replay()
    torch.cuda.synchronize()
    ctx.check_device_error()
    post = _stores(ctx, B, Hkv)
    stats = {}
    for u in range(B * Hkv):
        want, flags = oracle.split_drifted(pre[u], tau, seed, u, room=8)
        assert int(splits[u]) == int(flags.sum())
        _check_split_unit(pre[u], post[u], oracle.pad_clusters(want, C + 8), flags, seed, u, 10, stats)
        check_decode_unit(post[u], q[0, u * G:(u + 1) * G], budget, out[0, u * G:(u + 1) * G].cpu().numpy(),
                          sel[0, u].cpu().numpy(), int(cnt[0, u]), stats)
    del g


def test_split_then_window_recluster_and_decode():
    B, Hkv, n, C, seed, W = 1, 2, 2048, 16, 6, 320
    ctx, _, _ = _ctx(B, Hkv, n, C, 20, seed, max_clusters=48)
    pre = _stores(ctx, B, Hkv)
    tau = _threshold_in_gap([oracle.cluster_drift(st) for st in pre], 0.6)
    ctx.split_drifted_clusters(0, tau, 8)
    C1 = C + 8
    AK = np.empty((B, Hkv, W, 128), np.uint16)
    AV = np.empty_like(AK)
    for h in range(Hkv):
        AK[0, h], AV[0, h] = si.appended_tokens(seed, si.unit_id(0, 0, h, B, Hkv), W, 20)
    dk, dv = to_dev(AK), to_dev(AV)
    for j in range(W):
        ctx.append_kv(0, dk[:, :, j].contiguous(), dv[:, :, j].contiguous())
    mid = _stores(ctx, B, Hkv)
    ctx.recluster_increment(0)
    torch.cuda.synchronize()
    ctx.check_device_error()
    info = ctx.layer_info(0)
    assert (info.C, info.windows, info.pending) == (C1 + 4, 1, 0)
    post = _stores(ctx, B, Hkv, windows=1)
    for u in range(2):
        want, _ = oracle.recluster(mid[u], seed, u)
        np.testing.assert_array_equal(post[u].offsets[:C1 + 1], mid[u].offsets)
        np.testing.assert_array_equal(post[u].mu[:C1], mid[u].mu)
        assert post[u].offsets[-1] == want.offsets[-1]
    _decode_all(ctx, B, Hkv, 4, 600, seed, 1, {})
    # a second split pass uses the window number in its init key
    pre2 = _stores(ctx, B, Hkv, windows=1)
    tau2 = _threshold_in_gap([oracle.cluster_drift(st) for st in pre2], 0.5)
    room2 = 48 - pre2[0].C
    splits2 = _split(ctx, 0, tau2, room2)
    post2 = _stores(ctx, B, Hkv, windows=1)
    assert post2[0].C == 48
    stats = {}
    for u in range(2):
        want, flags = oracle.split_drifted(pre2[u], tau2, seed, u, room=room2)
        assert splits2[u] == int(flags.sum())
        want = oracle.pad_clusters(want, post2[u].C)
        _check_split_unit(pre2[u], post2[u], want, flags, seed, u, 10, stats)
    _decode_all(ctx, B, Hkv, 4, 600, seed, 1, {})


def test_split_argument_and_state_errors():
    import recallable_kv_cache_cosine_b200 as ckv
    ctx = ckv.ClusterKV(2, 1, 2, 8, capacity=2048 + 640, max_clusters=24, seed=1)
    with pytest.raises(ckv.CkvError) as e:
        ctx.split_drifted_clusters(0, 0.5, 4)   # layer not prefilled
    assert e.value.code == ckv.CKV_ESTATE
    K = to_dev(np.stack([np.stack([si.keys_values(1, h, 2048, 10)[0] for h in range(2)])]))
    ctx.cluster_prefill(0, K, K, 12)
    with pytest.raises(ckv.CkvError) as e:
        ctx.split_drifted_clusters(0, float("nan"), 4)
    assert e.value.code == ckv.CKV_EINVAL
    with pytest.raises(ckv.CkvError) as e:
        ctx.split_drifted_clusters(0, 0.5, -1)
    assert e.value.code == ckv.CKV_EINVAL
    with pytest.raises(ckv.CkvError) as e:
        ctx.split_drifted_clusters(5, 0.5, 4)
    assert e.value.code == ckv.CKV_EINVAL
    assert ctx.layer_info(0).C == 12
    ctx.check_device_error()
