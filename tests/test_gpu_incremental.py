"""GPU parity of append_kv + recluster_increment against the oracle (ClusterKV explainer,
section 3.2: incremental clustering every 320 new tokens).

recluster_increment_traced records the window's centroids before every iteration and
after the last, plus every iteration's assignment, so each stage is checked on
identical inputs:
* init: the centroids are the window keys chosen by the oracle's init on key
  (seed, unit, window number);
* assign: equal to the oracle's argmax on the same centroids, except cosine gaps < 1e-4;
* update: the next centroids within 1e-3 of the oracle's means of that assignment;
* append: the store gains the window's rows in cluster-major order with their token ids,
  4 more clusters, and unchanged old clusters. Decode before, during and after the window
  matches the oracle on the GPU's store.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_helpers import MU_TOL, check_assign, check_decode_unit, store_from_export, to_dev, to_u16

pytestmark = pytest.mark.gpu


def _decode_check(ctx, q, budget, B, Hkv, G, stats, windows):
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


@pytest.mark.parametrize("B,Hkv,n,C,n_centers", [(1, 2, 2048, 32, 32), (2, 1, 3000, 40, 30)])
def test_append_and_recluster_stage_by_stage(B, Hkv, n, C, n_centers):
    import recallable_kv_cache_cosine_b200 as ckv
    seed, G, W, iters = 5, 4, 320, 10
    U = B * Hkv
    K = np.empty((B, Hkv, n, 128), np.uint16)
    V = np.empty_like(K)
    AK = np.empty((B, Hkv, 2 * W, 128), np.uint16)
    AV = np.empty_like(AK)
    for b in range(B):
        for h in range(Hkv):
            u = si.unit_id(0, b, h, B, Hkv)
            K[b, h], V[b, h] = si.keys_values(seed, u, n, n_centers)
            AK[b, h], AV[b, h] = si.appended_tokens(seed, u, 2 * W, n_centers)
    ctx = ckv.ClusterKV(1, B, Hkv, Hkv * G, capacity=n + 2 * W, max_clusters=C + 8, seed=seed)
    ctx.cluster_prefill(0, to_dev(K), to_dev(V), C)
    stats = {}
    qs = np.stack([si.queries(seed, 0, b, 8, Hkv * G) for b in range(B)], axis=1)  # [8, B, Hq, 128]
    for window in range(2):
        m_old = n - 16 + window * W
        C_old = C + 4 * window
        for t in range(W):
            j = window * W + t
            ctx.append_kv(0, to_dev(np.ascontiguousarray(AK[:, :, j])), to_dev(np.ascontiguousarray(AV[:, :, j])))
            if t in (0, 17, W - 1):
                _decode_check(ctx, qs[t % 8], 512, B, Hkv, G, stats, window)
        info = ctx.layer_info(0)
        assert (info.pending, info.m, info.C) == (W, m_old, C_old)
        mu_tr = torch.empty(U, iters + 1, 4, 128, device="cuda", dtype=torch.float32)
        as_tr = torch.empty(U, iters, W, device="cuda", dtype=torch.int32)
        ctx.recluster_increment(0, mu_trace=mu_tr, assign_trace=as_tr)
        torch.cuda.synchronize()
        ctx.check_device_error()
        info = ctx.layer_info(0)
        assert (info.pending, info.m, info.C, info.windows) == (0, m_old + W, C_old + 4, window + 1)
        mu_tr, as_tr = mu_tr.cpu().numpy(), as_tr.cpu().numpy()
        astats = {}
        for b in range(B):
            for h in range(Hkv):
                u = si.unit_id(0, b, h, B, Hkv)
                wk = np.ascontiguousarray(AK[b, h, window * W:(window + 1) * W])
                wv = np.ascontiguousarray(AV[b, h, window * W:(window + 1) * W])
                mt, at = mu_tr[b * Hkv + h], as_tr[b * Hkv + h]
                init = oracle.init_indices(W, 4, oracle.stream_key(seed, u, window + 1))
                np.testing.assert_array_equal(mt[0], oracle.bf16_to_f64(wk[init]).astype(np.float32))
                for it in range(iters):
                    check_assign(wk, oracle.normalize(mt[it].astype(np.float64)), at[it], astats)
                    w_mu, w_off, w_perm = oracle.update(wk, at[it], 4, mt[it].astype(np.float64))
                    assert np.abs(mt[it + 1] - w_mu).max() <= MU_TOL
                ex = ctx.export_unit(0, b, h)
                st = store_from_export(ex, windows=window + 1)
                np.testing.assert_array_equal(st.offsets[C_old:], m_old + w_off)
                np.testing.assert_array_equal(st.ids[m_old:], 16 + m_old + w_perm)
                np.testing.assert_array_equal(st.kp[m_old:], wk[w_perm])
                np.testing.assert_array_equal(st.vp[m_old:], wv[w_perm])
                np.testing.assert_array_equal(ex["mu"].numpy()[C_old:], mt[iters])
                np.testing.assert_array_equal(np.sort(np.concatenate([np.arange(16), st.ids])),
                                              np.arange(n + (window + 1) * W))
        assert astats["near_tie"] <= 2
        for budget in (64, 700, n + 2 * W):
            _decode_check(ctx, qs[budget % 8], budget, B, Hkv, G, stats, window + 1)
    assert stats["near_tie"] <= 1
    print("decode stats", stats)


def test_window_full_and_order_errors():
    import recallable_kv_cache_cosine_b200 as ckv
    n, C = 600, 8
    K, V = si.keys_values(9, 0, n, 8)
    ctx = ckv.ClusterKV(1, 1, 1, 4, capacity=n + 320, max_clusters=C + 4, seed=9)
    with pytest.raises(ckv.CkvError) as e:
        ctx.recluster_increment(0)
    assert e.value.code == ckv.CKV_ESTATE
    ctx.cluster_prefill(0, to_dev(K[None, None]), to_dev(V[None, None]), C)
    with pytest.raises(ckv.CkvError) as e:
        ctx.recluster_increment(0)           # no full window yet
    assert e.value.code == ckv.CKV_ESTATE
    ka, va = si.appended_tokens(9, 0, 321, 8)
    for j in range(320):
        ctx.append_kv(0, to_dev(ka[j][None, None]), to_dev(va[j][None, None]))
    with pytest.raises(ckv.CkvError) as e:
        ctx.append_kv(0, to_dev(ka[320][None, None]), to_dev(va[320][None, None]))
    assert e.value.code == ckv.CKV_ECAPACITY
    ctx.recluster_increment(0)
    with pytest.raises(ckv.CkvError) as e:   # store full: capacity n + 320 reached
        ctx.append_kv(0, to_dev(ka[320][None, None]), to_dev(va[320][None, None]))
    assert e.value.code == ckv.CKV_ECAPACITY
    out = torch.empty(1, 4, 128, device="cuda")
    with pytest.raises(ckv.CkvError) as e:
        ctx.select_and_attend(0, to_dev(si.queries(9, 0, 0, 1, 4)), 15, out)  # below the sinks
    assert e.value.code == ckv.CKV_EINVAL
    torch.cuda.synchronize()
    ctx.check_device_error()


def _exports_equal(a, b):
    for key in ("mu", "offsets", "ids", "kp", "vp", "sp_k", "sp_v"):
        x, y = a[key], b[key]
        assert x.shape == y.shape, key
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y), key


def test_async_recluster_overlaps_decode():
    """recluster_begin on a second stream while appends and decode continue on the first
    (ClusterKV explainer, section 4.1: clustering runs asynchronously with decoding). During
    the overlap the layer attends its old clusters plus every pending token (the window being
    clustered and the tokens appended since); after recluster_finish the store equals the one
    the synchronous recluster_increment builds at the same position. Two windows are run, so
    the second overlap wraps around the pending ring."""
    import recallable_kv_cache_cosine_b200 as ckv
    seed, G, W = 9, 4, 320
    B, Hkv, n, C, n_centers = 1, 2, 2048, 32, 32
    extra = (50, 77)  # tokens appended during each overlap
    K = np.empty((B, Hkv, n, 128), np.uint16)
    V = np.empty_like(K)
    AK = np.empty((B, Hkv, 3 * W, 128), np.uint16)
    AV = np.empty_like(AK)
    for b in range(B):
        for h in range(Hkv):
            u = si.unit_id(0, b, h, B, Hkv)
            K[b, h], V[b, h] = si.keys_values(seed, u, n, n_centers)
            AK[b, h], AV[b, h] = si.appended_tokens(seed, u, 3 * W, n_centers)
    make = lambda: ckv.ClusterKV(1, B, Hkv, Hkv * G, capacity=n + 3 * W, max_clusters=C + 8, seed=seed)
    actx, sctx = make(), make()
    actx.cluster_prefill(0, to_dev(K), to_dev(V), C)
    sctx.cluster_prefill(0, to_dev(K), to_dev(V), C)
    # every appended token as its own device tensor, ready before any stream uses it
    tk = [to_dev(np.ascontiguousarray(AK[:, :, i])) for i in range(3 * W)]
    tv = [to_dev(np.ascontiguousarray(AV[:, :, i])) for i in range(3 * W)]
    tok = lambda a, i: tk[i] if a is AK else tv[i]
    qs = np.stack([si.queries(seed, 0, b, 8, Hkv * G) for b in range(B)], axis=1)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    stats = {}
    j = 0
    for window in range(2):
        C_old, m_old = C + 4 * window, n - 16 + window * W
        # fill the window (both contexts)
        while actx.layer_info(0).pending < W:
            actx.append_kv(0, tok(AK, j), tok(AV, j), stream=s1)
            sctx.append_kv(0, tok(AK, j), tok(AV, j))
            j += 1
        s2.wait_stream(s1)
        actx.recluster_begin(0, stream=s2)
        with pytest.raises(ckv.CkvError):
            actx.recluster_increment(0, stream=s1)
        sctx.recluster_increment(0)
        for t in range(extra[window]):
            actx.append_kv(0, tok(AK, j), tok(AV, j), stream=s1)
            sctx.append_kv(0, tok(AK, j), tok(AV, j))
            j += 1
            if t in (0, extra[window] - 1):
                info = actx.layer_info(0)
                assert (info.C, info.m, info.pending) == (C_old, m_old, W + t + 1)
                with torch.cuda.stream(s1):
                    _decode_check(actx, qs[t % 8], 512, B, Hkv, G, stats, window)
        actx.recluster_finish(0, stream=s1)
        info = actx.layer_info(0)
        assert (info.C, info.m, info.pending, info.windows) == (C_old + 4, m_old + W, extra[window], window + 1)
        with torch.cuda.stream(s1):
            _decode_check(actx, qs[window], 512, B, Hkv, G, stats, window + 1)
        torch.cuda.synchronize()
        actx.check_device_error()
        for b in range(B):
            for h in range(Hkv):
                _exports_equal(actx.export_unit(0, b, h), sctx.export_unit(0, b, h))
    with pytest.raises(ckv.CkvError):
        actx.recluster_finish(0)
    assert stats["near_tie"] <= 1
