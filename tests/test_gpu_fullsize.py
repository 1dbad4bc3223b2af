"""Full-size GPU parity on the workload configurations, on sampled units.

Each test runs the whole hot path at full size, with the launch shapes the library picks for
it. Units that a check reads are generated on the CPU by the seeded generator, so the oracle
sees the same inputs. Other units are filled on the device with the same recipe. For each
sampled unit:
* store invariants (ids permute the non-sink tokens; K/V rows are the inputs permuted);
* the final centroids are within 1e-3 of the oracle's means of the GPU's final clusters;
* the assignment stage: the stage kernel on the unit's full key set vs the oracle on
  sampled rows, on the same centroids (cosine-gap tolerance);
* decode: selection and attention vs the oracle on the GPU's store (near-tie and 2e-3
  tolerances).

Configurations: one Llama-3.1-8B-shaped layer at 32k (C=400, budget 1024); a 32-layer
batch-8 stack (budget 2048); batch-4 incremental decode (1280 generated tokens, 4 windows);
a 128k context (C=1600, budget 2048).
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_helpers import MU_TOL, check_assign, check_decode_unit, store_from_export, to_dev, to_u16

pytestmark = pytest.mark.gpu
HQ, HKV, G = 32, 8, 4


def _ckv():
    import recallable_kv_cache_cosine_b200 as ckv
    return ckv


def _fill_layer(K, V, seed, layer, B, n, n_centers, sampled):
    """K, V: device tensors [B, HKV, n, 128]; sampled (b, h) units come from the CPU generator."""
    for b in range(B):
        for h in range(HKV):
            u = si.unit_id(layer, b, h, B, HKV)
            if (b, h) in sampled:
                k, v = si.keys_values(seed, u, n, n_centers)
                K[b, h], V[b, h] = to_dev(k), to_dev(v)
            else:
                K[b, h], V[b, h] = si.keys_values_torch(seed, u, n, n_centers, K.device)


def _check_store(ctx, layer, b, h, Kn, Vn, C):
    ex = ctx.export_unit(layer, b, h)
    st = store_from_export(ex)
    n = Kn.shape[0]
    np.testing.assert_array_equal(np.sort(st.ids), np.arange(16, n))
    np.testing.assert_array_equal(st.kp, Kn[st.ids])
    np.testing.assert_array_equal(st.vp, Vn[st.ids])
    np.testing.assert_array_equal(st.sp_k, Kn[:16])
    a = np.empty(n - 16, np.int32)
    for c in range(C):
        a[st.ids[st.offsets[c]:st.offsets[c + 1]] - 16] = c
    w_mu, w_off, _ = oracle.update(Kn[16:], a, C, st.mu)
    np.testing.assert_array_equal(w_off, st.offsets)
    assert np.abs(w_mu - st.mu).max() <= MU_TOL
    return st


def _check_assign_stage(ctx, Kn, C, seed, rows=2048):
    """Stage kernels on one unit's full key set, checked on sampled rows."""
    n = Kn.shape[0]
    Kd = to_dev(Kn[None])
    mu, mh = ctx.kmeans_init(Kd, 16, n - 16, C, seed=seed)
    a = ctx.kmeans_assign(Kd, 16, n - 16, mh)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    pick = np.sort(rng.choice(n - 16, size=min(rows, n - 16), replace=False))
    stats = {}
    check_assign(np.ascontiguousarray(Kn[16:][pick]), to_u16(mh[0]), a[0].cpu().numpy()[pick], stats)
    assert stats["near_tie"] <= 2


def _decode(ctx, layer, q_u16, budget, B):
    out = torch.empty(B, HQ, 128, device="cuda", dtype=torch.float32)
    sel = torch.empty(B, HKV, budget, device="cuda", dtype=torch.int32)
    cnt = torch.empty(B, HKV, device="cuda", dtype=torch.int32)
    ctx.select_and_attend(layer, to_dev(q_u16), budget, out, sel, cnt)
    torch.cuda.synchronize()
    ctx.check_device_error()
    return out.cpu().numpy(), sel.cpu().numpy(), cnt.cpu().numpy()


def test_llama_layer_32k_budget_1k():
    ckv = _ckv()
    seed, n, C, budget, B = 21, 32768, 400, 1024, 1
    sampled = {(0, h) for h in range(HKV)}
    K = torch.empty(B, HKV, n, 128, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    _fill_layer(K, V, seed, 0, B, n, 400, sampled)
    ctx = ckv.ClusterKV(1, B, HKV, HQ, capacity=n, max_clusters=C, seed=seed)
    ctx.cluster_prefill(0, K, V, C)
    torch.cuda.synchronize()
    ctx.check_device_error()
    Kn, Vn = to_u16(K[0]), to_u16(V[0])
    stores = [_check_store(ctx, 0, 0, h, Kn[h], Vn[h], C) for h in range(HKV)]
    _check_assign_stage(ctx, Kn[3], C, seed)
    q = si.queries(seed, 0, 0, 64, HQ)
    stats = {}
    for step in (0, 17, 63):
        o, s, c = _decode(ctx, 0, q[step][None], budget, B)
        for h in range(HKV):
            check_decode_unit(stores[h], q[step, h * G:(h + 1) * G], budget, o[0, h * G:(h + 1) * G],
                              s[0, h], int(c[0, h]), stats)
    assert stats["near_tie"] <= 1
    print("32k/1k decode stats", stats)


def test_long_context_128k():
    ckv = _ckv()
    seed, n, C, budget, B = 25, 131072, 1600, 2048, 1
    sampled = {(0, 0), (0, 2), (0, 5), (0, 7)}
    K = torch.empty(B, HKV, n, 128, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    _fill_layer(K, V, seed, 0, B, n, 1600, sampled)
    ctx = ckv.ClusterKV(1, B, HKV, HQ, capacity=n, max_clusters=C, seed=seed)
    ctx.cluster_prefill(0, K, V, C)
    torch.cuda.synchronize()
    ctx.check_device_error()
    stats = {}
    q = si.queries(seed, 0, 0, 4, HQ)
    outs = [_decode(ctx, 0, q[s][None], budget, B) for s in range(4)]
    for (_, h) in sorted(sampled):
        Kn, Vn = to_u16(K[0, h]), to_u16(V[0, h])
        st = _check_store(ctx, 0, 0, h, Kn, Vn, C)
        for s in range(4):
            o, sel, c = outs[s]
            check_decode_unit(st, q[s, h * G:(h + 1) * G], budget, o[0, h * G:(h + 1) * G],
                              sel[0, h], int(c[0, h]), stats)
    _check_assign_stage(ctx, to_u16(K[0, 5]), C, seed, rows=8192)
    assert stats["near_tie"] <= 1
    print("128k decode stats", stats)


def test_incremental_batch4_four_windows():
    ckv = _ckv()
    seed, n, C, budget, B, W = 23, 32768, 400, 1024, 4, 320
    sampled = {(1, 3), (2, 6)}
    K = torch.empty(B, HKV, n, 128, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    _fill_layer(K, V, seed, 0, B, n, 400, sampled)
    AK = torch.empty(4 * W, B, HKV, 128, dtype=torch.bfloat16, device="cuda")
    AV = torch.empty_like(AK)
    for b in range(B):
        for h in range(HKV):
            u = si.unit_id(0, b, h, B, HKV)
            if (b, h) in sampled:
                ka, va = si.appended_tokens(seed, u, 4 * W, 400)
                AK[:, b, h], AV[:, b, h] = to_dev(ka), to_dev(va)
            else:
                AK[:, b, h], AV[:, b, h] = si.appended_tokens_torch(seed, u, 4 * W, 400, "cuda")
    ctx = ckv.ClusterKV(1, B, HKV, HQ, capacity=n + 4 * W, max_clusters=C + 16, seed=seed)
    ctx.cluster_prefill(0, K, V, C)
    qs = np.stack([si.queries(seed, 0, b, 8, HQ) for b in range(B)], axis=1)  # [8, B, HQ, 128]
    out = torch.empty(B, HQ, 128, device="cuda", dtype=torch.float32)
    stats = {}
    check_steps = {0, 100, 319, 320, 700, 1279}
    for t in range(4 * W):
        ctx.append_kv(0, AK[t], AV[t])
        if t in check_steps:
            o, s, c = _decode(ctx, 0, qs[t % 8], budget, B)
            for (b, h) in sorted(sampled):
                st = store_from_export(ctx.export_unit(0, b, h), windows=t // W)
                check_decode_unit(st, qs[t % 8][b, h * G:(h + 1) * G], budget, o[b, h * G:(h + 1) * G],
                                  s[b, h], int(c[b, h]), stats)
        else:
            ctx.select_and_attend(0, to_dev(qs[t % 8]), budget, out)
        if (t + 1) % W == 0:
            ctx.recluster_increment(0)
    torch.cuda.synchronize()
    ctx.check_device_error()
    info = ctx.layer_info(0)
    assert (info.C, info.m, info.pending, info.windows) == (C + 16, n - 16 + 4 * W, 0, 4)
    for (b, h) in sorted(sampled):
        st = store_from_export(ctx.export_unit(0, b, h), windows=4)
        np.testing.assert_array_equal(np.sort(st.ids), np.arange(16, n + 4 * W))
        full_k = np.concatenate([to_u16(K[b, h]), to_u16(AK[:, b, h])])
        np.testing.assert_array_equal(st.kp, full_k[st.ids])
    assert stats["near_tie"] <= 1
    print("incremental decode stats", stats)


def test_32_layer_batch8_stack_budget_2k():
    ckv = _ckv()
    seed, n, C, budget, B, L = 22, 32768, 400, 2048, 8, 32
    sampled = {(0, 0): None, (7, 3): None, (19, 5): None, (31, 7): None}  # (layer, b)
    ctx = ckv.ClusterKV(L, B, HKV, HQ, capacity=n, max_clusters=C, seed=seed)
    K = torch.empty(B, HKV, n, 128, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    host = {}
    for layer in range(L):
        units = {(b, h) for (l2, b) in sampled if l2 == layer for h in range(HKV)}
        _fill_layer(K, V, seed, layer, B, n, 400, units)
        ctx.cluster_prefill(layer, K, V, C)
        torch.cuda.synchronize()
        for (l2, b) in sampled:
            if l2 == layer:
                host[(layer, b)] = (to_u16(K[b]), to_u16(V[b]))
    ctx.check_device_error()
    stats = {}
    for step in range(2):
        for layer in range(L):
            q = si.queries(seed, layer, 0, 2, HQ)  # same queries for every sequence b
            qb = np.repeat(q[step][None], B, axis=0)
            o, s, c = _decode(ctx, layer, qb, budget, B)
            for (l2, b) in sampled:
                if l2 != layer:
                    continue
                for h in (0, 5):
                    if step == 0:
                        st = _check_store(ctx, layer, b, h, host[(layer, b)][0][h], host[(layer, b)][1][h], C)
                    else:
                        st = store_from_export(ctx.export_unit(layer, b, h))
                    check_decode_unit(st, qb[b, h * G:(h + 1) * G], budget, o[b, h * G:(h + 1) * G],
                                      s[b, h], int(c[b, h]), stats)
    assert stats["near_tie"] <= 1
    print("32-layer stack decode stats", stats)
