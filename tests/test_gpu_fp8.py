"""Far clusters attended from an fp8 copy (ClusterKV explainer section 7, outlook: lower
precision for clusters far from the query), against the oracle.

Reading (pinned on the CPU in test_oracle_fp8.py): every clustered row keeps an e4m3 copy
with one fp32 scale per row, scale = max|x| / 448, code = e4m3(x / scale); the selection is
unchanged, and a selected cluster at walk rank >= n_near (the cut cluster's partial rows
included) is attended from the copy.

Checks:
* the copy the library keeps equals the oracle's quantisation of the same bf16 rows, codes
  and scales bit for bit, after prefill, after an incremental re-clustering and after an
  import;
* select_and_attend_mixed equals ``oracle.attend_mixed`` element by element within 2e-3, at a
  2k-token store and a 32k-token store, with n_near placed so that the cut cluster is far
  (n_near = its rank) and near (n_near = its rank + 1), with every cluster far (n_near = 0),
  and on the resident and the ring paths of the cut cluster;
* n_near >= C gives exactly the output of select_and_attend (bit for bit), and the selection
  is the same in every case.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_helpers import OUT_TOL, rows_of_ids, selection_near_tie, store_from_export, to_dev

pytestmark = pytest.mark.gpu


def _ctx(B, Hkv, G, n, C_, seed, extra=0):
    import recallable_kv_cache_cosine_b200 as ckv
    K = np.stack([np.stack([si.keys_values(seed, si.unit_id(0, b, h, B, Hkv), n, C_)[0]
                            for h in range(Hkv)]) for b in range(B)])
    V = np.stack([np.stack([si.keys_values(seed, si.unit_id(0, b, h, B, Hkv), n, C_)[1]
                            for h in range(Hkv)]) for b in range(B)])
    ctx = ckv.ClusterKV(1, B, Hkv, Hkv * G, capacity=n + extra, max_clusters=C_ + 8, seed=seed)
    ctx.cluster_prefill(0, to_dev(K), to_dev(V), C_)
    ctx.enable_fp8()
    torch.cuda.synchronize()
    ctx.check_device_error()
    return ctx


def _check_copy(ctx, B, Hkv):
    for b in range(B):
        for h in range(Hkv):
            st = store_from_export(ctx.export_unit(0, b, h))
            f8 = ctx.export_unit_fp8(0, b, h)
            k8, ks = oracle.quantize_rows_e4m3(st.kp)
            v8, vs = oracle.quantize_rows_e4m3(st.vp)
            assert np.array_equal(f8["k8"].numpy(), k8)
            assert np.array_equal(f8["v8"].numpy(), v8)
            assert np.array_equal(f8["ks"].numpy().view(np.uint32), ks.view(np.uint32))
            assert np.array_equal(f8["vs"].numpy().view(np.uint32), vs.view(np.uint32))


def _mixed_and_check(ctx, q_u16, budget, n_near_of, B, Hkv, G, stats):
    """Runs select_and_attend_mixed with a per-call n_near (the same for every unit, chosen
    by n_near_of from unit (0, 0)'s oracle selection) and checks every unit."""
    qd = to_dev(q_u16)
    st00 = store_from_export(ctx.export_unit(0, 0, 0))
    sel00 = oracle.select(st00, q_u16[0, :G], budget)
    n_near = n_near_of(st00, sel00)
    out = torch.empty(B, Hkv * G, 128, device="cuda", dtype=torch.float32)
    sel = torch.empty(B, Hkv, budget, device="cuda", dtype=torch.int32)
    cnt = torch.empty(B, Hkv, device="cuda", dtype=torch.int32)
    ctx.select_and_attend_mixed(0, qd, budget, n_near, out, sel, cnt)
    torch.cuda.synchronize()
    ctx.check_device_error()
    outs, sels, cnts = out.cpu().numpy(), sel.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            st = store_from_export(ctx.export_unit(0, b, h))
            qh = q_u16[b, h * G:(h + 1) * G]
            want_sel = oracle.select(st, qh, budget)
            got = sels[b, h, : cnts[b, h]]
            assert cnts[b, h] == len(want_sel.ids)
            exact = set(got.tolist()) == set(want_sel.ids.tolist())
            if not exact:
                assert selection_near_tie(st, qh, want_sel)
                want_sel = oracle.Selection(got.copy(), rows_of_ids(st, got), 0, -1, 0, want_sel.scores)
            k8, ks = oracle.quantize_rows_e4m3(st.kp)
            v8, vs = oracle.quantize_rows_e4m3(st.vp)
            want = oracle.attend_mixed(st, qh, want_sel, n_near, k8, ks, v8, vs)
            err = float(np.abs(outs[b, h * G:(h + 1) * G] - want).max())
            assert err <= OUT_TOL, (n_near, err)
            stats["max_err"] = max(stats.get("max_err", 0.0), err)
            stats["units"] = stats.get("units", 0) + 1
    return out, sel, cnt, n_near


def _cut_rank(st, sel):
    rank = oracle.walk_rank(st, sel)
    return int(rank[sel.cut]) if sel.cut >= 0 else st.C


# (6016 tokens, 8 clusters): cut clusters of ~750 rows take the ring path, not the resident one
@pytest.mark.parametrize("B,Hkv,G,n,C_,budgets", [(1, 2, 4, 2048, 32, [100, 256, 700]),
                                                   (1, 1, 4, 6016, 8, [300, 2000]),
                                                   (1, 2, 4, 32768, 400, [1024, 2048])])
def test_mixed_precision_decode_matches_the_oracle(B, Hkv, G, n, C_, budgets):
    seed = 21
    ctx = _ctx(B, Hkv, G, n, C_, seed)
    try:
        _check_copy(ctx, B, Hkv)
        stats = {}
        for i, budget in enumerate(budgets):
            q = np.stack([si.queries(seed, 0, b, len(budgets), Hkv * G)[i] for b in range(B)])
            rules = [lambda st, s: _cut_rank(st, s),        # the cut cluster is far
                     lambda st, s: _cut_rank(st, s) + 1,    # the cut cluster is near
                     lambda st, s: 0,                       # every cluster is far
                     lambda st, s: max(1, _cut_rank(st, s) // 2)]
            for rule in rules:
                _mixed_and_check(ctx, q, budget, rule, B, Hkv, G, stats)
            # n_near >= C: bit for bit the bf16 path
            outm, selm, cntm, _ = _mixed_and_check(ctx, q, budget, lambda st, s: st.C, B, Hkv, G, stats)
            out = torch.empty_like(outm)
            sel = torch.empty_like(selm)
            cnt = torch.empty_like(cntm)
            ctx.select_and_attend(0, to_dev(q), budget, out, sel, cnt)
            torch.cuda.synchronize()
            assert torch.equal(out, outm) and torch.equal(sel, selm) and torch.equal(cnt, cntm)
        print("fp8 mixed decode", stats)
    finally:
        ctx.close()


def test_fp8_copy_follows_incremental_clustering_and_import():
    import recallable_kv_cache_cosine_b200 as ckv
    B, Hkv, G, n, C_, seed, W = 1, 2, 4, 3000, 40, 5, 320
    ctx = _ctx(B, Hkv, G, n, C_, seed, extra=W)
    try:
        ka = np.stack([si.appended_tokens(seed, h, W, 40)[0] for h in range(Hkv)])  # [Hkv, W, 128]
        va = np.stack([si.appended_tokens(seed, h, W, 40)[1] for h in range(Hkv)])
        for t in range(W):
            ctx.append_kv(0, to_dev(ka[:, t][None]), to_dev(va[:, t][None]))
        ctx.recluster_increment(0)
        torch.cuda.synchronize()
        ctx.check_device_error()
        _check_copy(ctx, B, Hkv)
        stats = {}
        q = si.queries(seed, 0, 0, 1, Hkv * G)[0][None]
        _mixed_and_check(ctx, q, 600, lambda st, s: _cut_rank(st, s), B, Hkv, G, stats)
        # import a unit's store: its copy is rebuilt
        st = store_from_export(ctx.export_unit(0, 0, 1))
        from gpu_helpers import store_to_import
        ctx.import_unit(0, 0, 0, store_to_import(st), pending=st.pending)
        torch.cuda.synchronize()
        _check_copy(ctx, B, Hkv)
        with pytest.raises(ckv.CkvError) as e:
            ctx.select_and_attend_mixed(0, to_dev(q), 600, -1, torch.empty(1, Hkv * G, 128, device="cuda"))
        assert e.value.code == ckv.CKV_EINVAL
    finally:
        ctx.close()


def test_mixed_precision_needs_the_copy():
    import recallable_kv_cache_cosine_b200 as ckv
    ctx = ckv.ClusterKV(1, 1, 1, 4, capacity=2048, max_clusters=32, seed=0)
    try:
        K, V = si.keys_values(0, 0, 2048, 32)
        ctx.cluster_prefill(0, to_dev(K[None, None]), to_dev(V[None, None]), 32)
        q = to_dev(si.queries(0, 0, 0, 1, 4)[0][None])
        with pytest.raises(ckv.CkvError) as e:
            ctx.select_and_attend_mixed(0, q, 256, 4, torch.empty(1, 4, 128, device="cuda"))
        assert e.value.code == ckv.CKV_ESTATE
    finally:
        ctx.close()
