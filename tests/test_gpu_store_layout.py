"""The order in which the library keeps a stored row's 16-byte chunks is internal to it.

Stored K/V rows keep logical chunk c of row r at chunk c ^ (r & 7) (the decode kernel copies
runs of rows into shared memory as they are and reads them without bank conflicts). Every
call that takes or gives rows works in logical order: what `import_unit` takes comes back
from `export_unit` bit for bit, a row `append_kv` takes comes back as it was, and the fp8 copy
exported after an import is the quantisation of the logical rows (checked against the
oracle's quantiser). Rows at every residue r & 7, odd row counts and a pending run are used.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _store(rng, m, C, n_sink, pending):
    cuts = np.sort(rng.choice(np.arange(1, m), size=C - 1, replace=False))
    offsets = np.concatenate([[0], cuts, [m]]).astype(np.int32)
    ids = (n_sink + rng.permutation(m + pending)[:m]).astype(np.int32)
    for c in range(C):  # ascending inside each cluster
        ids[offsets[c]:offsets[c + 1]] = np.sort(ids[offsets[c]:offsets[c + 1]])
    bf = lambda *s: torch.randn(*s).to(torch.bfloat16)
    return {"mu": torch.randn(C, 128), "offsets": torch.from_numpy(offsets),
            "ids": torch.from_numpy(ids), "kp": bf(m, 128), "vp": bf(m, 128),
            "sp_k": bf(n_sink + pending, 128), "sp_v": bf(n_sink + pending, 128)}


@pytest.mark.parametrize("m,C,pending", [(1501, 12, 37), (8, 1, 0), (777, 40, 320)])
def test_import_export_is_exact(m, C, pending):
    import recallable_kv_cache_cosine_b200 as ckv
    rng = np.random.default_rng(m)
    torch.manual_seed(m)
    ctx = ckv.ClusterKV(1, 2, 2, 8, capacity=2200, max_clusters=48, seed=5)
    try:
        stores = {}
        for b in range(2):
            for h in range(2):
                stores[b, h] = _store(rng, m, C, ctx.cfg.n_sink, pending)
                ctx.import_unit(0, b, h, stores[b, h], pending=pending)
        torch.cuda.synchronize()
        for (b, h), st in stores.items():
            ex = ctx.export_unit(0, b, h)
            for k in ("mu", "offsets", "ids", "kp", "vp", "sp_k", "sp_v"):
                assert torch.equal(ex[k].view(torch.int32) if ex[k].dtype == torch.float32 else ex[k],
                                   st[k].view(torch.int32) if st[k].dtype == torch.float32 else st[k]), k
        ctx.check_device_error()
    finally:
        ctx.close()


def test_appended_rows_come_back_as_given():
    import recallable_kv_cache_cosine_b200 as ckv
    rng = np.random.default_rng(11)
    torch.manual_seed(11)
    ctx = ckv.ClusterKV(1, 1, 2, 8, capacity=2400, max_clusters=16, seed=5)
    try:
        pending0 = 5
        for h in range(2):
            ctx.import_unit(0, 0, h, _store(rng, 1200, 9, ctx.cfg.n_sink, pending0), pending=pending0)
        new_k = torch.randn(13, 1, 2, 128, device="cuda").to(torch.bfloat16)
        new_v = torch.randn(13, 1, 2, 128, device="cuda").to(torch.bfloat16)
        for t in range(13):  # rows at every residue of the ring position
            ctx.append_kv(0, new_k[t], new_v[t])
        torch.cuda.synchronize()
        for h in range(2):
            ex = ctx.export_unit(0, 0, h)
            base = ctx.cfg.n_sink + pending0
            assert torch.equal(ex["sp_k"][base:base + 13], new_k[:, 0, h].cpu())
            assert torch.equal(ex["sp_v"][base:base + 13], new_v[:, 0, h].cpu())
        ctx.check_device_error()
    finally:
        ctx.close()


def test_fp8_copy_of_imported_rows_matches_the_oracle():
    import recallable_kv_cache_cosine_b200 as ckv
    rng = np.random.default_rng(21)
    torch.manual_seed(21)
    ctx = ckv.ClusterKV(1, 1, 1, 4, capacity=1200, max_clusters=8, seed=5)
    try:
        st = _store(rng, 999, 7, ctx.cfg.n_sink, 0)
        ctx.import_unit(0, 0, 0, st, pending=0)
        ctx.enable_fp8()
        ex = ctx.export_unit_fp8(0, 0, 0)
        for rows, codes, scales in ((st["kp"], ex["k8"], ex["ks"]), (st["vp"], ex["v8"], ex["vs"])):
            c_ref, s_ref = oracle.quantize_rows_e4m3(rows.view(torch.int16).numpy().view(np.uint16))
            assert np.array_equal(codes.numpy(), c_ref)
            assert np.array_equal(scales.numpy(), s_ref)
        ctx.check_device_error()
    finally:
        ctx.close()
