"""The allocation-free K-means update (ckv_kmeans_update_noalloc) against the context-based
ckv_kmeans_update and the oracle.

The no-alloc call is for callers that cannot allocate device memory (memory-pool engines,
decode loops that must not stall on cudaMalloc, plugins whose host owns the device memory).
It keeps its counting-sort scratch in a fixed array inside the library and runs the same
kernels as the context call, so its results must be bit-identical to that call's.

This test calls it through the C-ABI twice in a row, the second call on a larger shape
than the first, so the second call's counts land on scratch the first call left behind.
Each result must equal the context call's bit for bit, and the oracle's update (ClusterKV
explainer sections 3.1 and 4.1): offsets and perm exactly, mu within the 1e-3 centroid
tolerance. A third case feeds assignments outside [0, C): they are skipped, and
offsets[u][C] counts only the keys placed. The file is named so that pytest collects it
last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_helpers import MU_TOL, to_dev

pytestmark = pytest.mark.gpu


def _p(t):
    return C.c_void_p(t.data_ptr())


def _inputs(U, n, C_, seed):
    K = np.stack([si.keys_values(seed, u, n, max(C_, 8))[0] for u in range(U)])
    rng = np.random.default_rng(seed)
    m = n - 16
    assign = rng.integers(0, C_, size=(U, m)).astype(np.int32)
    mu0 = rng.standard_normal((U, C_, 128)).astype(np.float32)
    return K, assign, mu0


def _noalloc(L, Kd, n, m, U, assign_d, C_, mu0):
    mu = torch.from_numpy(mu0).cuda()
    mh = torch.empty(U, C_, 128, device="cuda", dtype=torch.bfloat16)
    off = torch.empty(U, C_ + 1, device="cuda", dtype=torch.int32)
    perm = torch.empty(U, m, device="cuda", dtype=torch.int32)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.ckv_kmeans_update_noalloc(_p(Kd), n, 16, m, U, _p(assign_d), C_, _p(mu), _p(mh),
                                     _p(off), _p(perm), stream)
    assert rc == 0, L.ckv_last_error()
    torch.cuda.synchronize()
    return mu, mh, off, perm


# the second call needs more scratch than the first (U * ceil(m / 1024) * C counts: 360,
# then 3000), so it reads and rewrites counts the first call left behind
CALLS = [(3, 2100, 40, 2), (2, 5016, 300, 1)]


def test_noalloc_update_matches_context_update_and_oracle_on_two_calls():
    import recallable_kv_cache_cosine_b200 as ckv
    L = ckv.lib()
    for U, n, C_, seed in CALLS:
        m = n - 16
        K, assign, mu0 = _inputs(U, n, C_, seed)
        Kd, assign_d = to_dev(K), torch.from_numpy(assign).cuda()
        ctx = ckv.ClusterKV(1, U, 1, 1, capacity=n, max_clusters=C_)
        mu_ref, mh_ref, off_ref, perm_ref = ctx.kmeans_update(Kd, 16, m, assign_d,
                                                              torch.from_numpy(mu0).cuda())
        torch.cuda.synchronize()
        ctx.check_device_error()
        ctx.close()
        mu, mh, off, perm = _noalloc(L, Kd, n, m, U, assign_d, C_, mu0)
        # the same deterministic kernels: bit-identical to the context call
        assert torch.equal(off, off_ref)
        assert torch.equal(perm, perm_ref)
        assert torch.equal(mu, mu_ref)
        assert torch.equal(mh, mh_ref)
        # and the oracle's update of the same inputs
        for u in range(U):
            mu_o, off_o, perm_o = oracle.update(K[u, 16:], assign[u], C_, mu0[u].astype(np.float64))
            assert np.array_equal(off[u].cpu().numpy(), off_o)
            assert np.array_equal(perm[u].cpu().numpy(), perm_o)
            assert np.abs(mu[u].cpu().numpy() - mu_o).max() <= MU_TOL
            # mu_hat is the normalised centroid rounded to bf16 (one bf16 step: the fp32
            # norm may round a halfway case the other way)
            nrm = (mu[u].double() / mu[u].double().norm(dim=1, keepdim=True)).cpu().numpy()
            got = mh[u].float().cpu().numpy()
            assert np.all(np.abs(got - nrm) <= np.abs(nrm) * 2.0 ** -8 + 1e-30)


def test_noalloc_update_skips_out_of_range_assignments():
    import recallable_kv_cache_cosine_b200 as ckv
    L = ckv.lib()
    U, n, C_, seed = 2, 3000, 50, 5
    m = n - 16
    K, assign, mu0 = _inputs(U, n, C_, seed)
    bad = np.zeros_like(assign, dtype=bool)
    bad[0, [0, 17, 1500, m - 1]] = True
    bad[1, [3, 2048]] = True
    assign[0, [0, 1500]] = -1
    assign[0, [17, m - 1]] = C_
    assign[1, 3] = -7
    assign[1, 2048] = C_ + 100
    Kd, assign_d = to_dev(K), torch.from_numpy(assign).cuda()
    mu, mh, off, perm = _noalloc(L, Kd, n, m, U, assign_d, C_, mu0)
    # the context call skips them too, and reports them through the device error word
    ctx = ckv.ClusterKV(1, U, 1, 1, capacity=n, max_clusters=C_)
    mu_ref, mh_ref, off_ref, perm_ref = ctx.kmeans_update(Kd, 16, m, assign_d,
                                                          torch.from_numpy(mu0).cuda())
    torch.cuda.synchronize()
    with pytest.raises(ckv.CkvError) as e:
        ctx.check_device_error()
    assert e.value.code == ckv.CKV_EINVAL
    ctx.check_device_error()  # the word was cleared
    ctx.close()
    assert torch.equal(off, off_ref) and torch.equal(mu, mu_ref) and torch.equal(mh, mh_ref)
    for u in range(U):
        keep = np.flatnonzero(~bad[u])
        placed = int(off[u, C_])
        assert placed == len(keep) < m  # offsets[C] counts the keys placed, not m
        assert torch.equal(perm[u, :placed], perm_ref[u, :placed])
        # equal to the oracle's update of the valid keys alone, with indices mapped back
        mu_o, off_o, perm_o = oracle.update(K[u, 16:][keep], assign[u, keep], C_,
                                            mu0[u].astype(np.float64))
        assert np.array_equal(off[u].cpu().numpy(), off_o)
        assert np.array_equal(perm[u, :placed].cpu().numpy(), keep[perm_o])
        assert np.abs(mu[u].cpu().numpy() - mu_o).max() <= MU_TOL


def test_noalloc_update_rejects_requests_beyond_its_scratch():
    import recallable_kv_cache_cosine_b200 as ckv
    L = ckv.lib()
    t = torch.zeros(64, device="cuda", dtype=torch.float32)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    # 8 units x 131056 keys x 4096 clusters needs 8 * 128 * 4096 counts > 2^21
    rc = L.ckv_kmeans_update_noalloc(_p(t), 131072, 16, 131056, 8, _p(t), 4096, _p(t), _p(t),
                                     _p(t), _p(t), stream)
    assert rc == ckv.CKV_EINVAL
    assert b"scratch" in L.ckv_last_error()
