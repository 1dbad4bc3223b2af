"""The allocation-free K-means update (ckv_kmeans_update_noalloc) matches the context-based
ckv_kmeans_update.

The no-alloc call is for callers that cannot allocate device memory (memory-pool engines,
decode loops that must not stall on cudaMalloc, plugins whose host owns the device memory).
It keeps its counting-sort scratch in a fixed array inside the library. This test calls it
through the C-ABI twice in a row with different shapes, so the second call runs on the
first call's leftovers. It compares both results with the regular entry point: offsets and
perm exactly, mu within the 1e-3 centroid tolerance, mu_hat within one bf16 step. The file
is named so that pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import synth_inputs as si
from gpu_helpers import MU_TOL, to_dev

pytestmark = pytest.mark.gpu


def _p(t):
    return C.c_void_p(t.data_ptr())


def _inputs(U, n, C_, seed):
    K = np.stack([si.keys_values(seed, u, n, max(C_, 8))[0] for u in range(U)])
    rng = np.random.default_rng(seed)
    m = n - 16
    assign = torch.from_numpy(rng.integers(0, C_, size=(U, m)).astype(np.int32)).cuda()
    mu0 = torch.from_numpy(rng.standard_normal((U, C_, 128)).astype(np.float32)).cuda()
    return to_dev(K), assign, mu0


@pytest.mark.parametrize("calls", [[(2, 5016, 300, 1), (3, 2100, 40, 2)]])
def test_noalloc_update_matches_context_update_on_two_calls(calls):
    import recallable_kv_cache_cosine_b200 as ckv
    L = ckv.lib()
    for U, n, C_, seed in calls:
        m = n - 16
        Kd, assign, mu0 = _inputs(U, n, C_, seed)
        ctx = ckv.ClusterKV(1, U, 1, 1, capacity=n, max_clusters=C_)
        mu_ref, mh_ref, off_ref, perm_ref = ctx.kmeans_update(Kd, 16, m, assign, mu0.clone())
        mu = mu0.clone()
        mh = torch.empty(U, C_, 128, device="cuda", dtype=torch.bfloat16)
        off = torch.empty(U, C_ + 1, device="cuda", dtype=torch.int32)
        perm = torch.empty(U, m, device="cuda", dtype=torch.int32)
        stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = L.ckv_kmeans_update_noalloc(_p(Kd), n, 16, m, U, _p(assign), C_, _p(mu), _p(mh),
                                         _p(off), _p(perm), stream)
        assert rc == 0, L.ckv_last_error()
        torch.cuda.synchronize()
        assert torch.equal(off, off_ref)
        assert torch.equal(perm, perm_ref)
        assert (mu - mu_ref).abs().max().item() <= MU_TOL
        a = mh.float()
        b = mh_ref.float()
        assert torch.all((a - b).abs() <= b.abs() * 2.0 ** -7 + 1e-30)
        ctx.close()


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
