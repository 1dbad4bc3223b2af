"""GPU parity of the prefill K-means stages against the oracle (stage by stage).

Each stage gets identical inputs on both sides: the GPU's own previous output, fed to the
oracle. One early assignment flip therefore cannot cascade and hide a kernel bug.
* init: exact init indices, centroids equal to the chosen keys, mu_hat within one bf16 step;
* assign (tcgen05): equal to the oracle's argmax on the same mu_hat, except cosine gaps < 1e-4;
* update: offsets and perm exact; mu within 1e-3; mu_hat within one bf16 step.
Shapes cover every path of the assignment kernel: one TMEM slot (C <= 256), two slots
(256 < C <= 512), chunked launches with merging (C > 512), ragged and sub-tile key counts.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_helpers import check_assign, check_mu_hat, to_dev, to_u16, MU_TOL

pytestmark = pytest.mark.gpu


def _ctx(U, n, C):
    import recallable_kv_cache_cosine_b200 as ckv
    return ckv.ClusterKV(n_layers=1, batch=U, n_kv_heads=1, n_q_heads=1, capacity=n,
                         max_clusters=C)


def _keys(U, n, n_centers, seed):
    K = np.stack([si.keys_values(seed, u, n, n_centers)[0] for u in range(U)])
    return K, to_dev(K)


@pytest.mark.parametrize("m,C", [(40, 3), (127, 8), (300, 4), (2032, 32), (5000, 200), (5000, 256),
                                 (5000, 257), (4000, 400), (3000, 512), (3000, 513), (6000, 1100),
                                 (60000, 40)])
def test_init_and_assign_stage(m, C):
    U, n = 2, m + 16
    Kn, Kd = _keys(U, n, max(C, 4), seed=m + C)
    ctx = _ctx(U, n, C)
    init_idx = torch.empty(U, C, dtype=torch.int32, device="cuda")
    mu, mu_hat = ctx.kmeans_init(Kd, 16, m, C, seed=99, unit_base=5, window=0, init_idx=init_idx)
    assign = ctx.kmeans_assign(Kd, 16, m, mu_hat)
    torch.cuda.synchronize()
    ctx.check_device_error()
    stats = {}
    for u in range(U):
        want_init = oracle.init_indices(m, C, oracle.stream_key(99, 5 + u, 0))
        np.testing.assert_array_equal(init_idx[u].cpu().numpy(), want_init)
        keys = Kn[u, 16:]
        np.testing.assert_array_equal(mu[u].cpu().numpy(),
                                      oracle.bf16_to_f64(keys[want_init]).astype(np.float32))
        check_mu_hat(mu[u].cpu().numpy(), to_u16(mu_hat[u]))
        check_assign(keys, to_u16(mu_hat[u]), assign[u].cpu().numpy(), stats)
    assert stats["near_tie"] <= max(2, stats["keys"] // 1000)


def test_assign_ties_go_to_lower_index():
    # duplicated centroids (exact ties) and a zero centroid
    U, m, C = 1, 1000, 300
    n = m + 16
    Kn, Kd = _keys(U, n, 50, seed=3)
    rng = np.random.default_rng(0)
    mh = rng.standard_normal((C, 128))
    mh[7] = 0.0
    mh[150:300] = mh[0:150]  # every centroid >= 150 duplicates one below it
    mh_u16 = oracle.normalize(mh)
    ctx = _ctx(U, n, C)
    assign = ctx.kmeans_assign(Kd, 16, m, to_dev(mh_u16[None]))
    got = assign[0].cpu().numpy()
    assert got.max() < 150
    check_assign(Kn[0, 16:], mh_u16, got)


@pytest.mark.parametrize("n,C,n_centers", [(2048, 32, 32), (9000, 300, 200), (6000, 600, 500)])
def test_ten_iterations_stage_by_stage(n, C, n_centers):
    U, m = 2, n - 16
    Kn, Kd = _keys(U, n, n_centers, seed=11)
    ctx = _ctx(U, n, C)
    mu, mu_hat = ctx.kmeans_init(Kd, 16, m, C, seed=1)
    stats = {}
    for it in range(10):
        assign = ctx.kmeans_assign(Kd, 16, m, mu_hat)
        mu_prev = mu.clone()
        mu_hat_used = mu_hat.clone()
        mu, mu_hat, offsets, perm = ctx.kmeans_update(Kd, 16, m, assign, mu)
        torch.cuda.synchronize()
        for u in range(U):
            keys = Kn[u, 16:]
            a = assign[u].cpu().numpy()
            # assign stage: same mu_hat on both sides
            check_assign(keys, to_u16(mu_hat_used[u]), a, stats)
            # update stage: same assignment and previous mu on both sides
            w_mu, w_off, w_perm = oracle.update(keys, a, C, mu_prev[u].cpu().numpy().astype(np.float64))
            np.testing.assert_array_equal(offsets[u].cpu().numpy(), w_off)
            np.testing.assert_array_equal(perm[u].cpu().numpy(), w_perm)
            err = np.abs(mu[u].cpu().numpy() - w_mu).max()
            assert err <= MU_TOL, err
            check_mu_hat(mu[u].cpu().numpy(), to_u16(mu_hat[u]))
    ctx.check_device_error()
    assert stats["near_tie"] <= max(2, stats["keys"] // 1000)
