"""No kernel writes past the end of a device buffer (canary check, in place of a sanitizer).

Every device allocation of a context is followed by 256 canary bytes of 0xA5. These tests run
every entry point of the hot path and its extensions on shapes that reach the edge cases
(budgets below, at and above the token count, cut clusters held in shared memory and in the
global key scratch, the pending ring at a window's end, splits, the fp8 copy, per-head
selection, selected-id outputs), then require every canary to be intact. The outputs are
checked against the oracle elsewhere; here the check is that nothing else was written.
"""
import numpy as np
import pytest
import torch

import synth_inputs as si
from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


def _layer(seed, B, Hkv, n, n_centers, layer=0):
    K = np.stack([np.stack([si.keys_values(seed, si.unit_id(layer, b, h, B, Hkv), n, n_centers)[0]
                            for h in range(Hkv)]) for b in range(B)])
    V = np.stack([np.stack([si.keys_values(seed, si.unit_id(layer, b, h, B, Hkv), n, n_centers)[1]
                            for h in range(Hkv)]) for b in range(B)])
    return to_dev(K), to_dev(V)


def _decode_all(ctx, B, Hkv, G, n, budgets, seed, mixed_C=None):
    for i, budget in enumerate(budgets):
        q = to_dev(np.stack([si.queries(seed, 0, b, len(budgets), Hkv * G)[i] for b in range(B)]))
        out = torch.empty(B, Hkv * G, 128, device="cuda", dtype=torch.float32)
        sel = torch.empty(B, Hkv, budget, device="cuda", dtype=torch.int32)
        cnt = torch.empty(B, Hkv, device="cuda", dtype=torch.int32)
        ctx.select_and_attend(0, q, budget, out, sel, cnt)
        outh = torch.empty(B, Hkv * G, 128, device="cuda", dtype=torch.float32)
        selh = torch.empty(B, Hkv * G, budget, device="cuda", dtype=torch.int32)
        cnth = torch.empty(B, Hkv * G, device="cuda", dtype=torch.int32)
        ctx.select_and_attend_per_head(0, q, budget, outh, selh, cnth)
        if mixed_C is not None:
            for n_near in (0, 3, mixed_C):
                ctx.select_and_attend_mixed(0, q, budget, n_near, out, sel, cnt)
    torch.cuda.synchronize()
    ctx.check_device_error()


@pytest.mark.parametrize("B,Hkv,G,n,C_,n_centers", [(2, 2, 4, 3000, 40, 40), (1, 2, 4, 6016, 8, 8)])
def test_no_kernel_writes_past_a_buffer(B, Hkv, G, n, C_, n_centers):
    import recallable_kv_cache_cosine_b200 as ckv
    seed, W = 31, 320
    ctx = ckv.ClusterKV(1, B, Hkv, Hkv * G, capacity=n + W, max_clusters=C_ + 8, seed=seed)
    try:
        assert ctx.damaged_canaries() == 0
        K, V = _layer(seed, B, Hkv, n, n_centers)
        ctx.cluster_prefill(0, K, V, C_)
        ctx.enable_fp8()
        # below, at and above the token count; cut clusters in shared and in global memory
        _decode_all(ctx, B, Hkv, G, n, [16, 17, 300, 2000, n - 1, n, n + 100], seed, mixed_C=C_)
        assert ctx.damaged_canaries() == 0
        # a full window of appends (the pending ring's end), decodes in between, re-clustering
        ka = torch.randn(W, B, Hkv, 128, device="cuda").to(torch.bfloat16)
        va = torch.randn(W, B, Hkv, 128, device="cuda").to(torch.bfloat16)
        for t in range(W):
            ctx.append_kv(0, ka[t], va[t])
            if t in (0, W // 2, W - 1):
                _decode_all(ctx, B, Hkv, G, n, [16 + t + 1, 600], seed + t)
        ctx.recluster_increment(0)
        _decode_all(ctx, B, Hkv, G, n, [400, n + W], seed + 1, mixed_C=C_)
        # splits up to the cluster capacity
        ctx.split_drifted_clusters(0, 0.0, 8)
        _decode_all(ctx, B, Hkv, G, n, [500], seed + 2, mixed_C=C_)
        torch.cuda.synchronize()
        ctx.check_device_error()
        assert ctx.damaged_canaries() == 0
    finally:
        ctx.close()
