"""Failure detection on the device: a bounded wait that runs out is reported, not hung.

Every wait inside the library's kernels gives up after a limit, sets the context's device
error word and lets its kernel unwind; ckv_check_device_error then returns CKV_ETIMEOUT.
The test hook ckv_debug_expire_wait makes one such wait run out on purpose (an mbarrier that
nothing completes, a 1 ms limit, no copy in flight), so the path is exercised without
faulting or hanging the GPU. Afterwards the same context must decode normally, and its
result must match the oracle.
"""
import numpy as np
import pytest
import torch

import synth_inputs as si
from gpu_helpers import check_decode_unit, store_from_export, to_dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_reports_timeout_and_context_stays_usable():
    import recallable_kv_cache_cosine_b200 as ckv
    B, Hkv, G, n, C_, budget, seed = 1, 2, 4, 1500, 20, 200, 3
    K = np.stack([si.keys_values(seed, h, n, 20)[0] for h in range(Hkv)])[None]
    V = np.stack([si.keys_values(seed, h, n, 20)[1] for h in range(Hkv)])[None]
    ctx = ckv.ClusterKV(1, B, Hkv, Hkv * G, capacity=n, max_clusters=C_, seed=seed)
    try:
        ctx.cluster_prefill(0, to_dev(K), to_dev(V), C_)
        ctx.check_device_error()
        waited = torch.zeros(1, dtype=torch.int32, device="cuda")
        ctx.debug_expire_wait(1_000_000, waited)  # 1 ms
        with pytest.raises(ckv.CkvError) as e:
            ctx.check_device_error()
        assert e.value.code == ckv.CKV_ETIMEOUT
        ns = int(waited.item()) & 0xFFFFFFFF
        assert 1_000_000 <= ns < 1_000_000_000, ns  # gave up after the limit, not at once
        ctx.check_device_error()  # reading the word cleared it
        # out-of-range limits are refused on the host, nothing is launched
        for bad in (0, 999, 2_000_000_000):
            with pytest.raises(ckv.CkvError) as e:
                ctx.debug_expire_wait(bad)
            assert e.value.code == ckv.CKV_EINVAL
        # the context still decodes, and matches the oracle
        q = si.queries(seed, 0, 0, 1, Hkv * G)[0]
        out = torch.empty(B, Hkv * G, 128, device="cuda", dtype=torch.float32)
        sel = torch.empty(B, Hkv, budget, device="cuda", dtype=torch.int32)
        cnt = torch.empty(B, Hkv, device="cuda", dtype=torch.int32)
        ctx.select_and_attend(0, to_dev(q[None]), budget, out, sel, cnt)
        torch.cuda.synchronize()
        ctx.check_device_error()
        for h in range(Hkv):
            st = store_from_export(ctx.export_unit(0, 0, h))
            check_decode_unit(st, q[h * G:(h + 1) * G], budget, out[0, h * G:(h + 1) * G].cpu().numpy(),
                              sel[0, h].cpu().numpy(), int(cnt[0, h]))
    finally:
        ctx.close()
