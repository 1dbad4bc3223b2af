"""The Python binding fails loudly (runs without a GPU): wrong tensor types are refused
before any library call, and a context cannot be created without a CUDA device (there is
no CPU fallback)."""
import ctypes as C

import pytest
import torch

import recallable_kv_cache_cosine_b200 as ckv


def _detached():
    """A binding object with a null context: any call that reached the library would fail
    with CKV_EINVAL, so a TypeError proves the check ran first."""
    obj = ckv.ClusterKV.__new__(ckv.ClusterKV)
    obj._ctx = C.c_void_p()
    cfg = ckv.Config()
    ckv.lib().ckv_config_default(C.byref(cfg))
    cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.n_q_heads = 1, 1, 8, 32
    obj.cfg = cfg
    return obj


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_no_context():
    with pytest.raises(ckv.CkvError):
        ckv.ClusterKV(1, 1, 8, 32, capacity=4096, max_clusters=64)


def test_host_or_mistyped_tensors_are_refused_before_the_library():
    obj = _detached()
    q = torch.zeros(1, 32, 128, dtype=torch.bfloat16)
    out = torch.zeros(1, 32, 128, dtype=torch.float32)
    with pytest.raises(TypeError):
        obj.select_and_attend(0, q, 1024, out)
    with pytest.raises(TypeError):
        obj.select_and_attend_per_head(0, q, 1024, out)
    with pytest.raises(TypeError):
        obj.select_and_attend(0, q, 1024, out.double())
    k = torch.zeros(1, 8, 128, dtype=torch.float16)
    with pytest.raises(TypeError):
        obj.append_kv(0, k, k)
    with pytest.raises(TypeError):
        obj.cluster_prefill(0, torch.zeros(1, 8, 64, 128), torch.zeros(1, 8, 64, 128), 4)
    with pytest.raises(TypeError):
        obj.split_drifted_clusters(0, 0.5, 4, drift=torch.zeros(8, 4))


def test_null_context_calls_raise_with_the_reason():
    obj = _detached()
    with pytest.raises(ckv.CkvError) as e:
        obj.recluster_increment(0, stream=0)  # an explicit (null) stream handle
    assert e.value.code == ckv.CKV_EINVAL and "context" in str(e.value)
    with pytest.raises(ckv.CkvError):
        obj.split_drifted_clusters(0, 0.5, 4, stream=0)
    with pytest.raises(ckv.CkvError):
        obj.layer_info(0)
