"""ClusterKV semantic-cluster KV recall on B200 (sm_100a): Python binding.

A thin ctypes layer over ``_lib/libckv.so``, whose C-ABI is declared in ``include/ckv.h``.
The binding only marshals arguments. Every step of the hot path runs in the library's
CUDA kernels. PyTorch supplies device memory (``data_ptr()``) and the current CUDA stream.

If the shared library is missing, importing this module raises. There is no CPU fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

__all__ = ["ClusterKV", "Config", "CkvError", "lib", "LIB_PATH", "kmeans_init", "kmeans_assign",
           "kmeans_update"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libckv.so")

CKV_OK, CKV_EINVAL, CKV_ENOMEM, CKV_ECUDA, CKV_ECAPACITY, CKV_ETIMEOUT, CKV_ESTATE = 0, -1, -2, -3, -4, -5, -6


class CkvError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {msg} (code {code})")
        self.code = code


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("batch", C.c_int32), ("n_kv_heads", C.c_int32),
                ("n_q_heads", C.c_int32), ("head_dim", C.c_int32), ("n_sink", C.c_int32),
                ("window", C.c_int32), ("new_clusters", C.c_int32), ("iters", C.c_int32),
                ("max_clusters", C.c_int32), ("capacity", C.c_int64), ("seed", C.c_uint64)]


class LayerInfo(C.Structure):
    _fields_ = [("n_total", C.c_int64), ("m", C.c_int64), ("C", C.c_int32), ("pending", C.c_int32),
                ("windows", C.c_int32), ("prefilled", C.c_int32)]


class UnitBuffers(C.Structure):
    _fields_ = [("mu", C.c_void_p), ("offsets", C.c_void_p), ("ids", C.c_void_p), ("kp", C.c_void_p),
                ("vp", C.c_void_p), ("sp_k", C.c_void_p), ("sp_v", C.c_void_p)]


# exported symbol -> (restype, argtypes); also the list the ABI test checks against ckv.h
P, I32, I64, U64 = C.c_void_p, C.c_int32, C.c_int64, C.c_uint64
SIGNATURES = {
    "ckv_config_default": (C.c_int, [P]),
    "ckv_create": (C.c_int, [P, P]),
    "ckv_destroy": (C.c_int, [P]),
    "ckv_strerror": (C.c_char_p, [C.c_int]),
    "ckv_last_error": (C.c_char_p, []),
    "ckv_device_bytes": (C.c_int64, [P]),
    "ckv_check_canaries": (C.c_int, [P, P]),
    "cluster_prefill": (C.c_int, [P, I32, P, P, I64, I32, P]),
    "select_and_attend": (C.c_int, [P, I32, P, I32, P, P, P, P]),
    "select_and_attend_per_head": (C.c_int, [P, I32, P, I32, P, P, P, P]),
    "ckv_append_kv": (C.c_int, [P, I32, P, P, P]),
    "recluster_increment": (C.c_int, [P, I32, P]),
    "recluster_increment_traced": (C.c_int, [P, I32, P, P, P]),
    "recluster_begin": (C.c_int, [P, I32, P]),
    "recluster_finish": (C.c_int, [P, I32, P]),
    "split_drifted_clusters": (C.c_int, [P, I32, C.c_float, I32, P, P, P]),
    "ckv_get_layer_info": (C.c_int, [P, I32, P]),
    "ckv_export_unit": (C.c_int, [P, I32, I32, I32, P, P]),
    "ckv_import_unit": (C.c_int, [P, I32, I32, I32, I64, I32, I32, P, P]),
    "ckv_check_device_error": (C.c_int, [P, P]),
    "ckv_debug_expire_wait": (C.c_int, [P, U64, P, P]),
    "ckv_enable_fp8": (C.c_int, [P, P]),
    "select_and_attend_mixed": (C.c_int, [P, I32, P, I32, I32, P, P, P, P]),
    "ckv_export_unit_fp8": (C.c_int, [P, I32, I32, I32, P, P, P, P, P]),
    "ckv_kmeans_init": (C.c_int, [P, P, I64, I64, I64, I32, I32, U64, I64, U64, P, P, P, P]),
    "ckv_kmeans_assign": (C.c_int, [P, P, I64, I64, I64, I32, P, I32, P, P]),
    "ckv_kmeans_update": (C.c_int, [P, P, I64, I64, I64, I32, P, I32, P, P, P, P, P]),
    "ckv_kmeans_update_noalloc": (C.c_int, [P, I64, I64, I64, I32, P, I32, P, P, P, P, P]),
}

_lib = None


def lib():
    """Load the CUDA library (built by ``recallable_kv_cache_cosine_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m recallable_kv_cache_cosine_b200.build` (no fallback exists)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(rc: int, where: str):
    if rc != CKV_OK:
        msg = lib().ckv_last_error().decode(errors="replace")
        raise CkvError(rc, where, msg or lib().ckv_strerror(rc).decode())


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _bf16(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
    return _ptr(t)


class ClusterKV:
    """One context: the cluster stores of ``n_layers`` layers of a GQA attention stack."""

    def __init__(self, n_layers: int, batch: int, n_kv_heads: int, n_q_heads: int,
                 capacity: int, max_clusters: int, seed: int = 0, n_sink: int = 16,
                 window: int = 320, new_clusters: int = 4, iters: int = 10):
        cfg = Config()
        _check(lib().ckv_config_default(C.byref(cfg)), "ckv_config_default")
        cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.n_q_heads = n_layers, batch, n_kv_heads, n_q_heads
        cfg.capacity, cfg.max_clusters, cfg.seed = capacity, max_clusters, seed
        cfg.n_sink, cfg.window, cfg.new_clusters, cfg.iters = n_sink, window, new_clusters, iters
        self.cfg = cfg
        self._ctx = C.c_void_p()
        _check(lib().ckv_create(C.byref(cfg), C.byref(self._ctx)), "ckv_create")

    # -- lifecycle
    def close(self):
        if self._ctx:
            lib().ckv_destroy(self._ctx)
            self._ctx = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def device_bytes(self) -> int:
        return lib().ckv_device_bytes(self._ctx)

    @property
    def group(self) -> int:
        return self.cfg.n_q_heads // self.cfg.n_kv_heads

    # -- the hot path
    def cluster_prefill(self, layer: int, K: torch.Tensor, V: torch.Tensor, C_: int, stream=None):
        """K, V: [batch, n_kv_heads, n, 128] bf16 on the device."""
        n = K.shape[2]
        _check(lib().cluster_prefill(self._ctx, layer, _bf16(K, "K"), _bf16(V, "V"), n, C_,
                                     _stream(stream)), "cluster_prefill")

    def select_and_attend(self, layer: int, q: torch.Tensor, budget: int, out: torch.Tensor,
                          sel_idx: torch.Tensor | None = None, sel_count: torch.Tensor | None = None,
                          stream=None):
        """q: [batch, n_q_heads, 128] bf16; out: same shape fp32."""
        if out.dtype != torch.float32 or not out.is_cuda:
            raise TypeError("out must be a CUDA float32 tensor")
        _check(lib().select_and_attend(self._ctx, layer, _bf16(q, "q"), budget, _ptr(out),
                                       _ptr(sel_idx), _ptr(sel_count), _stream(stream)),
               "select_and_attend")

    def select_and_attend_per_head(self, layer: int, q: torch.Tensor, budget: int, out: torch.Tensor,
                                   sel_idx: torch.Tensor | None = None,
                                   sel_count: torch.Tensor | None = None, stream=None):
        """One selection per query head; sel_idx [batch, n_q_heads, budget], sel_count [batch, n_q_heads]."""
        if out.dtype != torch.float32 or not out.is_cuda:
            raise TypeError("out must be a CUDA float32 tensor")
        _check(lib().select_and_attend_per_head(self._ctx, layer, _bf16(q, "q"), budget, _ptr(out),
                                                _ptr(sel_idx), _ptr(sel_count), _stream(stream)),
               "select_and_attend_per_head")

    def append_kv(self, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None):
        """k, v: [batch, n_kv_heads, 128] bf16."""
        _check(lib().ckv_append_kv(self._ctx, layer, _bf16(k, "k"), _bf16(v, "v"), _stream(stream)),
               "ckv_append_kv")

    def recluster_increment(self, layer: int, mu_trace=None, assign_trace=None, stream=None):
        _check(lib().recluster_increment_traced(self._ctx, layer, _ptr(mu_trace), _ptr(assign_trace),
                                                _stream(stream)), "recluster_increment")

    def recluster_begin(self, layer: int, stream=None):
        """Starts re-clustering the full pending window on `stream`, overlapped with decode."""
        _check(lib().recluster_begin(self._ctx, layer, _stream(stream)), "recluster_begin")

    def recluster_finish(self, layer: int, stream=None):
        """Makes `stream` wait for that re-clustering and switches the layer to its clusters."""
        _check(lib().recluster_finish(self._ctx, layer, _stream(stream)), "recluster_finish")

    def split_drifted_clusters(self, layer: int, threshold: float, max_splits: int,
                               drift: torch.Tensor | None = None, splits: torch.Tensor | None = None,
                               stream=None) -> torch.Tensor:
        """Splits the layer's clusters whose drift (mean cosine distance of the members to
        the centroid) is above `threshold`, at most `max_splits` per unit; the layer's
        cluster count grows by exactly min(max_splits, room left). drift: optional CUDA
        float32 [units, C] receiving every cluster's drift; splits: optional CUDA int32
        [units] receiving the clusters split per unit (both filled asynchronously). Returns
        `splits`."""
        if drift is not None and (drift.dtype != torch.float32 or not drift.is_cuda):
            raise TypeError("drift must be a CUDA float32 tensor")
        if splits is not None and (splits.dtype != torch.int32 or not splits.is_cuda):
            raise TypeError("splits must be a CUDA int32 tensor")
        _check(lib().split_drifted_clusters(self._ctx, layer, float(threshold), int(max_splits),
                                            _ptr(drift), _ptr(splits), _stream(stream)),
               "split_drifted_clusters")
        return splits

    # -- inspection
    def layer_info(self, layer: int) -> LayerInfo:
        info = LayerInfo()
        _check(lib().ckv_get_layer_info(self._ctx, layer, C.byref(info)), "ckv_get_layer_info")
        return info

    def export_unit(self, layer: int, b: int, h: int, stream=None) -> dict:
        """Copies one unit's store into new CPU tensors."""
        info = self.layer_info(layer)
        sp = self.cfg.n_sink + info.pending
        out = {
            "mu": torch.empty(info.C, 128, dtype=torch.float32),
            "offsets": torch.empty(info.C + 1, dtype=torch.int32),
            "ids": torch.empty(info.m, dtype=torch.int32),
            "kp": torch.empty(info.m, 128, dtype=torch.bfloat16),
            "vp": torch.empty(info.m, 128, dtype=torch.bfloat16),
            "sp_k": torch.empty(sp, 128, dtype=torch.bfloat16),
            "sp_v": torch.empty(sp, 128, dtype=torch.bfloat16),
        }
        buf = UnitBuffers(*[C.c_void_p(out[k].data_ptr()) if out[k].numel() else None
                            for k in ("mu", "offsets", "ids", "kp", "vp", "sp_k", "sp_v")])
        _check(lib().ckv_export_unit(self._ctx, layer, b, h, C.byref(buf), _stream(stream)),
               "ckv_export_unit")
        return out

    def import_unit(self, layer: int, b: int, h: int, store: dict, pending: int, stream=None):
        """Loads one unit's store from tensors (CPU or CUDA) with the export layout."""
        t = {k: store[k].contiguous() for k in ("mu", "offsets", "ids", "kp", "vp", "sp_k", "sp_v")}
        buf = UnitBuffers(*[C.c_void_p(t[k].data_ptr()) for k in ("mu", "offsets", "ids", "kp", "vp",
                                                                  "sp_k", "sp_v")])
        m, C_ = t["kp"].shape[0], t["mu"].shape[0]
        _check(lib().ckv_import_unit(self._ctx, layer, b, h, m, C_, pending, C.byref(buf),
                                     _stream(stream)), "ckv_import_unit")
        self._keep = t  # keep host memory alive until the next import

    def check_device_error(self, stream=None):
        _check(lib().ckv_check_device_error(self._ctx, _stream(stream)), "ckv_check_device_error")

    def damaged_canaries(self) -> int:
        """Number of device allocations whose trailing canary bytes changed (waits for the
        device)."""
        n = C.c_int32(0)
        _check(lib().ckv_check_canaries(self._ctx, C.byref(n)), "ckv_check_canaries")
        return int(n.value)

    def enable_fp8(self, stream=None):
        """Keep an fp8 (e4m3, per-row scale) copy of every layer's clustered rows."""
        _check(lib().ckv_enable_fp8(self._ctx, _stream(stream)), "ckv_enable_fp8")

    def select_and_attend_mixed(self, layer: int, q, budget: int, n_near: int, out, sel_idx=None,
                                sel_count=None, stream=None):
        """select_and_attend with clusters at walk rank >= n_near attended from the fp8 copy."""
        _check(lib().select_and_attend_mixed(self._ctx, layer, _bf16(q, "q"), budget, n_near, _ptr(out),
                                             _ptr(sel_idx), _ptr(sel_count), _stream(stream)),
               "select_and_attend_mixed")
        return out

    def export_unit_fp8(self, layer: int, b: int, h: int, stream=None):
        """One unit's fp8 copy as CPU tensors: k8, v8 uint8 [m, 128]; ks, vs float32 [m]."""
        m = self.layer_info(layer).m
        k8 = torch.empty(m, 128, dtype=torch.uint8)
        v8 = torch.empty_like(k8)
        ks = torch.empty(m, dtype=torch.float32)
        vs = torch.empty_like(ks)
        _check(lib().ckv_export_unit_fp8(self._ctx, layer, b, h, _ptr(k8), _ptr(ks), _ptr(v8), _ptr(vs),
                                         _stream(stream)), "ckv_export_unit_fp8")
        return {"k8": k8, "ks": ks, "v8": v8, "vs": vs}

    def debug_expire_wait(self, limit_ns: int, waited_ns=None, stream=None):
        """Test hook: one bounded device wait that nothing completes runs out after
        ``limit_ns``; the error word is then set (see ``check_device_error``)."""
        _check(lib().ckv_debug_expire_wait(self._ctx, int(limit_ns), _ptr(waited_ns), _stream(stream)),
               "ckv_debug_expire_wait")

    # -- stage-level K-means calls (same kernels as cluster_prefill)
    def kmeans_init(self, keys, row0, m, C_, seed, unit_base=0, window=0, init_idx=None, mu=None,
                    mu_hat=None, stream=None):
        U, n_rows = keys.shape[0], keys.shape[1]
        mu = mu if mu is not None else torch.empty(U, C_, 128, device=keys.device, dtype=torch.float32)
        mu_hat = mu_hat if mu_hat is not None else torch.empty(U, C_, 128, device=keys.device,
                                                               dtype=torch.bfloat16)
        _check(lib().ckv_kmeans_init(self._ctx, _bf16(keys, "keys"), n_rows, row0, m, U, C_, seed,
                                     unit_base, window, _ptr(init_idx), _ptr(mu), _ptr(mu_hat),
                                     _stream(stream)), "ckv_kmeans_init")
        return mu, mu_hat

    def kmeans_assign(self, keys, row0, m, mu_hat, assign=None, stream=None):
        U, n_rows, C_ = keys.shape[0], keys.shape[1], mu_hat.shape[1]
        assign = assign if assign is not None else torch.empty(U, m, device=keys.device,
                                                               dtype=torch.int32)
        _check(lib().ckv_kmeans_assign(self._ctx, _bf16(keys, "keys"), n_rows, row0, m, U,
                                       _bf16(mu_hat, "mu_hat"), C_, _ptr(assign), _stream(stream)),
               "ckv_kmeans_assign")
        return assign

    def kmeans_update(self, keys, row0, m, assign, mu, mu_hat=None, offsets=None, perm=None,
                      stream=None):
        U, n_rows, C_ = keys.shape[0], keys.shape[1], mu.shape[1]
        dev = keys.device
        mu_hat = mu_hat if mu_hat is not None else torch.empty(U, C_, 128, device=dev, dtype=torch.bfloat16)
        offsets = offsets if offsets is not None else torch.empty(U, C_ + 1, device=dev, dtype=torch.int32)
        perm = perm if perm is not None else torch.empty(U, m, device=dev, dtype=torch.int32)
        _check(lib().ckv_kmeans_update(self._ctx, _bf16(keys, "keys"), n_rows, row0, m, U,
                                       _ptr(assign), C_, _ptr(mu), _ptr(mu_hat), _ptr(offsets),
                                       _ptr(perm), _stream(stream)), "ckv_kmeans_update")
        return mu, mu_hat, offsets, perm


def kmeans_init(ctx: ClusterKV, *a, **k):
    return ctx.kmeans_init(*a, **k)


def kmeans_assign(ctx: ClusterKV, *a, **k):
    return ctx.kmeans_assign(*a, **k)


def kmeans_update(ctx: ClusterKV, *a, **k):
    return ctx.kmeans_update(*a, **k)
