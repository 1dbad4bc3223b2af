"""ClusterKV CPU oracle: TEST INFRASTRUCTURE ONLY.

This is a ctypes front end to ``ckv_oracle.c``, a plain fp64 C restatement of the
ClusterKV hot path. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it. The CUDA library never does, and it shares no code with
it.

bf16 tensors are passed as their raw ``uint16`` bit patterns. Section references are to
the ClusterKV explainer page "大模型KV Cache压缩技术：ClusterKV的语义空间优化".
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os

import numpy as np

from . import build as _build

D = 128
N_SINK = 16
WINDOW = 320
NEW_CLUSTERS = 4
ITERS = 10

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build.build())
        P = C.c_void_p
        i32, i64, u64, u16 = C.c_int32, C.c_int64, C.c_uint64, C.c_uint16
        sig = {
            "orc_bf16_to_double": (C.c_double, [u16]),
            "orc_bf16_from_double": (u16, [C.c_double]),
            "orc_bf16_from_double_array": (None, [P, i64, P]),
            "orc_splitmix64_next": (u64, [P]),
            "orc_bounded": (C.c_uint32, [u64, C.c_uint32]),
            "orc_stream_key": (u64, [u64, i64, u64]),
            "orc_init_indices": (None, [i64, i32, u64, P]),
            "orc_normalize": (None, [P, i32, P]),
            "orc_assign": (None, [P, i64, P, i32, P]),
            "orc_assign_gap": (None, [P, i64, P, i32, P, P]),
            "orc_update": (None, [P, i64, P, i32, P, P, P]),
            "orc_kmeans": (None, [P, i64, i32, i32, P, P, P, P, P]),
            "orc_prefill_unit": (None, [P, P, i64, i32, i32, i32, u64, P, P, P, P, P, P]),
            "orc_recluster_window": (None, [P, P, i64, i32, i32, u64, i64, P, P, P, P, P, P]),
            "orc_cluster_drift": (None, [P, P, P, i32, P]),
            "orc_split_key": (u64, [u64, i64, u64, i32]),
            "orc_split_drifted": (i32, [P, P, P, P, P, i32, C.c_double, i32, i32, u64, i64,
                                        u64, P, P, P, P, P, P]),
            "orc_e4m3_from_float": (C.c_uint8, [C.c_float]),
            "orc_e4m3_from_float_array": (None, [P, i64, P]),
            "orc_e4m3_to_double": (C.c_double, [C.c_uint8]),
            "orc_quantize_rows_e4m3": (None, [P, i64, P, P]),
            "orc_attend_mixed": (None, [P, P, i32, P, P, i32, i32, P, P, P, P, P]),
            "orc_group_query": (None, [P, i32, P]),
            "orc_select": (i32, [P, P, i32, P, P, P, P]),
            "orc_attend": (None, [P, P, i32, P, i32, P]),
            "orc_dense_attention": (None, [P, P, i64, P, i32, P]),
            "orc_set_threads": (i32, [i32]),
            "orc_prefill_batch": (None, [i32, P, P, i64, i32, i32, i32, P, P, P, P, P, P, P]),
            "orc_select_attend_batch": (None, [i32, i32, i32, i64, i32, P, P, P, P, P, P, P, P,
                                               i32, i32, P, P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(_lib, name)
            f.restype = res
            f.argtypes = args
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, f"expected bf16 bit patterns (uint16), got {a.dtype}"
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


# ------------------------------------------------------------------ primitives

def bf16_to_f64(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_from_f64(x) -> np.ndarray:
    x = _f64(x)
    out = np.empty(x.shape, np.uint16)
    lib().orc_bf16_from_double_array(_p(x), x.size, _p(out))
    return out


def splitmix64(state: int, count: int) -> list[int]:
    s = C.c_uint64(state)
    return [lib().orc_splitmix64_next(C.byref(s)) for _ in range(count)]


def bounded(x: int, r: int) -> int:
    return lib().orc_bounded(x, r)


def stream_key(seed: int, unit: int, window: int) -> int:
    return lib().orc_stream_key(seed, unit, window)


def init_indices(m: int, C_: int, key: int) -> np.ndarray:
    out = np.empty(C_, np.int32)
    lib().orc_init_indices(m, C_, key, _p(out))
    return out


def normalize(mu) -> np.ndarray:
    mu = _f64(mu)
    out = np.empty(mu.shape, np.uint16)
    lib().orc_normalize(_p(mu), mu.shape[0], _p(out))
    return out


def assign(keys, mu_hat) -> np.ndarray:
    keys, mu_hat = _u16(keys), _u16(mu_hat)
    out = np.empty(keys.shape[0], np.int32)
    lib().orc_assign(_p(keys), keys.shape[0], _p(mu_hat), mu_hat.shape[0], _p(out))
    return out


def assign_gap(keys, mu_hat, other) -> np.ndarray:
    keys, mu_hat, other = _u16(keys), _u16(mu_hat), _i32(other)
    out = np.empty(keys.shape[0], np.float64)
    lib().orc_assign_gap(_p(keys), keys.shape[0], _p(mu_hat), mu_hat.shape[0], _p(other), _p(out))
    return out


def update(keys, assignment, C_: int, mu_prev):
    """One centroid update. Returns (mu, offsets, perm)."""
    keys, assignment = _u16(keys), _i32(assignment)
    mu = _f64(mu_prev).copy()
    offsets = np.empty(C_ + 1, np.int32)
    perm = np.empty(keys.shape[0], np.int32)
    lib().orc_update(_p(keys), keys.shape[0], _p(assignment), C_, _p(mu), _p(offsets), _p(perm))
    return mu, offsets, perm


def kmeans(keys, C_: int, iters: int, init):
    """Returns (mu, offsets, perm, assign) after ``iters`` Lloyd iterations."""
    keys, init = _u16(keys), _i32(init)
    m = keys.shape[0]
    mu = np.empty((C_, D), np.float64)
    offsets = np.empty(C_ + 1, np.int32)
    perm = np.empty(m, np.int32)
    a = np.empty(m, np.int32)
    lib().orc_kmeans(_p(keys), m, C_, iters, _p(init), _p(mu), _p(offsets), _p(perm), _p(a))
    return mu, offsets, perm, a


# ------------------------------------------------------------------ unit store

@dataclasses.dataclass
class Store:
    """Cluster store of one unit (explainer section 4.1's cluster-contiguous layout)."""
    sp_k: np.ndarray      # [n_sink + pending, 128] sinks then pending rows
    sp_v: np.ndarray
    kp: np.ndarray        # [m, 128] clustered rows, cluster-major
    vp: np.ndarray
    ids: np.ndarray       # [m] original token id per clustered row
    offsets: np.ndarray   # [C + 1]
    mu: np.ndarray        # [C, 128] float64
    n_sink: int = N_SINK
    windows: int = 0      # incremental re-clusterings done so far

    @property
    def C(self) -> int:
        return self.mu.shape[0]

    @property
    def m(self) -> int:
        return self.kp.shape[0]

    @property
    def pending(self) -> int:
        return self.sp_k.shape[0] - self.n_sink

    @property
    def n_total(self) -> int:
        return self.n_sink + self.m + self.pending

    def _c(self):
        class _S(C.Structure):
            _fields_ = [("n_sink", C.c_int32), ("pending", C.c_int32), ("C", C.c_int32),
                        ("m", C.c_int64), ("sp_k", C.c_void_p), ("sp_v", C.c_void_p),
                        ("kp", C.c_void_p), ("vp", C.c_void_p), ("ids", C.c_void_p),
                        ("offsets", C.c_void_p), ("mu", C.c_void_p)]
        for name in ("sp_k", "sp_v", "kp", "vp"):
            setattr(self, name, _u16(getattr(self, name)))
        self.ids, self.offsets, self.mu = _i32(self.ids), _i32(self.offsets), _f64(self.mu)
        return _S(self.n_sink, self.pending, self.C, self.m, self.sp_k.ctypes.data,
                  self.sp_v.ctypes.data, self.kp.ctypes.data, self.vp.ctypes.data,
                  self.ids.ctypes.data, self.offsets.ctypes.data, self.mu.ctypes.data)


def prefill_unit(K, V, C_: int, key: int, iters: int = ITERS, n_sink: int = N_SINK):
    """Prefill clustering of one unit. Returns (Store, assign of the non-sink tokens)."""
    K, V = _u16(K), _u16(V)
    n = K.shape[0]
    m = n - n_sink
    kp = np.empty((m, D), np.uint16)
    vp = np.empty((m, D), np.uint16)
    ids = np.empty(m, np.int32)
    offsets = np.empty(C_ + 1, np.int32)
    mu = np.empty((C_, D), np.float64)
    a = np.empty(m, np.int32)
    lib().orc_prefill_unit(_p(K), _p(V), n, n_sink, C_, iters, key, _p(kp), _p(vp), _p(ids),
                           _p(offsets), _p(mu), _p(a))
    st = Store(K[:n_sink].copy(), V[:n_sink].copy(), kp, vp, ids, offsets, mu, n_sink)
    return st, a


def append(st: Store, k, v) -> Store:
    """Append one generated token's K/V row to the pending rows."""
    return dataclasses.replace(st, sp_k=np.concatenate([st.sp_k, _u16(k).reshape(1, D)]),
                               sp_v=np.concatenate([st.sp_v, _u16(v).reshape(1, D)]))


def recluster(st: Store, seed: int, unit: int, C_new: int = NEW_CLUSTERS,
              iters: int = ITERS, window: int = WINDOW):
    """Incremental clustering of a full pending window (explainer section 3.2).
    Returns (new Store, window assignment)."""
    assert st.pending == window, "recluster needs a full pending window"
    wk = np.ascontiguousarray(st.sp_k[st.n_sink:])
    wv = np.ascontiguousarray(st.sp_v[st.n_sink:])
    key = stream_key(seed, unit, st.windows + 1)
    kp = np.empty((window, D), np.uint16)
    vp = np.empty((window, D), np.uint16)
    ids = np.empty(window, np.int32)
    offs = np.empty(C_new + 1, np.int32)
    mu = np.empty((C_new, D), np.float64)
    a = np.empty(window, np.int32)
    first_id = st.n_sink + st.m
    lib().orc_recluster_window(_p(wk), _p(wv), window, C_new, iters, key, first_id, _p(kp),
                               _p(vp), _p(ids), _p(offs), _p(mu), _p(a))
    new = Store(st.sp_k[:st.n_sink].copy(), st.sp_v[:st.n_sink].copy(),
                np.concatenate([st.kp, kp]), np.concatenate([st.vp, vp]),
                np.concatenate([st.ids, ids]),
                np.concatenate([st.offsets, st.m + offs[1:]]).astype(np.int32),
                np.concatenate([st.mu, mu]), st.n_sink, st.windows + 1)
    return new, a


def cluster_drift(st: Store) -> np.ndarray:
    """Mean cosine distance of each cluster's members to its centroid (explainer section
    3.2, drift detection). Returns [C] float64."""
    s = st._c()
    out = np.empty(max(st.C, 1), np.float64)
    lib().orc_cluster_drift(s.kp, s.offsets, s.mu, st.C, _p(out))
    return out[: st.C].copy()


def split_key(seed: int, unit: int, window: int, c: int) -> int:
    return lib().orc_split_key(seed, unit, window, c)


def split_drifted(st: Store, threshold: float, seed: int, unit: int, room: int,
                  iters: int = ITERS):
    """One split pass (explainer section 3.2, decode phase): every cluster with drift above
    ``threshold`` and at least two members is split by 2-cluster cosine K-means, at most
    ``room`` of them (lowest index first). Returns (new Store, split flags [C])."""
    st._c()
    C_, m = st.C, st.m
    kp2 = np.empty_like(st.kp)
    vp2 = np.empty_like(st.vp)
    ids2 = np.empty_like(st.ids)
    offs2 = np.empty(C_ + max(room, 0) + 1, np.int32)
    mu2 = np.empty((C_ + max(room, 0), D), np.float64)
    flags = np.empty(max(C_, 1), np.int32)
    n = lib().orc_split_drifted(_p(st.kp), _p(st.vp), _p(st.ids), _p(st.offsets), _p(st.mu), C_,
                                float(threshold), room, iters, seed, unit, st.windows,
                                _p(kp2), _p(vp2), _p(ids2), _p(offs2), _p(mu2), _p(flags))
    assert offs2[n] == m
    new = dataclasses.replace(st, kp=kp2, vp=vp2, ids=ids2, offsets=offs2[: n + 1].copy(),
                              mu=mu2[:n].copy())
    return new, flags[:C_].copy()


def pad_clusters(st: Store, C_total: int) -> Store:
    """Appends empty clusters (zero centroid, no rows) up to ``C_total``. An empty cluster
    never adds a row to a selection."""
    extra = C_total - st.C
    assert extra >= 0
    return dataclasses.replace(
        st, offsets=np.concatenate([st.offsets, np.full(extra, st.m, np.int32)]).astype(np.int32),
        mu=np.concatenate([st.mu, np.zeros((extra, D))]))


@dataclasses.dataclass
class Selection:
    ids: np.ndarray       # original token ids, selection order
    rows: np.ndarray      # >= 0: clustered row; < 0: sink/pending row (-r - 1)
    n_whole: int
    cut: int              # cut cluster, -1 if none
    r: int                # tokens taken from the cut cluster
    scores: np.ndarray    # [C] qbar . mu_c


def group_query(q) -> np.ndarray:
    q = _u16(q)
    out = np.empty(D, np.float64)
    lib().orc_group_query(_p(q), q.shape[0], _p(out))
    return out


def select(st: Store, q, budget: int) -> Selection:
    """select_clusters of explainer section 3.3 for one KV head. q: [G, 128] bf16 bits."""
    return select_qbar(st, group_query(q), budget)


def select_qbar(st: Store, qbar, budget: int) -> Selection:
    qbar = _f64(qbar)
    s = st._c()
    cap = max(budget, 1)
    ids = np.empty(cap, np.int32)
    rows = np.empty(cap, np.int32)
    info = np.empty(4, np.int32)
    scores = np.empty(max(st.C, 1), np.float64)
    n = lib().orc_select(C.byref(s), _p(qbar), budget, _p(ids), _p(rows), _p(info), _p(scores))
    if n < 0:
        raise ValueError("budget smaller than sinks + pending")
    return Selection(ids[:n].copy(), rows[:n].copy(), int(info[0]), int(info[1]), int(info[2]),
                     scores[:st.C].copy())


def attend(st: Store, q, sel: Selection) -> np.ndarray:
    """Attention of each query head over the selected rows. Returns [G, 128] float64."""
    q = _u16(q)
    s = st._c()
    rows = _i32(sel.rows)
    out = np.empty((q.shape[0], D), np.float64)
    lib().orc_attend(C.byref(s), _p(q), q.shape[0], _p(rows), rows.shape[0], _p(out))
    return out


def select_and_attend(st: Store, q, budget: int):
    sel = select(st, q, budget)
    return attend(st, q, sel), sel


# ------------------------------------------------------------------ far clusters in fp8

def e4m3_from_f32(x) -> np.ndarray:
    """fp8 e4m3 codes of float32 values (ties to even, saturating at 448)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_from_float_array(_p(x), x.size, _p(out))
    return out


def e4m3_to_f64(codes) -> np.ndarray:
    table = np.array([lib().orc_e4m3_to_double(b) for b in range(256)])
    return table[np.asarray(codes, dtype=np.uint8)]


def quantize_rows_e4m3(rows) -> tuple[np.ndarray, np.ndarray]:
    """Per-row fp8 copy of bf16 rows [n, 128]: (codes uint8 [n, 128], scales float32 [n])."""
    rows = _u16(rows)
    n = rows.shape[0]
    codes = np.empty((n, D), np.uint8)
    scales = np.empty(max(n, 1), np.float32)
    lib().orc_quantize_rows_e4m3(_p(rows), n, _p(codes), _p(scales))
    return codes, scales[:n].copy()


def walk_rank(st: Store, sel: "Selection") -> np.ndarray:
    """Walk rank (0 = highest score, ties to the lower index) of every cluster."""
    order = sorted(range(st.C), key=lambda c: (-sel.scores[c], c))
    rank = np.empty(st.C, np.int32)
    rank[order] = np.arange(st.C, dtype=np.int32)
    return rank


def attend_mixed(st: Store, q, sel: "Selection", n_near: int, k8, ks, v8, vs) -> np.ndarray:
    """Attention like ``attend``, reading the selected rows of clusters at walk rank >= n_near
    from the fp8 copy (explainer section 7, mixed precision for far clusters)."""
    q = _u16(q)
    s = st._c()
    rows = _i32(sel.rows)
    rank = walk_rank(st, sel)
    clus = np.searchsorted(st.offsets, np.maximum(rows, 0), side="right") - 1
    row_rank = _i32(np.where(rows >= 0, rank[np.clip(clus, 0, max(st.C - 1, 0))], -1))
    k8, v8 = np.ascontiguousarray(k8, np.uint8), np.ascontiguousarray(v8, np.uint8)
    ks, vs = np.ascontiguousarray(ks, np.float32), np.ascontiguousarray(vs, np.float32)
    out = np.empty((q.shape[0], D), np.float64)
    lib().orc_attend_mixed(C.byref(s), _p(q), q.shape[0], _p(rows), _p(row_rank), rows.shape[0],
                           n_near, _p(k8), _p(ks), _p(v8), _p(vs), _p(out))
    return out


def dense_attention(K, V, q) -> np.ndarray:
    K, V, q = _u16(K), _u16(V), _u16(q)
    out = np.empty((q.shape[0], D), np.float64)
    lib().orc_dense_attention(_p(K), _p(V), K.shape[0], _p(q), q.shape[0], _p(out))
    return out


# ------------------------------------------------------------------ batched (timing)

def prefill_batch(K, V, C_: int, keys, iters: int = ITERS, n_sink: int = N_SINK):
    """Prefill of U units, OpenMP-parallel over units. K, V: [U, n, 128] bf16 bits."""
    K, V = _u16(K), _u16(V)
    U, n = K.shape[0], K.shape[1]
    m = n - n_sink
    keys = np.ascontiguousarray(keys, dtype=np.uint64)
    kp = np.empty((U, m, D), np.uint16)
    vp = np.empty_like(kp)
    ids = np.empty((U, m), np.int32)
    offsets = np.empty((U, C_ + 1), np.int32)
    mu = np.empty((U, C_, D), np.float64)
    a = np.empty((U, m), np.int32)
    lib().orc_prefill_batch(U, _p(K), _p(V), n, n_sink, C_, iters, _p(keys), _p(kp), _p(vp),
                            _p(ids), _p(offsets), _p(mu), _p(a))
    return kp, vp, ids, offsets, mu, a


def select_attend_batch(sp_k, sp_v, kp, vp, ids, offsets, mu, q, budget: int, n_sink: int = N_SINK):
    """select + attend of U units with equal shapes, OpenMP-parallel over units."""
    sp_k, sp_v, kp, vp, q = map(_u16, (sp_k, sp_v, kp, vp, q))
    ids, offsets, mu = _i32(ids), _i32(offsets), _f64(mu)
    U, G = q.shape[0], q.shape[1]
    out = np.empty((U, G, D), np.float64)
    sel = np.empty((U, budget), np.int32)
    cnt = np.empty(U, np.int32)
    lib().orc_select_attend_batch(U, n_sink, sp_k.shape[1] - n_sink, kp.shape[1], mu.shape[1],
                                  _p(sp_k), _p(sp_v), _p(kp), _p(vp), _p(ids), _p(offsets),
                                  _p(mu), _p(q), G, budget, _p(out), _p(sel), _p(cnt))
    return out, sel, cnt


def omp_threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def set_threads(n: int) -> int:
    """Threads of the batched (timing) calls; returns the previous setting."""
    return int(lib().orc_set_threads(n))
