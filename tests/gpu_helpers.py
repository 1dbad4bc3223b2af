"""Shared helpers for the GPU parity tests: device transfer, store conversion and
tolerance-aware comparisons against the oracle.

Tolerances:
* selected token sets: equal, except where two competing scores differ by less than 1e-5
  relative (a near-tie that fp32 scoring may break either way);
* K-means assignments: equal, except where the cosine gap between the oracle's best
  cluster and the GPU's choice is below 1e-4;
* centroids: 1e-3 max-abs;
* attention outputs: 2e-3 max-abs against the fp64 oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

SEL_REL_TOL = 1e-5
COS_GAP_TOL = 1e-4
MU_TOL = 1e-3
OUT_TOL = 2e-3


def to_dev(u16: np.ndarray, device="cuda") -> torch.Tensor:
    """bf16 bit patterns (uint16) -> CUDA bfloat16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).to(device)


def to_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def store_from_export(ex: dict, n_sink: int = 16, windows: int = 0) -> oracle.Store:
    """A GPU store exported by ClusterKV.export_unit, as an oracle Store (fp32 mu -> fp64)."""
    return oracle.Store(to_u16(ex["sp_k"]), to_u16(ex["sp_v"]), to_u16(ex["kp"]), to_u16(ex["vp"]),
                        ex["ids"].numpy().astype(np.int32), ex["offsets"].numpy().astype(np.int32),
                        ex["mu"].numpy().astype(np.float64), n_sink=n_sink, windows=windows)


def store_to_import(st: oracle.Store) -> dict:
    """An oracle Store as tensors for ClusterKV.import_unit (mu rounded to fp32)."""
    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return {"mu": torch.from_numpy(st.mu.astype(np.float32)),
            "offsets": torch.from_numpy(st.offsets.astype(np.int32)),
            "ids": torch.from_numpy(st.ids.astype(np.int32)),
            "kp": bf(st.kp), "vp": bf(st.vp), "sp_k": bf(st.sp_k), "sp_v": bf(st.sp_v)}


def fp32_store(st: oracle.Store) -> oracle.Store:
    """The same store with mu rounded to fp32 (what the GPU scores with)."""
    st2 = oracle.Store(st.sp_k, st.sp_v, st.kp, st.vp, st.ids, st.offsets,
                       st.mu.astype(np.float32).astype(np.float64), st.n_sink, st.windows)
    return st2


def _rel(a, b):
    return abs(a - b) / max(abs(a), abs(b), 1e-30)


def selection_near_tie(st: oracle.Store, q_u16: np.ndarray, sel: oracle.Selection) -> bool:
    """True if the oracle's selection hinges on a near-tie: two cluster scores near the cut,
    or the cut cluster's r-th and (r+1)-th token scores, differ by < 1e-5 relative."""
    s = sel.scores
    order = sorted(range(st.C), key=lambda c: (-s[c], c))
    if sel.cut < 0:
        return False
    k = order.index(sel.cut)
    for i in range(max(0, k - 2), min(st.C - 1, k + 2)):
        if _rel(s[order[i]], s[order[i + 1]]) < SEL_REL_TOL:
            return True
    lo, hi = st.offsets[sel.cut], st.offsets[sel.cut + 1]
    qbar = oracle.group_query(q_u16)
    t = np.sort(oracle.bf16_to_f64(st.kp[lo:hi]) @ qbar)[::-1]
    r = sel.r
    if 0 < r < len(t) and _rel(t[r - 1], t[r]) < SEL_REL_TOL:
        return True
    return False


def rows_of_ids(st: oracle.Store, ids: np.ndarray) -> np.ndarray:
    """Row references (oracle convention) of a set of original token ids."""
    pos = {int(t): j for j, t in enumerate(st.ids)}
    n_sp = st.n_sink + st.pending
    out = []
    for t in ids:
        t = int(t)
        if t < st.n_sink:
            out.append(-t - 1)
        elif t >= st.n_sink + st.m:
            out.append(-(st.n_sink + (t - st.n_sink - st.m)) - 1)
        else:
            out.append(pos[t])
    assert all(-n_sp <= r for r in out)
    return np.array(out, np.int32)


def check_decode_unit(st: oracle.Store, q_u16: np.ndarray, budget: int, gpu_out: np.ndarray,
                      gpu_ids: np.ndarray, gpu_count: int, stats: dict | None = None):
    """Checks one unit's select+attend result against the oracle on the same store."""
    sel = oracle.select(st, q_u16, budget)
    assert gpu_count == len(sel.ids), (gpu_count, len(sel.ids))
    got = gpu_ids[:gpu_count]
    assert np.all(gpu_ids[gpu_count:] == -1)
    assert len(set(got.tolist())) == gpu_count, "duplicate selected ids"
    exact = set(got.tolist()) == set(sel.ids.tolist())
    if not exact:
        assert selection_near_tie(st, q_u16, sel), "selection differs without a near-tie"
        sel = oracle.Selection(got.copy(), rows_of_ids(st, got), 0, -1, 0, sel.scores)
    want = oracle.attend(st, q_u16, sel)
    err = float(np.abs(gpu_out - want).max())
    assert err <= OUT_TOL, f"attention max-abs error {err}"
    if stats is not None:
        stats["units"] = stats.get("units", 0) + 1
        stats["near_tie"] = stats.get("near_tie", 0) + (0 if exact else 1)
        stats["max_err"] = max(stats.get("max_err", 0.0), err)
    return err


def check_assign(keys_u16: np.ndarray, mu_hat_u16: np.ndarray, gpu_assign: np.ndarray,
                 stats: dict | None = None):
    """GPU assignment vs the oracle on the same mu_hat; mismatches need a cosine gap < 1e-4."""
    want = oracle.assign(keys_u16, mu_hat_u16)
    bad = np.flatnonzero(want != gpu_assign)
    if len(bad):
        gap = oracle.assign_gap(keys_u16[bad], mu_hat_u16, gpu_assign[bad])
        assert np.all(gap < COS_GAP_TOL), f"assignment mismatch with cosine gap {gap.max()}"
        assert np.all((gpu_assign[bad] >= 0) & (gpu_assign[bad] < mu_hat_u16.shape[0]))
    if stats is not None:
        stats["keys"] = stats.get("keys", 0) + len(want)
        stats["near_tie"] = stats.get("near_tie", 0) + len(bad)
    return len(bad)


def check_mu_hat(mu_f32: np.ndarray, gpu_mu_hat_u16: np.ndarray):
    """GPU mu_hat vs the oracle's normalisation of the same mu: within one bf16 step and
    identical in all but a tiny fraction of components (fp32 vs fp64 rounding at ties)."""
    want = oracle.normalize(mu_f32.astype(np.float64))
    a = oracle.bf16_to_f64(want)
    b = oracle.bf16_to_f64(gpu_mu_hat_u16)
    diff = np.abs(a - b)
    ulp = np.maximum(np.abs(a), 1e-30) * 2.0 ** -7
    assert np.all(diff <= ulp * 1.01), "mu_hat differs by more than one bf16 step"
    frac = float((want != gpu_mu_hat_u16).mean())
    assert frac < 1e-3, f"mu_hat differs in {frac:.2e} of components"
    return frac
