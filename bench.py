#!/usr/bin/env python
"""Benchmark of the ClusterKV hot path on B200.

Metric: select+attend µs per layer-step at a 32k context and a 1k budget, with K-means
keys/s and the fraction of the HBM roofline.

Workload (one Llama-3.1-8B-shaped layer: 32 query / 8 KV heads, head_dim 128, n = 32768,
batch 1, C = 400, budget 1024), held as 32 distinct layer stores. Each decode pass then
reads ~190 MB of selected rows and centroids, more than the 126 MB L2. Inputs are
synthetic (seeded clustered mixture), already resident in HBM.

One bench step is one pass of the whole hot path:
  A. cluster_prefill of all 32 layers (sinks, seeded init, 10 Lloyd iterations of tcgen05
     assignment + counting-sort update, relayout of K and V);
  B. 64 decode steps x 32 layers of select_and_attend (queries only), one CUDA graph;
  C. one 320-token incremental window on layer 0: per token append_kv + select_and_attend,
     then recluster_increment.
`value` = device time of B / layer-steps (µs, lower is better). Per-section times, keys/s,
the roofline of the select+attend kernel, an end-to-end figure (eager API calls; per decode
step the queries copied in from pinned host memory and the outputs read back) and the
CPU oracle's time on a bounded sample of the same workload are added to the JSON line.

--impl reference times the CPU oracle instead, on the same metric.
N > 1 (torchrun): every rank runs the same workload on its own GPU (weak scaling, no
data-path collective). Times are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

METRIC = "select+attend µs per layer-step @32k ctx/1k budget; k-means keys/s; % HBM roofline"
UNIT = "us/layer-step"

# workload: one Llama-3.1-8B-shaped layer, 32 distinct layer stores
B, HKV, HQ, N_CTX, C_CLUSTERS, BUDGET, N_CENTERS = 1, 8, 32, 32768, 400, 1024, 400
N_SINK, WINDOW, ITERS, SEED = 16, 320, 10, 1
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0

# DRAM bytes per select+attend launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum)
# for the current kernel, or None when the kernel changed after the counters were taken.
SELECT_ATTEND_TRAFFIC = 6.099e6  # dram read + write per launch, ncu --set full of the headline layer (cold L2)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def select_attend_bytes(units, budget, C, m, G):
    """Algorithmic bytes of one select+attend launch: per unit the budget's K and V rows
    (256 B each), the fp32 centroids (512 B each), the offsets, the cut cluster's K rows
    (mean cluster size m/C, 256 B each), q (bf16) and o (fp32)."""
    per_unit = budget * 512 + C * 512 + (C + 1) * 4 + (m / C) * 256 + G * 128 * 2 + G * 128 * 4
    return units * per_unit


class Clocks:
    """nvidia-smi sampler running during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_index):
        # address the GPU by UUID: CUDA_VISIBLE_DEVICES may renumber devices
        try:
            u = str(torch.cuda.get_device_properties(local_index).uuid)
            self.index = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            self.index = str(local_index)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return False
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.rows.append(parts)
        return False

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[4 + i].lower() == "active"})
        busy = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)]
        return {"sm_mhz": statistics.median(busy or sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------- CPU oracle leg

def oracle_sample_stores(units=HKV):
    """Stores for a bounded CPU sample: layer-0 units of the workload whose clusters are the
    generator's mixture components, with centroids from one oracle mean update. The decode
    work is the same size as the GPU's (C = 400 clusters of ~82 tokens, budget 1024)."""
    import oracle
    stores = []
    for h in range(units):
        K, V, lab = si.keys_values_labeled(SEED, si.unit_id(0, 0, h, B, HKV), N_CTX, N_CENTERS)
        keys = np.ascontiguousarray(K[N_SINK:])
        mu, offs, perm = oracle.update(keys, lab[N_SINK:], C_CLUSTERS, np.zeros((C_CLUSTERS, 128)))
        stores.append((K[:N_SINK], V[:N_SINK], K[N_SINK:][perm], V[N_SINK:][perm],
                       (perm + N_SINK).astype(np.int32), offs, mu))
    st = [np.stack([s[i] for s in stores]) for i in range(7)]
    q = np.stack([si.queries(SEED, 0, 0, 64, HQ)[:, h * (HQ // HKV):(h + 1) * (HQ // HKV)]
                  for h in range(units)], axis=1)  # [steps, units, G, 128]
    return st, q


def oracle_time_layer_steps(st, q, n_layer_steps):
    import oracle
    t0 = time.perf_counter()
    for i in range(n_layer_steps):
        oracle.select_attend_batch(*st, q[i % q.shape[0]], BUDGET)
    return (time.perf_counter() - t0) / n_layer_steps


def workload_config(L, D, world):
    """The workload both arms report (the reference arm times a sample of it)."""
    return {"workload": "llama3.1-8b-shaped layer (32 q / 8 kv heads, d=128), n=32768, "
                        "batch 1, C=400, budget=1024, held as 32 distinct layer stores",
            "layer_stores": L, "decode_steps": D, "n": N_CTX, "batch": B, "kv_heads": HKV,
            "q_heads": HQ, "C": C_CLUSTERS, "budget": BUDGET, "iters": ITERS,
            "window": WINDOW, "parallelism": f"replicas x{world} (units independent)",
            "l2": "inputs larger than L2: 32 layer stores, ~193 MB selected per decode pass"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    cores = oracle.omp_threads()
    st, q = oracle_sample_stores()
    per_step = 8  # layer-steps per bench step
    for _ in range(args.warmup):
        oracle_time_layer_steps(st, q, per_step)
    times = [oracle_time_layer_steps(st, q, per_step) for _ in range(args.steps)]
    us = statistics.mean(times) * 1e6
    sample = (f"oracle select+attend of one 32k-token layer (8 KV heads, G=4, C=400, budget 1024), "
              f"{per_step} layer-steps per bench step, OpenMP over the 8 units on {cores} threads")
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us * per_step / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(args.layers, args.decode_steps, args.gpus),
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- GPU leg

def decode_shape(ckv, s, dev, hbm_gbs, B, L, D, budget, n, C, what, mixed_n_near=None):
    """µs per select+attend launch at one shape: L layer stores of B sequences x 8 KV heads,
    D decode steps x L layers as one CUDA graph of back-to-back launches, and the fraction of
    the HBM peak by the algorithmic bytes per launch."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    G = HQ // HKV
    try:
        cx = ckv.ClusterKV(n_layers=L, batch=B, n_kv_heads=HKV, n_q_heads=HQ, capacity=n,
                           max_clusters=C, seed=SEED)
    except Exception as exc:
        return {"error": f"{type(exc).__name__}: {exc}"[:300]}
    try:
        K = torch.empty(B, HKV, n, 128, dtype=torch.bfloat16, device=dev)
        V = torch.empty_like(K)
        qs = torch.empty(D, L, B, HQ, 128, dtype=torch.bfloat16, device=dev)
        os_ = torch.empty(D, L, B, HQ, 128, dtype=torch.float32, device=dev)
        for l in range(L):
            for b in range(B):
                for h in range(HKV):
                    K[b, h], V[b, h] = si.keys_values_torch(SEED + 7, si.unit_id(l, b, h, B, HKV), n,
                                                            C, dev)
                qs[:, l, b] = si.queries_torch(SEED + 7, l, b, D, HQ, dev)
            # the prefill on s reads K / V after they are written; the next layer's K / V
            # are written after it ends
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                cx.cluster_prefill(l, K, V, C, stream=s)
            torch.cuda.current_stream().wait_stream(s)
        if mixed_n_near is not None:
            cx.enable_fp8(stream=s)
        s.synchronize()
        del K, V

        def dec():
            for d in range(D):
                for l in range(L):
                    if mixed_n_near is None:
                        cx.select_and_attend(l, qs[d, l], budget, os_[d, l], stream=s)
                    else:
                        cx.select_and_attend_mixed(l, qs[d, l], budget, mixed_n_near, os_[d, l], stream=s)
        with torch.cuda.stream(s):
            dec()
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
            dec()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(5):
                g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        cx.check_device_error(stream=s)
        us = e0.elapsed_time(e1) * 1e3 / (5 * D * L)
        by = select_attend_bytes(B * HKV, budget, C, n - N_SINK, G)
        del g
        return {"us_per_layer_step": us, "units": B * HKV, "bytes_per_launch": by,
                "achieved_gbs": by / (us * 1e-6) / 1e9, "frac": by / (us * 1e-6) / 1e9 / hbm_gbs,
                "what": what + ", CUDA graph of %d launches" % (D * L)}
    except Exception as exc:
        return {"error": f"{type(exc).__name__}: {exc}"[:300]}
    finally:
        cx.close()


def extra_measurements(ckv, ctx, q, out, s, L, dev, hbm_gbs, bf16_tflops):
    """Single-launch latency with L2 flushed, the batch-8 / budget-2048 shape, and the prefill
    keys/s sweep over n in {8k, 32k, 128k}."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    G = HQ // HKV
    res = {}
    # one select+attend launch after a 256 MB write (more than the 126 MB L2)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    single = []
    for i in range(9):
        with torch.cuda.stream(s):
            flush.zero_()
            e0, e1 = ev(), ev()
            e0.record(s)
            ctx.select_and_attend(i % L, q[0, i % L], BUDGET, out[0, i % L], stream=s)
            e1.record(s)
        s.synchronize()
        single.append(e0.elapsed_time(e1) * 1e3)
    res["single_launch_us_l2_flushed"] = statistics.median(single[1:])
    del flush

    # the other decode shapes of the workload family, each as back-to-back launches over
    # distinct layer stores in one CUDA graph (inputs larger than L2)
    res["batch8_budget2k"] = decode_shape(ckv, s, dev, hbm_gbs, B=8, L=4, D=8, budget=2048, n=N_CTX,
                                          C=C_CLUSTERS, what="batch 8 x 8 KV heads, n=32768, C=400, "
                                          "budget 2048, 4 layer stores (320 MB per decode pass)")
    res["batch4_budget1k"] = decode_shape(ckv, s, dev, hbm_gbs, B=4, L=8, D=8, budget=1024, n=N_CTX,
                                          C=C_CLUSTERS, what="batch 4 x 8 KV heads, n=32768, C=400, "
                                          "budget 1024, 8 layer stores (189 MB per decode pass)")
    mix = decode_shape(ckv, s, dev, hbm_gbs, B=1, L=32, D=8, budget=BUDGET, n=N_CTX, C=C_CLUSTERS,
                       mixed_n_near=0, what="select_and_attend_mixed with n_near = 0 (every selected "
                       "cluster attended from the fp8 copy) at the headline shape, 32 layer stores")
    if "us_per_layer_step" in mix:
        # far rows move codes and scales (2 x 132 B) instead of 2 x 256 B
        by = mix["bytes_per_launch"] - B * HKV * (BUDGET - N_SINK) * (512 - 264)
        mix["bytes_per_launch"] = by
        mix["achieved_gbs"] = by / (mix["us_per_layer_step"] * 1e-6) / 1e9
        mix["frac"] = mix["achieved_gbs"] / hbm_gbs
    res["mixed_fp8"] = mix
    res["mixed_fp8_near6"] = decode_shape(ckv, s, dev, hbm_gbs, B=1, L=32, D=8, budget=BUDGET, n=N_CTX,
                                          C=C_CLUSTERS, mixed_n_near=6,
                                          what="select_and_attend_mixed with n_near = 6 at the "
                                          "headline shape (bytes counted as bf16 rows)")
    res["long_128k"] = decode_shape(ckv, s, dev, hbm_gbs, B=1, L=16, D=8, budget=2048, n=131072,
                                    C=1600, what="batch 1 x 8 KV heads, n=131072, C=1600, budget "
                                    "2048, 16 layer stores (242 MB per decode pass)")

    # prefill keys/s sweep, one layer of 8 KV heads each
    sweep = []
    for n_s, c_s in ((8192, 100), (32768, 400), (131072, 1600)):
        Ks = torch.empty(1, HKV, n_s, 128, dtype=torch.bfloat16, device=dev)
        Vs = torch.empty_like(Ks)
        for h in range(HKV):
            Ks[0, h], Vs[0, h] = si.keys_values_torch(SEED + 11, h, n_s, c_s, dev)
        cs = ckv.ClusterKV(n_layers=1, batch=1, n_kv_heads=HKV, n_q_heads=HQ, capacity=n_s,
                           max_clusters=c_s, seed=SEED)
        s.wait_stream(torch.cuda.current_stream())  # the inputs are written
        with torch.cuda.stream(s):
            cs.cluster_prefill(0, Ks, Vs, c_s, stream=s)
        s.synchronize()
        ts = []
        for _ in range(3):
            e0, e1 = ev(), ev()
            with torch.cuda.stream(s):
                e0.record(s)
                cs.cluster_prefill(0, Ks, Vs, c_s, stream=s)
                e1.record(s)
            s.synchronize()
            ts.append(e0.elapsed_time(e1) / 1e3)
        cs.check_device_error(stream=s)
        t = statistics.median(ts)
        kps = HKV * (n_s - N_SINK) / t
        roof, bound = kmeans_roofline(c_s, hbm_gbs, bf16_tflops)
        sweep.append({"n": n_s, "C": c_s, "ms_per_layer": t * 1e3, "keys_per_s": kps,
                      "roofline_keys_per_s": roof, "frac": kps / roof, "bound": bound})
        cs.close()
        del Ks, Vs
    res["prefill_sweep"] = sweep
    for key, fn in (("per_head", per_head_decode), ("split", split_pass)):
        try:
            res[key] = fn(ckv, ctx, q, s, L, dev, hbm_gbs)
        except Exception as exc:  # a failed extra never hides the headline line
            res[key] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    return res


def per_head_decode(ckv, ctx, q, s, L, dev, hbm_gbs):
    """One selection per query head (select_and_attend_per_head) against the grouped
    selection, both as eager calls over the 32 layer stores, 8 decode steps."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    steps = 8
    out = torch.empty(L, B, HQ, 128, dtype=torch.float32, device=dev)
    res = {}
    for name in ("select_and_attend", "select_and_attend_per_head"):
        call = getattr(ctx, name)
        with torch.cuda.stream(s):
            for l in range(L):
                call(l, q[0, l], BUDGET, out[l], stream=s)
        s.synchronize()
        e0, e1 = ev(), ev()
        with torch.cuda.stream(s):
            e0.record(s)
            for d in range(steps):
                for l in range(L):
                    call(l, q[d, l], BUDGET, out[l], stream=s)
            e1.record(s)
        s.synchronize()
        res[name] = e0.elapsed_time(e1) * 1e3 / (steps * L)
    ctx.check_device_error(stream=s)
    # rows, cut-cluster keys, q and o per query head (the rows as if the heads' selections were
    # disjoint: an upper bound of their union); centroids and offsets once per KV head
    m = N_CTX - N_SINK
    by = (B * HQ * (BUDGET * 512 + (m / C_CLUSTERS) * 256 + 128 * 2 + 128 * 4)
          + B * HKV * (C_CLUSTERS * 512 + (C_CLUSTERS + 1) * 4))
    us = res["select_and_attend_per_head"]
    return {"us_per_layer_step": us, "grouped_us_per_layer_step": res["select_and_attend"],
            "bytes_per_launch": by, "achieved_gbs": by / (us * 1e-6) / 1e9,
            "frac": by / (us * 1e-6) / 1e9 / hbm_gbs,
            "what": "32 query heads each select their own budget-1024 rows; eager calls over "
                    "32 layer stores x 8 steps, next to the grouped selection timed the same way; "
                    "bytes count each head's rows and each KV head's centroids once"}


def split_pass(ckv, ctx, q, s, L, dev, hbm_gbs):
    """split_drifted_clusters on one 32k layer (8 KV heads, C=400): the drift check alone
    (threshold +inf, max_splits 0) and a pass at the median drift (max_splits = the room left,
    624), each on a freshly prefilled store, timed with CUDA events around the call (which
    reads nothing back)."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    Ks = torch.empty(1, HKV, N_CTX, 128, dtype=torch.bfloat16, device=dev)
    Vs = torch.empty_like(Ks)
    for h in range(HKV):
        Ks[0, h], Vs[0, h] = si.keys_values_torch(SEED + 13, h, N_CTX, N_CENTERS, dev)
    cmax = 1024
    cs = ckv.ClusterKV(n_layers=1, batch=1, n_kv_heads=HKV, n_q_heads=HQ, capacity=N_CTX,
                       max_clusters=cmax, seed=SEED)
    drift = torch.empty(HKV, C_CLUSTERS, dtype=torch.float32, device=dev)
    cnt = torch.empty(HKV, dtype=torch.int32, device=dev)
    s.wait_stream(torch.cuda.current_stream())  # the inputs are written
    res = {}
    try:
        for label, tau, mx in (("detect_only", float("inf"), 0), ("median", None, cmax - C_CLUSTERS)):
            ts, n_split = [], 0
            for rep in range(4):
                with torch.cuda.stream(s):
                    cs.cluster_prefill(0, Ks, Vs, C_CLUSTERS, stream=s)
                    if tau is None:
                        cs.split_drifted_clusters(0, float("inf"), 0, drift, stream=s)
                        s.synchronize()
                        t = float(drift.median())
                    else:
                        t = tau
                    e0, e1 = ev(), ev()
                    e0.record(s)
                    cs.split_drifted_clusters(0, t, mx, drift, cnt, stream=s)
                    e1.record(s)
                s.synchronize()
                n_split = int(cnt.sum())
                if rep > 0:  # the first call allocates the scratch
                    ts.append(e0.elapsed_time(e1) * 1e3)
            res[label] = {"us": statistics.median(ts), "clusters_split": n_split, "max_splits": mx}
        cs.check_device_error(stream=s)
    finally:
        cs.close()
    res["drift_read_bytes"] = HKV * (N_CTX - N_SINK) * 256
    res["drift_floor_us"] = res["drift_read_bytes"] / (hbm_gbs * 1e3)
    res["what"] = ("one layer, 8 KV heads x 32752 keys, C=400; CUDA events around the call; "
                   "the call reads nothing back and can be captured in a CUDA graph")
    return res


def kmeans_roofline(C, hbm_gbs, bf16_tflops):
    """Keys/s bound of cluster_prefill: per key and Lloyd iteration 2*C*128 flops on the tensor
    cores and two 256-byte key reads (assignment, mean); the smaller rate binds."""
    tensor = bf16_tflops * 1e12 / (2 * C * 128)
    hbm = hbm_gbs * 1e9 / 512
    return min(tensor, hbm) / ITERS, ("tensor" if tensor < hbm else "hbm")


def launches_per_prefill(C, iters):
    # init; per Lloyd iteration the assignment launches (one per 512 centroids, the last one
    # also counting the chunk histograms), scan, scatter and mean; the sink copy
    assign_launches = (C + 511) // 512
    return 1 + iters * (assign_launches + 3) + 1


def run_gpu(args, world, rank, local):
    import recallable_kv_cache_cosine_b200 as ckv
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    L, D, W = args.layers, args.decode_steps, WINDOW
    G = HQ // HKV
    units = B * HKV
    hbm_gbs, bf16_tflops, peak_kind = peaks()

    # ------------------------------------------------------------ inputs (resident in HBM)
    K = torch.empty(L, B, HKV, N_CTX, 128, dtype=torch.bfloat16, device=dev)
    V = torch.empty_like(K)
    for l in range(L):
        for h in range(HKV):
            K[l, 0, h], V[l, 0, h] = si.keys_values_torch(SEED + rank, si.unit_id(l, 0, h, B, HKV),
                                                          N_CTX, N_CENTERS, dev)
    q = torch.empty(D, L, B, HQ, 128, dtype=torch.bfloat16, device=dev)
    for l in range(L):
        q[:, l, 0] = si.queries_torch(SEED + rank, l, 0, D, HQ, dev)
    out = torch.empty(D, L, B, HQ, 128, dtype=torch.float32, device=dev)
    app_k = torch.empty(W, B, HKV, 128, dtype=torch.bfloat16, device=dev)
    app_v = torch.empty_like(app_k)
    for h in range(HKV):
        app_k[:, 0, h], app_v[:, 0, h] = si.appended_tokens_torch(SEED + rank, si.unit_id(0, 0, h, B, HKV),
                                                                   W, N_CENTERS, dev)
    out_c = torch.empty(B, HQ, 128, dtype=torch.float32, device=dev)

    ctx = ckv.ClusterKV(n_layers=L, batch=B, n_kv_heads=HKV, n_q_heads=HQ, capacity=N_CTX + W,
                        max_clusters=C_CLUSTERS + 4, seed=SEED)
    s = torch.cuda.Stream(device=dev)
    launches = {"A": 0, "B": 0, "C": 0}

    def section_a():
        for l in range(L):
            ctx.cluster_prefill(l, K[l], V[l], C_CLUSTERS, stream=s)

    def section_b():
        for d in range(D):
            for l in range(L):
                ctx.select_and_attend(l, q[d, l], BUDGET, out[d, l], stream=s)

    def section_c():
        for t in range(W):
            ctx.append_kv(0, app_k[t], app_v[t], stream=s)
            ctx.select_and_attend(0, q[t % D, 0], BUDGET, out_c, stream=s)
        ctx.recluster_increment(0, stream=s)

    launches["A"] = L * launches_per_prefill(C_CLUSTERS, ITERS)
    launches["B"] = D * L
    launches["C"] = 2 * W + 1

    # ------------------------------------------------------------ capture B and C
    s.wait_stream(torch.cuda.current_stream())  # the inputs are written
    with torch.cuda.stream(s):
        section_a()
    s.synchronize()
    ctx.check_device_error(stream=s)
    gB, gC = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gB, stream=s, capture_error_mode="thread_local"):
        section_b()
    with torch.cuda.graph(gC, stream=s, capture_error_mode="thread_local"):
        section_c()
    torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def one_step(record):
        e = [ev() for _ in range(4)]
        with torch.cuda.stream(s):
            e[0].record(s)
            section_a()
            e[1].record(s)
            gB.replay()
            e[2].record(s)
            gC.replay()
            e[3].record(s)
        record.append(e)

    warm = []
    for _ in range(args.warmup):
        one_step(warm)
    torch.cuda.synchronize()
    ctx.check_device_error(stream=s)

    # ------------------------------------------------------------ timed region
    rec = []
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        for _ in range(args.steps):
            one_step(rec)
        torch.cuda.synchronize()
    barrier(world)
    ctx.check_device_error(stream=s)
    tA = sum(e[0].elapsed_time(e[1]) for e in rec) / 1e3
    tB = sum(e[1].elapsed_time(e[2]) for e in rec) / 1e3
    tC = sum(e[2].elapsed_time(e[3]) for e in rec) / 1e3
    t_step = sum(e[0].elapsed_time(e[3]) for e in rec) / 1e3
    tA, tB, tC, t_step = (max_over_ranks(x, world) for x in (tA, tB, tC, t_step))

    K_steps = args.steps
    layer_steps = K_steps * D * L * world
    value = tB / layer_steps * 1e6
    keys = K_steps * L * units * (N_CTX - N_SINK) * world
    keys_per_s = keys / tA
    keys_roof, keys_bound = kmeans_roofline(C_CLUSTERS, hbm_gbs, bf16_tflops)
    launch_us = tB / (K_steps * D * L) * 1e6
    m = N_CTX - N_SINK
    bytes_launch = select_attend_bytes(units, BUDGET, C_CLUSTERS, m, G)
    achieved = bytes_launch / (launch_us * 1e-6) / 1e9
    inc_us = tC / (K_steps * W * world) * 1e6

    # ------------------------------------------------------------ end to end (host buffers)
    with torch.cuda.stream(s):
        section_a()
    q_host = q[: min(D, 16)].cpu().pin_memory()  # [De, L, B, HQ, 128]
    o_host = torch.empty(q_host.shape[:3] + (HQ, 128), dtype=torch.float32).pin_memory()
    q_dev = torch.empty(q_host.shape[1:], dtype=torch.bfloat16, device=dev)
    o_dev = torch.empty(o_host.shape[1:], dtype=torch.float32, device=dev)
    De = q_host.shape[0]

    def e2e_pass():
        # per decode step: one copy of every layer's queries in, a select_and_attend per layer,
        # one copy of every layer's output back
        with torch.cuda.stream(s):
            for d in range(De):
                q_dev.copy_(q_host[d], non_blocking=True)
                for l in range(L):
                    ctx.select_and_attend(l, q_dev[l], BUDGET, o_dev[l], stream=s)
                o_host[d].copy_(o_dev, non_blocking=True)

    e2e_pass()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = ev(), ev()
    e0.record(s)
    for _ in range(max(1, args.steps)):
        e2e_pass()
    e1.record(s)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    e2e_value = t_e2e / (max(1, args.steps) * De * L * world) * 1e6
    launches_e2e = max(1, args.steps) * De * L
    ctx.check_device_error(stream=s)

    # ------------------------------------------------------------ more shapes (rank 0)
    extra = {}
    if rank == 0 and not args.no_extras:
        extra = extra_measurements(ckv, ctx, q, out, s, L, dev, hbm_gbs, bf16_tflops)

    # ------------------------------------------------------------ CPU baseline (rank 0, N = 1)
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        import oracle
        st, qo = oracle_sample_stores()
        oracle_time_layer_steps(st, qo, 2)
        n_ls = args.cpu_layer_steps
        t = oracle_time_layer_steps(st, qo, n_ls)
        cpu = {"value": t * 1e6, "unit": UNIT, "cores": oracle.omp_threads(), "kind": "oracle",
               "sample": (f"{n_ls} layer-steps of select+attend over one 32k-token layer (8 KV heads, "
                          f"G=4, C=400, budget 1024); clusters = the generator's mixture components "
                          f"with one oracle mean update; OpenMP over the 8 units")}
        try:  # the same sample on one thread
            prev = oracle.set_threads(1)
            n1 = max(8, n_ls // 16)
            try:
                cpu["single_thread"] = {"value": oracle_time_layer_steps(st, qo, n1) * 1e6,
                                        "unit": UNIT, "layer_steps": n1}
            finally:
                oracle.set_threads(prev)
        except Exception as exc:
            cpu["single_thread"] = {"error": f"{type(exc).__name__}: {exc}"[:200]}

    if rank == 0:
        clocks = clk.summary()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K_steps,
            "warmup": args.warmup, "ms_per_step": t_step / K_steps * 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(L, D, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "traffic": SELECT_ATTEND_TRAFFIC,
                         "kernel": "select_attend_kernel<4, false>", "bytes_per_launch": bytes_launch,
                         "us_per_launch": launch_us, "peak_kind": peak_kind},
            "kmeans": {"keys_per_s": keys_per_s, "roofline_keys_per_s": keys_roof,
                       "frac": keys_per_s / keys_roof, "prefill_ms_per_layer": tA / (K_steps * L) * 1e3,
                       "bound": keys_bound,
                       "roofline": "min(tensor at 2*C*128 flop/key, HBM at 2 key reads)/iters"},
            "incremental": {"us_per_token_layer": inc_us,
                            "what": "append_kv + select_and_attend per token, recluster every 320"},
            "sections_ms_per_step": {"prefill": tA / K_steps * 1e3, "decode": tB / K_steps * 1e3,
                                     "incremental": tC / K_steps * 1e3},
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": De * L * B * HQ * 128 * 2,
                    "d2h_bytes_per_step": De * L * B * HQ * 128 * 4,
                    "what": "eager API calls on one stream; per decode step the queries of all "
                            "layers are copied in from pinned host memory and all outputs are "
                            "read back"},
            "gpu_launches": (launches["A"] + launches["B"] + launches["C"]) * K_steps,
            "gpu_launches_e2e": launches_e2e,
            "cpu_baseline": cpu,
            "clocks": clocks,
        }
        line.update(extra)
        print(json.dumps(line), flush=True)
    del gB, gC
    ctx.close()


# Decode shapes that `--shape` runs alone (small, self-contained cases for profilers).
SHAPES = {
    "headline": dict(B=1, budget=BUDGET, n=N_CTX, C=C_CLUSTERS),
    "batch8_budget2k": dict(B=8, budget=2048, n=N_CTX, C=C_CLUSTERS),
    "batch4_budget1k": dict(B=4, budget=1024, n=N_CTX, C=C_CLUSTERS),
    "long_128k": dict(B=1, budget=2048, n=131072, C=1600),
}


def run_shape(args):
    """One decode shape only: --layers layer stores, --decode-steps steps, one JSON line."""
    import recallable_kv_cache_cosine_b200 as ckv
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm_gbs, _, peak_kind = peaks()
    sh = SHAPES[args.shape]
    s = torch.cuda.Stream(device=dev)
    r = decode_shape(ckv, s, dev, hbm_gbs, L=args.layers, D=args.decode_steps,
                     what=f"{args.shape}: batch {sh['B']} x 8 KV heads, n={sh['n']}, C={sh['C']}, "
                          f"budget {sh['budget']}, {args.layers} layer stores", **sh)
    r.update({"shape": args.shape, "peak_kind": peak_kind})
    print(json.dumps(r), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--decode-steps", type=int, default=64)
    ap.add_argument("--cpu-layer-steps", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other shapes, the sweep, per-head and split timings")
    ap.add_argument("--shape", choices=sorted(SHAPES), default=None,
                    help="time one decode shape alone (1 GPU) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_env()
    if args.shape and args.impl == "ours":
        if rank == 0:
            run_shape(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
