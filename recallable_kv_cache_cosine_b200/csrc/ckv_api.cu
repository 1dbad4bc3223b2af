// C-ABI of the ClusterKV hot path: context, argument checks and orchestration of the
// kernels. The ABI is declared and documented in include/ckv.h.
#include <algorithm>
#include <cudaTypedefs.h>
#include <stdio.h>

#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {

static thread_local std::string g_err;

void set_error(const std::string& msg) { g_err = msg; }

int cuda_fail(cudaError_t e, const char* what) {
    set_error(std::string(what) + ": " + cudaGetErrorString(e));
    return CKV_ECUDA;
}

int num_sms_of_current_device() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = v > 0 ? v : 148;
    }
    return cache[dev];
}

int ensure_smem(const void* func, size_t bytes, const char* what) {
    static std::mutex mtx;
    static std::map<std::pair<int, const void*>, size_t> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mtx);
    size_t& cur = done[std::make_pair(dev, func)];
    if (bytes <= cur) return CKV_OK;
    cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return cuda_fail(e, what);
    cur = bytes;
    return CKV_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    });
    return fn;
}

int encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1) {
    auto fn = encode_fn();
    if (!fn) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return CKV_ECUDA;
    }
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
        return CKV_ECUDA;
    }
    return CKV_OK;
}

}  // namespace ckv

using namespace ckv;

namespace {

bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

int einval(const std::string& m) {
    set_error(m);
    return CKV_EINVAL;
}

int check_ctx(const ckv_ctx* c) {
    if (!c) return einval("null context");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != reinterpret_cast<const Ctx*>(c)->device)
        return einval("the context's device is not the current device");
    return CKV_OK;
}

Ctx* C_(ckv_ctx* c) { return reinterpret_cast<Ctx*>(c); }
const Ctx* C_(const ckv_ctx* c) { return reinterpret_cast<const Ctx*>(c); }

int check_layer(const Ctx* c, int32_t layer) {
    if (layer < 0 || layer >= c->cfg.n_layers) return einval("layer out of range");
    return CKV_OK;
}

template <class T>
int dev_alloc(T** p, size_t count, Ctx* c) {
    const size_t bytes = count * sizeof(T);
    if (bytes == 0) {
        *p = nullptr;
        return CKV_OK;
    }
    // the allocation carries kCanaryBytes of a fixed pattern right after its end
    cudaError_t e = cudaMalloc((void**)p, bytes + kCanaryBytes);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        set_error("cudaMalloc of " + std::to_string(bytes) + " bytes failed");
        return CKV_ENOMEM;
    }
    uint8_t* canary = reinterpret_cast<uint8_t*>(*p) + bytes;
    e = cudaMemset(canary, kCanaryByte, kCanaryBytes);
    if (e != cudaSuccess) {
        cudaFree(*p);
        *p = nullptr;
        return cuda_fail(e, "canary memset");
    }
    c->canaries.emplace_back((void*)*p, canary);
    c->bytes += (int64_t)(bytes + kCanaryBytes);
    return CKV_OK;
}

void free_all(Ctx* c) {
    void* ptrs[] = {c->kp, c->vp, c->spk, c->spv, c->ids, c->offsets, c->mu, c->ws.mu_hat,
                    c->ws.assign, c->ws.best, c->ws.perm, c->ws.chunk, c->ws.part, c->err,
                    c->split.drift, c->split.plan, c->split.count, c->split.tasks, c->split.cmu, c->split.n0,
                    c->split.mu2, c->split.off2, c->split.lab, c->split.rk, c->split.rv,
                    c->split.rid, c->kp8, c->vp8, c->ks8, c->vs8};
    for (void* p : ptrs)
        if (p) cudaFree(p);
}

// Refreshes the fp8 copy of rows [r0, r0 + nrows) of every unit of a layer, when the copy is
// kept (ckv_enable_fp8). Launched last by every call that writes those rows.
int refresh_fp8(Ctx* c, int32_t layer, int64_t r0, int64_t nrows, cudaStream_t s) {
    if (!c->kp8 || nrows <= 0) return CKV_OK;
    const int64_t o = c->rows_kp(layer, 0);
    return launch_quantize_rows(c->kp + o * kD, c->vp + o * kD, c->kp8 + o * kD, c->vp8 + o * kD,
                                c->ks8 + o, c->vs8 + o, c->cap_c, r0, nrows, c->units, s);
}

// Checks and launches the re-clustering of layer's full window (the `window` oldest pending
// tokens, at ring position L.pstart). The host state is left to the caller.
int launch_window_recluster(Ctx* c, int32_t layer, float* mu_trace, int32_t* assign_trace,
                            cudaStream_t stream) {
    LayerState& L = c->layers[(size_t)layer];
    if (!L.prefilled || L.in_flight || L.pending != c->cfg.window) {
        set_error(L.in_flight ? "a re-clustering of this layer is in flight; call recluster_finish"
                              : "re-clustering needs exactly `window` pending tokens");
        return CKV_ESTATE;
    }
    if (L.m + c->cfg.window > c->cap_c || L.C + c->cfg.new_clusters > c->cfg.max_clusters) {
        set_error("cluster store full (tokens or clusters)");
        return CKV_ECAPACITY;
    }
    if ((mu_trace && ((uintptr_t)mu_trace & 15u)) || (assign_trace && ((uintptr_t)assign_trace & 3u)))
        return einval("misaligned trace buffer");
    ReclusterArgs a{};
    a.U = c->units;
    a.n_sink = c->cfg.n_sink;
    a.window = c->cfg.window;
    a.win_row0 = c->cfg.n_sink + L.pstart;
    a.C_new = c->cfg.new_clusters;
    a.iters = c->cfg.iters;
    a.C_old = L.C;
    a.m_old = L.m;
    a.seed = c->cfg.seed;
    a.unit_base = (int64_t)layer * c->units;
    a.window_no = (uint64_t)L.windows + 1;
    a.spk = c->spk + c->rows_sp(layer, 0) * kD;
    a.spv = c->spv + c->rows_sp(layer, 0) * kD;
    a.sp_ustride = c->sp_rows;
    a.kp = c->kp + c->rows_kp(layer, 0) * kD;
    a.vp = c->vp + c->rows_kp(layer, 0) * kD;
    a.ids = c->ids + c->rows_kp(layer, 0);
    a.kp_ustride = c->cap_c;
    a.offsets = c->offsets + c->off_base(layer, 0);
    a.off_ustride = c->cfg.max_clusters + 1;
    a.mu = c->mu + c->mu_rows(layer, 0) * kD;
    a.mu_ustride = c->cfg.max_clusters;
    a.mu_trace = mu_trace;
    a.assign_trace = assign_trace;
    int rc = launch_recluster(a, stream);
    if (rc) return rc;
    return refresh_fp8(c, layer, L.m, c->cfg.window, stream);
}

// The window's tokens join the cluster store: the layer's host state after a re-clustering.
void commit_window(Ctx* c, LayerState& L) {
    L.m += c->cfg.window;
    L.C += c->cfg.new_clusters;
    L.pending -= c->cfg.window;
    L.pstart = (L.pstart + c->cfg.window) % c->ring;
    L.windows += 1;
}
// Allocates the split scratch on first use (each buffer once; a failed call can be retried).
int ensure_split_scratch(Ctx* c) {
    SplitScratch& sp = c->split;
    const size_t U = (size_t)c->units, cmax = (size_t)c->cfg.max_clusters, cap = (size_t)c->cap_c;
    int rc = CKV_OK;
    if (!sp.drift) rc = dev_alloc(&sp.drift, U * cmax, c);
    if (!rc && !sp.plan) rc = dev_alloc(&sp.plan, U * cmax, c);
    if (!rc && !sp.count) rc = dev_alloc(&sp.count, U, c);
    if (!rc && !sp.tasks) rc = dev_alloc(&sp.tasks, U * cmax, c);
    if (!rc && !sp.cmu) rc = dev_alloc(&sp.cmu, U * cmax * 2 * kD, c);
    if (!rc && !sp.n0) rc = dev_alloc(&sp.n0, U * cmax, c);
    if (!rc && !sp.mu2) rc = dev_alloc(&sp.mu2, U * cmax * kD, c);
    if (!rc && !sp.off2) rc = dev_alloc(&sp.off2, U * (cmax + 1), c);
    if (!rc && !sp.lab) rc = dev_alloc(&sp.lab, U * cap, c);
    if (!rc && !sp.rk) rc = dev_alloc(&sp.rk, U * cap * kD, c);
    if (!rc && !sp.rv) rc = dev_alloc(&sp.rv, U * cap * kD, c);
    if (!rc && !sp.rid) rc = dev_alloc(&sp.rid, U * cap, c);
    return rc;
}

int decode_call(ckv_ctx* ctx, int32_t layer, const void* q, int32_t budget, float* out,
                int32_t* sel_idx, int32_t* sel_count, void* stream, bool per_head,
                int32_t n_near = -1) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    const LayerState& L = c->layers[(size_t)layer];
    if (!L.prefilled) {
        set_error("select_and_attend before cluster_prefill for this layer");
        return CKV_ESTATE;
    }
    if (!aligned16(q) || !aligned16(out)) return einval("q and out must be non-null and 16-byte aligned");
    if ((sel_idx && ((uintptr_t)sel_idx & 3u)) || (sel_count && ((uintptr_t)sel_count & 3u)))
        return einval("sel_idx / sel_count must be 4-byte aligned");
    if (budget < 1 || (int64_t)budget < (int64_t)c->cfg.n_sink + L.pending)
        return einval("budget must be >= n_sink + pending and >= 1");
    DecodeArgs a{};
    a.q = (const uint16_t*)q;
    a.out = out;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.budget = budget;
    a.B = c->cfg.batch;
    // per head: G = 1 over (b, query head) virtual units, each reading its KV head's store
    a.Hkv = per_head ? c->cfg.n_q_heads : c->cfg.n_kv_heads;
    a.G = per_head ? 1 : c->group;
    a.qsplit = per_head ? c->group : 1;
    a.n_sink = c->cfg.n_sink;
    a.pending = L.pending;
    a.pstart = L.pstart;
    a.pring = c->ring;
    a.C = L.C;
    a.m = L.m;
    a.kp = c->kp + c->rows_kp(layer, 0) * kD;
    a.vp = c->vp + c->rows_kp(layer, 0) * kD;
    a.spk = c->spk + c->rows_sp(layer, 0) * kD;
    a.spv = c->spv + c->rows_sp(layer, 0) * kD;
    a.ids = c->ids + c->rows_kp(layer, 0);
    a.offsets = c->offsets + c->off_base(layer, 0);
    a.mu = c->mu + c->mu_rows(layer, 0) * kD;
    a.kp_ustride = c->cap_c;
    a.sp_ustride = c->sp_rows;
    a.off_ustride = c->cfg.max_clusters + 1;
    a.mu_ustride = c->cfg.max_clusters;
    a.part_scratch = c->ws.part;
    a.part_ustride = c->cap_c;
    a.err = c->err;
    if (n_near >= 0) {  // mixed precision: far clusters from the fp8 copy
        if (!c->kp8) {
            set_error("select_and_attend_mixed needs the fp8 copy: call ckv_enable_fp8 first");
            return CKV_ESTATE;
        }
        const int64_t o = c->rows_kp(layer, 0);
        a.kp8 = c->kp8 + o * kD;
        a.vp8 = c->vp8 + o * kD;
        a.ks8 = c->ks8 + o;
        a.vs8 = c->vs8 + o;
        a.n_near = n_near;
        return launch_select_attend_mixed(a, c->num_sms, (cudaStream_t)stream);
    }
    return per_head ? launch_select_attend_per_head(a, c->num_sms, (cudaStream_t)stream)
                    : launch_select_attend(a, c->num_sms, (cudaStream_t)stream);
}

}  // namespace

extern "C" {

int ckv_config_default(ckv_config* cfg) {
    if (!cfg) return einval("null config");
    *cfg = ckv_config{};
    cfg->head_dim = CKV_HEAD_DIM;
    cfg->n_sink = 16;
    cfg->window = 320;
    cfg->new_clusters = 4;
    cfg->iters = 10;
    cfg->seed = 0;
    return CKV_OK;
}

const char* ckv_strerror(int code) {
    switch (code) {
        case CKV_OK: return "ok";
        case CKV_EINVAL: return "invalid argument";
        case CKV_ENOMEM: return "out of device memory";
        case CKV_ECUDA: return "CUDA error";
        case CKV_ECAPACITY: return "cluster store capacity exceeded";
        case CKV_ETIMEOUT: return "device wait timed out";
        case CKV_ESTATE: return "call out of order";
        default: return "unknown error";
    }
}

const char* ckv_last_error(void) { return g_err.c_str(); }

int ckv_create(const ckv_config* cfg, ckv_ctx** out) {
    if (!cfg || !out) return einval("null argument");
    *out = nullptr;
    const ckv_config& f = *cfg;
    if (f.head_dim != CKV_HEAD_DIM) return einval("head_dim must be 128");
    if (f.n_layers <= 0 || f.batch <= 0 || f.n_kv_heads <= 0 || f.n_q_heads <= 0)
        return einval("n_layers, batch, n_kv_heads and n_q_heads must be positive");
    if (f.n_q_heads % f.n_kv_heads != 0) return einval("n_q_heads must be a multiple of n_kv_heads");
    const int group = f.n_q_heads / f.n_kv_heads;
    if (group > CKV_MAX_GROUP) return einval("group size above 8");
    if (f.n_sink < 0 || f.window <= 0 || f.window > 768 || f.new_clusters <= 0 ||
        f.new_clusters > f.window || f.iters <= 0 || f.iters > 1000)
        return einval("bad n_sink/window/new_clusters/iters");
    if (f.max_clusters <= 0 || f.max_clusters > CKV_MAX_CLUSTERS)
        return einval("max_clusters must be in 1..4096");
    if (f.capacity <= f.n_sink || f.capacity - f.n_sink > (int64_t)INT32_MAX / 2)
        return einval("capacity out of range");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail(cudaGetLastError(), "cudaGetDevice");
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return einval("this library targets sm_100a (B200); current device differs");

    Ctx* c = new Ctx();
    c->cfg = f;
    c->units = f.batch * f.n_kv_heads;
    c->group = group;
    c->cap_c = f.capacity - f.n_sink;
    c->ring = 2 * f.window;
    c->sp_rows = f.n_sink + c->ring;
    c->device = dev;
    c->num_sms = num_sms_of_current_device();
    c->layers.assign((size_t)f.n_layers, LayerState{});
    const int64_t LU = (int64_t)f.n_layers * c->units;
    const int64_t U = c->units;
    const int64_t cmax = f.max_clusters;
    int rc = CKV_OK;
    rc = rc ? rc : dev_alloc(&c->kp, (size_t)(LU * c->cap_c * kD), c);
    rc = rc ? rc : dev_alloc(&c->vp, (size_t)(LU * c->cap_c * kD), c);
    rc = rc ? rc : dev_alloc(&c->spk, (size_t)(LU * c->sp_rows * kD), c);
    rc = rc ? rc : dev_alloc(&c->spv, (size_t)(LU * c->sp_rows * kD), c);
    rc = rc ? rc : dev_alloc(&c->ids, (size_t)(LU * c->cap_c), c);
    rc = rc ? rc : dev_alloc(&c->offsets, (size_t)(LU * (cmax + 1)), c);
    rc = rc ? rc : dev_alloc(&c->mu, (size_t)(LU * cmax * kD), c);
    rc = rc ? rc : dev_alloc(&c->ws.mu_hat, (size_t)(U * cmax * kD), c);
    rc = rc ? rc : dev_alloc(&c->ws.assign, (size_t)(U * c->cap_c), c);
    rc = rc ? rc : dev_alloc(&c->ws.best, (size_t)(U * c->cap_c), c);
    rc = rc ? rc : dev_alloc(&c->ws.perm, (size_t)(U * c->cap_c), c);
    rc = rc ? rc : dev_alloc(&c->ws.chunk, (size_t)(2 * U * n_chunks(c->cap_c) * cmax), c);  // two count buffers
    rc = rc ? rc : dev_alloc(&c->ws.part, (size_t)(U * c->group * c->cap_c), c);  // per query head
    rc = rc ? rc : dev_alloc(&c->err, 4, c);
    if (rc == CKV_OK) {
        cudaError_t e = cudaMemset(c->err, 0, 16);
        if (e == cudaSuccess) e = cudaMemset(c->offsets, 0, sizeof(int32_t) * LU * (cmax + 1));
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) rc = cuda_fail(e, "create: memset");
    }
    if (rc != CKV_OK) {
        free_all(c);
        delete c;
        return rc;
    }
    c->ws.U = c->units;
    c->ws.cap = c->cap_c;
    c->ws.cmax = f.max_clusters;
    *out = reinterpret_cast<ckv_ctx*>(c);
    return CKV_OK;
}

int ckv_destroy(ckv_ctx* ctx) {
    if (!ctx) return CKV_OK;
    Ctx* c = C_(ctx);
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(c->device);
    cudaDeviceSynchronize();
    for (LayerState& L : c->layers)
        if (L.done) cudaEventDestroy(L.done);
    free_all(c);
    cudaSetDevice(cur);
    delete c;
    return CKV_OK;
}

int64_t ckv_device_bytes(const ckv_ctx* ctx) { return ctx ? C_(ctx)->bytes : 0; }

int ckv_check_canaries(ckv_ctx* ctx, int32_t* n_damaged) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (!n_damaged) return einval("null n_damaged");
    Ctx* c = C_(ctx);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "check canaries: synchronize");
    std::vector<uint8_t> host(kCanaryBytes);
    int32_t bad = 0;
    for (const auto& pc : c->canaries) {
        e = cudaMemcpy(host.data(), pc.second, kCanaryBytes, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "check canaries: copy");
        for (size_t i = 0; i < kCanaryBytes; ++i)
            if (host[i] != kCanaryByte) {
                ++bad;
                break;
            }
    }
    *n_damaged = bad;
    return CKV_OK;
}

int cluster_prefill(ckv_ctx* ctx, int32_t layer, const void* K, const void* V, int64_t n,
                    int32_t C, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    if (!aligned16(K) || !aligned16(V)) return einval("K and V must be non-null and 16-byte aligned");
    if (c->layers[(size_t)layer].in_flight) {
        set_error("a re-clustering of this layer is in flight; call recluster_finish");
        return CKV_ESTATE;
    }
    const int32_t ns = c->cfg.n_sink;
    if (n > c->cfg.capacity) {
        set_error("n exceeds the context capacity");
        return CKV_ECAPACITY;
    }
    if (C < 1 || C > c->cfg.max_clusters) return einval("C must be in 1..max_clusters");
    if (n - ns < C) return einval("need n - n_sink >= C");
    cudaStream_t s = (cudaStream_t)stream;
    const int32_t U = c->units;
    const int64_t cmax = c->cfg.max_clusters;
    KeysView kv{(const uint16_t*)K, n, ns, n - ns, U};
    float* mu = c->mu + c->mu_rows(layer, 0) * kD;
    int32_t* offs = c->offsets + c->off_base(layer, 0);
    rc = launch_kmeans_init(kv, C, c->cfg.seed, (int64_t)layer * U, 0, nullptr, mu, cmax,
                            c->ws.mu_hat, cmax, c->err, s);
    if (rc) return rc;
    Relayout rl;
    rl.V = (const uint16_t*)V;
    rl.kp = c->kp + c->rows_kp(layer, 0) * kD;
    rl.vp = c->vp + c->rows_kp(layer, 0) * kD;
    rl.ids = c->ids + c->rows_kp(layer, 0);
    rl.ustride_rows = c->cap_c;
    rl.id_base = ns;
    // The assignment launch counts each key into its chunk's histogram. Iterations alternate
    // between two count buffers: the scatter of iteration i zeroes the one iteration i + 1
    // counts into (the first is zeroed here).
    const size_t cnt_elems = (size_t)U * (size_t)n_chunks(n - ns) * (size_t)C;
    int32_t* cnt[2] = {c->ws.chunk, c->ws.chunk + (size_t)U * n_chunks(c->cap_c) * cmax};
    cudaError_t ze = cudaMemsetAsync(cnt[0], 0, cnt_elems * sizeof(int32_t), s);
    if (ze != cudaSuccess) return cuda_fail(ze, "prefill: zero counts");
    AssignPlan plan[2];
    for (int b = 0; b < 2 && !rc; ++b)
        rc = prepare_kmeans_assign(kv, c->ws.mu_hat, cmax, C, c->ws.assign, c->cap_c, c->ws.best,
                                   c->cap_c, c->err, &plan[b], cnt[b]);
    if (rc) return rc;
    for (int it = 0; it < c->cfg.iters; ++it) {
        rc = run_kmeans_assign(plan[it & 1], s);
        if (rc) return rc;
        const bool last = it + 1 == c->cfg.iters;
        rc = launch_kmeans_update(kv, c->ws.assign, c->cap_c, C, mu, cmax, c->ws.mu_hat, cmax,
                                  offs, cmax + 1, c->ws.perm, c->cap_c, cnt[it & 1],
                                  last ? &rl : nullptr, c->err, s, true, last ? nullptr : cnt[(it + 1) & 1]);
        if (rc) return rc;
    }
    if (ns > 0) {
        rc = launch_copy_sinks((const uint16_t*)K, (const uint16_t*)V, n, U, ns,
                               c->spk + c->rows_sp(layer, 0) * kD,
                               c->spv + c->rows_sp(layer, 0) * kD, c->sp_rows, s);
        if (rc) return rc;
    }
    if ((rc = refresh_fp8(c, layer, 0, n - ns, s))) return rc;
    LayerState& L = c->layers[(size_t)layer];
    L.prefilled = 1;
    L.m = n - ns;
    L.C = C;
    L.pending = 0;
    L.windows = 0;
    L.pstart = 0;
    return CKV_OK;
}

int select_and_attend(ckv_ctx* ctx, int32_t layer, const void* q, int32_t budget, float* out,
                      int32_t* sel_idx, int32_t* sel_count, void* stream) {
    return decode_call(ctx, layer, q, budget, out, sel_idx, sel_count, stream, false);
}

int select_and_attend_per_head(ckv_ctx* ctx, int32_t layer, const void* q, int32_t budget,
                               float* out, int32_t* sel_idx, int32_t* sel_count, void* stream) {
    return decode_call(ctx, layer, q, budget, out, sel_idx, sel_count, stream, true);
}

int select_and_attend_mixed(ckv_ctx* ctx, int32_t layer, const void* q, int32_t budget,
                            int32_t n_near, float* out, int32_t* sel_idx, int32_t* sel_count,
                            void* stream) {
    if (n_near < 0) return einval("n_near must be >= 0");
    return decode_call(ctx, layer, q, budget, out, sel_idx, sel_count, stream, false, n_near);
}

int ckv_append_kv(ckv_ctx* ctx, int32_t layer, const void* k, const void* v, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    LayerState& L = c->layers[(size_t)layer];
    if (!L.prefilled) {
        set_error("append before cluster_prefill for this layer");
        return CKV_ESTATE;
    }
    if (!aligned16(k) || !aligned16(v)) return einval("k and v must be non-null and 16-byte aligned");
    if (L.pending >= (L.in_flight ? c->ring : c->cfg.window)) {
        set_error(L.in_flight ? "pending ring is full; call recluster_finish first"
                              : "pending window is full; call recluster_increment or recluster_begin first");
        return CKV_ECAPACITY;
    }
    if ((int64_t)c->cfg.n_sink + L.m + L.pending + 1 > c->cfg.capacity) {
        set_error("unit capacity exceeded");
        return CKV_ECAPACITY;
    }
    rc = launch_append((const uint16_t*)k, (const uint16_t*)v, c->units,
                       c->spk + c->rows_sp(layer, 0) * kD, c->spv + c->rows_sp(layer, 0) * kD,
                       c->sp_rows, c->cfg.n_sink + (L.pstart + L.pending) % c->ring,
                       (cudaStream_t)stream);
    if (rc) return rc;
    L.pending += 1;
    return CKV_OK;
}

int recluster_increment_traced(ckv_ctx* ctx, int32_t layer, float* mu_trace,
                               int32_t* assign_trace, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    rc = launch_window_recluster(c, layer, mu_trace, assign_trace, (cudaStream_t)stream);
    if (rc) return rc;
    commit_window(c, c->layers[(size_t)layer]);
    return CKV_OK;
}

int recluster_increment(ckv_ctx* ctx, int32_t layer, void* stream) {
    return recluster_increment_traced(ctx, layer, nullptr, nullptr, stream);
}

int recluster_begin(ckv_ctx* ctx, int32_t layer, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    LayerState& L = c->layers[(size_t)layer];
    if (!L.done) {
        cudaError_t e = cudaEventCreateWithFlags(&L.done, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            L.done = nullptr;
            return cuda_fail(e, "recluster_begin: event");
        }
    }
    rc = launch_window_recluster(c, layer, nullptr, nullptr, (cudaStream_t)stream);
    if (rc) return rc;
    cudaError_t e = cudaEventRecord(L.done, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "recluster_begin: record");
    L.in_flight = 1;
    return CKV_OK;
}

int recluster_finish(ckv_ctx* ctx, int32_t layer, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    LayerState& L = c->layers[(size_t)layer];
    if (!L.in_flight) {
        set_error("recluster_finish without recluster_begin");
        return CKV_ESTATE;
    }
    cudaError_t e = cudaStreamWaitEvent((cudaStream_t)stream, L.done, 0);
    if (e != cudaSuccess) return cuda_fail(e, "recluster_finish: wait");
    L.in_flight = 0;
    commit_window(c, L);
    return CKV_OK;
}

int split_drifted_clusters(ckv_ctx* ctx, int32_t layer, float threshold, int32_t max_splits,
                           float* drift, int32_t* splits, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    LayerState& L = c->layers[(size_t)layer];
    if (!L.prefilled || L.in_flight) {
        set_error(L.in_flight ? "a re-clustering of this layer is in flight; call recluster_finish"
                              : "split before cluster_prefill for this layer");
        return CKV_ESTATE;
    }
    if (threshold != threshold) return einval("threshold is NaN");
    if (max_splits < 0) return einval("max_splits must be >= 0");
    if (drift && ((uintptr_t)drift & 3u)) return einval("drift must be 4-byte aligned");
    if (splits && ((uintptr_t)splits & 3u)) return einval("splits must be 4-byte aligned");
    if (c->units > 65535) return einval("more than 65535 units per layer");
    if ((rc = ensure_split_scratch(c))) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    SplitArgs a{};
    a.U = c->units;
    a.C = L.C;
    a.Cmax = c->cfg.max_clusters;
    a.room = std::min(max_splits, c->cfg.max_clusters - L.C);
    a.iters = c->cfg.iters;
    a.m = L.m;
    a.tau = threshold;
    a.seed = c->cfg.seed;
    a.unit_base = (int64_t)layer * c->units;
    a.window_no = (uint64_t)L.windows;
    a.kp = c->kp + c->rows_kp(layer, 0) * kD;
    a.vp = c->vp + c->rows_kp(layer, 0) * kD;
    a.ids = c->ids + c->rows_kp(layer, 0);
    a.kp_ustride = c->cap_c;
    a.offsets = c->offsets + c->off_base(layer, 0);
    a.off_ustride = c->cfg.max_clusters + 1;
    a.mu = c->mu + c->mu_rows(layer, 0) * kD;
    a.mu_ustride = c->cfg.max_clusters;
    a.drift = c->split.drift;
    a.drift_out = drift;
    a.plan = c->split.plan;
    a.count = c->split.count;
    a.tasks = c->split.tasks;
    a.cmu = c->split.cmu;
    a.n0 = c->split.n0;
    a.mu2 = c->split.mu2;
    a.off2 = c->split.off2;
    a.lab = c->split.lab;
    a.rk = c->split.rk;
    a.rv = c->split.rv;
    a.rid = c->split.rid;
    a.err = c->err;
    if ((rc = launch_split(a, s))) return rc;
    if ((rc = refresh_fp8(c, layer, 0, L.m, s))) return rc;
    if (splits) {  // the per-unit split counts, left on the device
        cudaError_t e = cudaMemcpyAsync(splits, c->split.count, sizeof(int32_t) * (size_t)c->units,
                                        cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "split: copy split counts");
    }
    L.C += a.room;
    return CKV_OK;
}

int ckv_get_layer_info(const ckv_ctx* ctx, int32_t layer, ckv_layer_info* out) {
    if (!ctx || !out) return einval("null argument");
    const Ctx* c = C_(ctx);
    int rc = check_layer(c, layer);
    if (rc) return rc;
    const LayerState& L = c->layers[(size_t)layer];
    out->m = L.m;
    out->C = L.C;
    out->pending = L.pending;
    out->windows = L.windows;
    out->prefilled = L.prefilled;
    out->n_total = L.prefilled ? c->cfg.n_sink + L.m + L.pending : 0;
    return CKV_OK;
}

int ckv_export_unit(ckv_ctx* ctx, int32_t layer, int32_t b, int32_t h,
                    const ckv_unit_buffers* dst, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    if (!dst) return einval("null buffers");
    if (b < 0 || b >= c->cfg.batch || h < 0 || h >= c->cfg.n_kv_heads) return einval("unit out of range");
    const LayerState& L = c->layers[(size_t)layer];
    if (!L.prefilled) {
        set_error("layer not prefilled");
        return CKV_ESTATE;
    }
    const int u = b * c->cfg.n_kv_heads + h;
    cudaStream_t s = (cudaStream_t)stream;
    // sinks, then the pending tokens in append order (up to two runs of the ring)
    const int64_t ns = c->cfg.n_sink;
    const int64_t run1 = std::min<int64_t>(L.pending, c->ring - L.pstart), run2 = L.pending - run1;
    const uint16_t* spk_u = c->spk + c->rows_sp(layer, u) * kD;
    const uint16_t* spv_u = c->spv + c->rows_sp(layer, u) * kD;
    uint16_t* dk = (uint16_t*)dst->sp_k;
    uint16_t* dv = (uint16_t*)dst->sp_v;
    struct Item { void* d; const void* s; size_t n; } items[] = {
        {dst->mu, c->mu + c->mu_rows(layer, u) * kD, sizeof(float) * (size_t)L.C * kD},
        {dst->offsets, c->offsets + c->off_base(layer, u), sizeof(int32_t) * (size_t)(L.C + 1)},
        {dst->ids, c->ids + c->rows_kp(layer, u), sizeof(int32_t) * (size_t)L.m},
    };
    for (auto& it : items) {
        if (!it.d || it.n == 0) continue;
        cudaError_t e = cudaMemcpyAsync(it.d, it.s, it.n, cudaMemcpyDefault, s);
        if (e != cudaSuccess) return cuda_fail(e, "export: copy");
    }
    // K / V rows: stored rows r0 .. r0 + rows - 1, copied to a scratch buffer, put back in
    // logical chunk order there, then copied out
    struct Rows { void* d; const uint16_t* s; int64_t rows, r0; } rows[] = {
        {dst->kp, c->kp + c->rows_kp(layer, u) * kD, L.m, 0},
        {dst->vp, c->vp + c->rows_kp(layer, u) * kD, L.m, 0},
        {dk, spk_u, ns, 0},
        {dv, spv_u, ns, 0},
        {dk ? dk + ns * kD : nullptr, spk_u + (ns + L.pstart) * kD, run1, ns + L.pstart},
        {dv ? dv + ns * kD : nullptr, spv_u + (ns + L.pstart) * kD, run1, ns + L.pstart},
        {dk ? dk + (ns + run1) * kD : nullptr, spk_u + ns * kD, run2, ns},
        {dv ? dv + (ns + run1) * kD : nullptr, spv_u + ns * kD, run2, ns},
    };
    int64_t total = 0;
    for (auto& g : rows)
        if (g.d && g.rows > 0) total += g.rows;
    uint16_t* tmp = nullptr;
    cudaError_t e = cudaSuccess;
    if (total > 0) e = cudaMallocAsync((void**)&tmp, (size_t)total * kD * 2, s);
    if (e != cudaSuccess) return cuda_fail(e, "export: scratch");
    int64_t at = 0;
    for (auto& g : rows) {
        if (!g.d || g.rows <= 0 || rc) continue;
        uint16_t* t = tmp + at * kD;
        e = cudaMemcpyAsync(t, g.s, (size_t)g.rows * kD * 2, cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess) rc = launch_swizzle_rows(t, 16, g.r0, g.rows, s);
        if (e == cudaSuccess && !rc) e = cudaMemcpyAsync(g.d, t, (size_t)g.rows * kD * 2, cudaMemcpyDefault, s);
        if (e != cudaSuccess) rc = cuda_fail(e, "export: copy rows");
        at += g.rows;
    }
    if (tmp) cudaFreeAsync(tmp, s);
    e = cudaStreamSynchronize(s);
    if (rc) return rc;
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "export: sync");
}

int ckv_import_unit(ckv_ctx* ctx, int32_t layer, int32_t b, int32_t h, int64_t m, int32_t C,
                    int32_t pending, const ckv_unit_buffers* src, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    if (!src || !src->mu || !src->offsets || !src->ids || !src->kp || !src->vp || !src->sp_k || !src->sp_v)
        return einval("all seven buffers are required");
    if (b < 0 || b >= c->cfg.batch || h < 0 || h >= c->cfg.n_kv_heads) return einval("unit out of range");
    if (m < 0 || m > c->cap_c || C < 1 || C > c->cfg.max_clusters || pending < 0 ||
        pending > c->cfg.window || c->cfg.n_sink + m + pending > c->cfg.capacity)
        return einval("import sizes out of range");
    LayerState& L = c->layers[(size_t)layer];
    if (L.in_flight) {
        set_error("a re-clustering of this layer is in flight; call recluster_finish");
        return CKV_ESTATE;
    }
    const bool first = !L.prefilled || (L.m != m || L.C != C || L.pending != pending);
    const int64_t pstart = first ? 0 : L.pstart;  // pending rows go to ring position pstart
    cudaStream_t s = (cudaStream_t)stream;
    // content checks on a host copy of offsets and ids
    std::vector<int32_t> off((size_t)C + 1), ids((size_t)m);
    cudaError_t e = cudaMemcpy(off.data(), src->offsets, sizeof(int32_t) * (C + 1), cudaMemcpyDefault);
    if (e == cudaSuccess && m > 0) e = cudaMemcpy(ids.data(), src->ids, sizeof(int32_t) * m, cudaMemcpyDefault);
    if (e != cudaSuccess) return cuda_fail(e, "import: read offsets/ids");
    if (off[0] != 0 || off[(size_t)C] != m) return einval("offsets must run from 0 to m");
    for (int32_t i = 0; i < C; ++i) {
        if (off[(size_t)i + 1] < off[(size_t)i]) return einval("offsets must be non-decreasing");
        for (int32_t j = off[(size_t)i] + 1; j < off[(size_t)i + 1]; ++j)
            if (ids[(size_t)j] <= ids[(size_t)j - 1])
                return einval("ids must ascend inside each cluster (the lower-id tie rule)");
    }
    const int64_t n_total = c->cfg.n_sink + m + pending;
    for (int64_t i = 0; i < m; ++i)
        if (ids[(size_t)i] < c->cfg.n_sink || ids[(size_t)i] >= n_total) return einval("id out of range");
    const int u = b * c->cfg.n_kv_heads + h;
    const int64_t ns = c->cfg.n_sink;  // pending <= window and pstart is 0 or window: no wrap
    uint16_t* spk_u = c->spk + c->rows_sp(layer, u) * kD;
    uint16_t* spv_u = c->spv + c->rows_sp(layer, u) * kD;
    const uint16_t* sk = (const uint16_t*)src->sp_k;
    const uint16_t* sv = (const uint16_t*)src->sp_v;
    struct Item { void* d; const void* s; size_t n; } items[] = {
        {c->mu + c->mu_rows(layer, u) * kD, src->mu, sizeof(float) * (size_t)C * kD},
        {c->offsets + c->off_base(layer, u), src->offsets, sizeof(int32_t) * (size_t)(C + 1)},
        {c->ids + c->rows_kp(layer, u), src->ids, sizeof(int32_t) * (size_t)m},
        {c->kp + c->rows_kp(layer, u) * kD, src->kp, (size_t)(2 * m * kD)},
        {c->vp + c->rows_kp(layer, u) * kD, src->vp, (size_t)(2 * m * kD)},
        {spk_u, sk, (size_t)(2 * ns * kD)},
        {spv_u, sv, (size_t)(2 * ns * kD)},
        {spk_u + (ns + pstart) * kD, sk + ns * kD, (size_t)(2 * pending * kD)},
        {spv_u + (ns + pstart) * kD, sv + ns * kD, (size_t)(2 * pending * kD)},
    };
    for (auto& it : items) {
        if (it.n == 0) continue;
        e = cudaMemcpyAsync(it.d, it.s, it.n, cudaMemcpyDefault, s);
        if (e != cudaSuccess) return cuda_fail(e, "import: copy");
    }
    // the copied K / V rows into stored chunk order, in place
    const struct { uint16_t* p; int64_t rows, r0; } swz_rows[] = {
        {c->kp + c->rows_kp(layer, u) * kD, m, 0},
        {c->vp + c->rows_kp(layer, u) * kD, m, 0},
        {spk_u, ns, 0},
        {spv_u, ns, 0},
        {spk_u + (ns + pstart) * kD, pending, ns + pstart},
        {spv_u + (ns + pstart) * kD, pending, ns + pstart},
    };
    for (const auto& g : swz_rows)
        if ((rc = launch_swizzle_rows(g.p, 16, g.r0, g.rows, s))) return rc;
    if (c->kp8 && m > 0) {  // the unit's fp8 copy
        const int64_t o = c->rows_kp(layer, u);
        rc = launch_quantize_rows(c->kp + o * kD, c->vp + o * kD, c->kp8 + o * kD, c->vp8 + o * kD,
                                  c->ks8 + o, c->vs8 + o, c->cap_c, 0, m, 1, s);
        if (rc) return rc;
    }
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "import: sync");
    if (first) {
        L.prefilled = 1;
        L.m = m;
        L.C = C;
        L.pending = pending;
        L.windows = 0;
        L.pstart = 0;
    }
    return CKV_OK;
}

int ckv_check_device_error(ckv_ctx* ctx, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "check: sync");
    uint32_t w = 0;
    e = cudaMemcpy(&w, c->err, 4, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(c->err, 0, 4);
    if (e != cudaSuccess) return cuda_fail(e, "check: read error word");
    if (w & kErrTimeout) {
        set_error("a kernel wait timed out on the device (error word " + std::to_string(w) + ")");
        return CKV_ETIMEOUT;
    }
    if (w) {
        set_error("a kernel saw an out-of-range input and skipped it (error word " +
                  std::to_string(w) + ")");
        return CKV_EINVAL;
    }
    return CKV_OK;
}

int ckv_enable_fp8(ckv_ctx* ctx, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if (!c->kp8) {
        const size_t rows = (size_t)c->cfg.n_layers * c->units * c->cap_c;
        uint8_t *k8 = nullptr, *v8 = nullptr;
        float *ks = nullptr, *vs = nullptr;
        rc = dev_alloc(&k8, rows * kD, c);
        if (!rc) rc = dev_alloc(&v8, rows * kD, c);
        if (!rc) rc = dev_alloc(&ks, rows, c);
        if (!rc) rc = dev_alloc(&vs, rows, c);
        if (rc) {
            for (void* p : {(void*)k8, (void*)v8, (void*)ks, (void*)vs})
                if (p) {
                    for (size_t i = 0; i < c->canaries.size(); ++i)
                        if (c->canaries[i].first == p) {
                            c->canaries.erase(c->canaries.begin() + (ptrdiff_t)i);
                            break;
                        }
                    cudaFree(p);
                }
            return rc;
        }
        c->kp8 = k8;
        c->vp8 = v8;
        c->ks8 = ks;
        c->vs8 = vs;
    }
    for (int32_t l = 0; l < c->cfg.n_layers; ++l) {
        const LayerState& L = c->layers[(size_t)l];
        if (L.prefilled && (rc = refresh_fp8(c, l, 0, L.m, (cudaStream_t)stream))) return rc;
    }
    return CKV_OK;
}

int ckv_export_unit_fp8(ckv_ctx* ctx, int32_t layer, int32_t b, int32_t h, void* k8, float* ks,
                        void* v8, float* vs, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_layer(c, layer))) return rc;
    if (b < 0 || b >= c->cfg.batch || h < 0 || h >= c->cfg.n_kv_heads) return einval("unit out of range");
    if (!c->kp8) {
        set_error("no fp8 copy: call ckv_enable_fp8 first");
        return CKV_ESTATE;
    }
    const LayerState& L = c->layers[(size_t)layer];
    if (!L.prefilled) {
        set_error("layer not prefilled");
        return CKV_ESTATE;
    }
    const int64_t o = c->rows_kp(layer, b * c->cfg.n_kv_heads + h);
    cudaStream_t s = (cudaStream_t)stream;
    struct Item { void* d; const void* s; size_t n; } items[] = {
        {ks, c->ks8 + o, sizeof(float) * (size_t)L.m}, {vs, c->vs8 + o, sizeof(float) * (size_t)L.m}};
    for (auto& it : items) {
        if (!it.d || it.n == 0) continue;
        cudaError_t e = cudaMemcpyAsync(it.d, it.s, it.n, cudaMemcpyDefault, s);
        if (e != cudaSuccess) return cuda_fail(e, "export fp8: copy");
    }
    // the code rows (stored in 8-byte units of swizzled chunk order) through a scratch buffer
    uint8_t* tmp = nullptr;
    cudaError_t e = L.m > 0 ? cudaMallocAsync((void**)&tmp, (size_t)L.m * kD, s) : cudaSuccess;
    if (e != cudaSuccess) return cuda_fail(e, "export fp8: scratch");
    const struct { void* d; const uint8_t* s; } rows[] = {{k8, c->kp8 + o * kD}, {v8, c->vp8 + o * kD}};
    for (const auto& g : rows) {
        if (!g.d || L.m <= 0 || rc) continue;
        e = cudaMemcpyAsync(tmp, g.s, (size_t)L.m * kD, cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess) rc = launch_swizzle_rows(tmp, 8, 0, L.m, s);
        if (e == cudaSuccess && !rc) e = cudaMemcpyAsync(g.d, tmp, (size_t)L.m * kD, cudaMemcpyDefault, s);
        if (e != cudaSuccess) rc = cuda_fail(e, "export fp8: copy rows");
    }
    if (tmp) cudaFreeAsync(tmp, s);
    e = cudaStreamSynchronize(s);
    if (rc) return rc;
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "export fp8: sync");
}

int ckv_debug_expire_wait(ckv_ctx* ctx, uint64_t limit_ns, uint32_t* waited_ns, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (limit_ns < 1000 || limit_ns > 1000000000ull)
        return einval("limit_ns must be in [1 us, 1 s]");
    if (waited_ns && ((uintptr_t)waited_ns & 3u)) return einval("waited_ns must be 4-byte aligned");
    return launch_expire_wait(C_(ctx)->err, limit_ns, waited_ns, (cudaStream_t)stream);
}

static int check_stage(const Ctx* c, const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                       int32_t U, int32_t C) {
    if (!aligned16(keys)) return einval("keys must be non-null and 16-byte aligned");
    if (U < 1 || U > c->units) return einval("U must be in 1..batch*n_kv_heads");
    if (m < 1 || m > c->cap_c) return einval("m out of range");
    if (row0 < 0 || row0 + m > n_rows) return einval("rows [row0, row0+m) exceed n_rows");
    if (C < 1 || C > c->cfg.max_clusters || C > m) return einval("C must be in 1..min(max_clusters, m)");
    return CKV_OK;
}

int ckv_kmeans_init(ckv_ctx* ctx, const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                    int32_t U, int32_t C, uint64_t seed, int64_t unit_base, uint64_t window,
                    int32_t* init_idx, float* mu, void* mu_hat, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_stage(c, keys, n_rows, row0, m, U, C))) return rc;
    if (!aligned16(mu) || !aligned16(mu_hat)) return einval("mu and mu_hat must be 16-byte aligned");
    KeysView kv{(const uint16_t*)keys, n_rows, row0, m, U};
    return launch_kmeans_init(kv, C, seed, unit_base, window, init_idx, mu, C, (uint16_t*)mu_hat, C,
                              c->err, (cudaStream_t)stream);
}

int ckv_kmeans_assign(ckv_ctx* ctx, const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                      int32_t U, const void* mu_hat, int32_t C, int32_t* assign, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_stage(c, keys, n_rows, row0, m, U, C))) return rc;
    if (!aligned16(mu_hat) || !assign) return einval("mu_hat must be 16-byte aligned; assign non-null");
    KeysView kv{(const uint16_t*)keys, n_rows, row0, m, U};
    return launch_kmeans_assign(kv, (const uint16_t*)mu_hat, C, C, assign, m, c->ws.best, c->cap_c,
                                c->err, (cudaStream_t)stream);
}

int ckv_kmeans_update(ckv_ctx* ctx, const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                      int32_t U, const int32_t* assign, int32_t C, float* mu, void* mu_hat,
                      int32_t* offsets, int32_t* perm, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    Ctx* c = C_(ctx);
    if ((rc = check_stage(c, keys, n_rows, row0, m, U, C))) return rc;
    if (!assign || !aligned16(mu) || !aligned16(mu_hat) || !offsets || !perm)
        return einval("null or misaligned output");
    KeysView kv{(const uint16_t*)keys, n_rows, row0, m, U};
    return launch_kmeans_update(kv, assign, m, C, mu, C, (uint16_t*)mu_hat, C, offsets, C + 1, perm,
                                m, c->ws.chunk, nullptr, c->err, (cudaStream_t)stream);
}

}  // extern "C"
