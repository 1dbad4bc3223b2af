/*
 * ckv.h: C-ABI of the ClusterKV hot path on B200 (sm_100a).
 *
 * ClusterKV recalls KV-cache tokens at the granularity of semantic clusters. Sources:
 *   [EXPL] the ClusterKV explainer page "大模型KV Cache压缩技术：ClusterKV的语义空间优化",
 *          sections 3.1 (attention, centroid = mean of member keys), 3.2 (16 sink tokens,
 *          cosine K-means at prefill, incremental clustering every 320 new tokens),
 *          3.3 (select_clusters), 4.1 (half-precision distance matmul; each cluster's KV
 *          stored contiguously);
 *   [ABS]  "ClusterKV: Manipulating LLM KV Cache in Semantic Space for Recallable
 *          Compression" (arXiv 2412.03213), abstract.
 *
 * Conventions for every call:
 *   - Pointers named "device" are caller-owned CUDA device memory. The library never
 *     frees caller memory and never keeps a caller pointer past the call.
 *   - bf16 tensors are passed as `const void*` (IEEE bfloat16, row-major, rows of 128
 *     elements, 16-byte aligned base). fp32 and int32 tensors are 16-byte aligned too.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Work is enqueued
 *     asynchronously on it. No call synchronises the host, except ckv_create,
 *     ckv_destroy, ckv_check_device_error, ckv_export_unit, ckv_export_unit_fp8 and
 *     ckv_import_unit (and the first ckv_enable_fp8, which allocates).
 *   - Return 0 (CKV_OK) on success or a negative CKV_E* code. All arguments are checked on
 *     the host before anything is enqueued. A call that fails its checks leaves the
 *     cluster store unchanged. ckv_last_error() gives a one-line reason (per thread).
 *   - A "unit" is one (layer, sequence b, KV head). All units of a layer share the same
 *     token counts. Unit u = b * n_kv_heads + h inside a layer.
 */
#ifndef CKV_H
#define CKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CKV_API __attribute__((visibility("default")))
#else
#define CKV_API
#endif

#define CKV_OK 0
#define CKV_EINVAL (-1)     /* bad argument (null/misaligned pointer, size out of range) */
#define CKV_ENOMEM (-2)     /* device allocation failed (ckv_create only) */
#define CKV_ECUDA (-3)      /* a CUDA runtime call or kernel launch failed */
#define CKV_ECAPACITY (-4)  /* the cluster store is full (tokens or clusters) */
#define CKV_ETIMEOUT (-5)   /* a kernel's bounded wait gave up (see ckv_check_device_error) */
#define CKV_ESTATE (-6)     /* call out of order (e.g. select before prefill) */

#define CKV_HEAD_DIM 128
#define CKV_MAX_CLUSTERS 4096 /* upper bound of ckv_config.max_clusters */
#define CKV_MAX_GROUP 8       /* upper bound of n_q_heads / n_kv_heads */

typedef struct ckv_ctx ckv_ctx;

typedef struct ckv_config {
    int32_t n_layers;      /* layer stores held by the context */
    int32_t batch;         /* sequences per layer */
    int32_t n_kv_heads;    /* KV heads per layer */
    int32_t n_q_heads;     /* query heads; a multiple of n_kv_heads, group <= CKV_MAX_GROUP */
    int32_t head_dim;      /* must be 128 */
    int32_t n_sink;        /* uncompressed leading tokens, 16 in [EXPL] 3.2 */
    int32_t window;        /* tokens per incremental clustering, 320 in [EXPL] 3.2; <= 768 */
    int32_t new_clusters;  /* clusters made from each window (4) */
    int32_t iters;         /* Lloyd iterations per clustering run (10) */
    int32_t max_clusters;  /* capacity in clusters per unit, prefill + incremental */
    int64_t capacity;      /* capacity in tokens per unit (sinks + clustered + pending) */
    uint64_t seed;         /* K-means init seed */
} ckv_config;

/* Fills the defaults above: n_sink 16, window 320, new_clusters 4, iters 10, head_dim
 * 128, seed 0. Shape fields are zeroed and must be set by the caller. */
CKV_API int ckv_config_default(ckv_config* cfg);

/* Allocates the cluster stores of all layers (the cluster-contiguous layout of [EXPL]
 * 4.1) plus one layer's clustering workspace. Synchronous. CKV_ENOMEM if the device
 * allocation fails. *out receives the context. */
CKV_API int ckv_create(const ckv_config* cfg, ckv_ctx** out);

/* Frees everything ckv_create allocated. Waits for the device to go idle first. */
CKV_API int ckv_destroy(ckv_ctx* ctx);

CKV_API const char* ckv_strerror(int code);
CKV_API const char* ckv_last_error(void);

/* Device bytes held by the context (stores + workspace + canaries). */
CKV_API int64_t ckv_device_bytes(const ckv_ctx* ctx);

/* Out-of-bounds write check (a debugging aid, compute-sanitizer being unavailable). Every
 * device allocation of the context is followed by 256 canary bytes of 0xA5, written when it
 * is allocated. Waits for the device, copies every canary to the host and sets *n_damaged
 * to the number of allocations whose canary changed (0 when no kernel wrote past the end of
 * a buffer). Host-synchronizing. Errors: CKV_EINVAL (null ctx or n_damaged), CKV_ECUDA. */
CKV_API int ckv_check_canaries(ckv_ctx* ctx, int32_t* n_damaged);

/* Prefill clustering of one layer ([EXPL] 3.2; steps: sinks, seeded init, `iters` Lloyd
 * iterations of cosine assignment on tensor cores and mean update, then the relayout of
 * K and V into cluster-major order, [EXPL] 4.1).
 *   K, V : device bf16 [batch, n_kv_heads, n, 128].
 *   n    : tokens per sequence, n_sink + C <= n <= capacity.
 *   C    : clusters per unit, 1 <= C <= max_clusters.
 * Replaces whatever the layer held. Afterwards the layer has m = n - n_sink clustered
 * tokens and no pending tokens. Uses the context's workspace, so prefill calls on
 * different streams must not overlap in time. */
CKV_API int cluster_prefill(ckv_ctx* ctx, int32_t layer, const void* K, const void* V, int64_t n,
                    int32_t C, void* stream);

/* One decode step of one layer ([EXPL] 3.3 then 3.1), fused in one kernel launch:
 * qbar = sum of the group's query heads; score every cluster by qbar . mu_c; walk the
 * clusters by descending score (ties: lower index) taking whole clusters while they fit in
 * remaining = budget - n_sink - pending; fill the first cluster that does not fit with
 * its top-`remaining` tokens by qbar . k (ties: lower token id); then attend every query
 * head of the group over sinks + pending + selected rows: o = softmax(q K^T / sqrt(128)) V.
 *   q         : device bf16 [batch, n_q_heads, 128]; query head j uses KV head j / group.
 *   budget    : tokens attended per unit (sinks and pending included), >= n_sink + pending.
 *   out       : device fp32 [batch, n_q_heads, 128].
 *   sel_idx   : optional device int32 [batch, n_kv_heads, budget]. Original token ids of
 *               the selected rows in the kernel's order: sinks, pending, the whole clusters
 *               in walk order (descending centroid score, ties to the lower cluster index;
 *               each in store order), then the partial tokens (in store order). Entries past
 *               the count are -1. Without a cut (every token fits) the whole clusters come
 *               in cluster-index order.
 *   sel_count : optional device int32 [batch, n_kv_heads] = min(budget, n_total).
 * Reads the store only, so it can be captured in a CUDA graph. The token counts are read
 * at call time and baked into a captured launch. The kernel uses programmatic dependent
 * launch: it may start while the previous kernel of `stream` still runs and read the
 * layer's cluster store then (only this library writes the store, and its calls that do
 * let a following kernel start only once the store is complete); it waits for the previous
 * work before it reads q or the pending rows and before it writes any output. */
CKV_API int select_and_attend(ckv_ctx* ctx, int32_t layer, const void* q, int32_t budget, float* out,
                      int32_t* sel_idx, int32_t* sel_count, void* stream);

/* The same decode step with one selection per query head: query head j scores the clusters
 * of its KV head j / group by q_j . mu_c (instead of the group's qbar), fills its own
 * partial cluster by q_j . k and attends its own `budget` rows. This is the alternative
 * reading of the explainer's single-query select_clusters for grouped heads.
 *   q, out, budget : as for select_and_attend.
 *   sel_idx   : optional device int32 [batch, n_q_heads, budget], per query head.
 *   sel_count : optional device int32 [batch, n_q_heads].
 * Same errors as select_and_attend. */
CKV_API int select_and_attend_per_head(ckv_ctx* ctx, int32_t layer, const void* q, int32_t budget,
                               float* out, int32_t* sel_idx, int32_t* sel_count, void* stream);

/* Appends one generated token's K/V per unit to the layer's pending rows (the tokens a
 * later re-clustering will cluster). The pending rows form a ring of 2 x window rows per
 * unit: one window can be re-clustering (recluster_begin) while the next one fills.
 *   k, v : device bf16 [batch, n_kv_heads, 128].
 * CKV_ECAPACITY if the layer already holds `window` pending tokens and no re-clustering is
 * in flight (call recluster_increment or recluster_begin first), if it holds 2 x window
 * pending tokens (call recluster_finish first), or if the unit capacity would be exceeded. */
CKV_API int ckv_append_kv(ckv_ctx* ctx, int32_t layer, const void* k, const void* v, void* stream);

/* Incremental clustering of one layer ([EXPL] 3.2, every 320 new tokens): cosine K-means
 * with `new_clusters` clusters and `iters` iterations on the `window` pending rows of each
 * unit. The init stream is keyed by (seed, unit, window number). The new clusters, their
 * centroids and their permuted K/V rows are appended to the store. Existing clusters are
 * unchanged and the pending rows are emptied.
 * CKV_ESTATE unless exactly `window` tokens are pending. CKV_ECAPACITY if the store is full.
 *   mu_trace     : optional device fp32 [units, iters + 1, new_clusters, 128], the centroids
 *                  before each iteration and after the last (for stage-wise checks).
 *   assign_trace : optional device int32 [units, iters, window], each iteration's assignment. */
CKV_API int recluster_increment(ckv_ctx* ctx, int32_t layer, void* stream);
CKV_API int recluster_increment_traced(ckv_ctx* ctx, int32_t layer, float* mu_trace,
                               int32_t* assign_trace, void* stream);

/* The same incremental clustering, overlapped with decoding ([EXPL] 4.1: clustering runs
 * asynchronously with decode). recluster_begin launches it on `stream`, usually a second
 * stream. The caller orders `stream` after the appends that filled the window (an event or
 * a stream wait). Until recluster_finish, the layer keeps its clusters and still attends the
 * window as pending tokens. Tokens appended meanwhile join the pending rows in the ring's
 * other half. The decode kernels read only the existing clusters and rows, and the
 * re-clustering writes only rows, offsets and centroids past them, so the two never touch
 * the same memory.
 * recluster_finish makes `stream` wait for the re-clustering. The window's tokens then join
 * the cluster store (4 new clusters), and the tokens appended since begin stay pending. The
 * final store is identical to that of recluster_increment called at begin's position.
 * recluster_begin: CKV_ESTATE unless exactly `window` tokens are pending and none is in
 * flight. CKV_ECAPACITY if the store is full.
 * recluster_finish: CKV_ESTATE without a recluster_begin in flight.
 * While a re-clustering is in flight, cluster_prefill, recluster_increment and
 * ckv_import_unit of the layer return CKV_ESTATE. */
CKV_API int recluster_begin(ckv_ctx* ctx, int32_t layer, void* stream);
CKV_API int recluster_finish(ckv_ctx* ctx, int32_t layer, void* stream);

/* Drift check and split of one layer's clusters ([EXPL] 3.2, decode phase: a cluster whose
 * mean intra-cluster distance passes a threshold is split). Readings of the page, which
 * gives no formula: a cluster's drift is the mean over its members of 1 - cos(k_i, mu_c)
 * (a cosine with a zero vector counts as 0, an empty cluster has drift 0), computed in
 * fp32. A cluster with drift > threshold and at least two members is split by cosine
 * K-means with 2 clusters and `iters` iterations on its own rows (rows in store order;
 * init: the first two entries of the SplitMix64 Fisher-Yates shuffle keyed by
 * seed ^ (unit << 32) ^ windows ^ ((c + 1) * 0x9E3779B97F4A7C15), windows = the layer's
 * incremental clusterings so far), at most room = min(max_splits, max_clusters - C)
 * clusters per unit, lowest index first. The halves take indices c' and c' + 1, with
 * c' = c + (splits below c), and later clusters move up. A split cluster's rows are
 * reordered inside its own segment (first half, then second half, each in store order), so
 * ids stay ascending in every cluster. The layer's cluster count becomes exactly C + room:
 * a unit that split fewer than room clusters gets empty clusters (no rows, zero centroid) at
 * the end, which never add a selected row. The new count is therefore known on the host
 * without reading anything back: the call never synchronises and can be captured in a
 * CUDA graph. Pick max_splits near the number of splits expected; every padding cluster is
 * scored by later decode steps.
 *   threshold  : split when drift > threshold (+inf: never, -inf: every cluster of 2+ rows);
 *                NaN is CKV_EINVAL.
 *   max_splits : >= 0 (CKV_EINVAL otherwise); 0 only measures the drift.
 *   drift      : optional device fp32 [batch * n_kv_heads, C] (C before the call), every
 *                cluster's drift.
 *   splits     : optional device int32 [batch * n_kv_heads], clusters split per unit.
 * The first call allocates a scratch of about 520 bytes per token of capacity per unit of
 * one layer (CKV_ENOMEM if that fails). It shares no workspace with cluster_prefill, but all
 * split calls of a context share that scratch: calls whose work overlaps on the GPU must not
 * be issued. CKV_ESTATE before cluster_prefill or while a re-clustering of the layer is in
 * flight. */
CKV_API int split_drifted_clusters(ckv_ctx* ctx, int32_t layer, float threshold, int32_t max_splits,
                                   float* drift, int32_t* splits, void* stream);

typedef struct ckv_layer_info {
    int64_t n_total;   /* tokens per unit: n_sink + m + pending */
    int64_t m;         /* clustered tokens per unit */
    int32_t C;         /* clusters per unit */
    int32_t pending;   /* tokens appended since the last clustering */
    int32_t windows;   /* incremental clusterings done since prefill */
    int32_t prefilled; /* 1 once cluster_prefill (or ckv_import_unit) set the layer */
} ckv_layer_info;

CKV_API int ckv_get_layer_info(const ckv_ctx* ctx, int32_t layer, ckv_layer_info* out);

/* Copy of one unit's store. Any NULL pointer is skipped. Buffers may be host or device
 * memory (cudaMemcpyDefault). The call synchronises `stream` before it returns.
 *   mu      fp32 [C, 128]          offsets int32 [C + 1]        ids int32 [m]
 *   kp, vp  bf16 [m, 128]          sp_k, sp_v bf16 [n_sink + pending, 128]
 * Rows come out in plain element order. (Inside the context every stored row keeps its
 * 16-byte chunk c at chunk c ^ (r & 7), r = its row index in the unit; the copy puts the rows
 * back in order through a temporary device buffer, allocated on `stream`.) */
typedef struct ckv_unit_buffers {
    float* mu;
    int32_t* offsets;
    int32_t* ids;
    void* kp;
    void* vp;
    void* sp_k;
    void* sp_v;
} ckv_unit_buffers;

CKV_API int ckv_export_unit(ckv_ctx* ctx, int32_t layer, int32_t b, int32_t h,
                    const ckv_unit_buffers* dst, void* stream);

/* Loads one unit's store from caller buffers (all seven non-NULL; layouts as above, plain
 * element order), for decoding over stores built elsewhere. Synchronous, like ckv_export_unit. Sets the layer's counts to (m, C, pending),
 * which must then agree across the layer's units. Offsets must be non-decreasing from 0
 * to m, ids must lie in [n_sink, n_total) and ascend inside each cluster (the decode's
 * lower-id tie rule relies on store order). */
CKV_API int ckv_import_unit(ckv_ctx* ctx, int32_t layer, int32_t b, int32_t h, int64_t m, int32_t C,
                    int32_t pending, const ckv_unit_buffers* src, void* stream);

/* Reads and clears the device error word. Synchronises `stream`. Returns CKV_OK,
 * CKV_ETIMEOUT if a kernel's bounded wait gave up, or CKV_EINVAL if a kernel skipped an
 * out-of-range input (a caller-supplied assignment outside [0, C)). */
CKV_API int ckv_check_device_error(ckv_ctx* ctx, void* stream);

/* Lower precision for far clusters ([EXPL] section 7, outlook: a lower-precision KV cache for
 * clusters far from the current query). The page fixes no format; the reading: every
 * clustered row also keeps an fp8 e4m3 copy with one fp32 scale per row, scale = max|x| / 448,
 * code = e4m3(x / scale) (round to nearest, ties to even, saturating at 448; fp32
 * arithmetic; a zero row has scale 0). The dequantised value is e4m3(code) * scale.
 * ckv_enable_fp8 allocates the copy for every layer (about 264 bytes per clustered row of
 * capacity; CKV_ENOMEM if that fails), fills it for the layers already clustered, and from
 * then on every call that writes the store (cluster_prefill, recluster_increment,
 * recluster_begin, split_drifted_clusters, ckv_import_unit) refreshes the rows it wrote, on
 * the same stream. Calling it again only refreshes. Asynchronous on `stream` apart from the
 * first call's allocation. */
CKV_API int ckv_enable_fp8(ckv_ctx* ctx, void* stream);

/* select_and_attend with the far clusters attended from the fp8 copy ([EXPL] section 7).
 * The selection is exactly select_and_attend's. Then a selected cluster whose walk rank
 * (its position in the descending-score walk over all C clusters, ties to the lower index,
 * rank 0 first) is >= n_near is attended from its fp8 rows, x = e4m3(code) * scale; this
 * includes the partial rows of the cut cluster when its rank is >= n_near. Sinks, pending
 * rows and clusters of rank < n_near are attended in bf16 as usual. n_near >= C attends
 * everything in bf16 (the result then equals select_and_attend's); n_near = 0 attends every
 * clustered row from the copy. A far row moves 264 bytes (codes and scales of K and V)
 * instead of 512.
 *   n_near : >= 0 (CKV_EINVAL otherwise). Other arguments as for select_and_attend.
 * CKV_ESTATE without ckv_enable_fp8. */
CKV_API int select_and_attend_mixed(ckv_ctx* ctx, int32_t layer, const void* q, int32_t budget,
                                    int32_t n_near, float* out, int32_t* sel_idx,
                                    int32_t* sel_count, void* stream);

/* Copy of one unit's fp8 rows (layouts: k8, v8 uint8 [m, 128] in plain element order; ks, vs
 * fp32 [m]); any NULL pointer is skipped, host or device buffers. Synchronises `stream`. CKV_ESTATE without
 * ckv_enable_fp8 or before the layer is clustered. */
CKV_API int ckv_export_unit_fp8(ckv_ctx* ctx, int32_t layer, int32_t b, int32_t h, void* k8,
                                float* ks, void* v8, float* vs, void* stream);

/* Test hook for failure detection (the pages have no counterpart). Every wait inside the
 * library's kernels is bounded: when it runs out, the kernel sets the context's device error
 * word and unwinds, and ckv_check_device_error returns CKV_ETIMEOUT. This call makes one such
 * wait run out on purpose, with no fault: a one-thread kernel waits with the given limit on
 * an mbarrier that nothing completes, then sets the error word and returns.
 *   limit_ns  : the wait's limit, 1 us .. 1 s (CKV_EINVAL outside).
 *   waited_ns : optional device uint32 [1], the time the wait took (ns, saturating).
 * Asynchronous on `stream`; the context stays usable afterwards. */
CKV_API int ckv_debug_expire_wait(ckv_ctx* ctx, uint64_t limit_ns, uint32_t* waited_ns, void* stream);

/* ---- Stage-level K-means calls: the same kernels cluster_prefill runs, exposed so that
 * each stage can be checked on its own. They run on U units whose keys are rows
 * [row0, row0 + m) of `keys`, a device bf16 [U, n_rows, 128] tensor. They use the context's
 * workspace (U <= batch * n_kv_heads, m <= capacity, C <= max_clusters). ---- */

/* Seeded init ([EXPL] 3.2 "K-means", init reading: first C entries of a Fisher-Yates
 * shuffle of 0..m-1 driven by SplitMix64 with key seed ^ (unit << 32) ^ window,
 * unit = unit_base + u). Writes init_idx int32 [U, C] (optional), mu fp32 [U, C, 128]
 * (the chosen keys) and mu_hat bf16 [U, C, 128] = bf16(mu / |mu|). */
CKV_API int ckv_kmeans_init(ckv_ctx* ctx, const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                    int32_t U, int32_t C, uint64_t seed, int64_t unit_base, uint64_t window,
                    int32_t* init_idx, float* mu, void* mu_hat, void* stream);

/* Cosine assignment ([EXPL] 3.2 and 4.1): assign[u, i] = argmax_c keys[u, row0+i] . mu_hat[u, c]
 * (ties: lower c), as a bf16 tcgen05 contraction with fp32 accumulation in tensor memory.
 * mu_hat: bf16 [U, C, 128]. assign: int32 [U, m]. */
CKV_API int ckv_kmeans_assign(ckv_ctx* ctx, const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                      int32_t U, const void* mu_hat, int32_t C, int32_t* assign, void* stream);

/* Centroid update ([EXPL] 3.1 mean, 4.1 contiguous layout): stable counting sort by
 * cluster (offsets int32 [U, C + 1], perm int32 [U, m] = member indices in ascending
 * order per cluster), then mu[u, c] = mean of its members (fp32, summed in perm order),
 * empty clusters keep mu, and mu_hat = bf16(mu / |mu|). mu: fp32 [U, C, 128], in/out.
 * An assignment outside [0, C) is skipped: that key joins no cluster, offsets[u][C]
 * counts only the keys placed (below m), perm entries from there on are left unwritten,
 * and the device error word makes ckv_check_device_error return CKV_EINVAL. */
CKV_API int ckv_kmeans_update(ckv_ctx* ctx, const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                      int32_t U, const int32_t* assign, int32_t C, float* mu, void* mu_hat,
                      int32_t* offsets, int32_t* perm, void* stream);

/* ---- Allocation-free variant of ckv_kmeans_update. The pages have no counterpart for this
 * call: it exists for callers that cannot allocate device memory, such as an engine that
 * takes all of its memory from its own pool at start-up, a decode loop that must not stall
 * on cudaMalloc/cudaFree (they can synchronise the device), or a plugin whose host
 * application owns the device memory. It needs no context. The inputs and outputs are the
 * caller's, exactly as for ckv_kmeans_update (keys bf16 [U, n_rows, 128]; assign int32
 * [U, m]; mu fp32 [U, C, 128] in/out; mu_hat bf16 [U, C, 128]; offsets int32 [U, C + 1];
 * perm int32 [U, m]), and so are the results, bit for bit.
 * Having no context, it has no device error word: an assignment outside [0, C) is skipped
 * without a report. The key joins no cluster, and offsets[u][C] then counts only the keys
 * placed, so a caller detects bad input by comparing offsets[u][C] with m.
 * The kernels' scratch, the per-chunk cluster counts of the counting sort, is a fixed
 * array of 2^21 int32 (8 MiB) compiled into the library. Every GPU that loads the library
 * holds it until the process exits. A call needs U * ceil(m / 1024) * C counts. Larger
 * requests return CKV_EINVAL with the sizes in ckv_last_error(), and nothing is enqueued.
 * The call allocates nothing. On a device's first call it looks up the array's device
 * address (cudaGetSymbolAddress), so make that first call before any stream capture.
 * All calls on a device share the array: calls whose kernels overlap on the GPU (for
 * example on two streams) race. Each call writes every count it reads, so one call's
 * leftovers never reach the next call's results. */
CKV_API int ckv_kmeans_update_noalloc(const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                                      int32_t U, const int32_t* assign, int32_t C, float* mu,
                                      void* mu_hat, int32_t* offsets, int32_t* perm, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CKV_H */
