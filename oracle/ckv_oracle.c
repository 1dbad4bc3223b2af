/*
 * ClusterKV CPU oracle: TEST INFRASTRUCTURE ONLY.
 *
 * This is a plain, slow and direct restatement of what the ClusterKV hot path computes.
 * The tests, the smoke check and the bench's CPU-baseline leg use it to check the CUDA
 * library. The product path never calls it. It shares no code, header, table or
 * constant generator with the CUDA sources.
 *
 * Sources, cited by page title and section:
 *   [EXPL] "大模型KV Cache压缩技术：ClusterKV的语义空间优化" (ClusterKV explainer),
 *          section 3.1 (attention formula, centroid mean, cluster-importance relation),
 *          section 3.2 (16 sinks, cosine K-means at prefill, incremental clustering
 *          every 320 tokens, splitting of drifted clusters), section 3.3
 *          (select_clusters listing), section 7 (lower precision for far clusters),
 *          section 4.1
 *          (half-precision distance matmul, cluster-contiguous KV layout).
 *   [ABS]  "ClusterKV: Manipulating LLM KV Cache in Semantic Space for Recallable
 *          Compression" (arXiv 2412.03213 listing), abstract.
 *
 * Precision: every sum is in double. The bf16 rounding of the normalised centroid
 * follows [EXPL] 4.1 ("half-precision matmul" for the cosine distances). Inputs (keys,
 * values, queries) are bf16 bit patterns (uint16).
 *
 * Parity status: every function here is pinned by a CPU test (brute force, closed form,
 * invariant or published test vector). The end-to-end attention quality on real models
 * is not pinned (the pages print no numbers for it).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_D 128

/* ---------------------------------------------------------------- bf16 ---------- */

double orc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even (IEEE 754 roundTiesToEven on a
 * format with 8 significand bits and float32's exponent range). */
uint16_t orc_bf16_from_double(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double ax = fabs(x);
    if (ax == 0.0) return sign;
    if (isinf(ax)) return sign | 0x7F80;
    int e;
    frexp(ax, &e);              /* ax = f * 2^e, f in [0.5, 1) */
    int ex = e - 1;             /* ax in [2^ex, 2^(ex+1)) */
    if (ex < -126) ex = -126;   /* subnormal range keeps the fixed quantum 2^-133 */
    double quantum = ldexp(1.0, ex - 7);
    double r = nearbyint(ax / quantum) * quantum; /* default mode: nearest, ties to even */
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80;
    float f = (float)r;         /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

void orc_bf16_from_double_array(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_bf16_from_double(x[i]);
}

/* -------------------------------------------------------- seeded init ---------- */
/* The pages only say the K-means is seeded. The reading used here: the initial centroids
 * are the first C entries of a Fisher-Yates shuffle (Durstenfeld's form) of the candidate
 * token indices. The shuffle is driven by SplitMix64 (Steele, Lea & Flood, OOPSLA 2014),
 * and each draw is mapped into [0, r) by Lemire's multiply-shift (ACM TOMACS 2019,
 * without the rejection step). */

uint64_t orc_splitmix64_next(uint64_t* state) {
    uint64_t z = (*state += 0x9E3779B97F4A7C15ULL);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint32_t orc_bounded(uint64_t x, uint32_t r) {
    return (uint32_t)(((x >> 32) * (uint64_t)r) >> 32);
}

/* Stream key of one unit's clustering run: window 0 is the prefill, window w >= 1 is the
 * w-th incremental re-clustering of that unit. */
uint64_t orc_stream_key(uint64_t seed, int64_t unit, uint64_t window) {
    return seed ^ ((uint64_t)unit << 32) ^ window;
}

/* out[0..C) = first C entries of the shuffled sequence 0..m-1. Requires 1 <= C <= m. */
void orc_init_indices(int64_t m, int32_t C, uint64_t key, int32_t* out) {
    int32_t* a = (int32_t*)malloc(sizeof(int32_t) * (size_t)m);
    for (int64_t j = 0; j < m; j++) a[j] = (int32_t)j;
    uint64_t state = key;
    for (int32_t i = 0; i < C; i++) {
        uint64_t x = orc_splitmix64_next(&state);
        int64_t j = i + (int64_t)orc_bounded(x, (uint32_t)(m - i));
        int32_t t = a[i];
        a[i] = a[j];
        a[j] = t;
        out[i] = a[i];
    }
    free(a);
}

/* ---------------------------------------------------------- K-means ---------- */

static double dot_bf16_bf16(const uint16_t* a, const uint16_t* b) {
    double s = 0.0;
    for (int d = 0; d < ORC_D; d++) s += orc_bf16_to_double(a[d]) * orc_bf16_to_double(b[d]);
    return s;
}

/* Assignment operand: mu_hat_c = bf16(mu_c / ||mu_c||). A zero centroid maps to zero.
 * Cosine similarity of k with mu_c is (k . mu_hat_c) / ||k||, and ||k|| does not depend
 * on c, so the argmax over c of k . mu_hat_c is the argmax of the cosine ([EXPL] 3.2,
 * "cosine distance"). The bf16 rounding follows [EXPL] 4.1. */
void orc_normalize(const double* mu, int32_t C, uint16_t* mu_hat) {
    for (int32_t c = 0; c < C; c++) {
        const double* m = mu + (int64_t)c * ORC_D;
        double ss = 0.0;
        for (int d = 0; d < ORC_D; d++) ss += m[d] * m[d];
        double nrm = sqrt(ss);
        for (int d = 0; d < ORC_D; d++)
            mu_hat[(int64_t)c * ORC_D + d] = nrm > 0.0 ? orc_bf16_from_double(m[d] / nrm) : 0;
    }
}

/* a_i = argmax_c k_i . mu_hat_c, ties to the lower c. */
void orc_assign(const uint16_t* keys, int64_t m, const uint16_t* mu_hat, int32_t C,
                int32_t* assign) {
    for (int64_t i = 0; i < m; i++) {
        double best = -INFINITY;
        int32_t arg = 0;
        for (int32_t c = 0; c < C; c++) {
            double s = dot_bf16_bf16(keys + i * ORC_D, mu_hat + (int64_t)c * ORC_D);
            if (s > best) { best = s; arg = c; }
        }
        assign[i] = arg;
    }
}

/* Cosine gap between the oracle's best cluster and another assignment of the same key:
 * gap_i = (k_i . mu_hat_best - k_i . mu_hat_other_i) / ||k_i||. A zero gap means
 * other_i is also a correct answer. Tests use it to accept near-tie disagreements. */
void orc_assign_gap(const uint16_t* keys, int64_t m, const uint16_t* mu_hat, int32_t C,
                    const int32_t* other, double* gap) {
    for (int64_t i = 0; i < m; i++) {
        const uint16_t* k = keys + i * ORC_D;
        double best = -INFINITY, nk = 0.0;
        for (int32_t c = 0; c < C; c++) {
            double s = dot_bf16_bf16(k, mu_hat + (int64_t)c * ORC_D);
            if (s > best) best = s;
        }
        for (int d = 0; d < ORC_D; d++) {
            double x = orc_bf16_to_double(k[d]);
            nk += x * x;
        }
        int32_t o = other[i];
        double so = (o >= 0 && o < C) ? dot_bf16_bf16(k, mu_hat + (int64_t)o * ORC_D) : -INFINITY;
        gap[i] = (best - so) / (nk > 0.0 ? sqrt(nk) : 1.0);
    }
}

/* Update: counting sort of the keys by cluster, then mu_c = (1/|c|) sum of its members
 * (the raw mean of [EXPL] 3.1). sizes/offsets/perm describe the cluster-contiguous
 * layout of [EXPL] 4.1: perm[offsets[c] .. offsets[c+1]) lists the members of cluster c
 * in ascending key index. An empty cluster keeps its previous centroid. */
void orc_update(const uint16_t* keys, int64_t m, const int32_t* assign, int32_t C,
                double* mu, int32_t* offsets, int32_t* perm) {
    int64_t* fill = (int64_t*)calloc((size_t)C + 1, sizeof(int64_t));
    for (int32_t c = 0; c <= C; c++) offsets[c] = 0;
    for (int64_t i = 0; i < m; i++) offsets[assign[i] + 1]++;
    for (int32_t c = 0; c < C; c++) offsets[c + 1] += offsets[c];
    for (int64_t i = 0; i < m; i++) {
        int32_t c = assign[i];
        perm[offsets[c] + fill[c]++] = (int32_t)i;
    }
    for (int32_t c = 0; c < C; c++) {
        int32_t lo = offsets[c], hi = offsets[c + 1];
        if (hi == lo) continue;
        double acc[ORC_D] = {0};
        for (int32_t j = lo; j < hi; j++)
            for (int d = 0; d < ORC_D; d++) acc[d] += orc_bf16_to_double(keys[(int64_t)perm[j] * ORC_D + d]);
        for (int d = 0; d < ORC_D; d++) mu[(int64_t)c * ORC_D + d] = acc[d] / (double)(hi - lo);
    }
    free(fill);
}

/* Lloyd's K-means with cosine assignment ([EXPL] 3.2) from the given initial members.
 * Every iteration normalises, assigns, then updates. After the last iteration, mu holds
 * the means of the final assignment, and offsets/perm hold its layout. */
void orc_kmeans(const uint16_t* keys, int64_t m, int32_t C, int32_t iters,
                const int32_t* init, double* mu, int32_t* offsets, int32_t* perm,
                int32_t* assign) {
    uint16_t* mu_hat = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)C * ORC_D);
    for (int32_t c = 0; c < C; c++)
        for (int d = 0; d < ORC_D; d++)
            mu[(int64_t)c * ORC_D + d] = orc_bf16_to_double(keys[(int64_t)init[c] * ORC_D + d]);
    for (int32_t t = 0; t < iters; t++) {
        orc_normalize(mu, C, mu_hat);
        orc_assign(keys, m, mu_hat, C, assign);
        orc_update(keys, m, assign, C, mu, offsets, perm);
    }
    free(mu_hat);
}

/* --------------------------------------------------------- cluster store ---------- */
/* One unit = one (layer, sequence, KV head). Its store is the cluster-contiguous KV
 * layout of [EXPL] 4.1 plus the uncompressed rows:
 *   sp_k/sp_v   [n_sink + pending, 128]: sink rows (token ids 0..n_sink-1), then the
 *               pending rows appended since the last clustering (ids n_sink + m + j);
 *   kp/vp       [m, 128]: clustered rows, cluster-major;
 *   ids         [m]: original token id of each clustered row;
 *   offsets     [C + 1]: cluster c owns rows offsets[c] .. offsets[c+1];
 *   mu          [C, 128]: centroids (raw means). */
typedef struct {
    int32_t n_sink, pending, C;
    int64_t m;
    const uint16_t* sp_k;
    const uint16_t* sp_v;
    const uint16_t* kp;
    const uint16_t* vp;
    const int32_t* ids;
    const int32_t* offsets;
    const double* mu;
} orc_store;

/* Prefill of one unit ([EXPL] 3.2): the first n_sink tokens are kept as sinks. Cosine
 * K-means runs on the rest, and K and V are permuted into the cluster-major store.
 * K, V: [n, 128]. Outputs are sized by the caller: kp/vp [n - n_sink, 128],
 * ids [n - n_sink], offsets [C + 1], mu [C, 128], assign [n - n_sink]. */
void orc_prefill_unit(const uint16_t* K, const uint16_t* V, int64_t n, int32_t n_sink,
                      int32_t C, int32_t iters, uint64_t key, uint16_t* kp, uint16_t* vp,
                      int32_t* ids, int32_t* offsets, double* mu, int32_t* assign) {
    int64_t m = n - n_sink;
    const uint16_t* keys = K + (int64_t)n_sink * ORC_D;
    int32_t* init = (int32_t*)malloc(sizeof(int32_t) * (size_t)C);
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)m);
    orc_init_indices(m, C, key, init);
    orc_kmeans(keys, m, C, iters, init, mu, offsets, perm, assign);
    for (int64_t j = 0; j < m; j++) {
        int64_t src = (int64_t)n_sink + perm[j];
        memcpy(kp + j * ORC_D, K + src * ORC_D, sizeof(uint16_t) * ORC_D);
        memcpy(vp + j * ORC_D, V + src * ORC_D, sizeof(uint16_t) * ORC_D);
        ids[j] = (int32_t)src;
    }
    free(init);
    free(perm);
}

/* Incremental clustering of one full window ([EXPL] 3.2, "every 320 new tokens"). Cosine
 * K-means with C_new clusters runs on the window's rows alone, with the same init rule
 * and the given stream key. It writes the window's cluster-major rows, their token ids
 * (first_id + local index), the C_new + 1 offsets relative to the window start, and the
 * C_new centroids. Existing clusters are left unchanged. */
void orc_recluster_window(const uint16_t* wk, const uint16_t* wv, int64_t w, int32_t C_new,
                          int32_t iters, uint64_t key, int64_t first_id, uint16_t* kp,
                          uint16_t* vp, int32_t* ids, int32_t* offsets, double* mu,
                          int32_t* assign) {
    int32_t* init = (int32_t*)malloc(sizeof(int32_t) * (size_t)C_new);
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)w);
    orc_init_indices(w, C_new, key, init);
    orc_kmeans(wk, w, C_new, iters, init, mu, offsets, perm, assign);
    for (int64_t j = 0; j < w; j++) {
        memcpy(kp + j * ORC_D, wk + (int64_t)perm[j] * ORC_D, sizeof(uint16_t) * ORC_D);
        memcpy(vp + j * ORC_D, wv + (int64_t)perm[j] * ORC_D, sizeof(uint16_t) * ORC_D);
        ids[j] = (int32_t)(first_id + perm[j]);
    }
    free(init);
    free(perm);
}

/* --------------------------------------------------- drift check and split ---------- */
/* [EXPL] 3.2, decode phase: centroid drift is detected and a cluster whose mean
 * intra-cluster distance is above a threshold is split. The page gives neither the
 * distance, the threshold nor the way of splitting. Readings:
 *   - the distance of a member is its cosine distance to the cluster's centroid,
 *     1 - cos(k_i, mu_c), the same distance the clustering uses; a cosine with a zero
 *     vector counts as 0. An empty cluster has drift 0;
 *   - the threshold is a caller parameter;
 *   - a split is cosine K-means with 2 clusters on the cluster's own rows, the prefill's
 *     rule on a smaller set (same init rule, same iterations), and its two halves replace
 *     the cluster. */

/* drift[c] = (1/|c|) sum over the members of c of (1 - cos(k_i, mu_c)). */
void orc_cluster_drift(const uint16_t* kp, const int32_t* offsets, const double* mu, int32_t C,
                       double* drift) {
    for (int32_t c = 0; c < C; c++) {
        int32_t lo = offsets[c], hi = offsets[c + 1];
        if (hi == lo) {
            drift[c] = 0.0;
            continue;
        }
        const double* mc = mu + (int64_t)c * ORC_D;
        double mm = 0.0;
        for (int d = 0; d < ORC_D; d++) mm += mc[d] * mc[d];
        double acc = 0.0;
        for (int32_t j = lo; j < hi; j++) {
            double dot = 0.0, kk = 0.0;
            for (int d = 0; d < ORC_D; d++) {
                double x = orc_bf16_to_double(kp[(int64_t)j * ORC_D + d]);
                dot += x * mc[d];
                kk += x * x;
            }
            double cosv = (kk > 0.0 && mm > 0.0) ? dot / (sqrt(kk) * sqrt(mm)) : 0.0;
            acc += 1.0 - cosv;
        }
        drift[c] = acc / (double)(hi - lo);
    }
}

/* Init stream of the split of cluster c: the unit's stream key for the current window
 * number, mixed with (c + 1) times the 64-bit golden-ratio constant (the Weyl increment of
 * SplitMix64), so that every cluster of a split pass draws its own init. */
uint64_t orc_split_key(uint64_t seed, int64_t unit, uint64_t window, int32_t c) {
    return orc_stream_key(seed, unit, window) ^ ((uint64_t)(c + 1) * 0x9E3779B97F4A7C15ULL);
}

/* One split pass over a unit's store (offsets [C + 1], m = offsets[C]). Cluster c is split
 * when drift[c] > threshold and it has at least two members, for at most `room` clusters
 * (the lowest indices first). A split runs orc_kmeans with 2 clusters and `iters`
 * iterations on the cluster's rows in store order, from orc_init_indices(|c|, 2,
 * orc_split_key(seed, unit, window, c)). The rows are reordered inside the cluster's segment:
 * the first child's rows, then the second's, each in their previous order. The children
 * take indices c' and c' + 1, with c' = c + (number of split clusters below c), and their
 * centroids are the means of their rows. Any other cluster keeps its rows and centroid
 * and moves to index c + (number of split clusters below c).
 * Outputs: kp2, vp2 [m, 128], ids2 [m], offsets2 [C + room + 1], mu2 [C + room, 128] (only
 * the first (return value) clusters are written), split [C] (1 where c was split).
 * Returns the new cluster count. */
int32_t orc_split_drifted(const uint16_t* kp, const uint16_t* vp, const int32_t* ids,
                          const int32_t* offsets, const double* mu, int32_t C, double threshold,
                          int32_t room, int32_t iters, uint64_t seed, int64_t unit,
                          uint64_t window, uint16_t* kp2, uint16_t* vp2, int32_t* ids2,
                          int32_t* offsets2, double* mu2, int32_t* split) {
    double* drift = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    orc_cluster_drift(kp, offsets, mu, C, drift);
    int32_t n_split = 0, out = 0;
    for (int32_t c = 0; c < C; c++) {
        int32_t lo = offsets[c], hi = offsets[c + 1], size = hi - lo;
        split[c] = drift[c] > threshold && size >= 2 && n_split < room;
        if (!split[c]) {
            offsets2[out] = lo;
            memcpy(mu2 + (int64_t)out * ORC_D, mu + (int64_t)c * ORC_D, sizeof(double) * ORC_D);
            memcpy(kp2 + (int64_t)lo * ORC_D, kp + (int64_t)lo * ORC_D, sizeof(uint16_t) * (size_t)size * ORC_D);
            memcpy(vp2 + (int64_t)lo * ORC_D, vp + (int64_t)lo * ORC_D, sizeof(uint16_t) * (size_t)size * ORC_D);
            memcpy(ids2 + lo, ids + lo, sizeof(int32_t) * (size_t)size);
            out += 1;
            continue;
        }
        int32_t init[2], coff[3];
        double cmu[2 * ORC_D];
        int32_t* cperm = (int32_t*)malloc(sizeof(int32_t) * (size_t)size);
        int32_t* casg = (int32_t*)malloc(sizeof(int32_t) * (size_t)size);
        orc_init_indices(size, 2, orc_split_key(seed, unit, window, c), init);
        orc_kmeans(kp + (int64_t)lo * ORC_D, size, 2, iters, init, cmu, coff, cperm, casg);
        offsets2[out] = lo;
        offsets2[out + 1] = lo + coff[1];
        memcpy(mu2 + (int64_t)out * ORC_D, cmu, sizeof(double) * 2 * ORC_D);
        for (int32_t j = 0; j < size; j++) {
            int64_t src = (int64_t)lo + cperm[j], dst = (int64_t)lo + j;
            memcpy(kp2 + dst * ORC_D, kp + src * ORC_D, sizeof(uint16_t) * ORC_D);
            memcpy(vp2 + dst * ORC_D, vp + src * ORC_D, sizeof(uint16_t) * ORC_D);
            ids2[dst] = ids[src];
        }
        free(cperm);
        free(casg);
        out += 2;
        n_split++;
    }
    offsets2[out] = C > 0 ? offsets[C] : 0;
    free(drift);
    return out;
}

/* ------------------------------------------------------------- selection ---------- */

typedef struct { double score; int32_t idx; int32_t id; } orc_ranked;

/* Descending score, ties to the lower index. */
static int cmp_cluster(const void* a, const void* b) {
    const orc_ranked* x = (const orc_ranked*)a;
    const orc_ranked* y = (const orc_ranked*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* Descending score, ties to the lower original token id. */
static int cmp_token(const void* a, const void* b) {
    const orc_ranked* x = (const orc_ranked*)a;
    const orc_ranked* y = (const orc_ranked*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

/* Group query of one KV head: qbar = sum of its G query heads. One selection per KV head
 * is shared by the G query heads. Scoring one query against a centroid ([EXPL] 3.3) with
 * this sum gives the sum of the heads' own scores. q: [G, 128] bf16. */
void orc_group_query(const uint16_t* q, int32_t G, double* qbar) {
    for (int d = 0; d < ORC_D; d++) {
        double s = 0.0;
        for (int32_t g = 0; g < G; g++) s += orc_bf16_to_double(q[(int64_t)g * ORC_D + d]);
        qbar[d] = s;
    }
}

/* select_clusters of [EXPL] 3.3, for one KV head.
 * 1. score every cluster by qbar . mu_c;
 * 2. visit clusters by descending score (ties: lower cluster index);
 * 3. take a whole cluster while its size fits the remaining budget;
 * 4. the first cluster that does not fit gives its top-`remaining` tokens by qbar . k
 *    (descending; ties: lower token id), then the walk stops.
 * Two readings of the listing: the partial fill takes the highest-scoring tokens (the
 * printed ascending sort would take the lowest), and the sinks and pending rows are
 * always kept and counted against the budget: remaining = budget - n_sink - pending.
 *
 * Output: sel_ids[0..count) = original ids (sinks, pending, whole clusters in visit order,
 * then partial tokens in rank order). sel_rows encodes where each row sits:
 * r >= 0 is clustered row r of kp/vp, and r < 0 is row (-r - 1) of sp_k/sp_v.
 * info[0..4) = { number of whole clusters, cut cluster (-1 if none), partial count r,
 * selected count }. Returns the selected count, or -1 if budget < n_sink + pending. */
int32_t orc_select(const orc_store* s, const double* qbar, int32_t budget, int32_t* sel_ids,
                   int32_t* sel_rows, int32_t* info, double* scores_out) {
    int64_t remaining = (int64_t)budget - s->n_sink - s->pending;
    if (remaining < 0) return -1;
    int32_t count = 0;
    for (int32_t i = 0; i < s->n_sink + s->pending; i++) {
        sel_ids[count] = i < s->n_sink ? i : (int32_t)(s->n_sink + s->m + (i - s->n_sink));
        sel_rows[count] = -i - 1;
        count++;
    }
    orc_ranked* cl = (orc_ranked*)malloc(sizeof(orc_ranked) * (size_t)(s->C > 0 ? s->C : 1));
    for (int32_t c = 0; c < s->C; c++) {
        double sc = 0.0;
        for (int d = 0; d < ORC_D; d++) sc += qbar[d] * s->mu[(int64_t)c * ORC_D + d];
        cl[c].score = sc;
        cl[c].idx = c;
        cl[c].id = c;
        if (scores_out) scores_out[c] = sc;
    }
    qsort(cl, (size_t)s->C, sizeof(orc_ranked), cmp_cluster);
    int32_t n_whole = 0, cut = -1, r = 0;
    for (int32_t k = 0; k < s->C; k++) {
        int32_t c = cl[k].idx;
        int32_t lo = s->offsets[c], hi = s->offsets[c + 1];
        int64_t size = hi - lo;
        if (size <= remaining) {
            for (int32_t j = lo; j < hi; j++) {
                sel_ids[count] = s->ids[j];
                sel_rows[count] = j;
                count++;
            }
            remaining -= size;
            n_whole++;
        } else {
            orc_ranked* tk = (orc_ranked*)malloc(sizeof(orc_ranked) * (size_t)size);
            for (int32_t j = lo; j < hi; j++) {
                double t = 0.0;
                for (int d = 0; d < ORC_D; d++)
                    t += qbar[d] * orc_bf16_to_double(s->kp[(int64_t)j * ORC_D + d]);
                tk[j - lo].score = t;
                tk[j - lo].idx = j;
                tk[j - lo].id = s->ids[j];
            }
            qsort(tk, (size_t)size, sizeof(orc_ranked), cmp_token);
            for (int64_t j = 0; j < remaining; j++) {
                sel_ids[count] = tk[j].id;
                sel_rows[count] = tk[j].idx;
                count++;
            }
            cut = c;
            r = (int32_t)remaining;
            free(tk);
            break;
        }
    }
    free(cl);
    if (info) {
        info[0] = n_whole;
        info[1] = cut;
        info[2] = r;
        info[3] = count;
    }
    return count;
}

/* Attention over the selected rows ([EXPL] 3.1): o_g = softmax(q_g K_sel^T / sqrt(128)) V_sel
 * for each of the G query heads, all in double. */
void orc_attend(const orc_store* s, const uint16_t* q, int32_t G, const int32_t* sel_rows,
                int32_t count, double* out) {
    double* z = (double*)malloc(sizeof(double) * (size_t)(count > 0 ? count : 1));
    const double scale = 1.0 / sqrt((double)ORC_D);
    for (int32_t g = 0; g < G; g++) {
        const uint16_t* qg = q + (int64_t)g * ORC_D;
        double zmax = -INFINITY;
        for (int32_t i = 0; i < count; i++) {
            int32_t r = sel_rows[i];
            const uint16_t* k = r >= 0 ? s->kp + (int64_t)r * ORC_D : s->sp_k + (int64_t)(-r - 1) * ORC_D;
            z[i] = dot_bf16_bf16(qg, k) * scale;
            if (z[i] > zmax) zmax = z[i];
        }
        double den = 0.0;
        double acc[ORC_D] = {0};
        for (int32_t i = 0; i < count; i++) {
            int32_t r = sel_rows[i];
            const uint16_t* v = r >= 0 ? s->vp + (int64_t)r * ORC_D : s->sp_v + (int64_t)(-r - 1) * ORC_D;
            double p = exp(z[i] - zmax);
            den += p;
            for (int d = 0; d < ORC_D; d++) acc[d] += p * orc_bf16_to_double(v[d]);
        }
        for (int d = 0; d < ORC_D; d++) out[(int64_t)g * ORC_D + d] = acc[d] / den;
    }
    free(z);
}

/* Dense attention over all n rows of K, V ([EXPL] 3.1), the full-KV reference. */
void orc_dense_attention(const uint16_t* K, const uint16_t* V, int64_t n, const uint16_t* q,
                         int32_t G, double* out) {
    double* z = (double*)malloc(sizeof(double) * (size_t)n);
    const double scale = 1.0 / sqrt((double)ORC_D);
    for (int32_t g = 0; g < G; g++) {
        double zmax = -INFINITY, den = 0.0;
        double acc[ORC_D] = {0};
        for (int64_t i = 0; i < n; i++) {
            z[i] = dot_bf16_bf16(q + (int64_t)g * ORC_D, K + i * ORC_D) * scale;
            if (z[i] > zmax) zmax = z[i];
        }
        for (int64_t i = 0; i < n; i++) {
            double p = exp(z[i] - zmax);
            den += p;
            for (int d = 0; d < ORC_D; d++) acc[d] += p * orc_bf16_to_double(V[i * ORC_D + d]);
        }
        for (int d = 0; d < ORC_D; d++) out[(int64_t)g * ORC_D + d] = acc[d] / den;
    }
    free(z);
}

/* ------------------------------------------- far clusters in fp8 (e4m3) ---------- */
/* [EXPL] 7 (outlook) lists mixed precision: a lower-precision KV cache for the clusters far
 * from the current query. The page gives no format, scale or distance rule. Readings:
 *   - the low-precision copy is fp8 e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
 *     bits, no infinities, largest finite 448), one fp32 scale per row:
 *     scale = max_d |x_d| / 448 and code_d = e4m3(x_d / scale), both steps in fp32, the
 *     rounding to nearest with ties to even; a zero row has scale 0 and zero codes;
 *   - "far" is the walk order of the selection: whole clusters taken at rank >= n_near
 *     (rank 0 = highest score), and the cut cluster when its rank is >= n_near, are read
 *     from the fp8 copy; sinks, pending rows and the nearer clusters stay bf16. The
 *     selection itself is unchanged (it scores with the fp32 centroids and bf16 keys). */

/* e4m3 code of x, ties to even. Magnitudes above 448 saturate to 448 (the copy's scale keeps
 * every input at or below 448, so this rule only guards the format); NaN gives 0x7F. */
uint8_t orc_e4m3_from_float(float x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double ax = fabs((double)x);
    if (ax == 0.0) return sign;
    int e;
    frexp(ax, &e);            /* ax in [2^(e-1), 2^e) */
    int ex = e - 1;
    if (ex < -6) ex = -6;     /* subnormals: fixed quantum 2^-9 */
    double quantum = ldexp(1.0, ex - 3);
    double r = nearbyint(ax / quantum) * quantum;
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return sign;
    frexp(r, &e);
    int rex = e - 1;
    uint8_t code;
    if (rex < -6) {           /* subnormal: r = mant * 2^-9, mant in 1..7 */
        code = (uint8_t)(r / ldexp(1.0, -9));
    } else {                  /* normal: r = (1 + mant/8) * 2^rex */
        int mant = (int)(r / ldexp(1.0, rex - 3)) - 8;
        code = (uint8_t)(((rex + 7) << 3) | mant);
    }
    return sign | code;
}

void orc_e4m3_from_float_array(const float* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_e4m3_from_float(x[i]);
}

double orc_e4m3_to_double(uint8_t b) {
    int sign = b >> 7, ex = (b >> 3) & 15, mant = b & 7;
    if (ex == 15 && mant == 7) return NAN;
    double v = ex == 0 ? ldexp((double)mant, -9) : ldexp(1.0 + mant / 8.0, ex - 7);
    return sign ? -v : v;
}

/* Per-row fp8 copy of n rows of 128 bf16 values: codes [n, 128], scales [n]. */
void orc_quantize_rows_e4m3(const uint16_t* rows, int64_t n, uint8_t* codes, float* scales) {
    for (int64_t i = 0; i < n; i++) {
        float mx = 0.0f;
        for (int d = 0; d < ORC_D; d++) {
            float a = (float)fabs(orc_bf16_to_double(rows[i * ORC_D + d]));
            if (a > mx) mx = a;
        }
        float scale = mx / 448.0f;
        scales[i] = scale;
        for (int d = 0; d < ORC_D; d++) {
            float x = (float)orc_bf16_to_double(rows[i * ORC_D + d]);
            codes[i * ORC_D + d] = scale > 0.0f ? orc_e4m3_from_float(x / scale) : 0;
        }
    }
}

/* Attention over the selected rows like orc_attend, except that a clustered row whose
 * cluster has walk rank >= n_near (row_rank[i], -1 for sinks and pending) is read from the
 * fp8 copy: x = e4m3(code) * scale, in double. k8/v8 [m, 128], ks/vs [m]. */
void orc_attend_mixed(const orc_store* s, const uint16_t* q, int32_t G, const int32_t* sel_rows,
                      const int32_t* row_rank, int32_t count, int32_t n_near, const uint8_t* k8,
                      const float* ks, const uint8_t* v8, const float* vs, double* out) {
    double* z = (double*)malloc(sizeof(double) * (size_t)(count > 0 ? count : 1));
    const double scale = 1.0 / sqrt((double)ORC_D);
    for (int32_t g = 0; g < G; g++) {
        const uint16_t* qg = q + (int64_t)g * ORC_D;
        double zmax = -INFINITY;
        for (int32_t i = 0; i < count; i++) {
            int32_t r = sel_rows[i];
            double dot = 0.0;
            if (r >= 0 && row_rank[i] >= n_near) {
                for (int d = 0; d < ORC_D; d++)
                    dot += orc_bf16_to_double(qg[d]) *
                           (orc_e4m3_to_double(k8[(int64_t)r * ORC_D + d]) * (double)ks[r]);
            } else {
                const uint16_t* k = r >= 0 ? s->kp + (int64_t)r * ORC_D : s->sp_k + (int64_t)(-r - 1) * ORC_D;
                dot = dot_bf16_bf16(qg, k);
            }
            z[i] = dot * scale;
            if (z[i] > zmax) zmax = z[i];
        }
        double den = 0.0;
        double acc[ORC_D] = {0};
        for (int32_t i = 0; i < count; i++) {
            int32_t r = sel_rows[i];
            double p = exp(z[i] - zmax);
            den += p;
            if (r >= 0 && row_rank[i] >= n_near) {
                for (int d = 0; d < ORC_D; d++)
                    acc[d] += p * (orc_e4m3_to_double(v8[(int64_t)r * ORC_D + d]) * (double)vs[r]);
            } else {
                const uint16_t* v = r >= 0 ? s->vp + (int64_t)r * ORC_D : s->sp_v + (int64_t)(-r - 1) * ORC_D;
                for (int d = 0; d < ORC_D; d++) acc[d] += p * orc_bf16_to_double(v[d]);
            }
        }
        for (int d = 0; d < ORC_D; d++) out[(int64_t)g * ORC_D + d] = acc[d] / den;
    }
    free(z);
}

/* ---------------------------------------------------- batched (timing) ---------- */
/* Independent units run in parallel (OpenMP, when compiled with it). Each unit's
 * arithmetic is exactly the single-unit function above. */

#ifdef _OPENMP
#include <omp.h>
#endif

/* Sets the number of threads of the batched calls; returns the previous setting (1 without
 * OpenMP). */
int32_t orc_set_threads(int32_t n) {
#ifdef _OPENMP
    int32_t prev = (int32_t)omp_get_max_threads();
    if (n > 0) omp_set_num_threads(n);
    return prev;
#else
    (void)n;
    return 1;
#endif
}

void orc_prefill_batch(int32_t U, const uint16_t* K, const uint16_t* V, int64_t n,
                       int32_t n_sink, int32_t C, int32_t iters, const uint64_t* keys,
                       uint16_t* kp, uint16_t* vp, int32_t* ids, int32_t* offsets,
                       double* mu, int32_t* assign) {
    int64_t m = n - n_sink;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t u = 0; u < U; u++)
        orc_prefill_unit(K + (int64_t)u * n * ORC_D, V + (int64_t)u * n * ORC_D, n, n_sink, C,
                         iters, keys[u], kp + (int64_t)u * m * ORC_D, vp + (int64_t)u * m * ORC_D,
                         ids + (int64_t)u * m, offsets + (int64_t)u * (C + 1),
                         mu + (int64_t)u * C * ORC_D, assign + (int64_t)u * m);
}

/* select + attend for U units that share C, m, pending and budget (stores laid out back
 * to back). q: [U, G, 128]; out: [U, G, 128]; sel_ids: [U, budget]; counts: [U]. */
void orc_select_attend_batch(int32_t U, int32_t n_sink, int32_t pending, int64_t m, int32_t C,
                             const uint16_t* sp_k, const uint16_t* sp_v, const uint16_t* kp,
                             const uint16_t* vp, const int32_t* ids, const int32_t* offsets,
                             const double* mu, const uint16_t* q, int32_t G, int32_t budget,
                             double* out, int32_t* sel_ids, int32_t* counts) {
    int64_t sp = (int64_t)n_sink + pending;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t u = 0; u < U; u++) {
        orc_store s;
        s.n_sink = n_sink;
        s.pending = pending;
        s.C = C;
        s.m = m;
        s.sp_k = sp_k + (int64_t)u * sp * ORC_D;
        s.sp_v = sp_v + (int64_t)u * sp * ORC_D;
        s.kp = kp + (int64_t)u * m * ORC_D;
        s.vp = vp + (int64_t)u * m * ORC_D;
        s.ids = ids + (int64_t)u * m;
        s.offsets = offsets + (int64_t)u * (C + 1);
        s.mu = mu + (int64_t)u * C * ORC_D;
        double qbar[ORC_D];
        orc_group_query(q + (int64_t)u * G * ORC_D, G, qbar);
        int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)budget);
        int32_t cnt = orc_select(&s, qbar, budget, sel_ids + (int64_t)u * budget, rows, NULL, NULL);
        counts[u] = cnt;
        if (cnt > 0) orc_attend(&s, q + (int64_t)u * G * ORC_D, G, rows, cnt, out + (int64_t)u * G * ORC_D);
        free(rows);
    }
}
