// Host-side internals shared by the library's translation units: the context object and
// the kernel launchers. Not part of the public ABI.
#pragma once

#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <memory>
#include <string>
#include <vector>

#include "ckv.h"

namespace ckv {

struct LayerState {
    int prefilled = 0;
    int64_t m = 0;
    int32_t C = 0;
    int32_t pending = 0;    // pending tokens, in append order from ring position pstart
    int32_t windows = 0;
    int32_t pstart = 0;     // ring position of the oldest pending token (0 or window)
    int in_flight = 0;      // a re-clustering started by recluster_begin is not finished
    cudaEvent_t done = nullptr;  // recorded after that re-clustering
};

// Keys of U units: rows [row0, row0 + m) of a [U, n_rows, 128] bf16 tensor.
struct KeysView {
    const uint16_t* base;
    int64_t n_rows;
    int64_t row0;
    int64_t m;
    int32_t U;
};

struct Workspace {
    uint16_t* mu_hat = nullptr;  // [U][Cmax][128]
    int32_t* assign = nullptr;   // [U][cap_c]
    float* best = nullptr;       // [U][cap_c]
    int32_t* perm = nullptr;     // [U][cap_c]
    int32_t* chunk = nullptr;    // 2 x [U][n_chunks(cap_c)][Cmax] (two count buffers)
    float* part = nullptr;       // decode partial-cut scratch [U][cap_c] (keys of the cut cluster)
    int32_t U = 0;
    int64_t cap = 0;
    int32_t cmax = 0;
};

// Scratch of split_drifted_clusters, allocated by its first call.
struct SplitScratch {
    float* drift = nullptr;   // [U][Cmax] drift of every cluster
    int32_t* plan = nullptr;  // [U][Cmax] 2 * new index + split flag
    int32_t* count = nullptr; // [U] splits per unit
    int32_t* tasks = nullptr; // [U][Cmax] clusters to split, in index order
    float* cmu = nullptr;     // [U][Cmax][2][128] centroids of the two halves
    int32_t* n0 = nullptr;    // [U][Cmax] rows of the first half
    float* mu2 = nullptr;     // [U][Cmax][128] centroids at their new indices
    int32_t* off2 = nullptr;  // [U][Cmax + 1] offsets at their new indices
    int32_t* lab = nullptr;   // [U][cap_c] half of every row (segments above the staging size)
    uint16_t* rk = nullptr;   // [U][cap_c][128] row scratch of the stable partition
    uint16_t* rv = nullptr;
    int32_t* rid = nullptr;   // [U][cap_c]
};

struct Ctx {
    ckv_config cfg{};
    int32_t units = 0;   // batch * n_kv_heads
    int32_t group = 0;   // n_q_heads / n_kv_heads
    int64_t cap_c = 0;   // clustered-row capacity per unit
    int32_t sp_rows = 0; // n_sink + ring
    int32_t ring = 0;    // pending ring rows: 2 * window (one window re-clustering, one filling)
    int device = 0;
    int num_sms = 0;
    // Stores of all layers, [L][U][...].
    uint16_t* kp = nullptr;
    uint16_t* vp = nullptr;
    uint16_t* spk = nullptr;
    uint16_t* spv = nullptr;
    int32_t* ids = nullptr;
    int32_t* offsets = nullptr;
    float* mu = nullptr;
    // fp8 (e4m3) copy of the clustered rows with per-row scales, [L][U][cap_c] rows; allocated
    // by ckv_enable_fp8 and kept current by every call that writes the store afterwards.
    uint8_t* kp8 = nullptr;
    uint8_t* vp8 = nullptr;
    float* ks8 = nullptr;
    float* vs8 = nullptr;
    Workspace ws;
    SplitScratch split;
    uint32_t* err = nullptr;  // device error word
    std::vector<LayerState> layers;
    int64_t bytes = 0;
    // Canary bytes right after the end of every device allocation (kCanaryBytes of
    // kCanaryByte), checked by ckv_check_canaries: (allocation, canary start).
    std::vector<std::pair<void*, uint8_t*>> canaries;

    int64_t rows_kp(int layer, int u) const { return ((int64_t)layer * units + u) * cap_c; }
    int64_t rows_sp(int layer, int u) const { return ((int64_t)layer * units + u) * sp_rows; }
    int64_t off_base(int layer, int u) const {
        return ((int64_t)layer * units + u) * (cfg.max_clusters + 1);
    }
    int64_t mu_rows(int layer, int u) const {
        return ((int64_t)layer * units + u) * cfg.max_clusters;
    }
};

void set_error(const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);

constexpr int kD = 128;       // head dim
constexpr size_t kCanaryBytes = 256;
constexpr unsigned char kCanaryByte = 0xA5;
constexpr int kChunk = 1024;  // keys per counting-sort chunk
inline int64_t n_chunks(int64_t m) { return (m + kChunk - 1) / kChunk; }

// Tensor-map encoder from the driver, fetched through the runtime (no libcuda link).
int encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1);

int num_sms_of_current_device();

// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the current device.
// The attribute is set once per (device, kernel, size increase), not on every launch.
int ensure_smem(const void* func, size_t bytes, const char* what);

// ---- launchers (each returns CKV_OK or an error code; all asynchronous on `stream`)
int launch_kmeans_init(const KeysView& k, int32_t C, uint64_t seed, int64_t unit_base,
                       uint64_t window, int32_t* init_idx, float* mu, int64_t mu_ustride,
                       uint16_t* mu_hat, int64_t muhat_ustride, uint32_t* err, cudaStream_t s);

int launch_kmeans_assign(const KeysView& k, const uint16_t* mu_hat, int64_t muhat_ustride,
                         int32_t C, int32_t* assign, int64_t assign_ustride, float* best,
                         int64_t best_ustride, uint32_t* err, cudaStream_t s);

// The same launch split in two: prepare encodes the tensor maps and launch shapes once (they
// depend only on pointers and sizes), run launches them. cluster_prefill prepares once and
// runs once per Lloyd iteration.
struct AssignPlanImpl;
struct AssignPlan {
    std::shared_ptr<AssignPlanImpl> impl;
};
// counts (optional): [U][n_chunks(m)][C] integer counts, zero on entry; the launch adds one
// for every key to (its chunk, its cluster), which is what the update's count kernel computes.
int prepare_kmeans_assign(const KeysView& k, const uint16_t* mu_hat, int64_t muhat_ustride,
                          int32_t C, int32_t* assign, int64_t assign_ustride, float* best,
                          int64_t best_ustride, uint32_t* err, AssignPlan* out,
                          int32_t* counts = nullptr);
int run_kmeans_assign(const AssignPlan& plan, cudaStream_t s);

struct Relayout {  // final-iteration relayout of K and V into the cluster-major store
    const uint16_t* V = nullptr;  // same shape as the keys tensor
    uint16_t* kp = nullptr;
    uint16_t* vp = nullptr;
    int32_t* ids = nullptr;
    int64_t ustride_rows = 0;  // rows between units in kp/vp/ids
    int32_t id_base = 0;       // original id of local key 0
};

// chunk_ws: [U][n_chunks(m)][C] ints. counted: chunk_ws already holds the per-chunk counts of
// `assign` (from the assignment launch), so the count kernel is skipped. zero_next (optional):
// another [U][n_chunks(m)][C] buffer that the scatter sets to zero, ready for the next
// assignment launch to count into.
int launch_kmeans_update(const KeysView& k, const int32_t* assign, int64_t assign_ustride,
                         int32_t C, float* mu, int64_t mu_ustride, uint16_t* mu_hat,
                         int64_t muhat_ustride, int32_t* offsets, int64_t off_ustride,
                         int32_t* perm, int64_t perm_ustride, int32_t* chunk_ws,
                         const Relayout* relayout, uint32_t* err, cudaStream_t s,
                         bool counted = false, int32_t* zero_next = nullptr);

int launch_copy_sinks(const uint16_t* K, const uint16_t* V, int64_t n, int32_t U, int32_t n_sink,
                      uint16_t* spk, uint16_t* spv, int64_t sp_ustride_rows, cudaStream_t s);

struct DecodeArgs {
    const uint16_t* q;
    float* out;
    int32_t* sel_idx;
    int32_t* sel_count;
    int32_t budget;
    int32_t B, Hkv, G;
    int32_t n_sink, pending, C;
    int32_t pstart, pring;  // pending token j is in ring row n_sink + (pstart + j) % pring
    int32_t qsplit;         // per-head selection: virtual units per KV unit (query heads)
    int64_t m;
    const uint16_t* kp;
    const uint16_t* vp;
    const uint16_t* spk;
    const uint16_t* spv;
    const int32_t* ids;
    const int32_t* offsets;
    const float* mu;
    int64_t kp_ustride;   // rows
    int64_t sp_ustride;   // rows
    int64_t off_ustride;  // ints
    int64_t mu_ustride;   // rows of 128
    float* part_scratch;  // [U][cap]
    int64_t part_ustride;
    uint32_t* err;
    // mixed precision (select_and_attend_mixed): clusters at walk rank >= n_near are attended
    // from the fp8 copy (same row layout as kp / vp)
    const uint8_t* kp8;
    const uint8_t* vp8;
    const float* ks8;
    const float* vs8;
    int32_t n_near;
};
// Launch with programmatic dependent launch allowed: the kernel may be scheduled while the
// previous kernel in the stream is still running. Every kernel launched this way calls
// pdl_wait() before it touches memory that earlier work writes, so stream order holds. The
// one exception is the decode kernel, which reads the cluster store before its wait: the last
// kernel of every call that writes the store therefore does not trigger its dependents early
// (they start when it ends).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// fp8 copy of rows [r0, r0 + nrows) of U units (stride ustride rows); no early trigger.
int launch_quantize_rows(const uint16_t* kp, const uint16_t* vp, uint8_t* kp8, uint8_t* vp8,
                         float* ks, float* vs, int64_t ustride, int64_t r0, int64_t nrows,
                         int32_t U, cudaStream_t s);

// Rows [0, n) at `rows` are stored rows r0 .. r0 + n - 1 of a unit (16 units of unit_bytes
// each: 16 for bf16 rows, 8 for fp8 rows): swaps their order between logical and stored.
int launch_swizzle_rows(void* rows, int32_t unit_bytes, int64_t r0, int64_t n, cudaStream_t s);

// One bounded mbarrier wait that nothing completes, with the given limit (test hook).
int launch_expire_wait(uint32_t* err, uint64_t limit_ns, uint32_t* waited_ns, cudaStream_t s);

int launch_select_attend(const DecodeArgs& a, int num_sms, cudaStream_t s);
int launch_select_attend_per_head(const DecodeArgs& a, int num_sms, cudaStream_t s);
int launch_select_attend_mixed(const DecodeArgs& a, int num_sms, cudaStream_t s);

int launch_append(const uint16_t* k, const uint16_t* v, int32_t U, uint16_t* spk, uint16_t* spv,
                  int64_t sp_ustride_rows, int32_t row, cudaStream_t s);

struct ReclusterArgs {
    int32_t U;
    int32_t n_sink, window, C_new, iters;
    int32_t win_row0;  // row of the window's first token in a unit's sink / pending rows
    int32_t C_old;
    int64_t m_old;
    uint64_t seed;
    int64_t unit_base;
    uint64_t window_no;
    uint16_t* spk;
    uint16_t* spv;
    int64_t sp_ustride;
    uint16_t* kp;
    uint16_t* vp;
    int32_t* ids;
    int64_t kp_ustride;
    int32_t* offsets;
    int64_t off_ustride;
    float* mu;
    int64_t mu_ustride;
    float* mu_trace;
    int32_t* assign_trace;
};
int launch_recluster(const ReclusterArgs& a, cudaStream_t s);

struct SplitArgs {
    int32_t U, C, Cmax, room, iters;
    int64_t m;
    float tau;  // split when drift > tau
    uint64_t seed;
    int64_t unit_base;
    uint64_t window_no;
    uint16_t* kp;
    uint16_t* vp;
    int32_t* ids;
    int64_t kp_ustride;   // rows (also of lab, rk, rv, rid)
    int32_t* offsets;
    int64_t off_ustride;  // ints
    float* mu;
    int64_t mu_ustride;   // rows of 128
    float* drift;         // [U][Cmax]
    float* drift_out;     // optional [U][C]
    int32_t* plan;
    int32_t* count;
    int32_t* tasks;
    float* cmu;
    int32_t* n0;
    float* mu2;
    int32_t* off2;
    int32_t* lab;
    uint16_t* rk;
    uint16_t* rv;
    int32_t* rid;
    uint32_t* err;
};
// Drift, plan, 2-means split and renumbering of one layer (five launches on `s`). Every unit
// ends with C + room clusters (padding with empty clusters where it split fewer).
int launch_split(const SplitArgs& a, cudaStream_t s);

}  // namespace ckv
