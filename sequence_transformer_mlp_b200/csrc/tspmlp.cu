// tspmlp.cu -- the C ABI of libtspmlp (include/tspmlp.h): argument
// validation, the host schedule builder that turns (n, d_model, d_ff, P,
// schedule) into kernel launches, TMA descriptor encoding, and the launches.
//
// The method: "Tensor Parallelism: Splitting the Math" (column split of A,
// row split of B, partial outputs summed into the exact result) and "Folding
// Tensor and Sequence Parallelism for Memory-Efficient Transformer Training &
// Inference", Abstract (gated MLP; weight shards meet every sequence shard in
// ring order while partial outputs accumulate locally).  On one GPU the P
// shards are logical: the schedule visits them in order and adds each
// partial output into an fp32 accumulator in place.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/tspmlp.h"
#include "attn.cuh"
#include "bwd_pair.cuh"
#include "train_pair.cuh"
#include "grad_pair.cuh"
#include "fused.cuh"
#include "fused2.cuh"
#include "pipeline2.cuh"
#include "recipes.cuh"
#include "simt_f32.cuh"

namespace tspmlp {
namespace {

constexpr int kMaxDevices = 64;

// Scratch budgets.  The pass schedule's hidden buffer holds as many whole
// shards as fit in kFwdHiddenBudget: every extra chunk costs a read-modify-
// write pass of the fp32 [n][d_model] accumulator, which measured dearer than
// keeping the chunk's H resident in the 126 MB L2 (one 117 MB chunk beat two
// 59 MB chunks on the Llama-3-8B shape, and the 70B shape gained ~5% going
// from eight chunks to one or two).  The fused schedules keep their H ring
// (or two H chunk buffers) within L2-sized budgets: their consumers read H
// while it is being produced.
constexpr size_t kFwdHiddenBudget = 512ull << 20;  // one bf16 [rows][C] buffer
// The rotated TSP ring's sequence shards a launch, and the token rows a
// one-chunk pass takes: the down projection reads the group's H while that is
// still in L2.
constexpr size_t kRingGroupBudget = 512ull << 20;
constexpr size_t kRowGroupBudget = 128ull << 20;
constexpr size_t kFusedRingBudget = 96ull << 20;   // the fused schedule's H ring
constexpr size_t kFusedPassesBudget = 128ull << 20; // two H chunk buffers of the one-launch passes
// H, dG, dU (bf16) and the fp32 activation-derivative factors together.  The
// backward reads them from HBM anyway (the weight- and input-gradient kernels
// run after the whole chunk is produced), so the chunk is sized for few, large
// launches rather than for L2: one chunk at the Llama-3-8B shape.
constexpr size_t kBwdHiddenBudget = 1024ull << 20;

struct DevInfo {
    bool probed = false;
    bool arch_ok = false;
    int sms = 0;
};

std::mutex g_mu;
DevInfo g_dev[kMaxDevices];

tsp_status_t current_device(int* dev_out, DevInfo* info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TSP_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TSP_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo& di = g_dev[dev];
    if (!di.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return TSP_ERR_CUDA;
        di.arch_ok = (major == 10 && minor == 0);
        di.sms = sms;
        di.probed = true;
    }
    *dev_out = dev;
    *info = di;
    return di.arch_ok ? TSP_OK : TSP_ERR_ARCH;
}

// ---------------------------------------------------------------------------
// TMA descriptors through the driver entry point (no link against libcuda)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Row-major bf16 matrix [outer][inner] with row pitch `pitch` elements, box
// {box_in, box_out}; out-of-range elements read as zero.
bool tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
               uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch * 2};
    cuuint32_t box[2] = {box_in, box_out};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr CUtensorMapSwizzle SW128 = CU_TENSOR_MAP_SWIZZLE_128B;

// The same for an fp16 matrix.
bool tmap_f16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
              uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch * 2};
    cuuint32_t box[2] = {box_in, box_out};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// tracing: CUDA events around each launch, on the launching stream

struct TraceRec {
    const char* name;
    cudaEvent_t a, b;
};
struct TraceStat {
    const char* name;
    int64_t launches;
    double ms;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceRec> g_trace_pending;
std::vector<TraceStat> g_trace_stats;

// Records the start event of a traced launch; returns false if tracing is off.
bool trace_begin(cudaStream_t st, TraceRec* rec, const char* name) {
    {
        std::lock_guard<std::mutex> lk(g_trace_mu);
        if (!g_trace_on) return false;
    }
    rec->name = name;
    if (cudaEventCreate(&rec->a) != cudaSuccess) return false;
    if (cudaEventCreate(&rec->b) != cudaSuccess) {
        cudaEventDestroy(rec->a);
        return false;
    }
    cudaEventRecord(rec->a, st);
    return true;
}

void trace_end(cudaStream_t st, TraceRec* rec) {
    cudaEventRecord(rec->b, st);
    std::lock_guard<std::mutex> lk(g_trace_mu);
    g_trace_pending.push_back(*rec);
}

// ---------------------------------------------------------------------------
// launches

// Paired launch: clusters of two CTAs (cta_group::2 tiles), as many pairs as
// can be resident at once, each walking the tile list persistently.
// Pairs of recipe R that can be resident at once on device `dev` (sets the
// kernel's shared-memory attribute on first use); 0 on a CUDA error.
template <class R>
int pair_capacity(int dev, int sms) {
    constexpr int smem = pair_smem_bytes<R>();
    static_assert(smem <= 232448, "stage ring exceeds 227 KB of shared memory");
    static bool attr_set[kMaxDevices] = {};
    static int max_pairs[kMaxDevices] = {};
    std::lock_guard<std::mutex> lk(g_mu);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(umma_pair_pipeline_kernel<R>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return 0;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(static_cast<unsigned>(sms / 2 * 2));
        q.blockDim = dim3(kPipelineThreads);
        q.dynamicSmemBytes = smem;
        q.attrs = attr;
        q.numAttrs = 1;
        int nc = 0;
        if (cudaOccupancyMaxActiveClusters(&nc, umma_pair_pipeline_kernel<R>, &q) != cudaSuccess ||
            nc <= 0) {
            cudaGetLastError();
            nc = sms / 2;
        }
        max_pairs[dev] = nc;
        attr_set[dev] = true;
    }
    return max_pairs[dev];
}

template <class R>
tsp_status_t launch_pair(const typename R::Params& p, cudaStream_t st, int dev, int sms,
                         const char* trace_name = nullptr) {
    const int tiles = R::num_tiles(p);
    if (tiles <= 0) return TSP_OK;
    constexpr int smem = pair_smem_bytes<R>();
    const int cap = pair_capacity<R>(dev, sms);
    if (cap <= 0) return TSP_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    const int pairs = std::min(tiles, cap);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.blockDim = dim3(kPipelineThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TraceRec rec;
    const bool traced = trace_begin(st, &rec, trace_name ? trace_name : R::kName);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, umma_pair_pipeline_kernel<R>, p);
    if (traced) trace_end(st, &rec);
    return e == cudaSuccess ? TSP_OK : TSP_ERR_CUDA;
}

#define TSP_TRY(expr)                          \
    do {                                       \
        const tsp_status_t _s = (expr);        \
        if (_s != TSP_OK) return _s;           \
    } while (0)

// ---------------------------------------------------------------------------
// schedule builder

struct Chunk {
    int64_t col_base, width;
};

// Hidden-column chunks of the weight-shard schedule, in shard order, at most
// max_cols wide.  A chunk is a run of whole shards (the largest divisor G of P
// whose G shards fit) or, when one shard alone is too wide, an equal cut of a
// shard into 128-multiple sub-chunks.  Chunk edges always include the shard
// edges, so every chunk belongs to one shard or is a union of whole shards.
std::vector<Chunk> plan_chunks(int64_t f, int P, int64_t max_cols) {
    const int64_t fs = f / P;
    std::vector<Chunk> out;
    if (fs <= max_cols) {
        int G = 1;
        for (int g = P; g >= 1; --g)
            if (P % g == 0 && g * fs <= max_cols) {
                G = g;
                break;
            }
        for (int w = 0; w < P; w += G) out.push_back({w * fs, G * fs});
    } else {
        const int64_t k = (fs + max_cols - 1) / max_cols;
        const int64_t sub = ((fs + k - 1) / k + 127) / 128 * 128;
        for (int w = 0; w < P; ++w)
            for (int64_t c = 0; c < fs; c += sub) out.push_back({w * fs + c, std::min(sub, fs - c)});
    }
    return out;
}

// Widest chunk (a multiple of 128 columns, at least 128) whose hidden buffers
// fit `budget` bytes at `bytes_per_col` bytes a hidden column; 0 if none.
int64_t max_chunk_cols(size_t budget, size_t bytes_per_col) {
    const int64_t c = static_cast<int64_t>(budget / std::max<size_t>(bytes_per_col, 1)) / 128 * 128;
    return c >= 128 ? c : 0;
}

inline size_t align256(size_t b) { return (b + 255) / 256 * 256; }

int accum_mode(int pass, int npass) {
    if (npass == 1) return 3;          // bf16(tile)
    if (pass == 0) return 0;           // store fp32
    if (pass == npass - 1) return 2;   // bf16(acc + tile)
    return 1;                          // acc += tile
}

// ---------------------------------------------------------------------------
// validation

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = int64_t(1) << 30;

tsp_status_t validate_shape(int64_t n, int64_t d, int64_t f, int P, tsp_act_t act,
                            tsp_dtype_t dt, tsp_sched_t sched) {
    if (act != TSP_ACT_GELU && act != TSP_ACT_SWIGLU) return TSP_ERR_INVALID_ARG;
    if (dt != TSP_DT_BF16 && dt != TSP_DT_F32) return TSP_ERR_INVALID_ARG;
    if (sched < TSP_SCHED_WEIGHT_SHARDS || sched > TSP_SCHED_SHARD_PASSES_FUSED)
        return TSP_ERR_INVALID_ARG;
    if (n <= 0 || d <= 0 || f <= 0 || P <= 0) return TSP_ERR_INVALID_ARG;
    if (n > kMaxDim || d > kMaxDim || f > kMaxDim || P > 4096) return TSP_ERR_UNSUPPORTED_SHAPE;
    if (f % P != 0) return TSP_ERR_UNSUPPORTED_SHAPE;
    const bool ring = sched == TSP_SCHED_TSP_RING || sched == TSP_SCHED_TSP_RING_FUSED;
    if (ring && n % P != 0) return TSP_ERR_UNSUPPORTED_SHAPE;
    if ((sched == TSP_SCHED_FUSED || sched == TSP_SCHED_TSP_RING_FUSED ||
         sched == TSP_SCHED_SHARD_PASSES_FUSED) &&
        dt != TSP_DT_BF16)
        return TSP_ERR_UNSUPPORTED_SHAPE;
    if (sched == TSP_SCHED_SHARD_PASSES_FUSED && (f / P) % 64 != 0) return TSP_ERR_UNSUPPORTED_SHAPE;
    if (sched == TSP_SCHED_TSP_RING_FUSED && (f / P) % 64 != 0) return TSP_ERR_UNSUPPORTED_SHAPE;
    if (dt == TSP_DT_BF16 && (d % 8 != 0 || (f / P) % 8 != 0)) return TSP_ERR_UNSUPPORTED_SHAPE;
    return TSP_OK;
}

tsp_status_t validate_weights(const void* X, const void* Wg, const void* Wu, const void* Wd,
                              tsp_act_t act) {
    if (!X || !Wg || !Wd) return TSP_ERR_INVALID_ARG;
    if ((act == TSP_ACT_GELU) != (Wu == nullptr)) return TSP_ERR_INVALID_ARG;
    return TSP_OK;
}

tsp_status_t validate_forward(const void* X, const void* Wg, const void* Wu, const void* Wd,
                              int64_t n, int64_t d, int64_t f, int P, tsp_act_t act, tsp_dtype_t dt,
                              tsp_sched_t sched, const void* Y) {
    TSP_TRY(validate_shape(n, d, f, P, act, dt, sched));
    TSP_TRY(validate_weights(X, Wg, Wu, Wd, act));
    if (!Y) return TSP_ERR_INVALID_ARG;
    const size_t e = dt == TSP_DT_BF16 ? 2 : 4;
    const size_t xb = n * d * e, wb = d * f * e, yb = n * d * e;
    if (overlaps(Y, yb, X, xb) || overlaps(Y, yb, Wg, wb) || overlaps(Y, yb, Wu, wb) ||
        overlaps(Y, yb, Wd, wb))
        return TSP_ERR_INVALID_ARG;
    if (dt == TSP_DT_BF16 && (!aligned16(X) || !aligned16(Wg) || !aligned16(Wd) || !aligned16(Y) ||
                              (Wu && !aligned16(Wu))))
        return TSP_ERR_UNSUPPORTED_SHAPE;
    if (dt == TSP_DT_F32) {
        const void* ps[5] = {X, Wg, Wu, Wd, Y};
        for (const void* q : ps)
            if (q && (reinterpret_cast<uintptr_t>(q) & 3u)) return TSP_ERR_UNSUPPORTED_SHAPE;
    }
    return TSP_OK;
}

tsp_status_t validate_backward(const void* X, const void* Wg, const void* Wu, const void* Wd,
                               const void* dY, int64_t n, int64_t d, int64_t f, int P,
                               tsp_act_t act, const void* dX, const float* dWg, const float* dWu,
                               const float* dWd) {
    TSP_TRY(validate_shape(n, d, f, P, act, TSP_DT_BF16, TSP_SCHED_WEIGHT_SHARDS));
    TSP_TRY(validate_weights(X, Wg, Wu, Wd, act));
    if (!dY || !dX || !dWg || !dWd) return TSP_ERR_INVALID_ARG;
    if ((act == TSP_ACT_SWIGLU) != (dWu != nullptr)) return TSP_ERR_INVALID_ARG;
    const size_t xb = n * d * 2, wb = d * f * 2, gw = d * f * 4;
    const void* ins[5] = {X, Wg, Wu, Wd, dY};
    const size_t insz[5] = {xb, wb, wb, wb, xb};
    const void* outs[4] = {dX, dWg, dWu, dWd};
    const size_t outsz[4] = {xb, gw, gw, gw};
    for (int o = 0; o < 4; ++o) {
        for (int i = 0; i < 5; ++i)
            if (overlaps(outs[o], outsz[o], ins[i], insz[i])) return TSP_ERR_INVALID_ARG;
        for (int o2 = o + 1; o2 < 4; ++o2)
            if (overlaps(outs[o], outsz[o], outs[o2], outsz[o2])) return TSP_ERR_INVALID_ARG;
    }
    for (int i = 0; i < 5; ++i)
        if (ins[i] && !aligned16(ins[i])) return TSP_ERR_UNSUPPORTED_SHAPE;
    for (int o = 0; o < 4; ++o)
        if (outs[o] && !aligned16(outs[o])) return TSP_ERR_UNSUPPORTED_SHAPE;
    return TSP_OK;
}

// ---------------------------------------------------------------------------
// forward

struct FwdPlan {
    bool ok = true;
    bool ring = false;
    // TSP ring as whole-d_ff hidden blocks per sequence shard and a down
    // projection with each shard's K loop in ring order (bf16)
    bool ring_rotated = false;
    // the pass schedule in one paired launch (two H chunk buffers)
    bool fused_passes = false;
    // fused single-launch schedule (bf16)
    bool fused = false;
    int segs = 1, seg_rows = 0, mts = 0, MB = 0, GM = 1, R = 1;
    size_t ring_bytes = 0, sync_bytes = 0;
    // per-chunk pass schedule
    std::vector<Chunk> chunks;  // weight-shard passes
    int tsp_group = 1;          // ring passes: sequence shards per launch
    int64_t row_group = 0;      // > 0: one-chunk passes over groups of this many token rows
    size_t h_bytes = 0, acc_bytes = 0;
    // one-chunk passes: room for the down projection's tail split (the fp32
    // partial sums and flags of up to kMaxSplitTiles tiles); 0 = no split
    size_t split_bytes = 0;
    size_t total() const {
        if (fused) return align256(ring_bytes) + align256(sync_bytes);
        if (fused_passes) return 2 * align256(h_bytes) + align256(acc_bytes) + align256(sync_bytes);
        return align256(h_bytes) + align256(acc_bytes) + split_bytes;
    }
};

// The down projection's tail split: when a launch's last wave of 256 x 256
// tiles fills at most half the pairs, each of those tiles runs as two halves
// of its K loop on two pairs (DownAccum::Params::split_from).  The area holds
// the first halves' fp32 sums and one flag per epilogue warp.
constexpr int kMaxSplitTiles = 64;
constexpr size_t kSplitPartBytes = static_cast<size_t>(kMaxSplitTiles) * 256 * 256 * 4;
constexpr size_t kSplitFlagBytes = static_cast<size_t>(kMaxSplitTiles) * 8 * 4;
constexpr size_t kSplitBytes = kSplitPartBytes + 256 + kSplitFlagBytes + 256;

// The fused schedule: row blocks of 128 tokens per sequence segment, grouped
// GM at a time; the H ring holds three groups (R = 3*GM row-block slots, or one
// per row block when that is fewer).  Larger groups re-read the weights fewer
// times (once per group); GM is the largest of kFusedGroupRows that keeps the
// ring within the budget.
constexpr int kFusedGroupRows = 8;

bool plan_fused(int64_t n, int64_t d, int64_t f, int P, bool ring, size_t budget, FwdPlan* pl) {
    (void)d;
    pl->fused = true;
    pl->ring = ring;
    pl->segs = ring ? P : 1;
    pl->seg_rows = static_cast<int>(ring ? n / P : n);
    pl->mts = (pl->seg_rows + 127) / 128;
    pl->MB = pl->segs * pl->mts;
    const size_t slot = static_cast<size_t>(128) * f * 2;
    int GM = std::min(pl->MB, kFusedGroupRows);
    int R = std::min(pl->MB, 3 * GM);
    while (GM > 1 && static_cast<size_t>(R) * slot > budget) {
        --GM;
        R = std::min(pl->MB, 3 * GM);
    }
    pl->GM = GM;
    pl->R = R;
    pl->ring_bytes = static_cast<size_t>(R) * slot;
    pl->sync_bytes = static_cast<size_t>(1 + 2 * pl->MB) * 4;
    return pl->ring_bytes <= budget;
}

// Schedule of the forward pass for a hidden-buffer budget.  ok == false when
// not even the narrowest schedule fits.
FwdPlan plan_forward_budget(int64_t n, int64_t d, int64_t f, int P, tsp_dtype_t dt,
                            tsp_sched_t sched, size_t budget) {
    FwdPlan pl;
    const size_t e = dt == TSP_DT_BF16 ? 2 : 4;
    const int64_t fs = f / P;
    if (dt == TSP_DT_BF16 && (sched == TSP_SCHED_FUSED || sched == TSP_SCHED_TSP_RING_FUSED)) {
        pl.ok = plan_fused(n, d, f, P, sched == TSP_SCHED_TSP_RING_FUSED, budget, &pl);
        return pl;
    }
    if (sched == TSP_SCHED_TSP_RING) {
        pl.ring = true;
        // bf16 with 64-column shards: each sequence shard's hidden block for all
        // d_ff columns, and one down projection whose K loop visits the shards in
        // its ring order (no fp32 accumulator), for as many sequence shards a
        // launch as fit the budget
        const size_t per_seg_all = static_cast<size_t>(n / P) * f * e;
        if (dt == TSP_DT_BF16 && fs % 128 == 0 && budget >= per_seg_all) {
            pl.ring_rotated = true;
            pl.tsp_group = static_cast<int>(
                std::min<size_t>(P, std::max<size_t>(1, std::min(budget, kRingGroupBudget) / per_seg_all)));
            pl.h_bytes = static_cast<size_t>(pl.tsp_group) * per_seg_all;
            pl.acc_bytes = 0;
            return pl;
        }
        const size_t per_seg = static_cast<size_t>(n / P) * fs * e;
        pl.tsp_group = dt == TSP_DT_BF16
                           ? static_cast<int>(std::min<size_t>(P, budget / std::max<size_t>(per_seg, 1)))
                           : P;
        if (pl.tsp_group < 1) {
            pl.tsp_group = 1;
            pl.ok = budget >= per_seg;
        }
        pl.h_bytes = static_cast<size_t>(pl.tsp_group) * per_seg;
        pl.acc_bytes = (dt == TSP_DT_BF16 && P > 1) ? static_cast<size_t>(n) * d * 4 : 0;
        return pl;
    }
    if (dt == TSP_DT_BF16 && sched != TSP_SCHED_SHARD_PASSES_FUSED) {
        // Row groups: token rows are independent, so when all of H does not
        // fit in L2 the rows run in equal groups (multiples of 256) of at
        // most kRowGroupBudget of H, each a one-chunk pass summing every shard
        // in tensor memory -- no fp32 accumulator, H read back from L2.
        const size_t per_row = static_cast<size_t>(f) * e;
        const size_t rg = std::min(budget, kRowGroupBudget);
        const int64_t cap = static_cast<int64_t>(rg / per_row) / 256 * 256;
        if (static_cast<size_t>(n) * per_row > rg && cap >= 256) {
            const int64_t groups = (n + cap - 1) / cap;
            pl.row_group = ((n + groups - 1) / groups + 255) / 256 * 256;
            pl.chunks = {{0, f}};
            pl.h_bytes = static_cast<size_t>(pl.row_group) * per_row;
            pl.acc_bytes = 0;
            return pl;
        }
    }
    if (dt == TSP_DT_BF16) {
        // the one-launch pass schedule holds two H chunks; it needs chunk widths
        // that are whole 64-column k-blocks and at most kFusedMaxChunks chunks
        const bool try_fused = sched == TSP_SCHED_SHARD_PASSES_FUSED;
        const int64_t mc = max_chunk_cols(try_fused ? budget / 2 : budget, static_cast<size_t>(n) * 2);
        if (mc == 0) {
            pl.ok = false;
            return pl;
        }
        pl.chunks = plan_chunks(f, P, mc);
        if (try_fused) {
            pl.fused_passes = true;
            pl.ok = static_cast<int>(pl.chunks.size()) <= kFusedMaxChunks;
            pl.sync_bytes = static_cast<size_t>(1 + 2 * pl.chunks.size() * ((n + 255) / 256)) * 4;
        }
    } else {
        // fp32: chunks of whole shards within the same budget (no sub-shard cuts)
        const int64_t mc = max_chunk_cols(budget, static_cast<size_t>(n) * 4);
        pl.chunks = plan_chunks(f, P, std::max(mc, fs));
    }
    int64_t wmax = 0;
    for (auto& c : pl.chunks) wmax = std::max(wmax, c.width);
    pl.h_bytes = static_cast<size_t>(n) * wmax * e;
    pl.acc_bytes = (dt == TSP_DT_BF16 && pl.chunks.size() > 1) ? static_cast<size_t>(n) * d * 4 : 0;
    return pl;
}

// The preferred schedule: hidden buffers within their budgets.
FwdPlan plan_forward(int64_t n, int64_t d, int64_t f, int P, tsp_dtype_t dt, tsp_sched_t sched) {
    FwdPlan pl = plan_forward_budget(n, d, f, P, dt, sched, kFusedRingBudget);
    if (pl.fused) return pl;
    pl = plan_forward_budget(n, d, f, P, dt, sched,
                             sched == TSP_SCHED_SHARD_PASSES_FUSED ? kFusedPassesBudget
                                                                   : kFwdHiddenBudget);
    // one-chunk weight-shard passes write Y directly: room for the tail split
    if (dt == TSP_DT_BF16 && !pl.fused_passes && !pl.ring && pl.acc_bytes == 0 &&
        (pl.row_group > 0 || pl.chunks.size() == 1))
        pl.split_bytes = kSplitBytes;
    return pl;
}

// The schedule for a caller workspace of ws_bytes: the preferred one if it
// fits, otherwise a narrower one (bf16 only): fewer H-ring slots for the fused
// schedule, narrower hidden chunks for the pass schedules.
FwdPlan plan_forward_for(int64_t n, int64_t d, int64_t f, int P, tsp_dtype_t dt, tsp_sched_t sched,
                         size_t ws_bytes) {
    FwdPlan pl = plan_forward(n, d, f, P, dt, sched);
    if (pl.total() <= ws_bytes || dt != TSP_DT_BF16) return pl;
    if (pl.split_bytes > 0 && pl.total() - pl.split_bytes <= ws_bytes) {
        pl.split_bytes = 0;  // the same passes without the tail split
        return pl;
    }
    pl.split_bytes = 0;
    if (pl.fused) {
        const size_t sync = align256(pl.sync_bytes);
        if (ws_bytes <= sync + 256) {
            pl.ok = false;
            return pl;
        }
        pl = plan_forward_budget(n, d, f, P, dt, sched, ws_bytes - sync - 256);
        if (pl.total() > ws_bytes) pl.ok = false;
        return pl;
    }
    {
        // fewer sequence shards (ring) or token rows (row groups) a launch,
        // still without an accumulator
        FwdPlan r = plan_forward_budget(n, d, f, P, dt, sched, ws_bytes);
        if ((r.ring_rotated || r.row_group > 0) && r.ok && r.total() <= ws_bytes) return r;
    }
    const size_t acc = align256(static_cast<size_t>(n) * d * 4);
    if (sched == TSP_SCHED_SHARD_PASSES_FUSED) {
        // two H chunk buffers and the counters
        const size_t sync =
            align256(static_cast<size_t>(1 + 2 * kFusedMaxChunks * ((n + 255) / 256)) * 4);
        if (ws_bytes <= acc + sync + 512) {
            pl.ok = false;
            return pl;
        }
        pl = plan_forward_budget(n, d, f, P, dt, sched, ws_bytes - acc - sync - 512);
        if (pl.total() > ws_bytes) pl.ok = false;
        return pl;
    }
    if (ws_bytes <= acc + 256) {
        pl.ok = false;
        return pl;
    }
    pl = plan_forward_budget(n, d, f, P, dt, sched, ws_bytes - acc - 256);
    if (pl.total() > ws_bytes) pl.ok = false;
    return pl;
}

SegGeom seg_all_rows(int64_t n, int P, int64_t fs, int64_t col_base) {
    SegGeom g{};
    g.seg_rows = static_cast<int>(n);
    g.num_segs = 1;
    g.seg_begin = 0;
    g.ring = 0;
    g.ring_step = 0;
    g.P = P;
    g.fs = static_cast<int>(fs);
    g.col_base = static_cast<int>(col_base);
    return g;
}

SegGeom seg_ring(int64_t n, int P, int64_t fs, int seg_begin, int num_segs, int t) {
    SegGeom g{};
    g.seg_rows = static_cast<int>(n / P);
    g.num_segs = num_segs;
    g.seg_begin = seg_begin;
    g.ring = 1;
    g.ring_step = t;
    g.P = P;
    g.fs = static_cast<int>(fs);
    g.col_base = 0;
    return g;
}

// One pass of the bf16 forward: K1 over the segments' hidden chunk, then K2
// adding the chunk's partial output into the accumulator.
template <int ACT>
tsp_status_t fwd_pass_bf16(const void* X, const void* Wg, const void* Wu, const void* Wd,
                           int64_t n, int64_t d, int64_t f, const SegGeom& g, int64_t width,
                           int mode, __nv_bfloat16* H, float* acc, void* Y, cudaStream_t st,
                           int dev, int sms, int rot_P = 0, uint32_t* S1 = nullptr,
                           uint32_t* S2 = nullptr, char* split_area = nullptr) {
    using K1 = FwdHidden<ACT>;
    using K2 = DownAccum<true, 1>;
    typename K1::Params p1;
    std::memset(&p1, 0, sizeof(p1));
    if (!tmap_bf16(&p1.tmX, X, d, n, d, 64, 128, SW128) ||
        !tmap_bf16(&p1.tmG, Wg, f, d, f, 64, 128, SW128) ||
        (ACT == 1 && !tmap_bf16(&p1.tmU, Wu, f, d, f, 64, 128, SW128)))
        return TSP_ERR_CUDA;
    p1.g = g;
    p1.d = static_cast<int>(d);
    p1.width = static_cast<int>(width);
    p1.H = H;
    p1.ldh = width;
    if (S1) {
        // training forward: the same tiles, keeping the activation's factors
        FwdHiddenSaveParams<ACT> ps;
        std::memset(&ps, 0, sizeof(ps));
        static_cast<typename K1::Params&>(ps) = p1;
        ps.S1 = S1;
        ps.S2 = S2;
        TSP_TRY(launch_pair<FwdHiddenSavePair<ACT>>(ps, st, dev, sms));
    } else {
        TSP_TRY(launch_pair<FwdHiddenPair<ACT>>(p1, st, dev, sms));
    }

    typename K2::Params p2;
    std::memset(&p2, 0, sizeof(p2));
    const int64_t hrows = static_cast<int64_t>(g.num_segs) * g.seg_rows;
    if (!tmap_bf16(&p2.tmA0, H, width, hrows, width, 64, 128, SW128) ||
        !tmap_bf16(&p2.tmB0, Wd, d, f, d, 64, 128, SW128))
        return TSP_ERR_CUDA;
    p2.g = g;
    p2.kdim = static_cast<int>(width);
    p2.n_out = static_cast<int>(d);
    p2.mode = mode;
    p2.rot_P = rot_P;
    p2.acc = acc;
    p2.ldacc = d;
    p2.out = static_cast<__nv_bfloat16*>(Y);
    p2.ldo = d;
    using D2 = DownAccumPair<true, 1, 256>;
    if (split_area && mode == 3 && rot_P == 0) {
        // a last wave of r tiles on at most half the pairs: each of its tiles
        // as two halves of the K loop, so the wave takes half as long
        const int T = D2::whole_tiles(p2), cap = pair_capacity<D2>(dev, sms);
        const int r = cap > 0 ? T % cap : 0;
        if (T > cap && r > 0 && 2 * r <= cap && r <= kMaxSplitTiles && D2::kblocks(p2) >= 2) {
            p2.split_from = T - r;
            p2.part = reinterpret_cast<float*>(split_area);
            p2.flags = reinterpret_cast<int*>(split_area + kSplitPartBytes + 256);
            if (cudaMemsetAsync(p2.flags, 0, static_cast<size_t>(r) * 8 * sizeof(int), st) !=
                cudaSuccess)
                return TSP_ERR_CUDA;
        }
    }
    return launch_pair<D2>(p2, st, dev, sms);
}

// The whole forward as one persistent launch (fused.cuh).
template <int ACT>
tsp_status_t forward_bf16_fused(const void* X, const void* Wg, const void* Wu, const void* Wd,
                                int64_t n, int64_t d, int64_t f, int P, const FwdPlan& pl,
                                void* Y, void* ws, cudaStream_t st, int dev, int sms) {
    using C = FusedFwd<ACT>;
    char* w = static_cast<char*>(ws);
    auto* H = reinterpret_cast<__nv_bfloat16*>(w);
    auto* sync = reinterpret_cast<unsigned*>(w + align256(pl.ring_bytes));
    FusedFwdParams p;
    std::memset(&p, 0, sizeof(p));
    if (!tmap_bf16(&p.tmX, X, d, n, d, 64, 128, SW128) ||
        !tmap_bf16(&p.tmG, Wg, f, d, f, 64, 64, SW128) ||
        (ACT == 1 && !tmap_bf16(&p.tmU, Wu, f, d, f, 64, 64, SW128)) ||
        !tmap_bf16(&p.tmH, H, f, static_cast<uint64_t>(pl.R) * 128, f, 64, 128, SW128) ||
        !tmap_bf16(&p.tmD, Wd, d, f, d, 64, 64, SW128))
        return TSP_ERR_CUDA;
    p.n = static_cast<int>(n);
    p.d = static_cast<int>(d);
    p.f = static_cast<int>(f);
    p.seg_rows = pl.seg_rows;
    p.mts = pl.mts;
    p.ring = pl.ring ? 1 : 0;
    p.fs = static_cast<int>(f / P);
    p.MB = pl.MB;
    p.nJ = static_cast<int>((f + C::kOut - 1) / C::kOut);
    p.nC = static_cast<int>((d + 255) / 256);
    p.GM = pl.GM;
    p.G = (pl.MB + pl.GM - 1) / pl.GM;
    p.head = sms;
    p.R = pl.R;
    p.total = p.MB * (p.nJ + p.nC);
    p.H = H;
    p.Y = static_cast<__nv_bfloat16*>(Y);
    p.sync = sync;
    if (cudaMemsetAsync(sync, 0, pl.sync_bytes, st) != cudaSuccess) return TSP_ERR_CUDA;
    static bool attr_set[kMaxDevices] = {};
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(fused_mlp_fwd_kernel<ACT>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::kSmemBytes) != cudaSuccess)
                return TSP_ERR_CUDA;
            attr_set[dev] = true;
        }
    }
    const int grid = std::min(p.total, sms);
    TraceRec rec;
    const bool traced = trace_begin(st, &rec, C::kName);
    fused_mlp_fwd_kernel<ACT><<<grid, kPipelineThreads, C::kSmemBytes, st>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (traced) trace_end(st, &rec);
    return e == cudaSuccess ? TSP_OK : TSP_ERR_CUDA;
}

// The pass schedule as one persistent paired launch (fused2.cuh).
template <int ACT>
tsp_status_t forward_bf16_fused_passes(const void* X, const void* Wg, const void* Wu,
                                       const void* Wd, int64_t n, int64_t d, int64_t f,
                                       const FwdPlan& pl, void* Y, void* ws, cudaStream_t st,
                                       int dev, int sms) {
    using Cfg = FusedPassesCfg<ACT>;
    char* w = static_cast<char*>(ws);
    const size_t hb = align256(pl.h_bytes);
    int64_t wmax = 0;
    for (auto& c : pl.chunks) wmax = std::max(wmax, c.width);
    auto* H0 = reinterpret_cast<__nv_bfloat16*>(w);
    auto* H1 = reinterpret_cast<__nv_bfloat16*>(w + hb);
    float* acc = pl.acc_bytes ? reinterpret_cast<float*>(w + 2 * hb) : nullptr;
    auto* sync = reinterpret_cast<unsigned*>(w + 2 * hb + align256(pl.acc_bytes));
    FusedPassesParams p;
    std::memset(&p, 0, sizeof(p));
    if (!tmap_bf16(&p.tmX, X, d, n, d, 64, 128, SW128) ||
        !tmap_bf16(&p.tmG, Wg, f, d, f, 64, 64, SW128) ||
        (ACT == 1 && !tmap_bf16(&p.tmU, Wu, f, d, f, 64, 64, SW128)) ||
        !tmap_bf16(&p.tmH0, H0, wmax, n, wmax, 64, 128, SW128) ||
        !tmap_bf16(&p.tmH1, H1, wmax, n, wmax, 64, 128, SW128) ||
        !tmap_bf16(&p.tmD, Wd, d, f, d, 64, 64, SW128))
        return TSP_ERR_CUDA;
    p.n = static_cast<int>(n);
    p.d = static_cast<int>(d);
    p.f = static_cast<int>(f);
    p.MP = static_cast<int>((n + 255) / 256);
    p.C = static_cast<int>(pl.chunks.size());
    for (int i = 0; i < p.C; ++i) {
        p.cb[i] = static_cast<int>(pl.chunks[i].col_base);
        p.cw[i] = static_cast<int>(pl.chunks[i].width);
    }
    p.nN = static_cast<int>((d + 255) / 256);
    p.wmax = static_cast<int>(wmax);
    p.H0 = H0;
    p.H1 = H1;
    p.acc = acc;
    p.Y = static_cast<__nv_bfloat16*>(Y);
    p.sync = sync;
    int total = 0;
    for (int i = 0; i < p.C; ++i) total += pass_nj<Cfg::kOut>(p, i) * p.MP + p.nN * p.MP;
    p.total = total;
    const size_t sync_bytes = static_cast<size_t>(1 + 2 * p.C * p.MP) * 4;
    if (cudaMemsetAsync(sync, 0, sync_bytes, st) != cudaSuccess) return TSP_ERR_CUDA;
    static bool attr_set[kMaxDevices] = {};
    static int max_pairs[kMaxDevices] = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(fused_passes_pair_kernel<ACT>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg::kSmemBytes) != cudaSuccess)
                return TSP_ERR_CUDA;
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(static_cast<unsigned>(sms / 2 * 2));
            q.blockDim = dim3(kPipelineThreads);
            q.dynamicSmemBytes = Cfg::kSmemBytes;
            q.attrs = attr;
            q.numAttrs = 1;
            int nc = 0;
            if (cudaOccupancyMaxActiveClusters(&nc, fused_passes_pair_kernel<ACT>, &q) != cudaSuccess ||
                nc <= 0) {
                cudaGetLastError();
                nc = sms / 2;
            }
            max_pairs[dev] = nc;
            attr_set[dev] = true;
        }
    }
    const int pairs = std::min(total, max_pairs[dev]);
    p.head = pairs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.blockDim = dim3(kPipelineThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TraceRec rec;
    const bool traced = trace_begin(st, &rec, Cfg::kName);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fused_passes_pair_kernel<ACT>, p);
    if (traced) trace_end(st, &rec);
    return e == cudaSuccess ? TSP_OK : TSP_ERR_CUDA;
}

template <int ACT>
tsp_status_t forward_bf16(const void* X, const void* Wg, const void* Wu, const void* Wd, int64_t n,
                          int64_t d, int64_t f, int P, const FwdPlan& pl, void* Y, void* ws,
                          cudaStream_t st, int dev, int sms) {
    if (pl.fused) return forward_bf16_fused<ACT>(X, Wg, Wu, Wd, n, d, f, P, pl, Y, ws, st, dev, sms);
    if (pl.fused_passes)
        return forward_bf16_fused_passes<ACT>(X, Wg, Wu, Wd, n, d, f, pl, Y, ws, st, dev, sms);
    auto* H = static_cast<__nv_bfloat16*>(ws);
    float* acc = pl.acc_bytes ? reinterpret_cast<float*>(static_cast<char*>(ws) +
                                                         align256(pl.h_bytes))
                              : nullptr;
    char* split = pl.split_bytes ? static_cast<char*>(ws) + align256(pl.h_bytes) +
                                       align256(pl.acc_bytes)
                                 : nullptr;
    const int64_t fs = f / P;
    if (pl.row_group > 0) {
        // independent row groups: each a complete one-chunk pass on offset views
        const size_t xe = static_cast<size_t>(d) * 2;
        for (int64_t r0 = 0; r0 < n; r0 += pl.row_group) {
            const int64_t rows = std::min<int64_t>(pl.row_group, n - r0);
            const void* Xg = static_cast<const char*>(X) + r0 * xe;
            void* Yg = static_cast<char*>(Y) + r0 * xe;
            const SegGeom g = seg_all_rows(rows, P, fs, 0);
            TSP_TRY(fwd_pass_bf16<ACT>(Xg, Wg, Wu, Wd, rows, d, f, g, f, 3, H, nullptr, Yg, st, dev,
                                       sms, 0, nullptr, nullptr, split));
        }
        return TSP_OK;
    }
    if (!pl.ring) {
        const int np = static_cast<int>(pl.chunks.size());
        for (int i = 0; i < np; ++i) {
            const SegGeom g = seg_all_rows(n, P, fs, pl.chunks[i].col_base);
            TSP_TRY(fwd_pass_bf16<ACT>(X, Wg, Wu, Wd, n, d, f, g, pl.chunks[i].width,
                                       accum_mode(i, np), H, acc, Y, st, dev, sms, 0, nullptr,
                                       nullptr, split));
        }
    } else if (pl.ring_rotated) {
        for (int s0 = 0; s0 < P; s0 += pl.tsp_group) {
            const int cnt = std::min(pl.tsp_group, P - s0);
            SegGeom g = seg_all_rows(n, P, fs, 0);
            g.seg_rows = static_cast<int>(n / P);
            g.num_segs = cnt;
            g.seg_begin = s0;
            TSP_TRY(fwd_pass_bf16<ACT>(X, Wg, Wu, Wd, n, d, f, g, f, /*mode direct*/ 3, H, nullptr, Y,
                                       st, dev, sms, P));
        }
    } else {
        for (int t = 0; t < P; ++t)
            for (int s0 = 0; s0 < P; s0 += pl.tsp_group) {
                const int cnt = std::min(pl.tsp_group, P - s0);
                const SegGeom g = seg_ring(n, P, fs, s0, cnt, t);
                TSP_TRY(fwd_pass_bf16<ACT>(X, Wg, Wu, Wd, n, d, f, g, fs, accum_mode(t, P), H, acc,
                                           Y, st, dev, sms));
            }
    }
    return TSP_OK;
}

// ---------------------------------------------------------------------------
// training forward: the weight-shard pass schedule with its activations kept
//
// The block is the gated MLP of "Folding Tensor and Sequence Parallelism for
// Memory-Efficient Transformer Training & Inference" (Abstract) or the plain
// one of "Tensor Parallelism: Splitting the Math"; that page notes that the
// backward pass repeats the forward's split.  The backward needs, per hidden
// unit, the derivative of the activation at the pre-activation; the forward
// keeps those factors (train_pair.cuh) so that the backward need not run the
// gate/up projection again.

// Saved activations: H (bf16 [n][f]), then the bf16 factor regions S1 (and
// S2 for SwiGLU), each of whole 32-row blocks of f columns (the layout of
// train_pair.cuh: bf16x2 words of column pairs), every region 256-byte aligned.
struct SavedLayout {
    size_t h = 0, s = 0;
    int nfac = 1;
    // scratch for the down projection's tail split (as the forward's
    // workspace has), so that the training forward's Y is the forward's bit
    // for bit
    size_t split = kSplitBytes;
    size_t total() const { return h + nfac * s + split; }
    size_t split_offset() const { return h + nfac * s; }
};

SavedLayout saved_layout(int64_t n, int64_t f, tsp_act_t act) {
    SavedLayout l;
    l.h = align256(static_cast<size_t>(n) * f * 2);
    l.s = align256(static_cast<size_t>((n + 31) / 32 * 32) * f * 2);
    l.nfac = act == TSP_ACT_SWIGLU ? 2 : 1;
    return l;
}

// Token rows a launch pair of the training forward covers: the row groups of
// the pass schedule (at most kRowGroupBudget of H, equal multiples of 256
// rows), else all rows.
int64_t train_row_group(int64_t n, int64_t f) {
    const size_t per_row = static_cast<size_t>(f) * 2;
    const int64_t cap = static_cast<int64_t>(kRowGroupBudget / per_row) / 256 * 256;
    if (static_cast<size_t>(n) * per_row <= kRowGroupBudget || cap < 256) return n;
    const int64_t groups = (n + cap - 1) / cap;
    return ((n + groups - 1) / groups + 255) / 256 * 256;
}

template <int ACT>
tsp_status_t forward_train_bf16(const void* X, const void* Wg, const void* Wu, const void* Wd,
                                int64_t n, int64_t d, int64_t f, int P, void* Y, void* saved,
                                cudaStream_t st, int dev, int sms) {
    const SavedLayout sl = saved_layout(n, f, ACT == 1 ? TSP_ACT_SWIGLU : TSP_ACT_GELU);
    char* base = static_cast<char*>(saved);
    auto* H = reinterpret_cast<__nv_bfloat16*>(base);
    auto* S1 = reinterpret_cast<uint32_t*>(base + sl.h);
    uint32_t* S2 = ACT == 1 ? reinterpret_cast<uint32_t*>(base + sl.h + sl.s) : nullptr;
    const int64_t fs = f / P, rg = train_row_group(n, f);
    const size_t xe = static_cast<size_t>(d) * 2;
    for (int64_t r0 = 0; r0 < n; r0 += rg) {
        const int64_t rows = std::min<int64_t>(rg, n - r0);
        const void* Xg = static_cast<const char*>(X) + r0 * xe;
        void* Yg = static_cast<char*>(Y) + r0 * xe;
        const SegGeom g = seg_all_rows(rows, P, fs, 0);
        // row groups start on 256-row boundaries, so a group's factors begin
        // at element r0 x f, as its rows of H: word r0 x f / 2
        const int64_t ho = r0 * f, so = ho / 2;
        TSP_TRY(fwd_pass_bf16<ACT>(Xg, Wg, Wu, Wd, rows, d, f, g, f, /*mode direct*/ 3, H + ho,
                                   nullptr, Yg, st, dev, sms, 0, S1 + so, S2 ? S2 + so : nullptr,
                                   base + sl.split_offset()));
    }
    return TSP_OK;
}

// Grid of TM x TM output tiles over rows x cols for each segment.
template <int TM>
dim3 f32_grid(int64_t cols, int rows, int segs) {
    return dim3(static_cast<unsigned>((cols + TM - 1) / TM), static_cast<unsigned>((rows + TM - 1) / TM),
                static_cast<unsigned>(segs));
}

// Large tiles when they make at least one block per SM, small ones otherwise.
bool f32_small_tiles(int64_t cols, int rows, int segs, int sms) {
    const dim3 g = f32_grid<kF32TileLarge>(cols, rows, segs);
    return static_cast<int64_t>(g.x) * g.y * g.z < sms;
}

template <int ACT>
void launch_f32_hidden(const float* X, const float* Wg, const float* Wu, int64_t d, int64_t f,
                       const SegGeom& g, int64_t width, float* H, cudaStream_t st, int sms) {
    if (f32_small_tiles(width, g.seg_rows, g.num_segs, sms))
        f32_hidden_kernel<ACT, kF32TileSmall, kF32KSmall>
            <<<f32_grid<kF32TileSmall>(width, g.seg_rows, g.num_segs), 256, 0, st>>>(
                X, Wg, Wu, static_cast<int>(d), static_cast<int>(f), g, static_cast<int>(width), H, width);
    else
        f32_hidden_kernel<ACT, kF32TileLarge, kF32KLarge>
            <<<f32_grid<kF32TileLarge>(width, g.seg_rows, g.num_segs), 256, 0, st>>>(
                X, Wg, Wu, static_cast<int>(d), static_cast<int>(f), g, static_cast<int>(width), H, width);
}

tsp_status_t forward_f32(const float* X, const float* Wg, const float* Wu, const float* Wd,
                         int64_t n, int64_t d, int64_t f, int P, tsp_act_t act, const FwdPlan& pl,
                         float* Y, void* ws, cudaStream_t st, int sms) {
    float* H = static_cast<float*>(ws);
    const int64_t fs = f / P;
    auto run = [&](const SegGeom& g, int64_t width, int first) -> tsp_status_t {
        TraceRec rec;
        bool traced = trace_begin(st, &rec, act == TSP_ACT_SWIGLU ? "f32_hidden_swiglu" : "f32_hidden_gelu");
        if (act == TSP_ACT_SWIGLU)
            launch_f32_hidden<1>(X, Wg, Wu, d, f, g, width, H, st, sms);
        else
            launch_f32_hidden<0>(X, Wg, Wu, d, f, g, width, H, st, sms);
        if (traced) trace_end(st, &rec);
        if (cudaGetLastError() != cudaSuccess) return TSP_ERR_CUDA;
        traced = trace_begin(st, &rec, "f32_down");
        if (f32_small_tiles(d, g.seg_rows, g.num_segs, sms))
            f32_down_kernel<kF32TileSmall, kF32KSmall>
                <<<f32_grid<kF32TileSmall>(d, g.seg_rows, g.num_segs), 256, 0, st>>>(
                    H, width, Wd, static_cast<int>(d), g, static_cast<int>(width), first, Y);
        else
            f32_down_kernel<kF32TileLarge, kF32KLarge>
                <<<f32_grid<kF32TileLarge>(d, g.seg_rows, g.num_segs), 256, 0, st>>>(
                    H, width, Wd, static_cast<int>(d), g, static_cast<int>(width), first, Y);
        if (traced) trace_end(st, &rec);
        return cudaGetLastError() == cudaSuccess ? TSP_OK : TSP_ERR_CUDA;
    };
    if (!pl.ring) {
        for (size_t i = 0; i < pl.chunks.size(); ++i)
            TSP_TRY(run(seg_all_rows(n, P, fs, pl.chunks[i].col_base), pl.chunks[i].width, i == 0));
    } else {
        for (int t = 0; t < P; ++t) TSP_TRY(run(seg_ring(n, P, fs, 0, P, t), fs, t == 0));
    }
    return TSP_OK;
}

// ---------------------------------------------------------------------------
// backward (bf16, weight-shard schedule)

struct BwdPlan {
    bool ok = true;
    std::vector<Chunk> chunks;
    int n16 = 3, n32 = 1;     // bf16 buffers (H, dG, dU) and the fp32 dH buffer
    size_t b16 = 0, b32 = 0;  // bytes of one bf16 / fp32 chunk buffer
    size_t acc_bytes = 0;
    size_t total() const {
        return n16 * align256(b16) + n32 * align256(b32) + align256(acc_bytes);
    }
};

// saved: the backward from the training forward's activations, which needs
// only the dG (dU) chunk buffers -- no H, no fp32 dH.
BwdPlan plan_backward_budget(int64_t n, int64_t d, int64_t f, int P, tsp_act_t act, size_t budget,
                             bool saved) {
    BwdPlan pl;
    pl.n16 = (act == TSP_ACT_SWIGLU ? 3 : 2) - (saved ? 1 : 0);
    pl.n32 = saved ? 0 : 1;
    const size_t per_col = static_cast<size_t>(n) * (2 * pl.n16 + 4 * pl.n32);
    const int64_t mc = max_chunk_cols(budget, per_col);
    if (mc == 0) {
        pl.ok = false;
        return pl;
    }
    pl.chunks = plan_chunks(f, P, mc);
    int64_t wmax = 0;
    for (auto& c : pl.chunks) wmax = std::max(wmax, c.width);
    pl.b16 = static_cast<size_t>(n) * wmax * 2;
    pl.b32 = static_cast<size_t>(n) * wmax * 4;
    pl.acc_bytes = pl.chunks.size() > 1 ? static_cast<size_t>(n) * d * 4 : 0;
    return pl;
}

BwdPlan plan_backward(int64_t n, int64_t d, int64_t f, int P, tsp_act_t act, bool saved) {
    return plan_backward_budget(n, d, f, P, act, kBwdHiddenBudget, saved);
}

BwdPlan plan_backward_for(int64_t n, int64_t d, int64_t f, int P, tsp_act_t act, size_t ws_bytes,
                          bool saved) {
    BwdPlan pl = plan_backward(n, d, f, P, act, saved);
    if (pl.total() <= ws_bytes) return pl;
    const size_t acc = align256(static_cast<size_t>(n) * d * 4);
    if (ws_bytes <= acc + 2048) {
        pl.ok = false;
        return pl;
    }
    pl = plan_backward_budget(n, d, f, P, act, ws_bytes - acc - 2048, saved);
    if (pl.total() > ws_bytes) pl.ok = false;
    return pl;
}

// Activations kept by the training forward (see SavedLayout), row pitch ld.
struct SavedAct {
    const __nv_bfloat16* H;
    const uint32_t* S1;  // bf16x2 words (train_pair.cuh)
    const uint32_t* S2;
    int64_t ld;
};

template <int ACT>
tsp_status_t backward_bf16(const void* X, const void* Wg, const void* Wu, const void* Wd,
                           const void* dY, int64_t n, int64_t d, int64_t f, int P,
                           const BwdPlan& pl, void* dX, float* dWg, float* dWu, float* dWd,
                           void* ws, cudaStream_t st, int dev, int sms,
                           const SavedAct* sv = nullptr) {
    char* w = static_cast<char*>(ws);
    const size_t a16 = align256(pl.b16), a32 = align256(pl.b32);
    int slot = 0;
    auto* Hc = sv ? nullptr : reinterpret_cast<__nv_bfloat16*>(w + a16 * slot++);
    auto* dGc = reinterpret_cast<__nv_bfloat16*>(w + a16 * slot++);
    auto* dUc = ACT == 1 ? reinterpret_cast<__nv_bfloat16*>(w + a16 * slot++) : nullptr;
    auto* dHc = sv ? nullptr : reinterpret_cast<float*>(w + pl.n16 * a16);
    float* acc = pl.acc_bytes ? reinterpret_cast<float*>(w + pl.n16 * a16 + pl.n32 * a32) : nullptr;
    const int64_t fs = f / P;
    const int np = static_cast<int>(pl.chunks.size());
    for (int i = 0; i < np; ++i) {
        const int64_t cb = pl.chunks[i].col_base, C = pl.chunks[i].width;
        if (sv) {
            // K3 from the saved factors: dH = dY . W_down[chunk]^T, applied to
            // S1 (S2) in the epilogue, giving dG (dU) directly
            DhFactorParams p;
            std::memset(&p, 0, sizeof(p));
            if (!tmap_bf16(&p.tmDY, dY, d, n, d, 64, 128, SW128) ||
                !tmap_bf16(&p.tmD, Wd, d, f, d, 64, 128, SW128))
                return TSP_ERR_CUDA;
            p.n = static_cast<int>(n);
            p.d = static_cast<int>(d);
            p.col_base = static_cast<int>(cb);
            p.width = static_cast<int>(C);
            p.ld = C;
            p.S1 = sv->S1 + cb / 2 * 32;  // column cb (even) of every 32-row block
            p.S2 = ACT == 1 ? sv->S2 + cb / 2 * 32 : nullptr;
            p.lds = sv->ld;
            p.dG = dGc;
            p.dU = dUc;
            TSP_TRY(launch_pair<DhFactorPair<ACT>>(p, st, dev, sms));
        }
        // K3a: dH = dY . W_down[chunk]^T, kept in fp32
        if (!sv) {
            DhParams p;
            std::memset(&p, 0, sizeof(p));
            if (!tmap_bf16(&p.tmDY, dY, d, n, d, 64, 128, SW128) ||
                !tmap_bf16(&p.tmD, Wd, d, f, d, 64, 128, SW128))
                return TSP_ERR_CUDA;
            p.n = static_cast<int>(n);
            p.d = static_cast<int>(d);
            p.col_base = static_cast<int>(cb);
            p.width = static_cast<int>(C);
            p.dH = dHc;
            p.ld = C;
            TSP_TRY(launch_pair<DhPair<ACT>>(p, st, dev, sms));
        }
        // K3b: recompute G (U); emit H and, from dH, dG (dU)
        if (!sv) {
            BwdGateUpParams p;
            std::memset(&p, 0, sizeof(p));
            if (!tmap_bf16(&p.tmX, X, d, n, d, 64, 128, SW128) ||
                !tmap_bf16(&p.tmG, Wg, f, d, f, 64, 128, SW128) ||
                (ACT == 1 && !tmap_bf16(&p.tmU, Wu, f, d, f, 64, 128, SW128)))
                return TSP_ERR_CUDA;
            p.n = static_cast<int>(n);
            p.d = static_cast<int>(d);
            p.col_base = static_cast<int>(cb);
            p.width = static_cast<int>(C);
            p.dH = dHc;
            p.H = Hc;
            p.dG = dGc;
            p.dU = dUc;
            p.ld = C;
            TSP_TRY(launch_pair<BwdGateUpPair<ACT>>(p, st, dev, sms));
        }
        // K4a: dW_down[cb .. cb+C) = H^T . dY
        {
            using K = Wgrad<256, false>;
            typename K::Params p;
            std::memset(&p, 0, sizeof(p));
            // H: the recomputed chunk, or the chunk's columns of the saved H
            const __nv_bfloat16* Hs = sv ? sv->H + cb : Hc;
            if (!tmap_bf16(&p.tmA, Hs, C, n, sv ? sv->ld : C, 64, 64, SW128) ||
                !tmap_bf16(&p.tmB0, dY, d, n, d, 64, 64, SW128))
                return TSP_ERR_CUDA;
            p.ntok = static_cast<int>(n);
            p.m_valid = static_cast<int>(C);
            p.n_valid = static_cast<int>(d);
            p.out0 = dWd;
            p.ldo = d;
            p.out_row0 = static_cast<int>(cb);
            p.out_col0 = 0;
            TSP_TRY((launch_pair<WgradPair<256, false>>(p, st, dev, sms)));
        }
        if (ACT == 1) {
            // K4b + K5 in one launch (grad_pair.cuh): the input gradient's long
            // tiles first, the weight gradients' short ones filling each pair.
            // Both backward paths take it, so their dX, dW_gate and dW_up come
            // from the same kernel.
            DgradWgradParams p;
            std::memset(&p, 0, sizeof(p));
            if (!tmap_bf16(&p.w.tmA, X, d, n, d, 64, 128, SW128) ||
                !tmap_bf16(&p.w.tmB0, dGc, C, n, C, 64, 128, SW128) ||
                !tmap_bf16(&p.w.tmB1, dUc, C, n, C, 64, 128, SW128))
                return TSP_ERR_CUDA;
            p.w.ntok = static_cast<int>(n);
            p.w.m_valid = static_cast<int>(d);
            p.w.n_valid = static_cast<int>(C);
            p.w.out0 = dWg;
            p.w.out1 = dWu;
            p.w.ldo = f;
            p.w.out_row0 = 0;
            p.w.out_col0 = static_cast<int>(cb);
            p.d.g = seg_all_rows(n, P, fs, cb);
            if (!tmap_bf16(&p.d.tmA0, dGc, C, n, C, 64, 128, SW128) ||
                !tmap_bf16(&p.d.tmB0, Wg, f, d, f, 64, 128, SW128) ||
                !tmap_bf16(&p.d.tmA1, dUc, C, n, C, 64, 128, SW128) ||
                !tmap_bf16(&p.d.tmB1, Wu, f, d, f, 64, 128, SW128))
                return TSP_ERR_CUDA;
            p.d.kdim = static_cast<int>(C);
            p.d.n_out = static_cast<int>(d);
            p.d.mode = accum_mode(i, np);
            p.d.acc = acc;
            p.d.ldacc = d;
            p.d.out = static_cast<__nv_bfloat16*>(dX);
            p.d.ldo = d;
            TSP_TRY(launch_pair<DgradWgradPair>(p, st, dev, sms));
            continue;
        }
        // GeLU: K4b, dA[:, cb .. cb+C) = X^T . dG
        {
            using K = Wgrad<128, false>;
            typename K::Params p;
            std::memset(&p, 0, sizeof(p));
            if (!tmap_bf16(&p.tmA, X, d, n, d, 64, 64, SW128) ||
                !tmap_bf16(&p.tmB0, dGc, C, n, C, 64, 64, SW128))
                return TSP_ERR_CUDA;
            p.ntok = static_cast<int>(n);
            p.m_valid = static_cast<int>(d);
            p.n_valid = static_cast<int>(C);
            p.out0 = dWg;
            p.ldo = f;
            p.out_row0 = 0;
            p.out_col0 = static_cast<int>(cb);
            TSP_TRY((launch_pair<WgradPair<128, false>>(p, st, dev, sms)));
        }
        // GeLU: K5, dX (+)= dG . A[:, chunk]^T
        {
            using K = DownAccum<false, 1>;
            typename K::Params p;
            std::memset(&p, 0, sizeof(p));
            p.g = seg_all_rows(n, P, fs, cb);
            if (!tmap_bf16(&p.tmA0, dGc, C, n, C, 64, 128, SW128) ||
                !tmap_bf16(&p.tmB0, Wg, f, d, f, 64, 128, SW128))
                return TSP_ERR_CUDA;
            p.kdim = static_cast<int>(C);
            p.n_out = static_cast<int>(d);
            p.mode = accum_mode(i, np);
            p.acc = acc;
            p.ldacc = d;
            p.out = static_cast<__nv_bfloat16*>(dX);
            p.ldo = d;
            TSP_TRY((launch_pair<DownAccumPair<false, 1, 256>>(p, st, dev, sms)));
        }
    }
    return TSP_OK;
}


// ---------------------------------------------------------------------------
// TSP attention ("Folding Tensor and Sequence Parallelism ...", Abstract: the
// attention schedule).  Head dimension 128.

constexpr int kAttnHeadDim = 128;

tsp_status_t validate_attn_shape(int64_t n, int64_t d, int heads, int P) {
    if (n <= 0 || d <= 0 || heads <= 0 || P <= 0) return TSP_ERR_INVALID_ARG;
    if (n > (int64_t(1) << 28) || d > 65536 || P > 4096) return TSP_ERR_UNSUPPORTED_SHAPE;
    if (d != static_cast<int64_t>(heads) * kAttnHeadDim) return TSP_ERR_UNSUPPORTED_SHAPE;
    if (n % P != 0) return TSP_ERR_UNSUPPORTED_SHAPE;
    return TSP_OK;
}

// C[m][nout] = A[m][k] . B[k][nout] (bf16 A, B), fp32 accumulate in tensor
// memory: the paired down-projection recipe with one K segment, stored direct
// as bf16 (out_f16 false) or fp16 (true; magnitudes above 65504 saturate and
// raise the range bit of the device error word).
tsp_status_t gemm_bf16(const void* A, const void* B, int64_t m, int64_t k, int64_t nout, void* Cm,
                       bool out_f16, cudaStream_t st, int dev, int sms, const char* trace_name) {
    using K2 = DownAccum<true, 1>;
    typename K2::Params p2;
    std::memset(&p2, 0, sizeof(p2));
    if (!tmap_bf16(&p2.tmA0, A, k, m, k, 64, 128, SW128) ||
        !tmap_bf16(&p2.tmB0, B, nout, k, nout, 64, 128, SW128))
        return TSP_ERR_CUDA;
    p2.g = seg_all_rows(m, 1, k, 0);
    p2.kdim = static_cast<int>(k);
    p2.n_out = static_cast<int>(nout);
    p2.mode = out_f16 ? 4 : 3;
    p2.rot_P = 0;
    p2.acc = nullptr;
    p2.out = static_cast<__nv_bfloat16*>(Cm);
    p2.ldo = nout;
    return launch_pair<DownAccumPair<true, 1, 256>>(p2, st, dev, sms, trace_name);
}

// qk_f16: Q and K are fp16 (the block's own projections), else bf16.
tsp_status_t launch_attn_core(const void* Q, const void* K, const void* V, int64_t n, int64_t d,
                              int heads, int P, int causal, bool qk_f16, void* O, cudaStream_t st,
                              int dev, int sms) {
    AttnParams p;
    std::memset(&p, 0, sizeof(p));
    auto tmap_qk = qk_f16 ? tmap_f16 : tmap_bf16;
    if (!tmap_qk(&p.tmQ, Q, d, n, d, 64, 128, SW128) ||
        !tmap_qk(&p.tmK, K, d, n, d, 64, 128, SW128) ||
        !tmap_bf16(&p.tmV, V, d, n, d, 64, 128, SW128))
        return TSP_ERR_CUDA;
    p.O = static_cast<__nv_bfloat16*>(O);
    p.ldo = d;
    p.n = static_cast<int>(n);
    p.heads = heads;
    p.P = P;
    p.ns = static_cast<int>(n / P);
    p.nb = (p.ns + 127) / 128;
    p.npr = (p.ns + 255) / 256;
    p.causal = causal ? 1 : 0;
    p.items = heads * P * p.npr;
    p.sl2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kAttnHeadDim)));
    constexpr int smem = AttnCore::kSmemBytes;
    static_assert(smem <= 232448, "attention core exceeds 227 KB of shared memory");
    static bool attr_set[kMaxDevices] = {};
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(attn_core_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
                cudaFuncSetAttribute(attn_core_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
                return TSP_ERR_CUDA;
            attr_set[dev] = true;
        }
    }
    const int grid = std::min(p.items, sms);
    TraceRec rec;
    const bool traced = trace_begin(st, &rec, causal ? "attn_core_causal" : "attn_core");
    if (qk_f16)
        attn_core_kernel<true><<<grid, AttnCore::kThreads, smem, st>>>(p);
    else
        attn_core_kernel<false><<<grid, AttnCore::kThreads, smem, st>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (traced) trace_end(st, &rec);
    return e == cudaSuccess ? TSP_OK : TSP_ERR_CUDA;
}

}  // namespace
}  // namespace tspmlp

// ---------------------------------------------------------------------------
// Scratch of tsp_mlp_forward_noalloc: a static device array, so that entry
// point never allocates.  Host code must not hand the symbol itself to a
// kernel (on the host it is only a stand-in); its device address is looked up
// once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char tsp_noalloc_scratch[TSP_NOALLOC_SCRATCH_BYTES];

namespace tspmlp {
namespace {

void* g_noalloc_scratch_addr[kMaxDevices] = {};

// Device address of the static scratch on device `dev` (the current device).
tsp_status_t noalloc_scratch_address(int dev, void** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, tsp_noalloc_scratch) != cudaSuccess || !p) return TSP_ERR_CUDA;
        g_noalloc_scratch_addr[dev] = p;
    }
    *out = g_noalloc_scratch_addr[dev];
    return TSP_OK;
}

}  // namespace
}  // namespace tspmlp

using namespace tspmlp;

extern "C" {

const char* tsp_status_string(tsp_status_t s) {
    switch (s) {
        case TSP_OK: return "ok";
        case TSP_ERR_INVALID_ARG: return "invalid argument";
        case TSP_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case TSP_ERR_ARCH: return "device is not compute capability 10.0 (B200, sm_100a)";
        case TSP_ERR_CUDA: return "CUDA error";
        case TSP_ERR_TIMEOUT: return "a device-side wait timed out";
        case TSP_ERR_WORKSPACE: return "workspace missing or too small";
        case TSP_ERR_RANGE:
            return "a value left the range of an fp16 intermediate (saturated at 65504)";
        case TSP_ERR_SCRATCH_LIMIT:
            return "problem needs more scratch than the no-allocation entry point's static array";
    }
    return "unknown status";
}

tsp_status_t tsp_mlp_workspace_size(int64_t n, int64_t d, int64_t f, int P, tsp_act_t act,
                                    tsp_dtype_t dt, tsp_sched_t sched, int backward,
                                    size_t* bytes) {
    if (!bytes) return TSP_ERR_INVALID_ARG;
    TSP_TRY(validate_shape(n, d, f, P, act, dt, sched));
    if (backward) {
        if (dt != TSP_DT_BF16 || sched != TSP_SCHED_WEIGHT_SHARDS) return TSP_ERR_INVALID_ARG;
        *bytes = plan_backward(n, d, f, P, act, false).total();
    } else {
        *bytes = plan_forward(n, d, f, P, dt, sched).total();
    }
    return TSP_OK;
}

tsp_status_t tsp_mlp_forward_ex(const void* X, const void* Wg, const void* Wu, const void* Wd,
                                int64_t n, int64_t d, int64_t f, int P, tsp_act_t act,
                                tsp_dtype_t dt, tsp_sched_t sched, void* Y, void* ws,
                                size_t ws_bytes, tsp_stream_t stream) {
    TSP_TRY(validate_forward(X, Wg, Wu, Wd, n, d, f, P, act, dt, sched, Y));
    const FwdPlan pl = plan_forward_for(n, d, f, P, dt, sched, ws ? ws_bytes : 0);
    const size_t need = pl.total();
    if (!pl.ok) return TSP_ERR_WORKSPACE;
    if (need > 0) {
        if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TSP_ERR_WORKSPACE;
        const size_t e = dt == TSP_DT_BF16 ? 2 : 4;
        const size_t xb = n * d * e, wb = d * f * e;
        if (overlaps(ws, need, X, xb) || overlaps(ws, need, Wg, wb) || overlaps(ws, need, Wu, wb) ||
            overlaps(ws, need, Wd, wb) || overlaps(ws, need, Y, xb))
            return TSP_ERR_INVALID_ARG;
    }
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == TSP_DT_F32)
        return forward_f32(static_cast<const float*>(X), static_cast<const float*>(Wg),
                           static_cast<const float*>(Wu), static_cast<const float*>(Wd), n, d, f, P,
                           act, pl, static_cast<float*>(Y), ws, st, di.sms);
    if (act == TSP_ACT_SWIGLU)
        return forward_bf16<1>(X, Wg, Wu, Wd, n, d, f, P, pl, Y, ws, st, dev, di.sms);
    return forward_bf16<0>(X, Wg, Wu, Wd, n, d, f, P, pl, Y, ws, st, dev, di.sms);
}

tsp_status_t tsp_mlp_forward(const void* X, const void* Wg, const void* Wu, const void* Wd,
                             int64_t n, int64_t d, int64_t f, int P, tsp_act_t act, void* Y,
                             tsp_stream_t stream) {
    TSP_TRY(validate_forward(X, Wg, Wu, Wd, n, d, f, P, act, TSP_DT_BF16,
                             TSP_SCHED_WEIGHT_SHARDS, Y));
    const size_t need = plan_forward(n, d, f, P, TSP_DT_BF16, TSP_SCHED_WEIGHT_SHARDS).total();
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    if (need && cudaMallocAsync(&ws, need, st) != cudaSuccess) return TSP_ERR_CUDA;
    const tsp_status_t s = tsp_mlp_forward_ex(X, Wg, Wu, Wd, n, d, f, P, act, TSP_DT_BF16,
                                              TSP_SCHED_WEIGHT_SHARDS, Y, ws, need, stream);
    if (ws && cudaFreeAsync(ws, st) != cudaSuccess && s == TSP_OK) return TSP_ERR_CUDA;
    return s;
}

tsp_status_t tsp_mlp_backward_ex(const void* X, const void* Wg, const void* Wu, const void* Wd,
                                 const void* dY, int64_t n, int64_t d, int64_t f, int P,
                                 tsp_act_t act, void* dX, float* dWg, float* dWu, float* dWd,
                                 void* ws, size_t ws_bytes, tsp_stream_t stream) {
    TSP_TRY(validate_backward(X, Wg, Wu, Wd, dY, n, d, f, P, act, dX, dWg, dWu, dWd));
    const BwdPlan pl = plan_backward_for(n, d, f, P, act, ws ? ws_bytes : 0, false);
    const size_t need = pl.total();
    if (!pl.ok || !ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return TSP_ERR_WORKSPACE;
    const size_t xb = n * d * 2, wb = d * f * 2, gw = d * f * 4;
    const void* bufs[9] = {X, Wg, Wu, Wd, dY, dX, dWg, dWu, dWd};
    const size_t sz[9] = {xb, wb, wb, wb, xb, xb, gw, gw, gw};
    for (int i = 0; i < 9; ++i)
        if (overlaps(ws, need, bufs[i], sz[i])) return TSP_ERR_INVALID_ARG;
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (act == TSP_ACT_SWIGLU)
        return backward_bf16<1>(X, Wg, Wu, Wd, dY, n, d, f, P, pl, dX, dWg, dWu, dWd, ws, st, dev,
                                di.sms);
    return backward_bf16<0>(X, Wg, Wu, Wd, dY, n, d, f, P, pl, dX, dWg, dWu, dWd, ws, st, dev,
                            di.sms);
}

tsp_status_t tsp_mlp_backward(const void* X, const void* Wg, const void* Wu, const void* Wd,
                              const void* dY, int64_t n, int64_t d, int64_t f, int P,
                              tsp_act_t act, void* dX, float* dWg, float* dWu, float* dWd,
                              tsp_stream_t stream) {
    TSP_TRY(validate_backward(X, Wg, Wu, Wd, dY, n, d, f, P, act, dX, dWg, dWu, dWd));
    const size_t need = plan_backward(n, d, f, P, act, false).total();
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    if (cudaMallocAsync(&ws, need, st) != cudaSuccess) return TSP_ERR_CUDA;
    const tsp_status_t s = tsp_mlp_backward_ex(X, Wg, Wu, Wd, dY, n, d, f, P, act, dX, dWg, dWu,
                                               dWd, ws, need, stream);
    if (cudaFreeAsync(ws, st) != cudaSuccess && s == TSP_OK) return TSP_ERR_CUDA;
    return s;
}

tsp_status_t tsp_mlp_saved_size(int64_t n, int64_t d, int64_t f, int P, tsp_act_t act,
                                size_t* bytes) {
    if (!bytes) return TSP_ERR_INVALID_ARG;
    TSP_TRY(validate_shape(n, d, f, P, act, TSP_DT_BF16, TSP_SCHED_WEIGHT_SHARDS));
    *bytes = saved_layout(n, f, act).total();
    return TSP_OK;
}

tsp_status_t tsp_mlp_forward_train(const void* X, const void* Wg, const void* Wu, const void* Wd,
                                   int64_t n, int64_t d, int64_t f, int P, tsp_act_t act, void* Y,
                                   void* saved, size_t saved_bytes, tsp_stream_t stream) {
    TSP_TRY(validate_forward(X, Wg, Wu, Wd, n, d, f, P, act, TSP_DT_BF16,
                             TSP_SCHED_WEIGHT_SHARDS, Y));
    const size_t need = saved_layout(n, f, act).total();
    if (!saved || saved_bytes < need || (reinterpret_cast<uintptr_t>(saved) & 255u))
        return TSP_ERR_INVALID_ARG;
    const size_t xb = n * d * 2, wb = d * f * 2;
    if (overlaps(saved, need, X, xb) || overlaps(saved, need, Wg, wb) ||
        overlaps(saved, need, Wu, wb) || overlaps(saved, need, Wd, wb) ||
        overlaps(saved, need, Y, xb))
        return TSP_ERR_INVALID_ARG;
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (act == TSP_ACT_SWIGLU)
        return forward_train_bf16<1>(X, Wg, Wu, Wd, n, d, f, P, Y, saved, st, dev, di.sms);
    return forward_train_bf16<0>(X, Wg, Wu, Wd, n, d, f, P, Y, saved, st, dev, di.sms);
}

tsp_status_t tsp_mlp_backward_saved_workspace_size(int64_t n, int64_t d, int64_t f, int P,
                                                   tsp_act_t act, size_t* bytes) {
    if (!bytes) return TSP_ERR_INVALID_ARG;
    TSP_TRY(validate_shape(n, d, f, P, act, TSP_DT_BF16, TSP_SCHED_WEIGHT_SHARDS));
    *bytes = plan_backward(n, d, f, P, act, true).total();
    return TSP_OK;
}

tsp_status_t tsp_mlp_backward_saved(const void* X, const void* Wg, const void* Wu, const void* Wd,
                                    const void* dY, const void* saved, size_t saved_bytes,
                                    int64_t n, int64_t d, int64_t f, int P, tsp_act_t act,
                                    void* dX, float* dWg, float* dWu, float* dWd, void* ws,
                                    size_t ws_bytes, tsp_stream_t stream) {
    TSP_TRY(validate_backward(X, Wg, Wu, Wd, dY, n, d, f, P, act, dX, dWg, dWu, dWd));
    const SavedLayout sl = saved_layout(n, f, act);
    if (!saved || saved_bytes < sl.total() || (reinterpret_cast<uintptr_t>(saved) & 255u))
        return TSP_ERR_INVALID_ARG;
    const BwdPlan pl = plan_backward_for(n, d, f, P, act, ws ? ws_bytes : 0, true);
    const size_t need = pl.total();
    if (!pl.ok || !ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return TSP_ERR_WORKSPACE;
    const size_t xb = n * d * 2, wb = d * f * 2, gw = d * f * 4;
    const void* outs[4] = {dX, dWg, dWu, dWd};
    const size_t osz[4] = {xb, gw, gw, gw};
    for (int i = 0; i < 4; ++i)
        if (overlaps(saved, sl.total(), outs[i], osz[i])) return TSP_ERR_INVALID_ARG;
    if (overlaps(saved, sl.total(), ws, need)) return TSP_ERR_INVALID_ARG;
    const void* bufs[9] = {X, Wg, Wu, Wd, dY, dX, dWg, dWu, dWd};
    const size_t sz[9] = {xb, wb, wb, wb, xb, xb, gw, gw, gw};
    for (int i = 0; i < 9; ++i)
        if (overlaps(ws, need, bufs[i], sz[i])) return TSP_ERR_INVALID_ARG;
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const char* base = static_cast<const char*>(saved);
    const SavedAct sv{reinterpret_cast<const __nv_bfloat16*>(base),
                      reinterpret_cast<const uint32_t*>(base + sl.h),
                      act == TSP_ACT_SWIGLU ? reinterpret_cast<const uint32_t*>(base + sl.h + sl.s)
                                            : nullptr,
                      f};
    if (act == TSP_ACT_SWIGLU)
        return backward_bf16<1>(X, Wg, Wu, Wd, dY, n, d, f, P, pl, dX, dWg, dWu, dWd, ws, st, dev,
                                di.sms, &sv);
    return backward_bf16<0>(X, Wg, Wu, Wd, dY, n, d, f, P, pl, dX, dWg, dWu, dWd, ws, st, dev,
                            di.sms, &sv);
}

tsp_status_t tsp_attn_core(const void* Q, const void* K, const void* V, int64_t n, int64_t d,
                           int n_heads, int P, int causal, void* O, tsp_stream_t stream) {
    TSP_TRY(validate_attn_shape(n, d, n_heads, P));
    if (!Q || !K || !V || !O) return TSP_ERR_INVALID_ARG;
    const size_t b = n * d * 2;
    if (overlaps(O, b, Q, b) || overlaps(O, b, K, b) || overlaps(O, b, V, b))
        return TSP_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return TSP_ERR_UNSUPPORTED_SHAPE;
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    return launch_attn_core(Q, K, V, n, d, n_heads, P, causal, false, O,
                            reinterpret_cast<cudaStream_t>(stream), dev, di.sms);
}

tsp_status_t tsp_attn_workspace_size(int64_t n, int64_t d, int n_heads, int P, size_t* bytes) {
    if (!bytes) return TSP_ERR_INVALID_ARG;
    TSP_TRY(validate_attn_shape(n, d, n_heads, P));
    if (n_heads % P != 0) return TSP_ERR_UNSUPPORTED_SHAPE;
    *bytes = 4 * align256(static_cast<size_t>(n) * d * 2);
    return TSP_OK;
}

tsp_status_t tsp_attn_forward(const void* X, const void* Wq, const void* Wk, const void* Wv,
                              const void* Wo, int64_t n, int64_t d, int n_heads, int P, int causal,
                              void* Y, void* ws, size_t ws_bytes, tsp_stream_t stream) {
    TSP_TRY(validate_attn_shape(n, d, n_heads, P));
    if (n_heads % P != 0) return TSP_ERR_UNSUPPORTED_SHAPE;
    if (!X || !Wq || !Wk || !Wv || !Wo || !Y) return TSP_ERR_INVALID_ARG;
    const void* ins[5] = {X, Wq, Wk, Wv, Wo};
    for (const void* q : ins)
        if (!aligned16(q)) return TSP_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(Y)) return TSP_ERR_UNSUPPORTED_SHAPE;
    const size_t xb = n * d * 2, wb = d * d * 2;
    const size_t isz[5] = {xb, wb, wb, wb, wb};
    for (int i = 0; i < 5; ++i)
        if (overlaps(Y, xb, ins[i], isz[i])) return TSP_ERR_INVALID_ARG;
    const size_t one = align256(xb), need = 4 * one;
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TSP_ERR_WORKSPACE;
    for (int i = 0; i < 5; ++i)
        if (overlaps(ws, need, ins[i], isz[i])) return TSP_ERR_INVALID_ARG;
    if (overlaps(ws, need, Y, xb)) return TSP_ERR_INVALID_ARG;
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    void *Q = w, *K = w + one, *V = w + 2 * one, *O = w + 3 * one;
    // every parameter shard's columns of W_q, W_k, W_v, for every sequence
    // shard's tokens: the projections of all (shard, shard) pairs in one
    // launch each (no sum crosses shards)
    // (Q and K in fp16: their rounding is the largest term of the block's
    // error, and fp16 carries three more mantissa bits than bf16)
    TSP_TRY(gemm_bf16(X, Wq, n, d, d, Q, true, st, dev, di.sms, "attn_proj"));
    TSP_TRY(gemm_bf16(X, Wk, n, d, d, K, true, st, dev, di.sms, "attn_proj"));
    TSP_TRY(gemm_bf16(X, Wv, n, d, d, V, false, st, dev, di.sms, "attn_proj"));
    // each sequence shard's queries over the key/value shards in ring order
    TSP_TRY(launch_attn_core(Q, K, V, n, d, n_heads, P, causal, true, O, st, dev, di.sms));
    // Y_s = sum over parameter shards w (in order) of O_{s,w} . W_o[rows of w]:
    // the K loop runs over the head groups in order, summing in tensor memory
    return gemm_bf16(O, Wo, n, d, d, Y, false, st, dev, di.sms, "attn_out_proj");
}

tsp_status_t tsp_trace_enable(int enable) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    g_trace_on = enable != 0;
    return TSP_OK;
}

tsp_status_t tsp_trace_collect(tsp_kernel_stat_t* stats, int capacity, int* count) {
    if (!count || capacity < 0 || (capacity > 0 && !stats)) return TSP_ERR_INVALID_ARG;
    std::vector<TraceRec> pend;
    {
        std::lock_guard<std::mutex> lk(g_trace_mu);
        pend.swap(g_trace_pending);
    }
    tsp_status_t st = TSP_OK;
    std::vector<TraceStat> add;
    for (auto& r : pend) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            st = TSP_ERR_CUDA;
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
        add.push_back({r.name, 1, static_cast<double>(ms)});
    }
    std::lock_guard<std::mutex> lk(g_trace_mu);
    for (auto& a : add) {
        bool found = false;
        for (auto& t : g_trace_stats)
            if (std::strcmp(t.name, a.name) == 0) {
                t.launches += 1;
                t.ms += a.ms;
                found = true;
                break;
            }
        if (!found) g_trace_stats.push_back(a);
    }
    int k = 0;
    for (auto& t : g_trace_stats) {
        if (k < capacity) stats[k] = tsp_kernel_stat_t{t.name, t.launches, t.ms};
        ++k;
    }
    *count = std::min(k, capacity);
    return st;
}

tsp_status_t tsp_trace_reset(void) {
    std::vector<TraceRec> pend;
    {
        std::lock_guard<std::mutex> lk(g_trace_mu);
        pend.swap(g_trace_pending);
        g_trace_stats.clear();
    }
    for (auto& r : pend) {
        cudaEventSynchronize(r.b);
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    return TSP_OK;
}

tsp_status_t tsp_mlp_forward_noalloc(const void* X, const void* Wg, const void* Wu,
                                     const void* Wd, int64_t n, int64_t d, int64_t f, int P,
                                     tsp_act_t act, void* Y, tsp_stream_t stream) {
    // the fused schedule: its only scratch is the H ring and the counters
    TSP_TRY(validate_forward(X, Wg, Wu, Wd, n, d, f, P, act, TSP_DT_BF16, TSP_SCHED_FUSED, Y));
    const FwdPlan pl = plan_forward_for(n, d, f, P, TSP_DT_BF16, TSP_SCHED_FUSED,
                                        TSP_NOALLOC_SCRATCH_BYTES);
    if (!pl.ok || pl.total() > TSP_NOALLOC_SCRATCH_BYTES) return TSP_ERR_SCRATCH_LIMIT;
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    void* ws = nullptr;
    TSP_TRY(noalloc_scratch_address(dev, &ws));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (act == TSP_ACT_SWIGLU)
        return forward_bf16<1>(X, Wg, Wu, Wd, n, d, f, P, pl, Y, ws, st, dev, di.sms);
    return forward_bf16<0>(X, Wg, Wu, Wd, n, d, f, P, pl, Y, ws, st, dev, di.sms);
}

tsp_status_t tsp_selftest_timeout(int mode, tsp_stream_t stream) {
    if (mode != 0 && mode != 1) return TSP_ERR_INVALID_ARG;
    int dev = 0;
    DevInfo di;
    TSP_TRY(current_device(&dev, &di));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (mode == 0) {
        bounded_wait_selftest_kernel<<<1, 32, 0, st>>>();
        return cudaGetLastError() == cudaSuccess ? TSP_OK : TSP_ERR_CUDA;
    }
    // mode 1: a 128 x 256 x 128 gate/up problem -> one tile, four k-blocks
    using K = FwdHidden<1>;
    constexpr int64_t n = 128, d = 256, f = 128;
    const size_t xb = n * d * 2, wb = d * f * 2, hb = n * f * 2;
    char* buf = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void**>(&buf), xb + 2 * wb + hb, st) != cudaSuccess)
        return TSP_ERR_CUDA;
    tsp_status_t rc = TSP_OK;
    if (cudaMemsetAsync(buf, 0, xb + 2 * wb + hb, st) != cudaSuccess) rc = TSP_ERR_CUDA;
    typename K::Params p;
    std::memset(&p, 0, sizeof(p));
    if (rc == TSP_OK && (!tmap_bf16(&p.tmX, buf, d, n, d, 64, 128, SW128) ||
                         !tmap_bf16(&p.tmG, buf + xb, f, d, f, 64, 64, SW128) ||
                         !tmap_bf16(&p.tmU, buf + xb + wb, f, d, f, 64, 64, SW128)))
        rc = TSP_ERR_CUDA;
    if (rc == TSP_OK) {
        p.g = seg_all_rows(n, 1, f, 0);
        p.d = static_cast<int>(d);
        p.width = static_cast<int>(f);
        p.H = reinterpret_cast<__nv_bfloat16*>(buf + xb + 2 * wb);
        p.ldh = f;
        constexpr int smem = pipeline_smem_bytes<K>();
        if (cudaFuncSetAttribute(umma_pipeline_kernel<K, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            rc = TSP_ERR_CUDA;
        if (rc == TSP_OK) {
            umma_pipeline_kernel<K, true><<<1, kPipelineThreads, smem, st>>>(p);
            if (cudaGetLastError() != cudaSuccess) rc = TSP_ERR_CUDA;
        }
    }
    if (cudaFreeAsync(buf, st) != cudaSuccess && rc == TSP_OK) rc = TSP_ERR_CUDA;
    return rc;
}

tsp_status_t tsp_poll_device_error(tsp_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return TSP_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpyFromSymbol(&word, tspmlp::g_device_error, sizeof(word)) != cudaSuccess)
        return TSP_ERR_CUDA;
    if (word) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(tspmlp::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
            return TSP_ERR_CUDA;
        return (word & tspmlp::kDevErrTimeout) ? TSP_ERR_TIMEOUT : TSP_ERR_RANGE;
    }
    return TSP_OK;
}

}  // extern "C"
