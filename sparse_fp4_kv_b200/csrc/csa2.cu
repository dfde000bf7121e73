// csa2.cu -- the C ABI of libcsa2.so (declared in include/csa2.h): host-side
// argument checks, launch planning, tensor-map encoding and kernel launches.
// All kernels live in this one translation unit (append.cuh, indexer.cuh,
// attention.cuh) so the device error word is a single module variable.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <numeric>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <cstdint>
#include <array>
#include <map>
#include <mutex>
#include <set>
#include <utility>

#include "append.cuh"
#include "attention.cuh"
#include "attn_decode.cuh"
#include "indexer.cuh"
#include "indexer_fused.cuh"
#include "indexer_batch.cuh"

using namespace csa2;

namespace {

constexpr int32_t kVersion = 100;  // 0.1.0

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int max_smem_optin() {
    int dev = 0, n = 232448;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    return n;
}

// CSA2_FULL_PATH picks the Full indexer path where several apply: "multipass"
// (the multi-launch path), "fused" (never the batched path) or "batch" (the
// batched path whenever it applies); all are complete implementations and the
// switch lets tests exercise each at small sizes. Unset: the automatic choice.
enum FullPath { kPathAuto, kPathMultipass, kPathFused, kPathBatch };
FullPath full_path_env() {
    static const FullPath v = [] {
        const char *e = std::getenv("CSA2_FULL_PATH");
        if (!e) return kPathAuto;
        if (std::strcmp(e, "multipass") == 0) return kPathMultipass;
        if (std::strcmp(e, "fused") == 0) return kPathFused;
        if (std::strcmp(e, "batch") == 0) return kPathBatch;
        return kPathAuto;
    }();
    return v;
}
bool force_multipass() { return full_path_env() == kPathMultipass; }

// Batched Full path: CSA2_BATCH_MODE=exact skips the sampled threshold path
// (two exact passes for every query), =redo runs it and hands every query to
// the exact passes anyway (tests of the fallback). Default: sampled, with the
// exact passes for the queries it cannot settle.
enum BatchMode { kBatchSampled, kBatchExact, kBatchRedo };
BatchMode batch_mode_env() {
    static const BatchMode v = [] {
        const char *e = std::getenv("CSA2_BATCH_MODE");
        if (e == nullptr) return kBatchSampled;
        if (std::strcmp(e, "exact") == 0) return kBatchExact;
        if (std::strcmp(e, "redo") == 0) return kBatchRedo;
        return kBatchSampled;
    }();
    return v;
}

// CSA2_REINDEX=cluster: the one-launch Reindex (a cluster of CTAs per query
// scores into the first CTA's shared memory, which selects). It is correct
// and tested but measured slower than the two-launch path (22 against about
// 15 us cold on eight queries with 4096-id pools), so it is opt-in.
bool reindex_cluster() {
    static const bool v = [] {
        const char *e = std::getenv("CSA2_REINDEX");
        return e != nullptr && std::strcmp(e, "cluster") == 0;
    }();
    return v;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

csa2_status check_launch() {
    return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

csa2_status check_kv(const csa2_kv_desc *kv, bool need_kidx) {
    if (!kv) return CSA2_ERR_INVALID_ARG;
    if (kv->d != CSA2_D) return CSA2_ERR_UNSUPPORTED;
    if (!kv->codes || !kv->scales || !kv->page_table || !kv->seq_len) return CSA2_ERR_INVALID_ARG;
    if (!aligned(kv->codes, 16) || !aligned(kv->scales, 16) || !aligned(kv->page_table, 4) ||
        !aligned(kv->seq_len, 4))
        return CSA2_ERR_INVALID_ARG;
    if (kv->rows_cap <= 0 || kv->batch <= 0 || kv->max_pages <= 0 || kv->page_size <= 0) return CSA2_ERR_INVALID_ARG;
    if (kv->page_size % 32 != 0) return CSA2_ERR_UNSUPPORTED;
    if (kv->page_size < 128 && 128 % kv->page_size != 0) return CSA2_ERR_UNSUPPORTED;
    if (kv->page_size > 128 && kv->page_size % 128 != 0) return CSA2_ERR_UNSUPPORTED;
    if (kv->rows_cap > INT32_MAX) return CSA2_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
    if (need_kidx) {
        if (!kv->kidx || !aligned(kv->kidx, 16)) return CSA2_ERR_INVALID_ARG;
        if (kv->di != 64 && kv->di != 128) return CSA2_ERR_UNSUPPORTED;
        if ((kv->rows_cap * kv->di) % 128 != 0) return CSA2_ERR_UNSUPPORTED;  // keys are read as 128-byte rows
    }
    return CSA2_OK;
}

// cuTensorMapEncodeTiled, fetched through the runtime so that the library
// does not link the driver library directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// The indexer keys viewed as 128-byte rows (two entries per row when di is 64),
// loaded as boxes of box_rows rows with the 128B swizzle.
bool make_kidx_map(CUtensorMap *tm, const csa2_kv_desc *kv, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {128, (cuuint64_t)(kv->rows_cap * kv->di / 128)};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(kv->kidx), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- Full indexer workspace ------------------------------------------------
struct FullLayout {
    int64_t key_stride;
    int64_t c_chunk;       // keys per collecting CTA (part) of the multi-launch path
    int32_t c_parts;       // parts per query
    int32_t c_sure_stride;
    size_t off_keys, off_hist0, off_state, off_hist1, off_cnt, off_sure, off_cand, total;
    size_t b_hist, b_state, b_cnt, b_sure, b_cand;  // batched path
    size_t b_sstate, b_redo, b_samples;             // its sampled threshold path
    int64_t sample_stride;
};

// Split of the batched Full path: query groups of qg queries, chunks of
// whole tiles per group (one CTA each, about one CTA per SM in total). The
// workspace is sized with the bound over both group sizes (qg = 8 or 16) and
// both tile sizes (128 or 256 entries).
struct BatchSplit {
    int64_t nchunks, chunk;          // for a given qg and tile size
    int64_t max_chunks, max_span;    // bounds over every qg and tile size of chunks and chunks * chunk
};
BatchSplit batch_split(int32_t nq, int64_t n_max, int tile_entries, int sms, int qg = 16) {
    BatchSplit s{};
    auto one = [&](int q, int te, int64_t &nch, int64_t &chunk) {
        const int64_t ngroups = (nq + q - 1) / q;
        const int64_t tiles = std::max<int64_t>(1, (n_max + te - 1) / te);
        nch = std::max<int64_t>(1, std::min<int64_t>(tiles, std::min<int64_t>(kBatchMaxChunks, sms / ngroups)));
        chunk = (tiles + nch - 1) / nch * te;
    };
    one(qg, tile_entries, s.nchunks, s.chunk);
    s.max_chunks = 0;
    s.max_span = 0;
    for (int q : {8, 16})
        for (int te : {128, 256}) {
            int64_t a, c;
            one(q, te, a, c);
            s.max_chunks = std::max(s.max_chunks, a);
            s.max_span = std::max(s.max_span, a * c);
        }
    return s;
}

// Parts of the multi-launch path's selection: one round of the collecting
// CTA (16 keys per thread, 8192 keys) per part, so that parts are short and
// many, whatever the spread of the queries' lengths; more keys per part only
// beyond kBatchMaxChunks parts per query.
void collect_split(int32_t nq, int64_t n_max, int sms, int64_t &chunk, int32_t &parts) {
    (void)nq;
    (void)sms;
    constexpr int64_t kRound = 16 * kCollectThreads;
    const int64_t n = std::max<int64_t>(n_max, 1);
    chunk = std::max<int64_t>(kRound, ((n + kBatchMaxChunks - 1) / kBatchMaxChunks + kRound - 1) / kRound * kRound);
    parts = (int32_t)((n + chunk - 1) / chunk);
}

FullLayout full_layout(int32_t nq, int64_t n_max) {
    FullLayout L{};
    L.key_stride = (int64_t)align_up((size_t)std::max<int64_t>(n_max, 1), 128);
    collect_split(nq, n_max, num_sms(), L.c_chunk, L.c_parts);
    L.c_sure_stride = (int32_t)std::min<int64_t>(kBatchMaxK, L.c_chunk);  // a part holds < rank sure ids
    size_t off = 0;
    L.off_keys = off;
    off = align_up(off + (size_t)nq * L.key_stride * 4, 256);
    L.off_hist0 = off;
    off = align_up(off + (size_t)nq * kHist0Bins * 4, 256);
    L.off_state = off;
    off = align_up(off + (size_t)nq * kStateWords * 4, 256);
    L.off_hist1 = off;  // [2 targets][nq][2048]
    off = align_up(off + (size_t)2 * nq * 2048 * 4, 256);
    L.off_cnt = off;
    off = align_up(off + (size_t)nq * L.c_parts * 2 * 4, 256);
    L.off_sure = off;
    off = align_up(off + (size_t)nq * L.c_parts * L.c_sure_stride * 4, 256);
    L.off_cand = off;
    off = align_up(off + (size_t)nq * L.c_parts * L.c_chunk * 8, 256);
    // the batched path's region (the same bytes: one path runs per call),
    // sized for its largest split: chunks per query group, entries per chunk
    const BatchSplit bs = batch_split(nq, n_max, 256, num_sms());
    size_t b = 0;
    L.b_hist = b;
    b = align_up(b + (size_t)nq * kBatchBins * 4, 256);
    L.b_state = b;
    b = align_up(b + (size_t)nq * 2 * 4, 256);
    L.b_cnt = b;
    b = align_up(b + (size_t)nq * bs.max_chunks * 2 * 4, 256);
    L.b_sure = b;
    b = align_up(b + (size_t)nq * bs.max_chunks * kBatchMaxK * 4, 256);
    L.b_cand = b;
    b = align_up(b + (size_t)nq * bs.max_span * 8, 256);
    L.b_sstate = b;
    b = align_up(b + (size_t)nq * 2 * 4, 256);
    L.b_redo = b;
    b = align_up(b + (size_t)nq * 4, 256);
    L.b_samples = b;
    // every kSampleStride-th tile of 256 (di = 64) or 128 entries; sized for 256
    L.sample_stride = ((std::max<int64_t>(n_max, 1) + (int64_t)kSampleStride * 128 - 1) / ((int64_t)kSampleStride * 128) + 1) * 256;
    b = align_up(b + (size_t)nq * L.sample_stride * 4, 256);
    L.total = std::max(off, b);
    return L;
}

// ---- attention planning ------------------------------------------------------
// A query's attended rows are cut into `splits` runs of `tiles_per_split`
// tiles, one CTA each; split runs are merged through f32 partials in the
// workspace by a second kernel. Cost in tile-times: waves of CTAs times the
// tiles of a CTA plus a fixed charge for its prologue and epilogue, plus a
// charge per split for writing and merging the partials.
struct AttnPlan {
    int32_t tiles, tiles_per_split, splits;
    int32_t e_tiles = 0, e_splits = 0, tps_e = 0;  // NVFP4 variant: entry splits (see plan_attn_nvfp4)
};

AttnPlan plan_attn(int32_t nq, int32_t k, int32_t w_max, int sms) {
    AttnPlan P{};
    const int64_t rows = (int64_t)k + std::max(0, w_max);
    P.tiles = (int32_t)std::max<int64_t>(1, (rows + kAttnTile - 1) / kAttnTile);
    // a fixed split count (tuning and tests), else the cost model
    if (const char *e = std::getenv("CSA2_ATTN_SPLITS")) {
        const int32_t want = std::max(1, std::min(P.tiles, (int32_t)std::atoi(e)));
        P.tiles_per_split = (P.tiles + want - 1) / want;
        P.splits = (P.tiles + P.tiles_per_split - 1) / P.tiles_per_split;
        return P;
    }
    constexpr double kFixed = 1.2, kMergePerSplit = 0.1;
    double best = 1e30;
    for (int32_t tps = 1; tps <= P.tiles; ++tps) {
        const int32_t splits = (P.tiles + tps - 1) / tps;
        const double waves = (double)(((int64_t)nq * splits + sms - 1) / sms);
        const double cost = waves * (tps + kFixed) + (splits > 1 ? kMergePerSplit * splits : 0.0);
        if (cost < best - 1e-9) {
            best = cost;
            P.tiles_per_split = tps;
            P.splits = splits;
        }
    }
    return P;
}

// NVFP4 variant: the first floor(k / 128) tiles (selected entries only) go
// to entry splits whose S products are FP4; the rest (the last partial entry
// tile and the window) to splits on the f16 path. Both split lengths are
// chosen together with the same cost model, an FP4 tile charged kFp4Tile
// f16 tiles (measured on the 64-head, 2048 + 512-row step: about 6.3 us per
// FP4 tile against 5.1 us per f16 tile, from runs of 1 to 16 tiles a CTA).
AttnPlan plan_attn_nvfp4(int32_t nq, int32_t k, int32_t w_max, int sms) {
    const int32_t e_tiles = k / kAttnTile;
    if (e_tiles == 0) return plan_attn(nq, k, w_max, sms);
    AttnPlan P{};
    const int64_t rows = (int64_t)k + std::max(0, w_max);
    P.tiles = (int32_t)((rows + kAttnTile - 1) / kAttnTile);
    const int32_t w_tiles = P.tiles - e_tiles;
    // fixed tiles per entry split and per window split, "te,tw" (tuning, tests)
    if (const char *e = std::getenv("CSA2_ATTN_NV_TILES")) {
        int te = 1, tw = 1;
        if (std::sscanf(e, "%d,%d", &te, &tw) == 2 && te > 0 && tw > 0) {
            P.e_tiles = e_tiles;
            P.tps_e = std::min(te, e_tiles);
            P.e_splits = (e_tiles + P.tps_e - 1) / P.tps_e;
            P.tiles_per_split = w_tiles > 0 ? std::min(tw, w_tiles) : 1;
            P.splits = P.e_splits + (w_tiles > 0 ? (w_tiles + P.tiles_per_split - 1) / P.tiles_per_split : 0);
            return P;
        }
    }
    constexpr double kFp4Tile = 1.25, kFixed = 1.2, kMergePerSplit = 0.1;
    double best = 1e30;
    for (int32_t te = 1; te <= e_tiles; ++te) {
        const int32_t se = (e_tiles + te - 1) / te;
        for (int32_t tw = 1; tw <= std::max(1, w_tiles); ++tw) {
            const int32_t sw = w_tiles > 0 ? (w_tiles + tw - 1) / tw : 0;
            const int32_t splits = se + sw;
            const double waves = (double)(((int64_t)nq * splits + sms - 1) / sms);
            const double per = std::max(kFp4Tile * te, w_tiles > 0 ? (double)tw : 0.0) + kFixed;
            const double cost = waves * per + (splits > 1 ? kMergePerSplit * splits : 0.0);
            if (cost < best - 1e-9) {
                best = cost;
                P.e_tiles = e_tiles;
                P.tps_e = te;
                P.e_splits = se;
                P.tiles_per_split = w_tiles > 0 ? tw : 1;
                P.splits = splits;
            }
        }
    }
    return P;
}

struct AttnLayout {
    size_t off_o, off_lse, total;
    size_t off_q4 = 0, off_q4s = 0;  // NVFP4 variant: q codes [nq][h][256], scales [nq][h][32]
};

// Split partials: f32 [nq][S][H][512], then the log-sum-exp values [nq][S][H].
AttnLayout attn_layout(int32_t nq, int32_t h, const AttnPlan &P, bool nvfp4 = false) {
    AttnLayout L{};
    if (P.splits > 1) {
        L.off_o = 0;
        L.off_lse = align_up((size_t)nq * P.splits * h * CSA2_D * 4, 256);
        L.total = align_up(L.off_lse + (size_t)nq * P.splits * h * 4, 256);
    }
    if (nvfp4) {
        L.off_q4 = L.total;
        L.off_q4s = align_up(L.off_q4 + (size_t)nq * h * (CSA2_D / 2), 256);
        L.total = align_up(L.off_q4s + (size_t)nq * h * (CSA2_D / CSA2_BLOCK), 256);
    }
    return L;
}

// Persistent decode attention: tiles per query, tiles per CTA (each CTA
// one SM) and the number of partial slots of the split.
struct DecPlan {
    int32_t tpq, per, ctas, slots;
    int32_t max_parts;  // CTAs sharing one query, at most
    size_t off_o, off_lse, off_qslot, off_qcount, total;
};

DecPlan plan_decode(int32_t nq, int32_t h, int32_t k, int32_t w_max, int sms) {
    DecPlan P{};
    const int64_t rows = (int64_t)k + std::max(0, w_max);
    P.tpq = (int32_t)std::max<int64_t>(1, (rows + kAttnTile - 1) / kAttnTile);
    const int64_t T = (int64_t)nq * P.tpq;
    int64_t per = (T + sms - 1) / sms;
    if (const char *e = std::getenv("CSA2_ATTN_PER")) per = std::max<int64_t>(1, std::atoll(e));  // tuning, tests
    P.per = (int32_t)std::min<int64_t>(per, INT32_MAX);
    P.ctas = (int32_t)((T + P.per - 1) / P.per);
    const DecSplit sp{T, P.per, P.tpq};
    P.slots = 0;
    for (int32_t g = 0; g < P.ctas; ++g) P.slots += sp.nparts(g);
    // a query's tiles span at most ceil((tpq - 1) / per) + 1 CTAs
    P.max_parts = (int32_t)std::min<int64_t>(P.ctas, (P.tpq - 1 + (int64_t)P.per - 1) / P.per + 1);
    P.off_o = 0;
    P.off_lse = align_up((size_t)P.slots * h * CSA2_D * 4, 256);
    P.off_qslot = align_up(P.off_lse + (size_t)P.slots * h * 4, 256);
    P.off_qcount = align_up(P.off_qslot + (size_t)nq * 4, 256);
    P.total = P.slots > 0 ? align_up(P.off_qcount + (size_t)nq * 4, 256) : 0;
    return P;
}

// Dynamic shared memory limit of a kernel, and the maximal shared-memory
// carveout, which every kernel of the library requests so that consecutive
// launches do not change the L1 / shared split of the SMs.
// `bytes` is capped at the opt-in maximum minus the kernel's static shared
// memory. A failed attribute call is cleared from the runtime's last error.
template <typename K>
bool set_smem(K kernel, size_t bytes) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    const size_t cap = (size_t)max_smem_optin() - fa.sharedSizeBytes;
    const bool ok =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)std::min(bytes, cap)) ==
            cudaSuccess &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess;
    if (!ok) cudaGetLastError();
    return ok;
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while the previous kernel on the stream is still running; every kernel of
// the library waits (griddepcontrol.wait) for its predecessor's completion
// before it reads global memory, and lets its own dependents start early.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                   Args &&...args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Same, as a thread-block cluster of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                           unsigned cluster, Args &&...args) {
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Kernel attributes belong to a device: every (device, kernel) pair is set up
// once, with that device current, the first time a call on that device needs
// the kernel. `key` names the set-up (a kernel's address or another tag).
std::mutex g_attr_mu;
std::set<std::pair<int, const void *>> g_attr_done;

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return dev;
}

template <typename F>
bool once_per_device(const void *key, F &&setup) {
    const int dev = current_device();
    if (dev < 0) return false;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (g_attr_done.count({dev, key})) return true;
    if (!setup()) return false;
    g_attr_done.insert({dev, key});
    return true;
}

// set_smem once per device for this kernel.
template <typename K>
bool smem_attr(K kernel, size_t bytes) {
    return once_per_device(reinterpret_cast<const void *>(kernel), [&] { return set_smem(kernel, bytes); });
}

// Attributes of the single-launch Full kernel (maximal dynamic shared
// memory; clusters above 8 CTAs need the non-portable size), set once per
// device, and how many clusters of each size that device holds at once
// (0: not possible).
template <int DI>
const int *fused_cluster_caps() {
    static std::mutex mu;
    static std::map<int, std::array<int, kFusedClusterMax + 1>> per_dev;
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(mu);
    auto it = per_dev.find(dev);
    if (it != per_dev.end()) return it->second.data();
    std::array<int, kFusedClusterMax + 1> caps{};
    if (dev >= 0 && set_smem(k_index_full_fused<DI>, (size_t)max_smem_optin())) {
        if (cudaFuncSetAttribute(k_index_full_fused<DI>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess)
            cudaGetLastError();
        for (int c = kFusedClusterMin; c <= kFusedClusterMax; ++c) {
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)c;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)c, 1);
            cfg.blockDim = dim3(kFusedThreads);
            cfg.dynamicSmemBytes = (size_t)max_smem_optin() - 1024;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, k_index_full_fused<DI>, &cfg) != cudaSuccess) {
                cudaGetLastError();
                n = 0;
            }
            caps[c] = n;
        }
    }
    return per_dev.emplace(dev, caps).first->second.data();
}

// CTAs per query for the single-launch Full kernel: the largest size whose
// clusters the device holds for all queries at once, as long as every CTA
// keeps at least two tiles of entries; the portable 8 otherwise.
int fused_cluster_size(bool di64, int32_t nq, int64_t n_max, int tile_entries) {
    const int *caps = di64 ? fused_cluster_caps<64>() : fused_cluster_caps<128>();
    if (const char *e = std::getenv("CSA2_FULL_CLUSTER")) {
        const int c = std::atoi(e);
        if (c >= kFusedClusterMin && c <= kFusedClusterMax && caps[c] > 0) return c;
    }
    for (int c = kFusedClusterMax; c > kFusedClusterMin; --c)
        if (caps[c] >= nq && n_max >= (int64_t)c * 2 * tile_entries) return c;
    return kFusedClusterMin;
}

template <typename K>
bool prefer_shared(K kernel) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess;
}

// Attribute set-up of the kernels without large dynamic shared memory, once
// per device.
bool init_small_kernels() {
    static const char key = 0;
    return once_per_device(&key, [] {
        return prefer_shared(k_append_fp4) && prefer_shared(k_append_e4m3<kE4m3WindowPieces>) && prefer_shared(k_append_e4m3<1>) && prefer_shared(k_sel_collect) && prefer_shared(k_pad_heads) && prefer_shared(k_unpad_heads) && prefer_shared(k_batch_sthresh) && prefer_shared(k_batch_thresh) &&
               prefer_shared(k_reindex_score<64>) && prefer_shared(k_reindex_score<128>) &&
               prefer_shared(k_attn_combine<16, false>) && prefer_shared(k_attn_combine<32, false>) &&
               prefer_shared(k_attn_combine<64, false>) && prefer_shared(k_attn_combine<16, true>) &&
               prefer_shared(k_attn_combine<32, true>) && prefer_shared(k_attn_combine<64, true>) &&
               prefer_shared(k_attn_merge_parts<16, false>) && prefer_shared(k_attn_merge_parts<32, false>) &&
               prefer_shared(k_attn_merge_parts<64, false>) && prefer_shared(k_attn_merge_parts<16, true>) &&
               prefer_shared(k_attn_merge_parts<32, true>) && prefer_shared(k_attn_merge_parts<64, true>) &&
               prefer_shared(k_wait_selfcheck);
    });
}

}  // namespace

extern "C" {

int32_t csa2_version(void) { return kVersion; }

const char *csa2_status_string(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_INVALID_ARG: return "invalid argument";
        case CSA2_ERR_UNSUPPORTED: return "unsupported configuration";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA2_ERR_CUDA: return "CUDA error";
        case CSA2_ERR_DEVICE: return "device-side error recorded";
    }
    return "unknown status";
}

csa2_status csa2_device_status(cudaStream_t stream, uint32_t *code) {
    if (!code) return CSA2_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return CSA2_ERR_CUDA;
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof v) != cudaSuccess) return CSA2_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_dev_error, &z, sizeof z) != cudaSuccess) return CSA2_ERR_CUDA;
    *code = v;
    return v ? CSA2_ERR_DEVICE : CSA2_OK;
}

csa2_status csa2_check_wait_timeout(uint32_t limit_us, cudaStream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return CSA2_ERR_INVALID_ARG;
    k_wait_selfcheck<<<1, 32, 0, stream>>>((uint64_t)limit_us * 1000ull);
    return check_launch();
}

csa2_status csa2_append_fp4(const void *x_bf16, int32_t n, const int32_t *seq, const int64_t *pos,
                            const csa2_kv_desc *kv, cudaStream_t stream) {
    csa2_status st = check_kv(kv, false);
    if (st != CSA2_OK) return st;
    if (n < 0) return CSA2_ERR_INVALID_ARG;
    if (n == 0) return CSA2_OK;
    if (!x_bf16 || !seq || !pos || !aligned(x_bf16, 16) || !aligned(seq, 4) || !aligned(pos, 8))
        return CSA2_ERR_INVALID_ARG;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    // one wave of resident CTAs (each warp walks rows with a stride), fewer
    // when there are not enough rows for one per warp
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_append_fp4, kAppendWarps * 32, 0) != cudaSuccess ||
        per_sm < 1) {
        cudaGetLastError();
        per_sm = 1;
    }
    const int64_t want = (int64_t)num_sms() * per_sm;
    const unsigned grid =
        (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, ((int64_t)n + kAppendWarps - 1) / kAppendWarps));
    launch(k_append_fp4, dim3(grid), dim3(kAppendWarps * 32), 0, stream, static_cast<const uint16_t *>(x_bf16), n, seq, pos, *kv);
    return check_launch();
}

csa2_status csa2_append_swa_e4m3(const void *x_bf16, int32_t n, const int32_t *seq, const int64_t *pos,
                                 uint8_t *swa, int32_t batch, int64_t ring_rows, cudaStream_t stream) {
    if (n < 0 || batch <= 0 || ring_rows <= 0) return CSA2_ERR_INVALID_ARG;
    if (n == 0) return CSA2_OK;
    if (!x_bf16 || !seq || !pos || !swa || !aligned(x_bf16, 16) || !aligned(seq, 4) || !aligned(pos, 8) ||
        !aligned(swa, 8))
        return CSA2_ERR_INVALID_ARG;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    const int64_t threads = (int64_t)n * (CSA2_D / (8 * kE4m3WindowPieces));
    const unsigned grid = (unsigned)((threads + kE4m3Threads - 1) / kE4m3Threads);
    launch(k_append_e4m3<kE4m3WindowPieces>, dim3(grid), dim3(kE4m3Threads), 0, stream, static_cast<const uint16_t *>(x_bf16), n,
           (int32_t)CSA2_D, seq, pos, (int32_t)0, swa, batch, ring_rows, csa2_kv_desc{});
    return check_launch();
}

csa2_status csa2_append_kidx_e4m3(const void *x_bf16, int32_t n, const int32_t *seq, const int64_t *pos,
                                  const csa2_kv_desc *kv, cudaStream_t stream) {
    csa2_status st = check_kv(kv, true);
    if (st != CSA2_OK) return st;
    if (n < 0) return CSA2_ERR_INVALID_ARG;
    if (n == 0) return CSA2_OK;
    if (!x_bf16 || !seq || !pos || !aligned(x_bf16, 16) || !aligned(seq, 4) || !aligned(pos, 8))
        return CSA2_ERR_INVALID_ARG;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    const int64_t threads = (int64_t)n * (kv->di / 8);
    const unsigned grid = (unsigned)((threads + kE4m3Threads - 1) / kE4m3Threads);
    launch(k_append_e4m3<1>, dim3(grid), dim3(kE4m3Threads), 0, stream, static_cast<const uint16_t *>(x_bf16), n,
           kv->di, seq, pos, (int32_t)1, static_cast<uint8_t *>(nullptr), (int32_t)0, (int64_t)1, *kv);
    return check_launch();
}

size_t csa2_index_full_workspace_size(int32_t nq, int64_t n_max) {
    if (nq <= 0 || n_max < 0) return 0;
    return full_layout(nq, n_max).total;
}

csa2_status csa2_index_full(const uint8_t *qidx, const float *w, int32_t nq, int32_t q_per_seq, int32_t hi,
                            const int32_t *q_limit, int64_t n_max, const csa2_kv_desc *kv, int32_t k, int32_t p,
                            int32_t *topk, int32_t *pool, void *ws, size_t ws_bytes, cudaStream_t stream) {
    csa2_status st = check_kv(kv, true);
    if (st != CSA2_OK) return st;
    if (nq <= 0 || nq > 65535 || q_per_seq <= 0 || (nq + q_per_seq - 1) / q_per_seq > kv->batch)
        return CSA2_ERR_INVALID_ARG;
    if (hi < 1 || hi > kScanN) return CSA2_ERR_UNSUPPORTED;
    if (k < 1 || p < 0 || (p > 0 && p < k) || n_max < 0) return CSA2_ERR_INVALID_ARG;
    if (k > kBatchMaxK || p > kBatchMaxK) return CSA2_ERR_UNSUPPORTED;
    if (n_max > (int64_t)kv->max_pages * kv->page_size) return CSA2_ERR_INVALID_ARG;
    if (!qidx || !w || !topk || !aligned(qidx, 16) || !aligned(w, 4) || !aligned(topk, 4))
        return CSA2_ERR_INVALID_ARG;
    if ((p > 0) != (pool != nullptr) || (pool && !aligned(pool, 4))) return CSA2_ERR_INVALID_ARG;
    if (q_limit && !aligned(q_limit, 4)) return CSA2_ERR_INVALID_ARG;
    const FullLayout L = full_layout(nq, n_max);
    if (!ws || ws_bytes < L.total || !aligned(ws, 256)) return CSA2_ERR_WORKSPACE;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    uint8_t *wsb = static_cast<uint8_t *>(ws);

    const int epr = 128 / kv->di;                                  // entries per 128-byte row
    // rows per TMA box: a box holds gcd(page_size, tile) entries, so it never crosses a page
    const int box_rows = std::gcd((int)kv->page_size, 128 * epr) / epr;
    const int tile_entries = 128 * epr;
    CUtensorMap tm;
    if (!make_kidx_map(&tm, kv, box_rows)) return CSA2_ERR_CUDA;

    // Batched: many queries of one sequence share each key tile in one
    // tensor-core product (groups of 16 queries with up to 4 indexer heads, 8
    // with up to 8), two scans of the keys and an exact select per query.
    {
        const int hp = hi <= 4 ? 4 : 8;
        const int qg = batch_qg(hp);
        const FullPath fp = full_path_env();
        const bool applies = p == 0 && hi <= 8 && k <= kBatchMaxK && q_per_seq % qg == 0;
        if (applies && (fp == kPathBatch || (fp == kPathAuto && q_per_seq >= 64))) {
            CUtensorMap bm;
            if (!make_kidx_map(&bm, kv, box_rows)) return CSA2_ERR_CUDA;
            BatchParams bp{};
            bp.qidx = qidx;
            bp.w = w;
            bp.q_limit = q_limit;
            bp.kv = *kv;
            bp.hist = reinterpret_cast<uint32_t *>(wsb + L.b_hist);
            bp.state = reinterpret_cast<uint32_t *>(wsb + L.b_state);
            bp.state_stride = 2;
            bp.state_off = 0;
            bp.cnt = reinterpret_cast<uint32_t *>(wsb + L.b_cnt);
            bp.sure = reinterpret_cast<int32_t *>(wsb + L.b_sure);
            bp.cand = reinterpret_cast<unsigned long long *>(wsb + L.b_cand);
            bp.topk = topk;
            bp.k = k;
            bp.sure_stride = k;
            bp.q_per_seq = q_per_seq;
            bp.hi = hi;
            bp.hi_pad = hp;
            bp.nq = nq;
            bp.box_rows = box_rows;
            const int ngroups = (nq + qg - 1) / qg;
            const BatchSplit bsp = batch_split(nq, n_max, tile_entries, num_sms(), qg);
            bp.chunk = bsp.chunk;
            bp.nchunks = (int32_t)((std::max<int64_t>(n_max, 1) + bp.chunk - 1) / bp.chunk);
            if (bp.chunk / kv->page_size + 2 > kMaxScanPages) return CSA2_ERR_UNSUPPORTED;
            const dim3 sgrid((unsigned)bp.nchunks, (unsigned)ngroups);
            const size_t fsm = (size_t)max_smem_optin() - 1024;  // leaves room for the static shared words
            if (!smem_attr(k_batch_final, fsm)) return CSA2_ERR_CUDA;
            const size_t ffixed =
                2048 * 4 + (kBatchFinalThreads / 32 + 8) * 4 + 4 * kBatchMaxChunks * 4 + (size_t)kBatchMaxK * 4;
            const int32_t smem_keys = (int32_t)((fsm - ffixed) / 8);
            const BatchMode mode = batch_mode_env();
            // Sampled threshold path: sample pass (every kSampleStride-th tile),
            // per-query threshold, one collecting pass (every key at or above
            // the threshold), exact select; queries with too few candidates are
            // marked for the exact passes that follow.
            uint32_t *redo = reinterpret_cast<uint32_t *>(wsb + L.b_redo);
            if (mode != kBatchExact) {
                BatchParams sp = bp;
                sp.state = reinterpret_cast<uint32_t *>(wsb + L.b_sstate);
                sp.samples = reinterpret_cast<uint32_t *>(wsb + L.b_samples);
                sp.sample_stride = L.sample_stride;
                sp.tile_stride = kSampleStride;
                sp.sample_rank = (int32_t)((3 * (int64_t)k + 2 * kSampleStride - 1) / (2 * kSampleStride)) + 32;
                if (cudaMemsetAsync(redo, 0, (size_t)nq * 4, stream) != cudaSuccess) return CSA2_ERR_CUDA;
                auto spass = [&](auto k2, auto k3, size_t sm2, size_t sm3) -> csa2_status {
                    if (!smem_attr(k2, sm2) || !smem_attr(k3, sm3)) return CSA2_ERR_CUDA;
                    launch(k2, sgrid, dim3(kBatchThreads), sm2, stream, bm, sp);
                    launch(k_batch_sthresh, dim3((unsigned)nq), dim3(kSthreshThreads), 0, stream, sp);
                    launch(k3, sgrid, dim3(kBatchThreads), sm3, stream, bm, sp);
                    return CSA2_OK;
                };
                csa2_status ss;
                if (kv->di == 64 && hp == 4)
                    ss = spass(k_batch_scan<64, 4, 2>, k_batch_scan<64, 4, 3>, BatchCfg<64, 4, 2>::kSmem,
                               BatchCfg<64, 4, 3>::kSmem);
                else if (kv->di == 64)
                    ss = spass(k_batch_scan<64, 8, 2>, k_batch_scan<64, 8, 3>, BatchCfg<64, 8, 2>::kSmem,
                               BatchCfg<64, 8, 3>::kSmem);
                else if (hp == 4)
                    ss = spass(k_batch_scan<128, 4, 2>, k_batch_scan<128, 4, 3>, BatchCfg<128, 4, 2>::kSmem,
                               BatchCfg<128, 4, 3>::kSmem);
                else
                    ss = spass(k_batch_scan<128, 8, 2>, k_batch_scan<128, 8, 3>, BatchCfg<128, 8, 2>::kSmem,
                               BatchCfg<128, 8, 3>::kSmem);
                if (ss != CSA2_OK) return ss;
                sp.redo = redo;
                sp.redo_mark = mode == kBatchRedo ? 2 : 1;
                launch(k_batch_final, dim3((unsigned)nq), dim3(kBatchFinalThreads), fsm, stream, sp, smem_keys);
                bp.redo = redo;  // the exact passes below take only the marked queries
            }
            // Exact path: two scans with a digit-0 histogram and threshold bin.
            if (cudaMemsetAsync(bp.hist, 0, (size_t)nq * kBatchBins * 4, stream) != cudaSuccess) return CSA2_ERR_CUDA;
            auto scan = [&](auto k0, auto k1, size_t sm0, size_t sm1) -> csa2_status {
                if (!smem_attr(k0, sm0) || !smem_attr(k1, sm1)) return CSA2_ERR_CUDA;
                launch(k0, sgrid, dim3(kBatchThreads), sm0, stream, bm, bp);
                launch(k_batch_thresh, dim3((unsigned)nq), dim3(kBatchThreshThreads), 0, stream, bp);
                launch(k1, sgrid, dim3(kBatchThreads), sm1, stream, bm, bp);
                return CSA2_OK;
            };
            csa2_status bs;
            if (kv->di == 64 && hp == 4)
                bs = scan(k_batch_scan<64, 4, 0>, k_batch_scan<64, 4, 1>, BatchCfg<64, 4, 0>::kSmem,
                          BatchCfg<64, 4, 1>::kSmem);
            else if (kv->di == 64)
                bs = scan(k_batch_scan<64, 8, 0>, k_batch_scan<64, 8, 1>, BatchCfg<64, 8, 0>::kSmem,
                          BatchCfg<64, 8, 1>::kSmem);
            else if (hp == 4)
                bs = scan(k_batch_scan<128, 4, 0>, k_batch_scan<128, 4, 1>, BatchCfg<128, 4, 0>::kSmem,
                          BatchCfg<128, 4, 1>::kSmem);
            else
                bs = scan(k_batch_scan<128, 8, 0>, k_batch_scan<128, 8, 1>, BatchCfg<128, 8, 0>::kSmem,
                          BatchCfg<128, 8, 1>::kSmem);
            if (bs != CSA2_OK) return bs;
            launch(k_batch_final, dim3((unsigned)nq), dim3(kBatchFinalThreads), fsm, stream, bp, smem_keys);
            return check_launch();
        }
    }

    // Single launch: one cluster per query, every score kept in shared
    // memory, when a query's entries fit. Clusters of 16 CTAs when the device
    // holds one for every query at once, else 8.
    {
        const bool di64 = kv->di == 64;
        const int cl = fused_cluster_size(di64, nq, n_max, tile_entries);
        const int64_t slice = (int64_t)align_up((size_t)((std::max<int64_t>(n_max, 1) + cl - 1) / cl),
                                                (size_t)tile_entries);
        const size_t stage_bytes = 128 * 128;
        const size_t fixed = (di64 ? FusedCfg<64>::kFixed : FusedCfg<128>::kFixed) + 64 * 8 + 16;
        const size_t budget = (size_t)max_smem_optin();
        int stages = 0;
        if (fixed + (size_t)slice * 4 < budget) stages = (int)std::min<size_t>(16, (budget - fixed - slice * 4) / stage_bytes);
        const bool pages_fit = slice / kv->page_size + 2 <= kMaxScanPages;
        // the emission's chunk masks (16 B per 32 keys and warp) reuse the TMA ring
        const bool masks_fit = (size_t)slice / 2 + 128 <= (size_t)stages * stage_bytes;
        if (stages >= 3 && pages_fit && masks_fit && !force_multipass()) {
            FusedParams fp{};
            fp.qidx = qidx;
            fp.w = w;
            fp.q_limit = q_limit;
            fp.kv = *kv;
            fp.out[0] = topk;
            fp.out[1] = pool;
            fp.rank[0] = k;
            fp.rank[1] = p;
            fp.q_per_seq = q_per_seq;
            fp.hi = hi;
            fp.box_rows = box_rows;
            fp.slice = (int32_t)slice;
            fp.stages = stages;
            const dim3 fgrid((unsigned)cl, (unsigned)nq);
            const size_t smem = di64 ? FusedCfg<64>::smem((int)slice, stages) : FusedCfg<128>::smem((int)slice, stages);
            fp.csize = cl;
            if (di64)
                launch_cluster(k_index_full_fused<64>, fgrid, dim3(kFusedThreads), smem, stream, (unsigned)cl, tm, fp);
            else
                launch_cluster(k_index_full_fused<128>, fgrid, dim3(kFusedThreads), smem, stream, (unsigned)cl, tm,
                               fp);
            return check_launch();
        }
    }

    if (cudaMemsetAsync(wsb + L.off_hist0, 0, L.off_cnt - L.off_hist0, stream) != cudaSuccess) return CSA2_ERR_CUDA;

    ScanParams sp{};
    sp.qidx = qidx;
    sp.w = w;
    sp.q_limit = q_limit;
    sp.kv = *kv;
    sp.keys = reinterpret_cast<uint32_t *>(wsb + L.off_keys);
    sp.hist0 = reinterpret_cast<uint32_t *>(wsb + L.off_hist0);
    sp.state = reinterpret_cast<uint32_t *>(wsb + L.off_state);
    sp.rank[0] = k;
    sp.rank[1] = p;
    sp.key_stride = L.key_stride;
    sp.q_per_seq = q_per_seq;
    sp.hi = hi;
    sp.box_rows = box_rows;
    const int64_t tiles_max = std::max<int64_t>(1, (n_max + tile_entries - 1) / tile_entries);
    // several waves of two resident CTAs per SM when every query had n_max
    // entries: queries of ragged lengths then leave short CTAs behind instead
    // of a few long ones, and the hardware scheduler evens the SMs out
    const int64_t target = (int64_t)num_sms() * 2 * 4;
    int64_t chunk = std::max<int64_t>(16, ((int64_t)nq * tiles_max + target - 1) / target);
    chunk = std::min<int64_t>(chunk, 256);
    chunk = std::min<int64_t>(chunk, std::max<int64_t>(1, ((int64_t)(kMaxScanPages - 2) * kv->page_size) / tile_entries));
    sp.chunk_tiles = (int32_t)chunk;
    const dim3 sgrid((unsigned)((tiles_max + chunk - 1) / chunk), (unsigned)nq);
    if (kv->di == 64) {
        if (!smem_attr(k_index_scan<64>, ScanCfg<64>::kSmem)) return CSA2_ERR_CUDA;
        launch(k_index_scan<64>, sgrid, dim3(kScanThreads), ScanCfg<64>::kSmem, stream, tm, sp);
    } else {
        if (!smem_attr(k_index_scan<128>, ScanCfg<128>::kSmem)) return CSA2_ERR_CUDA;
        launch(k_index_scan<128>, sgrid, dim3(kScanThreads), ScanCfg<128>::kSmem, stream, tm, sp);
    }
    if ((st = check_launch()) != CSA2_OK) return st;

    // per target (Top-K, then the pool): collect each query's sure ids and
    // threshold-bin candidates in parts, then the exact select and sort of
    // the batched path
    BatchParams cp{};
    cp.q_limit = q_limit;
    cp.kv = *kv;
    cp.state = sp.state;
    cp.state_stride = kStateWords;
    cp.cnt = reinterpret_cast<uint32_t *>(wsb + L.off_cnt);
    cp.sure = reinterpret_cast<int32_t *>(wsb + L.off_sure);
    cp.cand = reinterpret_cast<unsigned long long *>(wsb + L.off_cand);
    cp.chunk = L.c_chunk;
    cp.nchunks = L.c_parts;
    cp.sure_stride = L.c_sure_stride;
    cp.shift1 = kCollectShift1;
    cp.parts_sorted = 1;
    cp.q_per_seq = q_per_seq;
    cp.nq = nq;
    const size_t fsm = (size_t)max_smem_optin() - 1024;  // leaves room for the static shared words
    if (!smem_attr(k_batch_final, fsm)) return CSA2_ERR_CUDA;
    const size_t ffixed = 2048 * 4 + (kBatchFinalThreads / 32 + 8) * 4 + 4 * kBatchMaxChunks * 4 + (size_t)kBatchMaxK * 4;
    const int32_t smem_keys = (int32_t)((fsm - ffixed) / 8);
    for (int tau = 0; tau < 2; ++tau) {
        const int32_t rank = tau == 0 ? k : p;
        if (rank <= 0) continue;
        cp.state_off = 8 * tau;
        cp.hist1 = reinterpret_cast<uint32_t *>(wsb + L.off_hist1) + (size_t)tau * nq * 2048;
        cp.k = rank;
        cp.topk = tau == 0 ? topk : pool;
        launch(k_sel_collect, dim3((unsigned)L.c_parts, (unsigned)nq), dim3(kCollectThreads), 0, stream, cp,
               (const uint32_t *)sp.keys, L.key_stride, rank);
        launch(k_batch_final, dim3((unsigned)nq), dim3(kBatchFinalThreads), fsm, stream, cp, smem_keys);
    }
    return check_launch();
}

size_t csa2_index_reindex_workspace_size(int32_t nq, int32_t p) {
    if (nq <= 0 || p <= 0) return 0;
    return align_up((size_t)nq * p * 8, 256);
}

csa2_status csa2_index_reindex(const uint8_t *qidx, const float *w, int32_t nq, int32_t q_per_seq, int32_t hi,
                               const int32_t *pool, int32_t p, const csa2_kv_desc *kv, int32_t k, int32_t *topk,
                               void *ws, size_t ws_bytes, cudaStream_t stream) {
    csa2_status st = check_kv(kv, true);
    if (st != CSA2_OK) return st;
    if (nq <= 0 || nq > 65535 || q_per_seq <= 0 || (nq + q_per_seq - 1) / q_per_seq > kv->batch)
        return CSA2_ERR_INVALID_ARG;
    if (hi < 1 || hi > kScanN) return CSA2_ERR_UNSUPPORTED;
    if (k < 1 || p < 1) return CSA2_ERR_INVALID_ARG;
    if (p > kReindexMaxPool) return CSA2_ERR_UNSUPPORTED;
    if (!qidx || !w || !pool || !topk || !aligned(qidx, 16) || !aligned(w, 4) || !aligned(pool, 4) ||
        !aligned(topk, 4))
        return CSA2_ERR_INVALID_ARG;
    if (!ws || ws_bytes < csa2_index_reindex_workspace_size(nq, p) || !aligned(ws, 256)) return CSA2_ERR_WORKSPACE;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    ReindexParams rp{};
    rp.qidx = qidx;
    rp.w = w;
    rp.pool = pool;
    rp.kv = *kv;
    rp.k64 = static_cast<unsigned long long *>(ws);
    rp.topk = topk;
    rp.p = p;
    rp.k = k;
    rp.hi = hi;
    rp.q_per_seq = q_per_seq;
    // one launch (opt-in, see reindex_cluster): a cluster of CTAs per query
    // scores the pool into the first CTA's shared memory, which selects
    const int cl = (p + kRcThreads - 1) / kRcThreads;
    if (cl <= kRcMaxCluster && reindex_cluster()) {
        const size_t rsm = 2048 * 4 + (kRcThreads / 32 + 8) * 4 + (size_t)p * 8;
        const dim3 rgrid((unsigned)cl, (unsigned)nq);
        if (kv->di == 64) {
            if (!smem_attr(k_reindex_cluster<64>, (size_t)max_smem_optin())) return CSA2_ERR_CUDA;
            launch_cluster(k_reindex_cluster<64>, rgrid, dim3(kRcThreads), rsm, stream, (unsigned)cl, rp);
        } else {
            if (!smem_attr(k_reindex_cluster<128>, (size_t)max_smem_optin())) return CSA2_ERR_CUDA;
            launch_cluster(k_reindex_cluster<128>, rgrid, dim3(kRcThreads), rsm, stream, (unsigned)cl, rp);
        }
        return check_launch();
    }
    const dim3 grid((unsigned)((p + kReindexScoreThreads - 1) / kReindexScoreThreads), (unsigned)nq);
    if (kv->di == 64)
        launch(k_reindex_score<64>, grid, dim3(kReindexScoreThreads), 0, stream, rp);
    else
        launch(k_reindex_score<128>, grid, dim3(kReindexScoreThreads), 0, stream, rp);
    if ((st = check_launch()) != CSA2_OK) return st;
    const size_t smem = 2048 * 4 + (kReindexSelectThreads / 32 + 8) * 4 + (size_t)p * 8;
    if (!smem_attr(k_reindex_select<false>, (size_t)max_smem_optin())) return CSA2_ERR_CUDA;
    launch(k_reindex_select<false>, dim3(nq), dim3(kReindexSelectThreads), smem, stream, rp);
    return check_launch();
}

size_t csa2_sparse_attn_workspace_size(int32_t nq, int32_t h, int32_t k, int32_t w_max) {
    if (nq <= 0 || h <= 0 || k < 0) return 0;
    if (h != 16 && h != 32 && h != 64) return 0;
    return plan_decode(nq, h, k, w_max, num_sms()).total;
}

}  // extern "C"

namespace {

template <bool F32>
void launch_combine(int32_t h, int32_t nq, const CombineArgs &ca, cudaStream_t stream) {
    const dim3 cgrid((unsigned)(h / kCombineHeads), (unsigned)nq);
    const size_t csmem = (size_t)(ca.n_splits + 1) * 4;
    switch (h) {
        case 64: launch(k_attn_combine<64, F32>, cgrid, dim3(kCombineThreads), csmem, stream, ca); break;
        case 32: launch(k_attn_combine<32, F32>, cgrid, dim3(kCombineThreads), csmem, stream, ca); break;
        default: launch(k_attn_combine<16, F32>, cgrid, dim3(kCombineThreads), csmem, stream, ca); break;
    }
}

template <int H>
csa2_status launch_decode(const DecParams &dp, const DecPlan &P, bool out_f32, cudaStream_t stream) {
    // the merge reads slot numbers the decode kernel writes: it is not
    // launched after a failed launch of that kernel
    if (dp.inline_merge && cudaMemsetAsync(dp.qcount, 0, (size_t)dp.nq * 4, stream) != cudaSuccess) {
        cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    if (launch(k_attn_decode<H>, dim3((unsigned)P.ctas), dim3(kDecThreads), DecCfg<H>::kSmem, stream, dp) !=
        cudaSuccess) {
        cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    if (P.slots > 0 && !dp.inline_merge) {
        const dim3 mgrid((unsigned)H, (unsigned)dp.nq);
        if (out_f32)
            launch(k_attn_merge_parts<H, true>, mgrid, dim3(kMergeThreads), 0, stream, dp);
        else
            launch(k_attn_merge_parts<H, false>, mgrid, dim3(kMergeThreads), 0, stream, dp);
    }
    return CSA2_OK;
}

// The exact decode attention (arguments already checked by attn_impl):
// the persistent kernel, then the merge of the queries split across CTAs.
csa2_status decode_impl(const void *q_bf16, int32_t nq, int32_t q_per_seq, int32_t h, const csa2_kv_desc *kv,
                        const int32_t *topk, int32_t k, const uint8_t *swa, int64_t swa_seq_stride,
                        const int32_t *swa_begin, const int32_t *swa_end, int32_t w_max, float softmax_scale, void *o,
                        bool out_f32, float *lse, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const DecPlan P = plan_decode(nq, h, k, w_max, num_sms());
    if (P.total > 0 && (!ws || ws_bytes < P.total || !aligned(ws, 256))) return CSA2_ERR_WORKSPACE;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    DecParams dp{};
    dp.q = static_cast<const uint16_t *>(q_bf16);
    dp.kv = *kv;
    dp.topk = topk;
    dp.swa = swa;
    dp.swa_seq_stride = swa_seq_stride;
    dp.swa_begin = swa_begin;
    dp.swa_end = swa_end;
    dp.o = out_f32 ? nullptr : static_cast<uint16_t *>(o);
    dp.o32 = out_f32 ? static_cast<float *>(o) : nullptr;
    dp.lse = lse;
    dp.o_part = P.slots > 0 ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + P.off_o) : nullptr;
    dp.lse_part = P.slots > 0 ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + P.off_lse) : nullptr;
    dp.qslot = P.slots > 0 ? reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + P.off_qslot) : nullptr;
    dp.scale_log2 = softmax_scale * 1.4426950408889634f;
    dp.k = k;
    dp.w_max = w_max;
    dp.q_per_seq = q_per_seq;
    dp.nq = nq;
    dp.tpq = P.tpq;
    dp.per = P.per;
    dp.nslots = P.slots;
    // queries split over at most kInlineMergeParts CTAs are merged inside the
    // kernel by the CTA that finishes their last part; wider splits by the
    // merge kernel (CSA2_ATTN_MERGE=kernel forces the merge kernel)
    const char *mk = std::getenv("CSA2_ATTN_MERGE");
    dp.inline_merge = P.slots > 0 && P.max_parts <= kInlineMergeParts && !(mk && std::strcmp(mk, "kernel") == 0);
    dp.qcount = P.slots > 0 ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + P.off_qcount) : nullptr;
    switch (h) {
        case 64:
            if (!smem_attr(k_attn_decode<64>, DecCfg<64>::kSmem)) return CSA2_ERR_CUDA;
            if (launch_decode<64>(dp, P, out_f32, stream) != CSA2_OK) return CSA2_ERR_CUDA;
            break;
        case 32:
            if (!smem_attr(k_attn_decode<32>, DecCfg<32>::kSmem)) return CSA2_ERR_CUDA;
            if (launch_decode<32>(dp, P, out_f32, stream) != CSA2_OK) return CSA2_ERR_CUDA;
            break;
        default:
            if (!smem_attr(k_attn_decode<16>, DecCfg<16>::kSmem)) return CSA2_ERR_CUDA;
            if (launch_decode<16>(dp, P, out_f32, stream) != CSA2_OK) return CSA2_ERR_CUDA;
            break;
    }
    return check_launch();
}

// Workspace of the NVFP4 variant for fewer than 64 heads: the 64-head call's
// region, then q padded to 64 heads, its bf16 o and its lse.
struct NvPad {
    size_t inner, off_q, off_o, off_lse, total;
};
NvPad nvfp4_pad_layout(int32_t nq, int32_t k, int32_t w_max) {
    NvPad d{};
    const AttnPlan P = plan_attn_nvfp4(nq, k, w_max, num_sms());
    d.inner = attn_layout(nq, 64, P, true).total;
    d.off_q = align_up(d.inner, 256);
    d.off_o = align_up(d.off_q + (size_t)nq * 64 * CSA2_D * 2, 256);
    d.off_lse = align_up(d.off_o + (size_t)nq * 64 * CSA2_D * 2, 256);
    d.total = align_up(d.off_lse + (size_t)nq * 64 * 4, 256);
    return d;
}

// Shared body of the decode entry points: o is bf16 (out_f32 false) or the
// normalised f32 o of this call's rows (out_f32 true, lse required).
csa2_status attn_impl(const void *q_bf16, int32_t nq, int32_t q_per_seq, int32_t h, const csa2_kv_desc *kv,
                      const int32_t *topk, int32_t k, const uint8_t *swa, int64_t swa_seq_stride,
                      const int32_t *swa_begin, const int32_t *swa_end, int32_t w_max, float softmax_scale, void *o,
                      bool out_f32, float *lse, void *ws, size_t ws_bytes, cudaStream_t stream, bool nvfp4 = false) {
    csa2_status st = check_kv(kv, false);
    if (st != CSA2_OK) return st;
    if (h != 16 && h != 32 && h != 64) return CSA2_ERR_UNSUPPORTED;
    // the block-scaled S product runs at N = 64 only (its scale-factor layout in
    // TMEM is established for that shape): 16 and 32 heads run as 64 heads with
    // q padded by zero heads (the h != 64 branch below)
    if (nvfp4 && h != 64 && out_f32) return CSA2_ERR_UNSUPPORTED;
    if (nq <= 0 || nq > 65535 || q_per_seq <= 0 || (nq + q_per_seq - 1) / q_per_seq > kv->batch)
        return CSA2_ERR_INVALID_ARG;
    if (k < 0 || w_max < 0 || (k > 0 && !topk) || (topk && !aligned(topk, 4))) return CSA2_ERR_INVALID_ARG;
    if (!q_bf16 || !o || !aligned(q_bf16, 16) || !aligned(o, 16) || (lse && !aligned(lse, 4)))
        return CSA2_ERR_INVALID_ARG;
    if (out_f32 && !lse) return CSA2_ERR_INVALID_ARG;
    const bool has_swa = swa_begin != nullptr;
    if (has_swa && (!swa || !swa_end || !aligned(swa, 16) || !aligned(swa_begin, 4) || !aligned(swa_end, 4)))
        return CSA2_ERR_INVALID_ARG;
    if (!has_swa && w_max > 0) return CSA2_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return CSA2_ERR_INVALID_ARG;
    if (!nvfp4) return decode_impl(q_bf16, nq, q_per_seq, h, kv, topk, k, swa, swa_seq_stride, has_swa ? swa_begin : nullptr,
                                   has_swa ? swa_end : nullptr, has_swa ? w_max : 0, softmax_scale, o, out_f32, lse,
                                   ws, ws_bytes, stream);
    if (h != 64) {
        // 16 or 32 heads: q padded to 64 heads in the workspace (after the
        // 64-head call's own region), the padded call, then its first h heads
        const NvPad pd = nvfp4_pad_layout(nq, k, has_swa ? w_max : 0);
        if (!ws || ws_bytes < pd.total || !aligned(ws, 256)) return CSA2_ERR_WORKSPACE;
        if (!init_small_kernels()) return CSA2_ERR_CUDA;
        uint8_t *wsb = static_cast<uint8_t *>(ws);
        const int64_t pieces_in = (int64_t)nq * 64 * (CSA2_D * 2 / 16);
        launch(k_pad_heads, dim3((unsigned)((pieces_in + 255) / 256)), dim3(256), 0, stream,
               static_cast<const uint4 *>(q_bf16), h, nq, reinterpret_cast<uint4 *>(wsb + pd.off_q));
        if ((st = check_launch()) != CSA2_OK) return st;
        st = attn_impl(wsb + pd.off_q, nq, q_per_seq, 64, kv, topk, k, swa, swa_seq_stride, swa_begin, swa_end,
                       w_max, softmax_scale, wsb + pd.off_o, false, lse ? reinterpret_cast<float *>(wsb + pd.off_lse) : nullptr,
                       ws, pd.inner, stream, true);
        if (st != CSA2_OK) return st;
        const int64_t pieces_out = (int64_t)nq * h * (CSA2_D * 2 / 16);
        launch(k_unpad_heads, dim3((unsigned)((pieces_out + 255) / 256)), dim3(256), 0, stream,
               reinterpret_cast<const uint4 *>(wsb + pd.off_o), reinterpret_cast<const float *>(wsb + pd.off_lse), h, nq,
               static_cast<uint4 *>(o), lse);
        return check_launch();
    }
    const AttnPlan P = plan_attn_nvfp4(nq, k, has_swa ? w_max : 0, num_sms());
    const AttnLayout L = attn_layout(nq, h, P, nvfp4);
    if (L.total > 0 && (!ws || ws_bytes < L.total || !aligned(ws, 256))) return CSA2_ERR_WORKSPACE;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;

    AttnParams ap{};
    ap.q = static_cast<const uint16_t *>(q_bf16);
    ap.kv = *kv;
    ap.topk = topk;
    ap.swa = swa;
    ap.swa_seq_stride = swa_seq_stride;
    ap.swa_begin = has_swa ? swa_begin : nullptr;
    ap.swa_end = has_swa ? swa_end : nullptr;
    ap.o = out_f32 ? nullptr : static_cast<uint16_t *>(o);
    ap.lse = lse;
    const bool parts = P.splits > 1;
    ap.o_part = parts ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + L.off_o) : nullptr;
    ap.lse_part = parts ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + L.off_lse) : nullptr;
    if (nvfp4) {
        ap.q4 = static_cast<uint8_t *>(ws) + L.off_q4;
        ap.q4s = static_cast<uint8_t *>(ws) + L.off_q4s;
    }
    ap.out_f32 = out_f32 ? 1 : 0;
    if (out_f32 && P.splits == 1) {
        // one split: the kernel's f32 partial is the result
        ap.o_part = static_cast<float *>(o);
        ap.lse_part = lse;
    }
    ap.scale_log2 = softmax_scale * 1.4426950408889634f;
    ap.k = k;
    ap.q_per_seq = q_per_seq;
    ap.n_splits = P.splits;
    ap.tiles_per_split = P.tiles_per_split;
    ap.e_splits = P.e_splits;
    ap.e_tiles = P.e_tiles;
    ap.tps_e = P.tps_e;
    const dim3 grid((unsigned)P.splits, (unsigned)nq);
    auto go = [&](auto kernel, size_t smem) { launch(kernel, grid, dim3(kAttnThreads), smem, stream, ap); };
    if (nvfp4) {
        if (!smem_attr(k_sparse_attn<64, true>, AttnCfg<64, true>::kSmem)) return CSA2_ERR_CUDA;
        // q -> NVFP4 once per call (codes and scales into the workspace)
        const int32_t n_blocks = nq * h * (CSA2_D / CSA2_BLOCK);
        launch(k_quant_rows_nvfp4, dim3((unsigned)((n_blocks + kQuantThreads - 1) / kQuantThreads)),
               dim3(kQuantThreads), 0, stream, static_cast<const uint16_t *>(q_bf16), n_blocks, ap.q4, ap.q4s);
        if ((st = check_launch()) != CSA2_OK) return st;
        go(k_sparse_attn<64, true>, AttnCfg<64, true>::kSmem);
    }
    if ((st = check_launch()) != CSA2_OK) return st;
    if (P.splits > 1) {
        CombineArgs ca{};
        ca.o_part = ap.o_part;
        ca.lse_part = ap.lse_part;
        ca.q_stride = (int64_t)P.splits * h * CSA2_D;
        ca.s_stride = (int64_t)h * CSA2_D;
        ca.lq_stride = (int64_t)P.splits * h;
        ca.ls_stride = h;
        ca.o = o;
        ca.lse = lse;
        ca.n_splits = P.splits;
        if (out_f32)
            launch_combine<true>(h, nq, ca, stream);
        else
            launch_combine<false>(h, nq, ca, stream);
        st = check_launch();
    }
    return st;
}

}  // namespace

extern "C" {

csa2_status csa2_sparse_attn_decode(const void *q_bf16, int32_t nq, int32_t q_per_seq, int32_t h,
                                    const csa2_kv_desc *kv, const int32_t *topk, int32_t k, const uint8_t *swa,
                                    int64_t swa_seq_stride, const int32_t *swa_begin, const int32_t *swa_end,
                                    int32_t w_max, float softmax_scale, void *o_bf16, float *lse, void *ws,
                                    size_t ws_bytes, cudaStream_t stream) {
    return attn_impl(q_bf16, nq, q_per_seq, h, kv, topk, k, swa, swa_seq_stride, swa_begin, swa_end, w_max,
                     softmax_scale, o_bf16, false, lse, ws, ws_bytes, stream);
}

csa2_status csa2_sparse_attn_partial(const void *q_bf16, int32_t nq, int32_t q_per_seq, int32_t h,
                                     const csa2_kv_desc *kv, const int32_t *topk, int32_t k, const uint8_t *swa,
                                     int64_t swa_seq_stride, const int32_t *swa_begin, const int32_t *swa_end,
                                     int32_t w_max, float softmax_scale, float *o_f32, float *lse, void *ws,
                                     size_t ws_bytes, cudaStream_t stream) {
    return attn_impl(q_bf16, nq, q_per_seq, h, kv, topk, k, swa, swa_seq_stride, swa_begin, swa_end, w_max,
                     softmax_scale, o_f32, true, lse, ws, ws_bytes, stream);
}

size_t csa2_sparse_attn_nvfp4_workspace_size(int32_t nq, int32_t h, int32_t k, int32_t w_max) {
    if (nq <= 0 || k < 0 || (h != 16 && h != 32 && h != 64)) return 0;
    if (h != 64) return nvfp4_pad_layout(nq, k, w_max).total;
    const AttnPlan P = plan_attn_nvfp4(nq, k, w_max, num_sms());
    return attn_layout(nq, h, P, true).total;
}

csa2_status csa2_sparse_attn_decode_nvfp4(const void *q_bf16, int32_t nq, int32_t q_per_seq, int32_t h,
                                          const csa2_kv_desc *kv, const int32_t *topk, int32_t k, const uint8_t *swa,
                                          int64_t swa_seq_stride, const int32_t *swa_begin, const int32_t *swa_end,
                                          int32_t w_max, float softmax_scale, void *o_bf16, float *lse, void *ws,
                                          size_t ws_bytes, cudaStream_t stream) {
    return attn_impl(q_bf16, nq, q_per_seq, h, kv, topk, k, swa, swa_seq_stride, swa_begin, swa_end, w_max,
                     softmax_scale, o_bf16, false, lse, ws, ws_bytes, stream, true);
}

csa2_status csa2_attn_merge(const float *o_parts, const float *lse_parts, int32_t g, int32_t nq, int32_t h,
                            void *o_bf16, float *lse, cudaStream_t stream) {
    if (h != 16 && h != 32 && h != 64) return CSA2_ERR_UNSUPPORTED;
    if (g < 1 || nq <= 0 || nq > 65535) return CSA2_ERR_INVALID_ARG;
    if (!o_parts || !lse_parts || !o_bf16 || !aligned(o_parts, 16) || !aligned(lse_parts, 4) ||
        !aligned(o_bf16, 16) || (lse && !aligned(lse, 4)))
        return CSA2_ERR_INVALID_ARG;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    CombineArgs ca{};
    ca.o_part = o_parts;
    ca.lse_part = lse_parts;
    ca.q_stride = (int64_t)h * CSA2_D;
    ca.s_stride = (int64_t)nq * h * CSA2_D;
    ca.lq_stride = h;
    ca.ls_stride = (int64_t)nq * h;
    ca.o = o_bf16;
    ca.lse = lse;
    ca.n_splits = g;
    launch_combine<false>(h, nq, ca, stream);
    return check_launch();
}

csa2_status csa2_score_ids(const uint8_t *qidx, const float *w, int32_t nq, int32_t q_per_seq, int32_t hi,
                           const int32_t *ids, int32_t m, const csa2_kv_desc *kv, int32_t id_offset,
                           unsigned long long *keys, cudaStream_t stream) {
    csa2_status st = check_kv(kv, true);
    if (st != CSA2_OK) return st;
    if (nq <= 0 || nq > 65535 || q_per_seq <= 0 || (nq + q_per_seq - 1) / q_per_seq > kv->batch)
        return CSA2_ERR_INVALID_ARG;
    if (hi < 1 || hi > kScanN) return CSA2_ERR_UNSUPPORTED;
    if (m < 1 || id_offset < 0) return CSA2_ERR_INVALID_ARG;
    if (!qidx || !w || !ids || !keys || !aligned(qidx, 16) || !aligned(w, 4) || !aligned(ids, 4) ||
        !aligned(keys, 8))
        return CSA2_ERR_INVALID_ARG;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    ReindexParams rp{};
    rp.qidx = qidx;
    rp.w = w;
    rp.pool = ids;
    rp.kv = *kv;
    rp.k64 = keys;
    rp.p = m;
    rp.hi = hi;
    rp.q_per_seq = q_per_seq;
    rp.id_offset = id_offset;
    const dim3 grid((unsigned)((m + kReindexScoreThreads - 1) / kReindexScoreThreads), (unsigned)nq);
    if (kv->di == 64)
        launch(k_reindex_score<64>, grid, dim3(kReindexScoreThreads), 0, stream, rp);
    else
        launch(k_reindex_score<128>, grid, dim3(kReindexScoreThreads), 0, stream, rp);
    return check_launch();
}

csa2_status csa2_select_keys(const unsigned long long *keys, int32_t nq, int32_t m, int32_t k, int32_t *ids,
                             cudaStream_t stream) {
    if (nq <= 0 || nq > 65535 || m < 1 || k < 1) return CSA2_ERR_INVALID_ARG;
    if (m > kSelectKeysMax) return CSA2_ERR_UNSUPPORTED;
    if (!keys || !ids || !aligned(keys, 8) || !aligned(ids, 4)) return CSA2_ERR_INVALID_ARG;
    if (!init_small_kernels()) return CSA2_ERR_CUDA;
    ReindexParams rp{};
    rp.k64 = const_cast<unsigned long long *>(keys);
    rp.topk = ids;
    rp.p = m;
    rp.k = k;
    const size_t base = 2048 * 4 + (kReindexSelectThreads / 32 + 8) * 4;
    const size_t smem = base + (size_t)m * 8;
    if (!smem_attr(k_reindex_select<false>, (size_t)max_smem_optin())) return CSA2_ERR_CUDA;
    if (smem <= (size_t)max_smem_optin())
        launch(k_reindex_select<false>, dim3(nq), dim3(kReindexSelectThreads), smem, stream, rp);
    else  // keys larger than shared memory: every pass reads them from L2
        launch(k_reindex_select<true>, dim3(nq), dim3(kReindexSelectThreads), base, stream, rp);
    return check_launch();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention without a caller workspace, for callers that cannot
// allocate device memory. The split partials go to a fixed array in device
// global memory, one copy per device (the module is loaded per device). Its
// address is looked up once per device, with that device current, and then
// handed to the regular attention path as its workspace, so the kernels and
// their arithmetic are exactly those of csa2_sparse_attn_decode. Each call
// writes every partial before the combine reads it, so the array needs no
// clearing. Calls on one device share the array: overlapping calls race.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) uint8_t g_attn_scratch[CSA2_ATTN_STATIC_SCRATCH_BYTES];

constexpr int kMaxScratchDevices = 64;
std::mutex g_attn_scratch_mu;
void *g_attn_scratch_ptr[kMaxScratchDevices] = {};
CUcontext g_attn_scratch_ctx[kMaxScratchDevices] = {};

// cuCtxGetCurrent, fetched through the runtime like cuTensorMapEncodeTiled.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of this device's copy of g_attn_scratch, or null on error.
// The address belongs to the context the module was loaded into: it is looked
// up again whenever the device's current context is not the one it was
// looked up in (after cudaDeviceReset, for example, the module is loaded
// anew and the old address is gone).
void *attn_scratch_of_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) {
        cudaGetLastError();
        return nullptr;
    }
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (!get_ctx) return nullptr;
    CUcontext ctx = nullptr;  // stays null while no context is current on this thread
    if (get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
    std::lock_guard<std::mutex> lock(g_attn_scratch_mu);
    if (!g_attn_scratch_ptr[dev] || ctx == nullptr || g_attn_scratch_ctx[dev] != ctx) {
        void *ptr = nullptr;
        // with the device current; makes the runtime's context current if none was
        if (cudaGetSymbolAddress(&ptr, g_attn_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
        g_attn_scratch_ptr[dev] = ptr;
        g_attn_scratch_ctx[dev] = ctx;
    }
    return g_attn_scratch_ptr[dev];
}

}  // namespace

extern "C" csa2_status csa2_sparse_attn_decode_static(const void *q_bf16, int32_t nq, int32_t q_per_seq, int32_t h,
                                                      const csa2_kv_desc *kv, const int32_t *topk, int32_t k,
                                                      const uint8_t *swa, int64_t swa_seq_stride,
                                                      const int32_t *swa_begin, const int32_t *swa_end, int32_t w_max,
                                                      float softmax_scale, void *o_bf16, float *lse,
                                                      cudaStream_t stream) {
    // the same workspace the regular path would ask for (no window: w_max 0)
    const size_t need = csa2_sparse_attn_workspace_size(nq, h, k, swa_begin ? w_max : 0);
    if (need > CSA2_ATTN_STATIC_SCRATCH_BYTES) return CSA2_ERR_WORKSPACE;
    void *scratch = attn_scratch_of_current_device();
    if (!scratch) return CSA2_ERR_CUDA;
    return csa2_sparse_attn_decode(q_bf16, nq, q_per_seq, h, kv, topk, k, swa, swa_seq_stride, swa_begin, swa_end,
                                   w_max, softmax_scale, o_bf16, lse, scratch, CSA2_ATTN_STATIC_SCRATCH_BYTES,
                                   stream);
}
