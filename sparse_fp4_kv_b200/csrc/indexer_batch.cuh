// indexer_batch.cuh -- Full-mode indexer for many queries of one sequence
// (the chunked-prefill workload: hundreds of causal queries over one cache),
// with the key tiles shared by a group of queries in each tensor-core
// product.
//
// Same method as indexer.cuh (DeepSeek V4.1-Flash Cuts KV Cache by 437x,
// paragraph "CSA2 assigns each layer one of three static operating modes":
// Full mode scores the whole visible context and keeps its Top-K):
//     score(t) = sum_h w_h * max(0, <q_h, kidx_t>),
// order score descending, entry id ascending on ties; output ids ascending.
//
// The queries are taken in groups of QG (16 with up to 4 indexer heads, 8
// with up to 8; all of one sequence). One
// product per tile of 128 key rows scores every entry of the tile for every
// query of the group: B holds the group's heads (kEpr copies side by side
// as in the single-query scan, so that a 128-byte key row can hold two
// 64-byte entries), N = kEpr * QG * HP = 128 / (DI / 64). The selection runs in
// two scans of the keys plus two small per-query kernels:
//   1. k_batch_scan<0>: the score keys' top 11 bits counted per query
//      (histograms in shared memory, added to a global histogram);
//   2. k_batch_thresh: per query, the bin b0 holding its k-th largest key and
//      how many keys of b0 are still needed;
//   3. k_batch_scan<1>: the scores again (the same products, so the same
//      keys): entries above b0 go to the query's "sure" list, entries in b0
//      to its candidate list as unique 64-bit keys (score key << 32 | ~id);
//      every CTA fills its own part of each list (shared-memory counters)
//      and records how many it wrote;
//   4. k_batch_final: the needed number of largest candidates by an exact
//      radix select, merged with the sure ids and sorted ascending.
#pragma once

#include "indexer.cuh"

namespace csa2 {

constexpr int kBatchBins = 2048;   // digit 0: the key's top 11 bits
constexpr int kBatchShift = 21;
constexpr int kBatchEpiWarps = 16;  // 4 per TMEM lane quarter
constexpr int kBatchThreads = 64 + kBatchEpiWarps * 32;
constexpr int kBatchFinalThreads = 1024;
constexpr int kBatchMaxK = 8192;   // ids staged and sorted in shared memory
constexpr int kSampleStride = 32;  // the sampled threshold path reads every 32nd tile first
constexpr uint32_t kBatchAll = 0xFFFFFFFFu;  // b0 marker: every visible entry is taken

struct BatchParams {
    const uint8_t *qidx;  // [nq][hi][DI] E4M3
    const float *w;       // [nq][hi]
    const int32_t *q_limit;
    csa2_kv_desc kv;
    uint32_t *hist;             // [nq][kBatchBins]
    uint32_t *state;            // b0, rem of query qi at state[qi * state_stride + state_off + 0 / 1]
    int32_t state_stride, state_off;
    int32_t *sure;              // [nq][nchunks][sure_stride]: ids above b0 found by each CTA (part)
    unsigned long long *cand;   // [nq][nchunks][chunk]: keys in b0 found by each part
    uint32_t *cnt;              // [nq][nchunks][2]: how many of each
    int32_t *topk;              // [nq][k]: the selected ids, ascending, -1 padded
    int64_t chunk;              // entries per part
    int32_t nchunks;            // parts per query (gridDim.x of the collecting kernel)
    int32_t sure_stride;        // >= min(k, chunk): a part holds fewer than k sure ids
    uint32_t *hist1;            // [nq][2048] digit-1 histogram of the candidates, or null
    int32_t shift1;             // digit 1 = bits shift1 .. shift1 + 10 of the score key
    int32_t parts_sorted;       // every part's lists are in ascending id order
    // sampled threshold path
    uint32_t *samples;          // [nq][sample_stride]: score keys of every tile_stride-th tile (0: not visible)
    int64_t sample_stride;
    int32_t tile_stride;
    int32_t sample_rank;        // the threshold is the sample_rank-th largest sampled key
    uint32_t *redo;             // [nq]: 1 where the sampled path could not settle the query, or null
    int32_t redo_mark;          // final: mark (instead of writing) queries with too few candidates
    int32_t k, q_per_seq, hi, hi_pad, nq, box_rows;
};

template <int DI>
struct BatchGeom {
    static constexpr int kEpr = 128 / DI;   // entries per 128-byte key row
    static constexpr int kTile = 128 * kEpr;
    static constexpr int kStageBytes = 128 * 128;
};

// Queries per group for HP padded heads (N = kEpr * QG * HP stays 64 or 128).
__host__ __device__ constexpr int batch_qg(int hp) { return hp == 4 ? 16 : 8; }

// Queries of group gq: [gq * QG, min(nq, (gq + 1) * QG)); the largest visible
// limit among them bounds the group's scan.
template <int QG>
__device__ __forceinline__ int64_t group_limit(const BatchParams &p, int32_t gq, int32_t *lim /*[QG]*/) {
    int64_t mx = 0;
    for (int j = 0; j < QG; ++j) {
        const int32_t qi = gq * QG + j;
        const int64_t l = qi < p.nq ? query_limit(p.q_limit, p.kv, qi, p.q_per_seq) : 0;
        if (lim) lim[j] = (int32_t)min(l, (int64_t)INT32_MAX);
        mx = max(mx, l);
    }
    return mx;
}

// HP: indexer heads padded to 4 or 8.
template <int DI, int HP, int PASS>
struct BatchCfg {
    using G = BatchGeom<DI>;
    static constexpr int QG = batch_qg(HP);
    static constexpr int N = G::kEpr * QG * HP;
    static constexpr int kStages = PASS == 0 || PASS == 2 ? 4 : 8;
    // TMEM accumulators: the products run up to three tiles ahead (two for the
    // sample pass, two of whose CTAs can share an SM)
    static constexpr int kAcc = PASS == 2 ? 2 : 4;
    static constexpr uint32_t kTmemCols = kAcc * N <= 128 ? 128u : (kAcc * N <= 256 ? 256u : 512u);
    static constexpr size_t kSmem = 1024 + (size_t)kStages * G::kStageBytes + (size_t)N * 128 +
                                    (PASS == 0 ? (size_t)QG * kBatchBins * 4 : 0) + 16 * 16 * 4 + 16 * 4 * 4 +
                                    (size_t)kMaxScanPages * 4 + 256;
};

template <int DI, int HP, int PASS>
__global__ void __launch_bounds__(kBatchThreads, 1)
    k_batch_scan(const __grid_constant__ CUtensorMap tm, BatchParams p) {
    using G = BatchGeom<DI>;
    using Cfg = BatchCfg<DI, HP, PASS>;
    static_assert(HP == 4 || HP == 8, "heads padded to 4 or 8");
    constexpr int QG = Cfg::QG, N = Cfg::N, kStages = Cfg::kStages;
    constexpr uint32_t tcols = Cfg::kTmemCols;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = base;
    uint8_t *btile = stages + kStages * G::kStageBytes;  // N rows x 128 B
    uint32_t *hist = reinterpret_cast<uint32_t *>(btile + N * 128);          // PASS 0: [QG][bins]
    float *wq = reinterpret_cast<float *>(hist + (PASS == 0 ? QG * kBatchBins : 0));  // [16][16]
    int32_t *lim = reinterpret_cast<int32_t *>(wq + 16 * 16);                 // [16]
    uint32_t *b0s = reinterpret_cast<uint32_t *>(lim + 16);                   // [16] (PASS 1)
    uint32_t *lcnt = b0s + 16;                                                // [16][2] (PASS 1)
    int32_t *ptab = reinterpret_cast<int32_t *>(lcnt + 32);                   // [kMaxScanPages]
    uint64_t *full_b = reinterpret_cast<uint64_t *>(ptab + kMaxScanPages);
    uint64_t *empty_b = full_b + kStages;
    uint64_t *tfull = empty_b + kStages;
    uint64_t *tempty = tfull + Cfg::kAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + Cfg::kAcc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t gq = blockIdx.y;
    const int32_t q0 = gq * QG;
    const int32_t b = q0 / p.q_per_seq;

    pdl_trigger();
    if (PASS == 0)
        for (int i = tid; i < QG * kBatchBins; i += kBatchThreads) hist[i] = 0u;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
        }
        for (int a = 0; a < Cfg::kAcc; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], kBatchEpiWarps);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tcols);
        tmem_relinquish();
    }
    pdl_wait();
    if (tid == 0) group_limit<QG>(p, gq, lim);
    if (p.redo != nullptr && tid < QG) {
        // fallback run of the exact passes: only the queries the sampled path
        // could not settle are scanned (the others look empty)
        if (q0 + tid >= p.nq || __ldcg(p.redo + q0 + tid) == 0u) lim[tid] = 0;
    }
    __syncthreads();
    int64_t gl = 0;
    for (int j = 0; j < QG; ++j) gl = max(gl, (int64_t)lim[j]);
    // PASS 2 takes every tile_stride-th tile of its range (a sample)
    const int tstride = PASS == 2 ? p.tile_stride : 1;
    const int64_t start = (int64_t)blockIdx.x * p.chunk;
    const int64_t n_loc = max((int64_t)0, min(gl, start + p.chunk) - start);
    const int ntiles = (int)((n_loc + (int64_t)tstride * G::kTile - 1) / ((int64_t)tstride * G::kTile));
    // B: rows (u, j, h) = u * QG * HP + j * HP + h hold query j's head h
    // in the 64-byte half u of a 128-byte row (DI = 64), zero elsewhere
    for (int i = tid; i < N * 8; i += kBatchThreads) {
        const int r = i / 8, c = i % 8;
        const int u = r / (QG * HP), jh = r % (QG * HP);
        const int j = jh / HP, h = jh % HP;
        const int32_t qi = q0 + j;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (qi < p.nq && h < p.hi) {
            const uint8_t *q = p.qidx + ((int64_t)qi * p.hi + h) * DI;
            if (DI == 128)
                v = *reinterpret_cast<const uint4 *>(q + c * 16);
            else if (c / 4 == u)
                v = *reinterpret_cast<const uint4 *>(q + (c % 4) * 16);
        }
        *reinterpret_cast<uint4 *>(btile + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) = v;
    }
    for (int i = tid; i < QG * 16; i += kBatchThreads) {
        const int j = i / 16, h = i % 16;
        const int32_t qi = q0 + j;
        wq[i] = (qi < p.nq && h < p.hi) ? p.w[(int64_t)qi * p.hi + h] : 0.0f;
    }
    if ((PASS == 1 || PASS == 3) && tid < QG) {
        b0s[tid] = q0 + tid < p.nq ? __ldcg(p.state + (int64_t)(q0 + tid) * p.state_stride + p.state_off) : 0u;
        lcnt[2 * tid] = lcnt[2 * tid + 1] = 0u;
    }
    if (ntiles > 0 && PASS != 2) stage_pages(p.kv, b, start, n_loc, ptab, kBatchThreads);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        scan_tma_loop<DI>(p.kv, ptab, start, gl, ntiles, kStages, p.box_rows, stages, &tm, full_b, empty_b, tstride,
                          p.kv.page_table + (int64_t)b * p.kv.max_pages);
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_e4m3_f32(128, N);
            const uint32_t qaddr = smem_u32(btile);
            int s = 0;
            uint32_t phase = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int a = i % Cfg::kAcc;
                if (!mbar_wait(&tempty[a], ((i / Cfg::kAcc) & 1) ^ 1)) break;
                if (!mbar_wait(&full_b[s], phase)) break;
                tc_fence_after();
                const uint32_t aaddr = smem_u32(stages + (size_t)s * G::kStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_e4m3(tmem + (uint32_t)(a * N), make_sdesc(aaddr + kk * 32, 16, 1024, kSw128),
                             make_sdesc(qaddr + kk * 32, 16, 1024, kSw128), idesc, kk > 0 ? 1u : 0u);
                tc_commit(&empty_b[s]);
                tc_commit(&tfull[a]);
                if (++s == kStages) {
                    s = 0;
                    phase ^= 1u;
                }
            }
        }
        __syncwarp();
    } else {
        // epilogue: TMEM lane quarter (warp & 3), queries [sub * QW, sub * QW + QW)
        constexpr int QW = QG / 4;  // queries of one warp: QW * HP = 16 columns per half row
        const int ew = warp - 2;
        const int quarter = warp & 3, sub = ew >> 2;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        // this warp's queries: head weights, visible limits (relative to the
        // CTA's range) and thresholds in registers for the whole loop
        float wr[QW][HP];
        int32_t limr[QW];
        uint32_t b0r[QW];
#pragma unroll
        for (int jj = 0; jj < QW; ++jj) {
            const int j = sub * QW + jj;
#pragma unroll
            for (int h = 0; h < HP; ++h) wr[jj][h] = wq[j * 16 + h];
            limr[jj] = (int32_t)max((int64_t)-1, min((int64_t)lim[j] - start, (int64_t)INT32_MAX));
            b0r[jj] = PASS == 1 || PASS == 3 ? b0s[j] : 0u;
        }
        for (int i = 0; i < ntiles; ++i) {
            const int a = i % Cfg::kAcc;
            const bool got = mbar_wait(&tfull[a], (i / Cfg::kAcc) & 1);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            tc_fence_after();
            // both halves' 16 columns of this warp's queries in flight at once
            uint32_t rr[G::kEpr][16];
#pragma unroll
            for (int u = 0; u < G::kEpr; ++u)
                tmem_ld16(lane_base + (uint32_t)(a * N + u * QG * HP + sub * QW * HP), rr[u]);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < G::kEpr; ++u) {
                const uint32_t(&r)[16] = rr[u];
                const int64_t tile0 = start + (int64_t)i * tstride * G::kTile;
                const int64_t t = tile0 + (int64_t)G::kEpr * (quarter * 32 + lane) + u;
                const int32_t trel = (int32_t)(t - start);  // < chunk
#pragma unroll
                for (int jj = 0; jj < QW; ++jj) {
                    const int j = sub * QW + jj;
                    float sc = 0.0f;
#pragma unroll
                    for (int h = 0; h < HP; ++h) sc = fmaf(wr[jj][h], fmaxf(__uint_as_float(r[jj * HP + h]), 0.0f), sc);
                    const uint32_t key = score_key(sc + 0.0f);
                    const bool vis = trel < limr[jj];
                    const int32_t qi = q0 + j;
                    if (PASS == 0) {
                        if (vis) atomicAdd(&hist[j * kBatchBins + (key >> kBatchShift)], 1u);
                    } else if (PASS == 2) {
                        // sample slot: sample tile (tile0 / kTile / tstride), entry in tile;
                        // 0 (no score has it) where the entry is not visible
                        if (qi < p.nq) {
                            const int64_t js = tile0 / ((int64_t)tstride * G::kTile);
                            p.samples[(int64_t)qi * p.sample_stride + js * G::kTile + (t - tile0)] = vis ? key : 0u;
                        }
                    } else if (PASS == 3) {
                        const bool cand = vis && key >= b0r[jj];
                        const uint32_t mc = __ballot_sync(0xFFFFFFFFu, cand);
                        if (mc) {
                            const int64_t part = (int64_t)qi * p.nchunks + blockIdx.x;
                            uint32_t base0 = 0;
                            if (lane == 0) base0 = atomicAdd(&lcnt[2 * j + 1], (uint32_t)__popc(mc));
                            base0 = __shfl_sync(0xFFFFFFFFu, base0, 0);
                            if (cand) {
                                const uint32_t at = base0 + __popc(mc & ((1u << lane) - 1u));
                                if ((int64_t)at < p.chunk)
                                    p.cand[part * p.chunk + at] =
                                        ((unsigned long long)key << 32) | (unsigned long long)(~(uint32_t)t);
                                else
                                    set_error(CSA2_DEVERR_SELECT);
                            }
                        }
                    } else {
                        const uint32_t b0 = b0r[jj];
                        const uint32_t d = key >> kBatchShift;
                        const bool sure = vis && (b0 == kBatchAll || d > b0);
                        const bool cand = vis && b0 != kBatchAll && d == b0;
                        const uint32_t ms = __ballot_sync(0xFFFFFFFFu, sure);
                        const uint32_t mc = __ballot_sync(0xFFFFFFFFu, cand);
                        const uint32_t lt = (1u << lane) - 1u;
                        const int64_t part = (int64_t)qi * p.nchunks + blockIdx.x;  // this CTA's part
                        if (ms) {
                            uint32_t base0 = 0;
                            if (lane == 0) base0 = atomicAdd(&lcnt[2 * j], (uint32_t)__popc(ms));
                            base0 = __shfl_sync(0xFFFFFFFFu, base0, 0);
                            if (sure) {
                                const uint32_t at = base0 + __popc(ms & lt);
                                if (at < (uint32_t)p.sure_stride)
                                    p.sure[part * p.sure_stride + at] = (int32_t)t;
                                else
                                    set_error(CSA2_DEVERR_SELECT);
                            }
                        }
                        if (mc) {
                            uint32_t base0 = 0;
                            if (lane == 0) base0 = atomicAdd(&lcnt[2 * j + 1], (uint32_t)__popc(mc));
                            base0 = __shfl_sync(0xFFFFFFFFu, base0, 0);
                            if (cand) {
                                const uint32_t at = base0 + __popc(mc & lt);
                                if ((int64_t)at < p.chunk)
                                    p.cand[part * p.chunk + at] =
                                        ((unsigned long long)key << 32) | (unsigned long long)(~(uint32_t)t);
                                else
                                    set_error(CSA2_DEVERR_SELECT);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[a]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
    if ((PASS == 1 || PASS == 3) && tid < QG && q0 + tid < p.nq &&
        (p.redo == nullptr || __ldcg(p.redo + q0 + tid) != 0u)) {
        uint32_t *c = p.cnt + ((int64_t)(q0 + tid) * p.nchunks + blockIdx.x) * 2;
        c[0] = min(lcnt[2 * tid], (uint32_t)p.sure_stride);
        c[1] = lcnt[2 * tid + 1];
    }
    if (PASS == 0) {
        for (int i = tid; i < QG * kBatchBins; i += kBatchThreads) {
            const int j = i / kBatchBins;
            const uint32_t v = hist[i];
            if (v && q0 + j < p.nq) atomicAdd(p.hist + (int64_t)(q0 + j) * kBatchBins + (i % kBatchBins), v);
        }
    }
}

// Per query: the digit-0 bin of its k-th largest key, how many keys of that
// bin are needed, and zeroed list counts (or "take all" when k covers every
// visible entry).
constexpr int kBatchThreshThreads = 256;
__global__ void __launch_bounds__(kBatchThreshThreads) k_batch_thresh(BatchParams p) {
    __shared__ uint32_t scratch[kBatchThreshThreads / 32 + 4];
    pdl_trigger();
    pdl_wait();
    const int32_t qi = blockIdx.x;
    if (p.redo != nullptr && __ldcg(p.redo + qi) == 0u) return;  // settled by the sampled path
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    uint32_t bin = kBatchAll, rem = 0;
    if ((int64_t)p.k < limit)
        find_rank_bin<kBatchThreshThreads, kBatchBins / kBatchThreshThreads, true>(
            p.hist + (int64_t)qi * kBatchBins, kBatchBins, (uint32_t)p.k, scratch, bin, rem);
    if (threadIdx.x == 0) {
        uint32_t *st = p.state + (int64_t)qi * p.state_stride + p.state_off;
        st[0] = bin;
        st[1] = rem;
    }
}

// Sampled threshold path, per query: the sample_rank-th largest of the keys
// the sampling pass recorded (every tile_stride-th tile of the query's
// range), by an exact radix select in three digits (11, 11, 10 bits) over
// those keys (read through L2 in every pass). Every visible entry whose key
// is at least that threshold becomes a candidate in the collecting pass, so
// about sample_rank * tile_stride entries do; with fewer sampled keys than
// sample_rank the threshold is 0 and every visible entry is a candidate.
// state: [0] the threshold, [1] k.
constexpr int kSthreshThreads = 512;
__global__ void __launch_bounds__(kSthreshThreads) k_batch_sthresh(BatchParams p) {
    constexpr int NT = kSthreshThreads;
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t scratch[NT / 32 + 4];
    pdl_trigger();
    pdl_wait();
    const int32_t qi = blockIdx.x;
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    const int64_t tile = 128 * (128 / p.kv.di);
    const int64_t span = (int64_t)p.tile_stride * tile;
    const int64_t ns = min((limit + span - 1) / span * tile, p.sample_stride);
    const uint32_t *src = p.samples + (int64_t)qi * p.sample_stride;
    uint32_t prefix = 0u, pmask = 0u, rem = (uint32_t)p.sample_rank;
    bool enough = true;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int d = 0; d < 3 && enough; ++d) {
        const int sh = shifts[d], nb = 1 << widths[d];
        for (int i = threadIdx.x; i < 2048; i += NT) hist[i] = 0u;
        __syncthreads();
        for (int64_t i0 = threadIdx.x; i0 < ns; i0 += 4 * NT) {
            uint32_t v[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) v[r] = i0 + r * NT < ns ? __ldcg(src + i0 + r * NT) : 0u;
#pragma unroll
            for (int r = 0; r < 4; ++r)
                if (v[r] != 0u && (v[r] & pmask) == prefix) atomicAdd(&hist[(v[r] >> sh) & (uint32_t)(nb - 1)], 1u);
        }
        __syncthreads();
        if (d == 0) {
            uint32_t c = 0;
            for (int i = threadIdx.x; i < nb; i += NT) c += hist[i];
            uint32_t total;
            block_excl_scan<NT>(c, scratch, &total);
            enough = total >= rem;
            if (!enough) break;
        }
        uint32_t bin, inbin;
        find_rank_bin<NT, 2048 / NT, false>(hist, nb, rem, scratch, bin, inbin);
        prefix |= bin << sh;
        pmask |= (uint32_t)(nb - 1) << sh;
        rem = inbin;
    }
    if (threadIdx.x == 0) {
        uint32_t *st = p.state + (int64_t)qi * p.state_stride + p.state_off;
        st[0] = enough ? prefix : 0u;
        st[1] = (uint32_t)p.k;
    }
}

// Per query: the rem largest of its candidate keys (unique 64-bit keys, in
// the parts the collecting CTAs wrote; copied into shared memory when they
// fit, else re-read from those parts through L2 in every radix pass), merged
// with its sure ids in ascending order, padded with -1. Parts are read with
// flattened indices (a binary search over the parts' offsets), so that every
// thread's loads are in flight at once whatever the number of parts. With a
// digit-1 histogram of the candidates (p.hist1), the radix select starts
// below digit 1. With p.parts_sorted, every part lists its ids in ascending
// order and the parts cover ascending id ranges, so the sure ids and the
// taken candidates are two sorted runs that are merged; otherwise they are
// sorted (bitonic) in shared memory.
constexpr int kBatchMaxChunks = 256;

// Largest part c in [0, nch) whose exclusive offset poff[2c + w] is <= j:
// the part holding flattened item j.
__device__ __forceinline__ int find_part(const uint32_t *poff, int nch, int w, uint32_t j) {
    int lo = 0, hi = nch - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (poff[2 * mid + w] <= j)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Number of elements of the ascending run a[0..n) below x.
__device__ __forceinline__ uint32_t count_below(const int32_t *a, uint32_t n, int32_t x) {
    uint32_t lo = 0, hi = n;
    while (lo < hi) {
        const uint32_t mid = (lo + hi) >> 1;
        if (a[mid] < x)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kBatchFinalThreads, 1) k_batch_final(BatchParams p, int32_t smem_keys) {
    constexpr int NT = kBatchFinalThreads;
    extern __shared__ uint8_t smem_raw[];
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem_raw);              // [2048]
    uint32_t *scratch = hist + 2048;                                      // [NT/32 + 8]
    uint32_t *pcnt = scratch + NT / 32 + 8;                               // [kBatchMaxChunks][2]
    uint32_t *poff = pcnt + 2 * kBatchMaxChunks;                          // [kBatchMaxChunks][2] exclusive prefixes
    int32_t *ids = reinterpret_cast<int32_t *>(poff + 2 * kBatchMaxChunks);  // [kBatchMaxK]: sure, then taken
    unsigned long long *k64 = reinterpret_cast<unsigned long long *>(ids + kBatchMaxK);  // [smem_keys]
    __shared__ unsigned long long and_acc, or_acc;
    __shared__ uint32_t tot[2];
    const int32_t qi = blockIdx.x;
    const int nch = min(p.nchunks, kBatchMaxChunks);
    pdl_trigger();
    if (p.redo != nullptr && !p.redo_mark) {
        pdl_wait();
        if (__ldcg(p.redo + qi) == 0u) return;  // settled by the sampled path
    }
    if (threadIdx.x == 0) {
        and_acc = ~0ull;
        or_acc = 0ull;
    }
    pdl_wait();
    for (int c = threadIdx.x; c < nch; c += NT) {
        // clamped to the parts' capacities: no read outside them whatever the counts say
        const uint32_t *cc = p.cnt + ((int64_t)qi * p.nchunks + c) * 2;
        pcnt[2 * c] = min(__ldcg(cc), (uint32_t)p.sure_stride);
        pcnt[2 * c + 1] = (uint32_t)min((int64_t)__ldcg(cc + 1), p.chunk);
    }
    __syncthreads();
    if (threadIdx.x < 2) {
        uint32_t acc = 0;
        for (int c = 0; c < nch; ++c) {
            poff[2 * c + threadIdx.x] = acc;
            acc += pcnt[2 * c + threadIdx.x];
        }
        tot[threadIdx.x] = acc;
    }
    __syncthreads();
    const uint32_t *stq = p.state + (int64_t)qi * p.state_stride + p.state_off;
    const uint32_t b0 = __ldcg(stq), need = __ldcg(stq + 1);
    const uint32_t n_sure = min(tot[0], (uint32_t)p.k);
    const uint32_t n_cand = tot[1];
    if (p.redo_mark) {
        // sampled path: fewer candidates than the query needs (the sample put
        // the threshold too high) -> left to the exact passes
        const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
        if ((int64_t)(n_sure + n_cand) < min((int64_t)p.k, limit) || p.redo_mark > 1) {
            if (threadIdx.x == 0) p.redo[qi] = 1u;
            return;
        }
    }
    const int64_t part0 = (int64_t)qi * p.nchunks;
    // the sure ids first, flattened over the parts
    for (uint32_t j0 = threadIdx.x; j0 < n_sure; j0 += 4 * NT) {
        int32_t v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint32_t j = j0 + r * NT;
            v[r] = 0;
            if (j < n_sure) {
                const int c = find_part(poff, nch, 0, j);
                v[r] = __ldcg(p.sure + (part0 + c) * p.sure_stride + (j - poff[2 * c]));
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
            if (j0 + r * NT < n_sure) ids[j0 + r * NT] = v[r];
    }
    // candidate j, flattened over the parts
    auto cand_at = [&](uint32_t j) -> unsigned long long {
        const int c = find_part(poff, nch, 1, j);
        return __ldcg(p.cand + (part0 + c) * p.chunk + (j - poff[2 * c + 1]));
    };
    uint32_t take = 0;
    const bool G = n_cand > (uint32_t)smem_keys;  // re-read the parts from L2 in every pass
    if (b0 != kBatchAll && need > 0 && n_cand > 0) {
        take = min(need, n_cand);
        // fn(key) over every candidate, each once, four loads in flight per thread
        auto each = [&](auto fn) {
            if (!G) {
                for (uint32_t j = threadIdx.x; j < n_cand; j += NT) fn(k64[j]);
            } else {
                for (uint32_t j0 = threadIdx.x; j0 < n_cand; j0 += 4 * NT) {
                    unsigned long long v[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) v[r] = j0 + r * NT < n_cand ? cand_at(j0 + r * NT) : 0ull;
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        if (j0 + r * NT < n_cand) fn(v[r]);
                }
            }
        };
        unsigned long long a_loc = ~0ull, o_loc = 0ull;
        for (uint32_t j0 = threadIdx.x; j0 < n_cand; j0 += 4 * NT) {
            unsigned long long v[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) v[r] = j0 + r * NT < n_cand ? cand_at(j0 + r * NT) : 0ull;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const uint32_t j = j0 + r * NT;
                if (j < n_cand) {
                    if (!G) k64[j] = v[r];
                    a_loc &= v[r];
                    o_loc |= v[r];
                }
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            a_loc &= __shfl_xor_sync(0xFFFFFFFFu, a_loc, o);
            o_loc |= __shfl_xor_sync(0xFFFFFFFFu, o_loc, o);
        }
        if ((threadIdx.x & 31) == 0) {
            atomicAnd(&and_acc, a_loc);
            atomicOr(&or_acc, o_loc);
        }
        __syncthreads();
        unsigned long long T = 0ull;  // take the keys >= T
        if (take < n_cand) {
            const unsigned long long diff = and_acc ^ or_acc;  // keys are unique: diff != 0
            int top = 63 - __clzll((long long)diff);
            unsigned long long prefix = top == 63 ? 0ull : (and_acc & ~((2ull << top) - 1ull));
            unsigned long long pmask = top == 63 ? 0ull : ~((2ull << top) - 1ull);
            uint32_t rem = take;
            bool done = false;
            if (p.hist1 != nullptr) {
                // digits 0 and 1 of the key's top word from the collecting pass's
                // histogram of the candidates' digit 1
                uint32_t b1, r1;
                find_rank_bin<NT, 2048 / NT, true>(p.hist1 + (int64_t)qi * 2048, 2048, take, scratch, b1, r1);
                const int lo = 32 + p.shift1;
                pmask = ~0ull << lo;
                prefix = (and_acc & pmask & ~(2047ull << lo)) | ((unsigned long long)b1 << lo);
                rem = r1;
                const unsigned long long below = diff & ((1ull << lo) - 1ull);
                if (below == 0ull)
                    done = true;
                else
                    top = 63 - __clzll((long long)below);
            }
            while (!done) {
                const int nbits = top + 1 < 11 ? top + 1 : 11;
                const int shift = top + 1 - nbits;
                const int nb = 1 << nbits;
                for (int i = threadIdx.x; i < 2048; i += NT) hist[i] = 0u;
                __syncthreads();
                each([&](unsigned long long v) {
                    if ((v & pmask) == prefix) atomicAdd(&hist[(uint32_t)(v >> shift) & (uint32_t)(nb - 1)], 1u);
                });
                __syncthreads();
                uint32_t bin, inbin;
                find_rank_bin<NT, 2048 / NT, false>(hist, nb, rem, scratch, bin, inbin);
                prefix |= (unsigned long long)bin << shift;
                pmask |= (unsigned long long)(nb - 1) << shift;
                rem = inbin;
                const bool all_taken = hist[bin] == rem;
                __syncthreads();
                if (all_taken || shift == 0) break;
                const unsigned long long below = diff & ((1ull << shift) - 1ull);
                if (below == 0ull) break;
                top = 63 - __clzll((long long)below);
            }
            T = prefix | (and_acc & ~diff & ~pmask);
        }
        // the taken candidates after the sure ids: in candidate order (each
        // thread a contiguous run) when the parts are sorted
        const uint32_t per = (n_cand + NT - 1) / NT;
        const uint32_t j0 = min(n_cand, threadIdx.x * per), j1 = min(n_cand, j0 + per);
        // fn(key) over candidates j0 .. j1-1 in order; from L2 eight loads at a
        // time, the part index walked forward
        auto run = [&](auto fn) {
            if (!G) {
                for (uint32_t j = j0; j < j1; ++j) fn(k64[j]);
                return;
            }
            int c = j0 < j1 ? find_part(poff, nch, 1, j0) : 0;
            for (uint32_t jb = j0; jb < j1; jb += 8) {
                unsigned long long v[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const uint32_t j = jb + r;
                    v[r] = 0ull;
                    if (j < j1) {
                        while (c + 1 < nch && poff[2 * (c + 1) + 1] <= j) ++c;
                        v[r] = __ldcg(p.cand + (part0 + c) * p.chunk + (j - poff[2 * c + 1]));
                    }
                }
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    if (jb + r < j1) fn(v[r]);
            }
        };
        uint32_t mine = 0;
        run([&](unsigned long long v) { mine += v >= T; });
        uint32_t pos = n_sure + block_excl_scan<NT>(mine, scratch, nullptr);
        run([&](unsigned long long v) {
            if (v < T) return;
            if (pos < (uint32_t)kBatchMaxK && pos < (uint32_t)p.k)
                ids[pos] = (int32_t)(~(uint32_t)v);
            else
                set_error(CSA2_DEVERR_SELECT);
            ++pos;
        });
    }
    __syncthreads();
    const uint32_t n_take = min(take, (uint32_t)p.k - n_sure);
    const uint32_t total = n_sure + n_take;
    int32_t *out = p.topk + (int64_t)qi * p.k;
    if (p.parts_sorted) {
        // two ascending runs: ids[0, n_sure) and ids[n_sure, total)
        for (uint32_t i = threadIdx.x; i < total; i += NT) {
            const int32_t x = ids[i];
            const uint32_t at = i < n_sure ? i + count_below(ids + n_sure, n_take, x)
                                           : (i - n_sure) + count_below(ids, n_sure, x);
            out[at] = x;
        }
        for (int j = (int)total + threadIdx.x; j < p.k; j += NT) out[j] = -1;
        return;
    }
    // bitonic sort of the ids ascending (padding above total sorts last)
    int P2 = 1;
    while (P2 < p.k) P2 <<= 1;
    for (int j = (int)total + threadIdx.x; j < P2; j += NT) ids[j] = INT32_MAX;
    __syncthreads();
    for (int size = 2; size <= P2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < P2 / 2; i += NT) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const int32_t x = ids[lo], y = ids[hi];
                if ((x > y) == up) {
                    ids[lo] = y;
                    ids[hi] = x;
                }
            }
            __syncthreads();
        }
    }
    for (int j = threadIdx.x; j < p.k; j += NT) out[j] = j < (int)total ? ids[j] : -1;
}

// ---------------------------------------------------------------------------
// Selection of the multi-launch Full path (one query per sequence, its score
// keys in the workspace after k_index_scan): part c of query qi reads keys
// [c * chunk, (c + 1) * chunk) of the query's visible range; keys whose
// digit 0 (top 12 bits) is above the target's threshold bin go to the
// part's sure list, keys in the bin to its candidates (64-bit keys) and to a
// histogram of their digit 1 (the next 11 bits), as in the batched path,
// whose k_batch_final then selects and merges. Every key is read once per
// target; each thread takes 16 consecutive keys per round, and one block
// scan per round places them, so every part's lists are in ascending id
// order.
// ---------------------------------------------------------------------------
constexpr int kCollectThreads = 512;
constexpr int kCollectShift1 = 9;  // digit 1: bits 19..9 of the score key

__global__ void __launch_bounds__(kCollectThreads) k_sel_collect(BatchParams p, const uint32_t *keys,
                                                                 int64_t key_stride, int32_t rank) {
    constexpr int NT = kCollectThreads;
    __shared__ uint32_t h1[2048];
    __shared__ uint32_t scratch[NT / 32 + 4];
    pdl_trigger();
    for (int i = threadIdx.x; i < 2048; i += NT) h1[i] = 0u;
    pdl_wait();
    const int32_t qi = blockIdx.y;
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    const bool all = (int64_t)rank >= limit;  // every visible entry is taken
    uint32_t *stq = p.state + (int64_t)qi * p.state_stride + p.state_off;
    const uint32_t b0 = all ? kBatchAll : __ldcg(stq);
    if (all && blockIdx.x == 0 && threadIdx.x == 0) {
        stq[0] = kBatchAll;
        stq[1] = 0u;
    }
    const int64_t c0 = (int64_t)blockIdx.x * p.chunk;
    const int64_t c1 = min(limit, c0 + p.chunk);
    const int64_t part = (int64_t)qi * p.nchunks + blockIdx.x;
    const uint32_t *kq = keys + (int64_t)qi * key_stride;
    uint32_t n_s = 0, n_c = 0;  // written so far (block-uniform)
    for (int64_t base = c0; base < c1; base += 16 * NT) {
        const int64_t t0 = base + 16 * threadIdx.x;
        uint4 k4[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
            k4[r] = t0 + 4 * r < c1 ? __ldcg(reinterpret_cast<const uint4 *>(kq + t0 + 4 * r)) : make_uint4(0u, 0u, 0u, 0u);
        // bit i: key t0 + i is sure / a candidate
        const int64_t left = c1 - t0;
        const uint32_t inmask = left >= 16 ? 0xFFFFu : (left > 0 ? (1u << left) - 1u : 0u);
        uint32_t ms = 0, mc = 0;
        if (all) {
            ms = inmask;
        } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const uint32_t kk[4] = {k4[r].x, k4[r].y, k4[r].z, k4[r].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t d = kk[j] >> 20;
                    ms |= (uint32_t)(d > b0) << (4 * r + j);
                    mc |= (uint32_t)(d == b0) << (4 * r + j);
                }
            }
            ms &= inmask;
            mc &= inmask;
        }
        // counts packed as sure | cand << 16 (each below 2^16 per round)
        uint32_t tot_r;
        const uint32_t ex = block_excl_scan<NT>((uint32_t)__popc(ms) | ((uint32_t)__popc(mc) << 16), scratch, &tot_r);
        uint32_t ps = n_s + (ex & 0xFFFFu), pc = n_c + (ex >> 16);
        const int32_t tl = (int32_t)t0;
        for (uint32_t m = ms; m; m &= m - 1u) {
            if (ps < (uint32_t)p.sure_stride)
                p.sure[part * p.sure_stride + ps] = tl + (int32_t)(__ffs(m) - 1);
            else
                set_error(CSA2_DEVERR_SELECT);
            ++ps;
        }
        if (mc) {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const uint32_t kk[4] = {k4[r].x, k4[r].y, k4[r].z, k4[r].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (!(mc & (1u << (4 * r + j)))) continue;
                    const uint32_t t = (uint32_t)(tl + 4 * r + j);
                    if ((int64_t)pc < p.chunk)
                        p.cand[part * p.chunk + pc] = ((unsigned long long)kk[j] << 32) | (unsigned long long)(~t);
                    else
                        set_error(CSA2_DEVERR_SELECT);
                    atomicAdd(&h1[(kk[j] >> kCollectShift1) & 2047u], 1u);
                    ++pc;
                }
            }
        }
        n_s += tot_r & 0xFFFFu;
        n_c += tot_r >> 16;
    }
    __syncthreads();
    if (p.hist1 != nullptr && n_c > 0)
        for (int i = threadIdx.x; i < 2048; i += NT)
            if (h1[i]) atomicAdd(p.hist1 + (int64_t)qi * 2048 + i, h1[i]);
    if (threadIdx.x == 0) {
        uint32_t *c = p.cnt + part * 2;
        c[0] = min(n_s, (uint32_t)p.sure_stride);
        c[1] = n_c;
    }
}

}  // namespace csa2
