// indexer.cuh -- Full and Reindex indexer modes and exact Top-k selection.
//
// DeepSeek V4.1-Flash Cuts KV Cache by 437x (ainewsfeed.tech), paragraph
// "CSA2 assigns each layer one of three static operating modes": Full mode
// reads the whole context, generates index data and selects Top-K; Reindex
// re-filters the entries a Full layer kept; the hierarchical sparse indexer
// lets later layers score only inside the Full layer's condensed pool.
// DeepSeek V4.1 Flash Architecture Breakdown (nashnova.com), section "How
// does the cache compress along three dimensions at once?": the first Full
// layer builds a shared candidate pool, later layers search only within it.
//
// Score (the pages give no formula; reading used throughout):
//     score(t) = sum_h w_h * max(0, <q_h, kidx_t>)
// Order: score descending, entry id ascending on ties.
//
// Full scan (k_index_scan): per CTA a chunk of one query's entries, streamed
// 128 entries at a time by TMA (64B / 128B swizzle, no multicast) into a
// shared-memory ring; one thread issues tcgen05.mma kind::f8f6f4
// (E4M3 x E4M3 -> f32, M = 128 entries, N = 16 padded heads, K = di) into a
// double-buffered TMEM accumulator; four epilogue warps read it back with
// tcgen05.ld, apply ReLU and the head weights, write the 32-bit ordered key
// of every score and histogram its top 12 bits. HBM-bound: di bytes per
// entry.
//
// Selection (indexer_batch.cuh): the scan's last CTA of a query finds the
// digit-0 bin of each target rank; k_sel_collect then splits the query's
// keys into ids certainly selected and candidates in that bin, and
// k_batch_final selects among the candidates on the unique 64-bit key
// (score key, ~id), so equal scores go to the lower id, and sorts the ids.
// Reindex (indexer_fused.cuh) keeps the pool's 64-bit keys
// (score key, ~id), which are unique, in shared memory.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kScanTile = 128;
constexpr int kScanThreads = 192;
constexpr int kScanN = 16;  // MMA N: indexer heads padded to 16
constexpr int kHist0Bins = 4096;

// Scan geometry. The indexer keys reach the tensor cores as 128-byte
// shared-memory rows (128B swizzle). With di = 64 a row holds two
// consecutive entries (kEpr = 2): the B operand carries two copies of the
// query heads, [q_h | 0] in rows 0..15 and [0 | q_h] in rows 16..31, so
// output column h scores a row's first entry and column 16 + h its second.
// TMA then moves 128-byte rows, which it does at full speed. With di = 128
// a row is one entry (kEpr = 1). A tile is 128 rows (256 or 128 entries).
template <int DI>
struct ScanGeom {
    static constexpr int kEpr = 128 / DI;
    static constexpr int kTile = 128 * kEpr;     // entries per tile
    static constexpr int kN = kScanN * kEpr;     // MMA N
    static constexpr int kStageBytes = 128 * 128;
    static constexpr int kQBytes = kN * 128;     // B operand tile
};

template <int DI>
struct ScanCfg {
    static constexpr int kStages = 4;
    static constexpr int kStageBytes = ScanGeom<DI>::kStageBytes;
    static constexpr size_t kSmem = 1024 /*align slack*/ + (size_t)kStages * kStageBytes + 4096 /*q tile*/ +
                                    kHist0Bins * 4 + 256 /*barriers + tmem slot*/ + 4 * 2048 /*page table*/;
};

struct ScanParams {
    const uint8_t *qidx;
    const float *w;
    const int32_t *q_limit;
    csa2_kv_desc kv;
    uint32_t *keys;    // [nq][key_stride]
    uint32_t *hist0;   // [nq][4096]
    uint32_t *state;   // [nq][kStateWords]
    int64_t key_stride;
    int32_t q_per_seq;
    int32_t hi;
    int32_t chunk_tiles;
    int32_t box_rows;
    int32_t rank[2];   // k, p (0 = no pool)
};

// Per-query selection state, per target tau (0 = Top-k, 1 = pool):
//   [8 tau + 0] digit-0 bin, [+1] rank left inside it, [+2] digit-1 bin,
//   [+3] rank left, [+4] digit-2 bin, [+5] equal keys to take, [+6] key T
// and counters of finished CTAs: [16] scan, [17] pass 1, [18] pass 2.
constexpr int kStateWords = 32;
constexpr int kCtrScan = 16;

__device__ __forceinline__ int64_t query_limit(const int32_t *q_limit, const csa2_kv_desc &kv, int32_t qi,
                                               int32_t q_per_seq) {
    int64_t lim = q_limit ? (int64_t)q_limit[qi] : (int64_t)kv.seq_len[qi / q_per_seq];
    return lim < 0 ? 0 : lim;
}

// Build the B operand (query heads, K-major, 128B swizzle) of one query:
// kN rows of 128 bytes (see ScanGeom), zero where no head.
template <int DI>
__device__ __forceinline__ void build_q_tile(uint8_t *qt, const uint8_t *q /*[hi][DI]*/, int hi, int nthreads) {
    using G = ScanGeom<DI>;
    for (int i = threadIdx.x; i < G::kN * 8; i += nthreads) {
        const int r = i / 8, c = i % 8;
        const int h = r % kScanN, half = r / kScanN;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (h < hi) {
            if (DI == 128) {
                v = *reinterpret_cast<const uint4 *>(q + h * DI + c * 16);
            } else if (c / 4 == half) {
                v = *reinterpret_cast<const uint4 *>(q + h * DI + (c % 4) * 16);
            }
        }
        *reinterpret_cast<uint4 *>(qt + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) = v;
    }
}

// Shared-memory histogram increment (bin 0xFFFFFFFF = skip).
__device__ __forceinline__ void hist_add_warp(uint32_t *hist, uint32_t bin) {
    // a shared-memory atomic per lane: lanes of a warp that hit the same bin
    // are serialised by the hardware, which measured cheaper than grouping
    // them with __match_any_sync first
    if (bin != 0xFFFFFFFFu) atomicAdd(&hist[bin], 1u);
}

// ---------------------------------------------------------------------------
// Block-wide helpers for the selection kernels
// ---------------------------------------------------------------------------
// Exclusive prefix sum over the block (NT threads); scratch holds NT/32 + 1
// words. Returns the exclusive prefix, *total gets the block sum.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *scratch, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < NT / 32 ? scratch[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < NT / 32) scratch[lane] = s;  // inclusive warp prefix
        if (lane == NT / 32 - 1) scratch[NT / 32] = s;
    }
    __syncthreads();
    const uint32_t warp_excl = warp ? scratch[warp - 1] : 0u;
    const uint32_t res = warp_excl + x - v;
    if (total) *total = scratch[NT / 32];
    __syncthreads();
    return res;
}

// Bins are ordered by key; the r-th largest key (r >= 1, r <= sum of the
// histogram) lies in the bin b with above(b) < r <= above(b) + h[b], where
// above(b) counts keys in bins > b. Returns b and r - above(b).
// Thread i owns PER consecutive bins from the top (nbins <= NT * PER); its
// loads are all issued before any is used. kGlobal: the histogram lives in
// global memory (filled by other CTAs' atomics, read through L2) rather than
// in this CTA's shared memory.
template <int NT, int PER, bool kGlobal>
__device__ __forceinline__ void find_rank_bin(const uint32_t *h, int nbins, uint32_t r, uint32_t *scratch,
                                              uint32_t &bin, uint32_t &rank_in_bin) {
    const int top = nbins - 1 - (int)threadIdx.x * PER;
    uint32_t v[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const int b = top - j;
        v[j] = b >= 0 ? (kGlobal ? __ldcg(h + b) : h[b]) : 0u;
    }
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) sum += v[j];
    const uint32_t excl = block_excl_scan<NT>(sum, scratch, nullptr);
    if (excl < r && r <= excl + sum) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            if (acc < r && acc + v[j] >= r) {
                scratch[NT / 32 + 1] = (uint32_t)(top - j);
                scratch[NT / 32 + 2] = r - acc;
            }
            acc += v[j];
        }
    }
    __syncthreads();
    bin = scratch[NT / 32 + 1];
    rank_in_bin = scratch[NT / 32 + 2];
    __syncthreads();
}

// True in every thread of the CTA that is the last of n CTAs to arrive on
// *counter; the global writes of all n CTAs are then visible to it. No CTA
// waits for another.
__device__ __forceinline__ bool last_block(uint32_t *counter, uint32_t n, uint32_t *flag_smem) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *flag_smem = (atomicAdd(counter, 1u) == n - 1) ? 1u : 0u;
    __syncthreads();
    const bool last = *flag_smem != 0u;
    if (last) __threadfence();
    return last;
}

// ---------------------------------------------------------------------------
// Scan pipeline pieces shared by the multi-launch and the cluster Full paths.
// The MMA thread commits kScanBatch tiles at a time into one of two
// kScanBatch*16-column TMEM buffers, so the epilogue pays one barrier
// round trip per kScanBatch tiles.
// ---------------------------------------------------------------------------
constexpr int kScanBatch = 4;

// Page-table entries of the pages that hold entries [start, start + n) of
// sequence b, staged in shared memory by the whole CTA so that the TMA
// producer never waits on a global load (entries outside the table read -1).
constexpr int kMaxScanPages = 2048;
__device__ __forceinline__ int stage_pages(const csa2_kv_desc &kv, int32_t b, int64_t start, int64_t n,
                                           int32_t *ptab, int nthreads) {
    if (n <= 0) return 0;
    const int64_t pg0 = start / kv.page_size;
    const int npg = (int)((start + n - 1) / kv.page_size - pg0 + 1);
    for (int i = threadIdx.x; i < npg && i < kMaxScanPages; i += nthreads) {
        const int64_t pg = pg0 + i;
        ptab[i] = pg < kv.max_pages ? kv.page_table[(int64_t)b * kv.max_pages + pg] : -1;
    }
    return npg;
}

// TMA producer, run by a whole warp (lane 0 issues): tile i = 128 smem rows =
// kTile entries, loaded as boxes of box_rows rows. A box never crosses a
// page (box_rows * kEpr divides the page size), so the page index and the
// offset inside the page advance by whole boxes without any division. Boxes
// whose first entry is past the limit are skipped (their rows are not read).
// Physical rows come from the staged page-table entries.
template <int DI>
__device__ __forceinline__ void scan_tma_loop(const csa2_kv_desc &kv, const int32_t *ptab, int64_t start,
                                              int64_t limit, int ntiles, int nstages, int box_rows,
                                              uint8_t *stage_base, const CUtensorMap *tm, uint64_t *full_b,
                                              uint64_t *empty_b, int tile_stride = 1,
                                              const int32_t *pt_row = nullptr) {
    using G = ScanGeom<DI>;
    const bool leader = (threadIdx.x & 31) == 0;
    const int nbox = 128 / box_rows;
    const int32_t step = box_rows * G::kEpr;  // entries per box
    const int32_t ps = kv.page_size;
    if (tile_stride > 1) {
        // every tile_stride-th tile from start (a sample of the range): the
        // page of each box is read from the sequence's page-table row
        int s = 0;
        uint32_t phase = 0;
        const int64_t lim = limit;
        for (int i = 0; i < ntiles; ++i) {
            if (!mbar_wait(&empty_b[s], phase ^ 1)) return;
            const int64_t t0 = start + (int64_t)i * tile_stride * G::kTile;
            int nvalid = 0;
            for (int j = 0; j < nbox; ++j) nvalid += (t0 + (int64_t)j * step < lim);
            if (leader) mbar_arrive_expect_tx(&full_b[s], (uint32_t)(nvalid * box_rows * 128));
            for (int j = 0; j < nvalid; ++j) {
                if (!leader) break;
                const int64_t pos = t0 + (int64_t)j * step;
                const int64_t pg = pos / ps;
                const int64_t phys = pg < kv.max_pages ? (int64_t)pt_row[pg] : -1;
                int64_t row = phys * ps + pos % ps;
                if (phys < 0 || row + step > kv.rows_cap) {
                    set_error(CSA2_DEVERR_BAD_ROW);
                    row = 0;
                }
                tma_load_2d(stage_base + (size_t)s * G::kStageBytes + j * box_rows * 128, tm, &full_b[s], 0,
                            (int32_t)(row / G::kEpr));
            }
            if (++s == nstages) {
                s = 0;
                phase ^= 1u;
            }
        }
        return;
    }
    // entry positions fit in 32 bits (sequence lengths are int32)
    int32_t pi = 0, off = (int32_t)(start % ps);
    int32_t t = (int32_t)start;
    const int32_t lim = (int32_t)min(limit, (int64_t)INT32_MAX);
    // ring slot and phase advance without divisions (this loop is latency-bound)
    int s = 0;
    uint32_t phase = 0;
    // Fast path: one box per tile and the whole range inside one page (every
    // contiguous cache): consecutive tiles are consecutive rows.
    const int64_t span = (int64_t)ntiles * G::kTile;
    if (nbox == 1 && ntiles > 0 && off + span <= ps && ptab[0] >= 0 &&
        (int64_t)ptab[0] * ps + off + span <= kv.rows_cap) {
        int32_t y = (int32_t)(((int64_t)ptab[0] * ps + off) / G::kEpr);
        for (int i = 0; i < ntiles; ++i) {
            if (!mbar_wait(&empty_b[s], phase ^ 1)) return;
            if (leader) {
                mbar_arrive_expect_tx(&full_b[s], (uint32_t)G::kStageBytes);
                tma_load_2d(stage_base + (size_t)s * G::kStageBytes, tm, &full_b[s], 0, y);
            }
            y += 128;
            if (++s == nstages) {
                s = 0;
                phase ^= 1u;
            }
        }
        return;
    }
    // Several boxes per tile: lane j issues box j, so the tile's loads go out
    // together instead of one after another from a single thread.
    const int lane = threadIdx.x & 31;
    for (int i = 0; i < ntiles; ++i) {
        if (!mbar_wait(&empty_b[s], phase ^ 1)) return;
        int nvalid = 0;
        for (int j = 0; j < nbox; ++j) nvalid += (t + j * step < lim);
        if (leader) mbar_arrive_expect_tx(&full_b[s], (uint32_t)(nvalid * box_rows * 128));
        __syncwarp();
        if (lane < nvalid) {
            const int32_t o = off + lane * step;  // from the start of page pi
            const int32_t pj = pi + o / ps;
            const int64_t phys = pj < kMaxScanPages ? ptab[pj] : -1;
            int64_t row = phys * ps + o % ps;
            if (phys < 0 || row + step > kv.rows_cap) {
                set_error(CSA2_DEVERR_BAD_ROW);
                row = 0;
            }
            tma_load_2d(stage_base + (size_t)s * G::kStageBytes + lane * box_rows * 128, tm, &full_b[s], 0,
                        (int32_t)(row / G::kEpr));
        }
        t += nbox * step;
        off += nbox * step;
        pi += off / ps;
        off %= ps;
        if (++s == nstages) {
            s = 0;
            phase ^= 1u;
        }
    }
}

template <int DI>
__device__ __forceinline__ void scan_mma_loop(int ntiles, int nstages, const uint8_t *stage_base, uint32_t qaddr,
                                              uint64_t *full_b, uint64_t *empty_b, uint64_t *tfull,
                                              uint64_t *tempty, uint32_t tmem) {
    using G = ScanGeom<DI>;
    const uint32_t idesc = idesc_e4m3_f32(128, G::kN);
    const int nbatch = (ntiles + kScanBatch - 1) / kScanBatch;
    int s = 0;
    uint32_t phase = 0;
    for (int g = 0; g < nbatch; ++g) {
        const int a = g & 1;
        if (!mbar_wait(&tempty[a], ((g >> 1) & 1) ^ 1)) return;
        for (int j = 0; j < kScanBatch; ++j) {
            const int i = g * kScanBatch + j;
            if (i >= ntiles) break;
            if (!mbar_wait(&full_b[s], phase)) return;
            tc_fence_after();
            const uint32_t aaddr = smem_u32(stage_base + (size_t)s * G::kStageBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = make_sdesc(aaddr + kk * 32, 16, 1024, kSw128);
                const uint64_t bd = make_sdesc(qaddr + kk * 32, 16, 1024, kSw128);
                mma_e4m3(tmem + a * (kScanBatch * G::kN) + j * G::kN, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            tc_commit(&empty_b[s]);
            if (++s == nstages) {
                s = 0;
                phase ^= 1u;
            }
        }
        tc_commit(&tfull[a]);
    }
}

// Epilogue of one TMEM lane quarter (a whole warp): for every entry of every
// tile it computes the score and calls consume(tile, entry_in_tile, key) with
// all 32 lanes (kEpr calls per tile).
template <int DI, typename Consume>
__device__ __forceinline__ void scan_epilogue_loop(int ntiles, const float (&wv)[kScanN], int hi, uint64_t *tfull,
                                                   uint64_t *tempty, uint32_t tmem, int quarter, Consume consume) {
    using G = ScanGeom<DI>;
    const int lane = threadIdx.x & 31;
    const int nbatch = (ntiles + kScanBatch - 1) / kScanBatch;
    for (int g = 0; g < nbatch; ++g) {
        const int a = g & 1;
        const bool ok = mbar_wait(&tfull[a], (g >> 1) & 1);
        if (!__all_sync(0xFFFFFFFFu, ok)) break;
        tc_fence_after();
        float sc[kScanBatch][G::kEpr];
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
            uint32_t r[G::kN];
            const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + a * (kScanBatch * G::kN) + j * G::kN;
            if (G::kN == 32) {
                tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(r));
            } else {
                tmem_ld16(ta, *reinterpret_cast<uint32_t(*)[16]>(r));
            }
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < G::kEpr; ++u) {
                float v = 0.0f;
#pragma unroll
                for (int h = 0; h < kScanN; ++h)
                    if (h < hi) v = fmaf(wv[h], fmaxf(__uint_as_float(r[u * kScanN + h]), 0.0f), v);
                sc[j][u] = v + 0.0f;
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
            const int i = g * kScanBatch + j;
            if (i >= ntiles) break;
#pragma unroll
            for (int u = 0; u < G::kEpr; ++u) consume(i, G::kEpr * (quarter * 32 + lane) + u, score_key(sc[j][u]));
        }
    }
}

template <int DI>
__global__ void __launch_bounds__(kScanThreads) k_index_scan(const __grid_constant__ CUtensorMap tm, ScanParams p) {
    using Cfg = ScanCfg<DI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = base;
    uint8_t *qt = stages + Cfg::kStages * Cfg::kStageBytes;
    uint32_t *hist = reinterpret_cast<uint32_t *>(qt + 4096);
    uint64_t *full = reinterpret_cast<uint64_t *>(hist + kHist0Bins);
    uint64_t *empty = full + Cfg::kStages;
    uint64_t *tfull = empty + Cfg::kStages;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    int32_t *ptab = reinterpret_cast<int32_t *>(tmem_slot + 2);  // [kMaxScanPages]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t qi = blockIdx.y;
    const int32_t b = qi / p.q_per_seq;
    pdl_trigger();
    pdl_wait();
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    using G = ScanGeom<DI>;
    const int64_t start = (int64_t)blockIdx.x * p.chunk_tiles * G::kTile;
    if (start >= limit) return;
    const int64_t rem = limit - start;
    const int ntiles = (int)min((int64_t)p.chunk_tiles, (rem + G::kTile - 1) / G::kTile);

    for (int i = tid; i < kHist0Bins; i += kScanThreads) hist[i] = 0u;
    build_q_tile<DI>(qt, p.qidx + (int64_t)qi * p.hi * DI, p.hi, kScanThreads);
    stage_pages(p.kv, b, start, min(rem, (int64_t)ntiles * G::kTile), ptab, kScanThreads);
    if (tid == 0) {
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * kScanBatch * G::kN);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        scan_tma_loop<DI>(p.kv, ptab, start, limit, ntiles, Cfg::kStages, p.box_rows, stages, &tm, full, empty);
    } else if (warp == 1) {
        if (lane == 0)
            scan_mma_loop<DI>(ntiles, Cfg::kStages, stages, smem_u32(qt), full, empty, tfull, tempty, tmem);
    } else {
        // epilogue: warps 2..5 cover TMEM lane quarters 2, 3, 0, 1
        float wv[kScanN];
#pragma unroll
        for (int h = 0; h < kScanN; ++h) wv[h] = h < p.hi ? p.w[(int64_t)qi * p.hi + h] : 0.0f;
        uint32_t *keys = p.keys + (int64_t)qi * p.key_stride;
        scan_epilogue_loop<DI>(ntiles, wv, p.hi, tfull, tempty, tmem, warp & 3, [&](int i, int e, uint32_t key) {
            const int64_t t = start + (int64_t)i * G::kTile + e;
            const bool valid = t < limit;
            if (valid) keys[t] = key;
            hist_add_warp(hist, valid ? (key >> 20) : 0xFFFFFFFFu);
        });
    }
    tc_fence_before();
    __syncthreads();
    for (int i = tid; i < kHist0Bins; i += kScanThreads)
        if (hist[i]) atomicAdd(&p.hist0[(int64_t)qi * kHist0Bins + i], hist[i]);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kScanBatch * G::kN);
    }
    // the last CTA of this query locates the digit-0 bin of each target rank
    const int64_t chunk = (int64_t)p.chunk_tiles * G::kTile;
    uint32_t *scratch = hist;  // the shared histogram is no longer needed
    if (last_block(&p.state[(int64_t)qi * kStateWords + kCtrScan], (uint32_t)((limit + chunk - 1) / chunk),
                   scratch + 64)) {
        for (int tau = 0; tau < 2; ++tau) {
            const int64_t r = p.rank[tau];
            if (r <= 0 || r >= limit) continue;
            uint32_t bin, rem;
            find_rank_bin<kScanThreads, (kHist0Bins + kScanThreads - 1) / kScanThreads, true>(p.hist0 + (int64_t)qi * kHist0Bins, kHist0Bins, (uint32_t)r, scratch, bin,
                                        rem);
            if (tid == 0) {
                p.state[(int64_t)qi * kStateWords + 8 * tau + 0] = bin;
                p.state[(int64_t)qi * kStateWords + 8 * tau + 1] = rem;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Reindex parameters (kernel in indexer_fused.cuh)
// ---------------------------------------------------------------------------
constexpr int kReindexMaxPool = 16384;
constexpr int kSelectKeysMax = 1 << 20;  // keys per query taken by csa2_select_keys

struct ReindexParams {
    const uint8_t *qidx;
    const float *w;
    const int32_t *pool;
    csa2_kv_desc kv;
    unsigned long long *k64;  // [nq][p] workspace: (score key << 32 | ~id), 0 = empty
    int32_t *topk;   // [nq][k]
    int32_t p, k, hi, q_per_seq;
    int32_t id_offset;  // added to every id in the keys (entry-range shards)
};

}  // namespace csa2
