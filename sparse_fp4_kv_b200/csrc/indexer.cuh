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
// Selection: exact radix select on the 32-bit key in three digits
// (12 + 10 + 10 bits) with global histograms, then an ordered emission in
// which equal keys are taken in ascending id order, so the output lists are
// sorted by id. Reindex keeps (key, id) pairs of one pool in shared memory
// and selects on the 64-bit key (score key, ~id), which is unique.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kScanTile = 128;
constexpr int kScanThreads = 192;
constexpr int kScanN = 16;  // MMA N: indexer heads padded to 16
constexpr int kHist0Bins = 4096;
constexpr int kHistBins = 1024;
constexpr int kSelThreads = 512;
constexpr int kSelChunk = 8192;  // entries per selection CTA
constexpr int kSelPer = kSelChunk / kSelThreads;

template <int DI>
struct ScanCfg {
    static constexpr int kStages = DI == 64 ? 6 : 4;
    static constexpr int kStageBytes = kScanTile * DI;
    static constexpr uint32_t kSwizzle = DI == 64 ? kSw64 : kSw128;
    static constexpr int kQBytes = kScanN * DI;
    static constexpr size_t kSmem = 1024 /*align slack*/ + (size_t)kStages * kStageBytes + 2048 /*q tile*/ +
                                    kHist0Bins * 4 + 256 /*barriers + tmem slot*/;
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

// Byte offset of 16-byte chunk c of row r inside a K-major swizzled tile
// whose rows are DI bytes (DI = 64: 64B swizzle, DI = 128: 128B swizzle).
template <int DI>
__device__ __forceinline__ uint32_t kmajor_chunk_offset(int r, int c) {
    const int rr = r & 7;
    const int sw = DI == 128 ? rr : ((rr >> 1) & 3);
    return (uint32_t)((r >> 3) * (8 * DI) + rr * DI + ((c ^ sw) << 4));
}

// Warp-aggregated shared-memory histogram increment (bin 0xFFFFFFFF = skip).
__device__ __forceinline__ void hist_add_warp(uint32_t *hist, uint32_t bin) {
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
    const int lane = threadIdx.x & 31;
    if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
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

template <int DI>
__global__ void __launch_bounds__(kScanThreads) k_index_scan(const __grid_constant__ CUtensorMap tm, ScanParams p) {
    using Cfg = ScanCfg<DI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = base;
    uint8_t *qt = stages + Cfg::kStages * Cfg::kStageBytes;
    uint32_t *hist = reinterpret_cast<uint32_t *>(qt + 2048);
    uint64_t *full = reinterpret_cast<uint64_t *>(hist + kHist0Bins);
    uint64_t *empty = full + Cfg::kStages;
    uint64_t *tfull = empty + Cfg::kStages;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t qi = blockIdx.y;
    const int32_t b = qi / p.q_per_seq;
    pdl_trigger();
    pdl_wait();
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    const int64_t start = (int64_t)blockIdx.x * p.chunk_tiles * kScanTile;
    if (start >= limit) return;
    const int64_t rem = limit - start;
    const int ntiles = (int)min((int64_t)p.chunk_tiles, (rem + kScanTile - 1) / kScanTile);

    for (int i = tid; i < kHist0Bins; i += kScanThreads) hist[i] = 0u;
    // B operand: query heads as rows 0..hi-1 of a [16][DI] K-major tile
    for (int i = tid; i < Cfg::kQBytes / 16; i += kScanThreads) {
        const int r = i / (DI / 16), c = i % (DI / 16);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < p.hi) v = *reinterpret_cast<const uint4 *>(p.qidx + ((int64_t)qi * p.hi + r) * DI + c * 16);
        *reinterpret_cast<uint4 *>(qt + kmajor_chunk_offset<DI>(r, c)) = v;
    }
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
        tmem_alloc(tmem_slot, 32);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // TMA producer
            const int nbox = kScanTile / p.box_rows;
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % Cfg::kStages;
                if (!mbar_wait(&empty[s], ((i / Cfg::kStages) & 1) ^ 1)) break;
                const int64_t t0 = start + (int64_t)i * kScanTile;
                int nvalid = 0;
                for (int j = 0; j < nbox; ++j) nvalid += (t0 + (int64_t)j * p.box_rows < limit);
                mbar_arrive_expect_tx(&full[s], (uint32_t)(nvalid * p.box_rows * DI));
                for (int j = 0; j < nvalid; ++j) {
                    int64_t row = physical_row(p.kv, b, t0 + (int64_t)j * p.box_rows);
                    if (row < 0) {
                        set_error(CSA2_DEVERR_BAD_ROW);
                        row = 0;
                    }
                    tma_load_2d(stages + s * Cfg::kStageBytes + j * p.box_rows * DI, &tm, &full[s], 0, (int32_t)row);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer
            const uint32_t idesc = idesc_e4m3_f32(128, kScanN);
            const uint32_t qaddr = smem_u32(qt);
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % Cfg::kStages, a = i & 1;
                if (!mbar_wait(&full[s], (i / Cfg::kStages) & 1)) break;
                if (!mbar_wait(&tempty[a], ((i >> 1) & 1) ^ 1)) break;
                tc_fence_after();
                const uint32_t aaddr = smem_u32(stages + s * Cfg::kStageBytes);
#pragma unroll
                for (int kk = 0; kk < DI / 32; ++kk) {
                    const uint64_t ad = make_sdesc(aaddr + kk * 32, 16, 8 * DI, Cfg::kSwizzle);
                    const uint64_t bd = make_sdesc(qaddr + kk * 32, 16, 8 * DI, Cfg::kSwizzle);
                    mma_e4m3(tmem + a * kScanN, ad, bd, idesc, kk > 0 ? 1u : 0u);
                }
                tc_commit(&empty[s]);
                tc_commit(&tfull[a]);
            }
        }
    } else {
        // epilogue: warps 2..5 cover TMEM lane quarters 2, 3, 0, 1
        const int quarter = warp & 3;
        float wv[kScanN];
#pragma unroll
        for (int h = 0; h < kScanN; ++h) wv[h] = h < p.hi ? p.w[(int64_t)qi * p.hi + h] : 0.0f;
        for (int i = 0; i < ntiles; ++i) {
            const int a = i & 1;
            const bool ok = mbar_wait(&tfull[a], (i >> 1) & 1);
            if (!__all_sync(0xFFFFFFFFu, ok)) break;
            tc_fence_after();
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + a * kScanN, r);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[a]);
            float sc = 0.0f;
#pragma unroll
            for (int h = 0; h < kScanN; ++h)
                if (h < p.hi) sc = fmaf(wv[h], fmaxf(__uint_as_float(r[h]), 0.0f), sc);
            sc += 0.0f;
            const int64_t t = start + (int64_t)i * kScanTile + quarter * 32 + lane;
            const bool valid = t < limit;
            const uint32_t key = score_key(sc);
            if (valid) p.keys[(int64_t)qi * p.key_stride + t] = key;
            hist_add_warp(hist, valid ? (key >> 20) : 0xFFFFFFFFu);
        }
    }
    tc_fence_before();
    __syncthreads();
    for (int i = tid; i < kHist0Bins; i += kScanThreads)
        if (hist[i]) atomicAdd(&p.hist0[(int64_t)qi * kHist0Bins + i], hist[i]);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 32);
    }
    // the last CTA of this query locates the digit-0 bin of each target rank
    const int64_t chunk = (int64_t)p.chunk_tiles * kScanTile;
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

struct SelParams {
    const uint32_t *keys;
    const int32_t *q_limit;
    csa2_kv_desc kv;
    uint32_t *hist1;  // [nq][2][1024]
    uint32_t *hist2;  // [nq][2][1024]
    uint32_t *cnt;    // [nq][2][n_chunks][2]
    uint32_t *state;  // [nq][kStateWords]
    int32_t *out[2];  // topk [nq][k], pool [nq][p]
    int32_t rank[2];  // k, p (0 = no pool)
    int64_t key_stride;
    int32_t q_per_seq;
    int32_t n_chunks;
};

// A target needs a threshold only when fewer than all visible entries are
// asked for; otherwise every visible entry is taken.
__device__ __forceinline__ bool sel_active(const SelParams &p, int tau, int64_t limit) {
    return p.rank[tau] > 0 && (int64_t)p.rank[tau] < limit;
}

// The kSelPer consecutive keys t0 .. t0+kSelPer-1 of this thread (64-byte
// aligned; keys at or beyond `end` read as 0 and must be masked by the
// caller), loaded with four 16-byte loads in flight together.
__device__ __forceinline__ void load_key_slice(const uint32_t *keys, int64_t t0, int64_t end,
                                               uint32_t (&k)[kSelPer]) {
    const uint4 *src = reinterpret_cast<const uint4 *>(keys + t0);
    uint4 v[kSelPer / 4];
#pragma unroll
    for (int i = 0; i < kSelPer / 4; ++i) v[i] = t0 + 4 * i < end ? __ldcg(src + i) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < kSelPer / 4; ++i) {
        k[4 * i + 0] = v[i].x;
        k[4 * i + 1] = v[i].y;
        k[4 * i + 2] = v[i].z;
        k[4 * i + 3] = v[i].w;
    }
}

// PASS 1: histogram of digit 1 (bits 19..10) among keys whose digit 0 is the
// threshold bin; PASS 2: digit 2 (bits 9..0) among keys matching digits 0
// and 1. The last CTA of each query then locates the next threshold digit.
template <int PASS>
__global__ void __launch_bounds__(kSelThreads) k_sel_hist(SelParams p) {
    pdl_trigger();
    pdl_wait();
    __shared__ uint32_t nh[2][kHistBins];
    __shared__ uint32_t scratch[kSelThreads / 32 + 4];
    const int32_t qi = blockIdx.y;
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    const int64_t c0 = (int64_t)blockIdx.x * kSelChunk;
    if (c0 >= limit) return;
    const int64_t c1 = min(limit, c0 + kSelChunk);
    const uint32_t *st = p.state + (int64_t)qi * kStateWords;
    bool act[2];
    uint32_t b0[2], b1[2];
    for (int tau = 0; tau < 2; ++tau) {
        act[tau] = sel_active(p, tau, limit);
        b0[tau] = act[tau] ? __ldcg(st + 8 * tau + 0) : 0u;
        b1[tau] = act[tau] ? __ldcg(st + 8 * tau + 2) : 0u;
    }
    if (!act[0] && !act[1]) return;
    for (int i = threadIdx.x; i < 2 * kHistBins; i += kSelThreads) (&nh[0][0])[i] = 0u;
    __syncthreads();
    const uint32_t *keys = p.keys + (int64_t)qi * p.key_stride;
    const int64_t s0 = c0 + (int64_t)threadIdx.x * kSelPer;
    uint32_t kreg[kSelPer];
    load_key_slice(keys, s0, c1, kreg);
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) {
        const uint32_t key = kreg[j];
        const bool in = s0 + j < c1;
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
            if (!act[tau]) continue;
            bool match = in && (key >> 20) == b0[tau];
            if (PASS == 2) match = match && ((key >> 10) & 1023u) == b1[tau];
            hist_add_warp(nh[tau], match ? (PASS == 1 ? (key >> 10) & 1023u : key & 1023u) : 0xFFFFFFFFu);
        }
    }
    __syncthreads();
    uint32_t *dst = (PASS == 1 ? p.hist1 : p.hist2) + (int64_t)qi * 2 * kHistBins;
    for (int i = threadIdx.x; i < 2 * kHistBins; i += kSelThreads) {
        const uint32_t v = (&nh[0][0])[i];
        if (v) atomicAdd(&dst[i], v);
    }
    const uint32_t n_part = (uint32_t)((limit + kSelChunk - 1) / kSelChunk);
    if (last_block(p.state + (int64_t)qi * kStateWords + kCtrScan + PASS, n_part, scratch + kSelThreads / 32 + 3)) {
        uint32_t *stw = p.state + (int64_t)qi * kStateWords;
        for (int tau = 0; tau < 2; ++tau) {
            if (!act[tau]) continue;
            const uint32_t r = __ldcg(stw + 8 * tau + (PASS == 1 ? 1 : 3));
            uint32_t bin, rem;
            find_rank_bin<kSelThreads, kHistBins / kSelThreads, true>(dst + tau * kHistBins, kHistBins, r, scratch, bin, rem);
            if (threadIdx.x == 0) {
                if (PASS == 1) {
                    stw[8 * tau + 2] = bin;
                    stw[8 * tau + 3] = rem;
                } else {
                    stw[8 * tau + 4] = bin;
                    stw[8 * tau + 5] = rem;
                    stw[8 * tau + 6] = (b0[tau] << 20) | (b1[tau] << 10) | bin;
                }
            }
        }
    }
}

// Counts, per chunk, the keys above and equal to each target's threshold.
__global__ void __launch_bounds__(kSelThreads) k_sel_count(SelParams p) {
    pdl_trigger();
    pdl_wait();
    __shared__ uint32_t scratch[kSelThreads / 32 + 4];
    const int32_t qi = blockIdx.y;
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    const int64_t c0 = (int64_t)blockIdx.x * kSelChunk;
    const int64_t c1 = min(limit, c0 + kSelChunk);
    const uint32_t *keys = p.keys + (int64_t)qi * p.key_stride;
    const int64_t s0 = c0 + (int64_t)threadIdx.x * kSelPer;
    uint32_t kreg[kSelPer];
    if (sel_active(p, 0, limit) || sel_active(p, 1, limit)) load_key_slice(keys, s0, c1, kreg);
    for (int tau = 0; tau < 2; ++tau) {
        if (!sel_active(p, tau, limit)) continue;
        const uint32_t T = __ldcg(p.state + (int64_t)qi * kStateWords + 8 * tau + 6);
        uint32_t gt = 0, eq = 0;
#pragma unroll
        for (int j = 0; j < kSelPer; ++j) {
            const bool in = s0 + j < c1;
            gt += in && kreg[j] > T;
            eq += in && kreg[j] == T;
        }
        uint32_t tgt, teq;
        block_excl_scan<kSelThreads>(gt, scratch, &tgt);
        block_excl_scan<kSelThreads>(eq, scratch, &teq);
        if (threadIdx.x == 0) {
            uint32_t *c = p.cnt + (((int64_t)qi * 2 + tau) * p.n_chunks + blockIdx.x) * 2;
            c[0] = tgt;
            c[1] = teq;
        }
    }
}

// Writes the selected ids of each target in ascending id order.
__global__ void __launch_bounds__(kSelThreads) k_sel_emit(SelParams p) {
    pdl_trigger();
    pdl_wait();
    __shared__ uint32_t scratch[kSelThreads / 32 + 4];
    const int32_t qi = blockIdx.y;
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    const int64_t c0 = (int64_t)blockIdx.x * kSelChunk;
    const int64_t c1 = min(limit, c0 + kSelChunk);
    const uint32_t *keys = p.keys + (int64_t)qi * p.key_stride;
    // this thread's contiguous slice of the chunk
    const int64_t s0 = c0 + (int64_t)threadIdx.x * kSelPer;
    uint32_t kreg[kSelPer];
    load_key_slice(keys, s0, c1, kreg);
    for (int tau = 0; tau < 2; ++tau) {
        const int32_t r_out = p.rank[tau];
        if (r_out <= 0 || p.out[tau] == nullptr) continue;
        int32_t *out = p.out[tau] + (int64_t)qi * r_out;
        if (blockIdx.x == 0) {
            const int64_t nsel = min((int64_t)r_out, limit);
            for (int64_t j = nsel + threadIdx.x; j < r_out; j += kSelThreads) out[j] = -1;
        }
        if (!sel_active(p, tau, limit)) {
            // no more visible entries than requested: take every visible entry
            for (int j = 0; j < kSelPer; ++j)
                if (s0 + j < c1) out[s0 + j] = (int32_t)(s0 + j);
            continue;
        }
        const uint32_t *st = p.state + (int64_t)qi * kStateWords + 8 * tau;
        const uint32_t T = __ldcg(st + 6);
        const uint32_t need = __ldcg(st + 5);
        // counts of the chunks before this one
        const uint32_t *cnt = p.cnt + ((int64_t)qi * 2 + tau) * p.n_chunks * 2;
        uint32_t bgt = 0, beq = 0;
        for (int c = threadIdx.x; c < (int)blockIdx.x; c += kSelThreads) {
            bgt += __ldcg(cnt + 2 * c);
            beq += __ldcg(cnt + 2 * c + 1);
        }
        uint32_t base_gt, base_eq;
        block_excl_scan<kSelThreads>(bgt, scratch, &base_gt);
        block_excl_scan<kSelThreads>(beq, scratch, &base_eq);
        uint32_t myeq = 0;
        for (int j = 0; j < kSelPer; ++j) myeq += (s0 + j < c1) && kreg[j] == T;
        uint32_t eq_rank = base_eq + block_excl_scan<kSelThreads>(myeq, scratch, nullptr);
        uint32_t selmask = 0, nsel = 0;
        for (int j = 0; j < kSelPer; ++j) {
            if (s0 + j >= c1) break;
            bool sel = kreg[j] > T;
            if (kreg[j] == T) {
                sel = eq_rank < need;
                ++eq_rank;
            }
            if (sel) {
                selmask |= 1u << j;
                ++nsel;
            }
        }
        uint32_t pos = base_gt + min(base_eq, need) + block_excl_scan<kSelThreads>(nsel, scratch, nullptr);
        for (int j = 0; j < kSelPer; ++j) {
            if (!(selmask & (1u << j))) continue;
            if (pos < (uint32_t)r_out) {
                out[pos] = (int32_t)(s0 + j);
            } else {
                set_error(CSA2_DEVERR_SELECT);
            }
            ++pos;
        }
    }
}

// ---------------------------------------------------------------------------
// Reindex: score the pool ids of a Full layer, then exact Top-k of the pool
// ---------------------------------------------------------------------------
constexpr int kReindexThreads = 128;
constexpr int kReindexSelThreads = 1024;
constexpr int kReindexMaxPool = 16384;

struct ReindexParams {
    const uint8_t *qidx;
    const float *w;
    const int32_t *pool;
    csa2_kv_desc kv;
    uint32_t *keys;  // [nq][p]
    int32_t *ids;    // [nq][p]
    int32_t *topk;   // [nq][k]
    int32_t p, k, hi, q_per_seq;
};

template <int DI>
__global__ void __launch_bounds__(kReindexThreads) k_reindex_score(ReindexParams p) {
    pdl_trigger();
    pdl_wait();
    __shared__ float qf[kScanN][DI];
    __shared__ float wf[kScanN];
    const int32_t qi = blockIdx.y;
    for (int i = threadIdx.x; i < p.hi * DI; i += kReindexThreads) {
        const uint8_t v = p.qidx[(int64_t)qi * p.hi * DI + i];
        qf[i / DI][i % DI] = e4m3x2_to_float2((uint16_t)v).x;
    }
    if (threadIdx.x < p.hi) wf[threadIdx.x] = p.w[(int64_t)qi * p.hi + threadIdx.x];
    __syncthreads();
    const int32_t j = blockIdx.x * kReindexThreads + threadIdx.x;
    if (j >= p.p) return;
    int32_t id = p.pool[(int64_t)qi * p.p + j];
    uint32_t key = 0u;
    if (id >= 0) {
        const int64_t row = physical_row(p.kv, qi / p.q_per_seq, id);
        if (row < 0) {
            set_error(CSA2_DEVERR_BAD_ROW);
            id = -1;
        } else {
            float kf[DI];
            const uint4 *src = reinterpret_cast<const uint4 *>(p.kv.kidx + row * DI);
#pragma unroll
            for (int c = 0; c < DI / 16; ++c) {
                const uint4 v = __ldg(src + c);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 lo = e4m3x2_to_float2((uint16_t)(wv[u] & 0xFFFFu));
                    const float2 hi2 = e4m3x2_to_float2((uint16_t)(wv[u] >> 16));
                    kf[c * 16 + u * 4 + 0] = lo.x;
                    kf[c * 16 + u * 4 + 1] = lo.y;
                    kf[c * 16 + u * 4 + 2] = hi2.x;
                    kf[c * 16 + u * 4 + 3] = hi2.y;
                }
            }
            float sc = 0.0f;
            for (int h = 0; h < p.hi; ++h) {
                float dot = 0.0f;
#pragma unroll
                for (int i = 0; i < DI; ++i) dot = fmaf(qf[h][i], kf[i], dot);
                sc = fmaf(wf[h], fmaxf(dot, 0.0f), sc);
            }
            key = score_key(sc + 0.0f);
        }
    }
    p.keys[(int64_t)qi * p.p + j] = key;
    p.ids[(int64_t)qi * p.p + j] = id;
}

// One CTA per query: radix select of the k largest 64-bit keys
// (score key << 32 | ~id) among the valid pool entries, emitted in pool
// order.
__global__ void __launch_bounds__(kReindexSelThreads) k_reindex_select(ReindexParams p) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ uint8_t smem_raw[];
    uint64_t *k64 = reinterpret_cast<uint64_t *>(smem_raw);   // [p]
    uint32_t *hist = reinterpret_cast<uint32_t *>(k64 + p.p); // [2048]
    uint32_t *scratch = hist + 2048;                          // [NT/32 + 4]
    const int32_t qi = blockIdx.x;
    const int NT = kReindexSelThreads;
    const uint32_t *keys = p.keys + (int64_t)qi * p.p;
    const int32_t *ids = p.ids + (int64_t)qi * p.p;
    uint32_t nvalid_t = 0;
    for (int j = threadIdx.x; j < p.p; j += NT) {
        const int32_t id = ids[j];
        uint64_t v = 0;
        if (id >= 0) {
            v = ((uint64_t)keys[j] << 32) | (uint64_t)(~(uint32_t)id);
            ++nvalid_t;
        }
        k64[j] = v;
    }
    uint32_t nvalid;
    block_excl_scan<NT>(nvalid_t, scratch, &nvalid);
    const uint32_t r = min((uint32_t)p.k, nvalid);
    uint64_t T = 0;  // select valid keys >= T
    if (nvalid > (uint32_t)p.k) {
        // bits every valid key shares need no radix pass: start at the highest
        // bit in which two keys differ
        __shared__ unsigned long long and_acc, or_acc;
        if (threadIdx.x == 0) {
            and_acc = ~0ull;
            or_acc = 0ull;
        }
        __syncthreads();
        unsigned long long a = ~0ull, o = 0ull;
        for (int j = threadIdx.x; j < p.p; j += NT)
            if (ids[j] >= 0) {
                a &= k64[j];
                o |= k64[j];
            }
        atomicAnd(&and_acc, a);
        atomicOr(&or_acc, o);
        __syncthreads();
        const unsigned long long diff = and_acc ^ or_acc;  // nonzero: keys are unique
        const int hb = 63 - __clzll((long long)diff);
        uint64_t prefix = hb == 63 ? 0ull : (and_acc & ~((1ull << (hb + 1)) - 1ull));
        uint64_t pmask = hb == 63 ? 0ull : ~((1ull << (hb + 1)) - 1ull);
        uint32_t rem = r;
        for (int top = hb; top >= 0; top -= 11) {
            const int nbits = top + 1 < 11 ? top + 1 : 11;
            const int shift = top + 1 - nbits;
            const int nb = 1 << nbits;
            for (int i = threadIdx.x; i < 2048; i += NT) hist[i] = 0u;
            __syncthreads();
            for (int j = threadIdx.x; j < p.p; j += NT) {
                const uint64_t v = k64[j];
                if (ids[j] >= 0 && (v & pmask) == prefix)
                    atomicAdd(&hist[(uint32_t)(v >> shift) & (uint32_t)(nb - 1)], 1u);
            }
            __syncthreads();
            uint32_t bin, inbin;
            find_rank_bin<NT, 2048 / NT, false>(hist, nb, rem, scratch, bin, inbin);
            prefix |= (uint64_t)bin << shift;
            pmask |= (uint64_t)(nb - 1) << shift;
            rem = inbin;
            const bool all_taken = hist[bin] == rem;  // every key of this bin is taken
            __syncthreads();
            if (all_taken) break;
        }
        T = prefix;
        __syncthreads();
    }
    // ordered emission (pool order)
    const int per = (p.p + NT - 1) / NT;
    const int j0 = threadIdx.x * per;
    uint32_t mine = 0;
    for (int j = j0; j < min(p.p, j0 + per); ++j) mine += (ids[j] >= 0 && k64[j] >= T);
    uint32_t pos = block_excl_scan<NT>(mine, scratch, nullptr);
    int32_t *out = p.topk + (int64_t)qi * p.k;
    for (int j = j0; j < min(p.p, j0 + per); ++j) {
        if (!(ids[j] >= 0 && k64[j] >= T)) continue;
        if (pos < (uint32_t)p.k) {
            out[pos] = ids[j];
        } else {
            set_error(CSA2_DEVERR_SELECT);
        }
        ++pos;
    }
    for (int j = (int)r + threadIdx.x; j < p.k; j += NT) out[j] = -1;
}

}  // namespace csa2
