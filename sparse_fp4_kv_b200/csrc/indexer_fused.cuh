// indexer_fused.cuh -- Full-mode indexer in one launch: score scan and exact
// Top-k / pool selection of a query by one thread-block cluster.
//
// Same method as indexer.cuh (DeepSeek V4.1-Flash Cuts KV Cache by 437x,
// paragraph "CSA2 assigns each layer one of three static operating modes":
// Full mode scores the whole context and keeps its Top-K; the first Full
// layer also builds the pool of the hierarchical indexer), for sequences of
// up to (cluster size) * slice entries.
//
// CTA r of a query's cluster owns entries [r*S, (r+1)*S). It streams their
// indexer keys by TMA through a deep shared-memory ring into tcgen05 FP8
// MMAs (as k_index_scan) and keeps every 32-bit score key in shared memory
// together with a 4096-bin histogram of the keys' top 12 bits. The radix
// select (digits 12/10/10) then runs on shared memory: for each digit every
// CTA adds its nonzero bins into the first CTA's histogram with distributed
// shared-memory atomics, the first CTA locates the bins of both target
// ranks, and every CTA reads them back (three cluster barriers a digit). The emission is ordered by
// CTA rank and, inside a CTA, by entry, so the output ids are ascending and
// ties at the threshold go to the lowest ids. No global scratch, no memset,
// no second launch.
#pragma once

#include "indexer.cuh"

namespace csa2 {

// CTAs per query: the largest cluster size up to kFusedClusterMax that the
// device holds for every query at once (8, the portable size, otherwise).
constexpr int kFusedClusterMin = 8;
constexpr int kFusedClusterMax = 16;
constexpr int kFusedThreads = 256;


// Cluster-wide rank bins: every CTA adds its nonzero local bins into the
// first CTA's accumulator acc (distributed shared-memory atomics, so only
// the few bins a CTA filled travel); the first CTA finds, for each active
// target tau, the bin holding rank rem[tau] of the TB bins at
// acc + hoff[tau] and the rank left inside it, clears acc for the next
// digit, and every CTA reads the results back. h and acc are at the same
// shared-memory offsets in every CTA; acc must be zero on entry.
template <int TB>
__device__ __forceinline__ void cluster_rank_bins(const uint32_t *h, int nbins, uint32_t *acc, const int (&hoff)[2],
                                                  const bool (&act)[2], uint32_t (&rem)[2], uint32_t (&bin)[2],
                                                  uint32_t *scratch, uint32_t *res, uint32_t crank) {
    cluster_sync_all();  // every CTA's local histogram is complete
    for (int i = threadIdx.x; i < nbins; i += kFusedThreads) {
        const uint32_t v = h[i];
        if (v) asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(cluster_smem_addr(acc + i, 0)), "r"(v) : "memory");
    }
    cluster_sync_all();  // every addition has landed in the first CTA
    if (crank == 0) {
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
            if (!act[tau]) continue;
            uint32_t b, r;
            find_rank_bin<kFusedThreads, TB / kFusedThreads, false>(acc + hoff[tau], TB, rem[tau], scratch, b, r);
            if (threadIdx.x == 0) {
                res[2 * tau] = b;
                res[2 * tau + 1] = r;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nbins; i += kFusedThreads) acc[i] = 0u;
    }
    cluster_sync_all();  // the results are written
#pragma unroll
    for (int tau = 0; tau < 2; ++tau) {
        if (!act[tau]) continue;
        uint32_t b, r;
        asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(b) : "r"(cluster_smem_addr(res + 2 * tau, 0)) : "memory");
        asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(r) : "r"(cluster_smem_addr(res + 2 * tau + 1, 0)) : "memory");
        bin[tau] = b;
        rem[tau] = r;
    }
}

struct FusedParams {
    const uint8_t *qidx;
    const float *w;
    const int32_t *q_limit;
    csa2_kv_desc kv;
    int32_t *out[2];  // topk [nq][k], pool [nq][p]
    int32_t rank[2];  // k, p (0 = no pool)
    int32_t q_per_seq;
    int32_t hi;
    int32_t box_rows;
    int32_t slice;    // entries per CTA (multiple of 128)
    int32_t stages;   // TMA ring depth
    int32_t csize;    // CTAs per query (cluster size)
};

template <int DI>
struct FusedCfg {
    static constexpr int kStageBytes = ScanGeom<DI>::kStageBytes;
    // fixed part: q tile, hist0, full, slice, local digit hists, small words
    static constexpr size_t kFixed = 1024 + 4096 + 4096 * 4 + 4096 * 4 + 512 * 4 + 2048 * 4 + 512 + 4 * kMaxScanPages;
    static size_t smem(int slice, int stages) {
        return kFixed + (size_t)stages * kStageBytes + (size_t)slice * 4 + 64 * 8 + 16;
    }
};

template <int DI>
__global__ void __launch_bounds__(kFusedThreads, 1)
    k_index_full_fused(const __grid_constant__ CUtensorMap tm, FusedParams p) {
    using Cfg = FusedCfg<DI>;
    using G = ScanGeom<DI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = base;
    uint8_t *qt = stages + (size_t)p.stages * Cfg::kStageBytes;
    uint32_t *hist0 = reinterpret_cast<uint32_t *>(qt + 4096);
    uint32_t *full = hist0 + 4096;
    uint32_t *slice = full + 4096;
    uint32_t *nh = slice + 512;            // [2][1024] local digit-1/2 histograms
    uint32_t *words = nh + 2048;           // 128 words: scratch + counts
    uint32_t *scratch = words;             // block-scan scratch (kFusedThreads/32 + 4)
    uint32_t *cnt = words + 32;            // [2 targets][gt, eq] of this CTA
    uint32_t *keys = words + 128;          // [slice]
    uint64_t *bars = reinterpret_cast<uint64_t *>(keys + p.slice);
    uint64_t *full_b = bars;
    uint64_t *empty_b = bars + p.stages;
    uint64_t *tfull = empty_b + p.stages;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    int32_t *ptab = reinterpret_cast<int32_t *>(tmem_slot + 2);  // [kMaxScanPages]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_rank();
    const int32_t qi = blockIdx.y;
    const int32_t b = qi / p.q_per_seq;

    // ---- set-up that reads no global memory ----
    pdl_trigger();
    for (int i = tid; i < 4096; i += kFusedThreads) hist0[i] = full[i] = 0u;
    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
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
    pdl_wait();
    const int64_t limit = query_limit(p.q_limit, p.kv, qi, p.q_per_seq);
    const int64_t start = (int64_t)crank * p.slice;
    const int64_t n_loc = max((int64_t)0, min(limit, start + p.slice) - start);
    const int ntiles = (int)((n_loc + G::kTile - 1) / G::kTile);
    build_q_tile<DI>(qt, p.qidx + (int64_t)qi * p.hi * DI, p.hi, kFusedThreads);
    stage_pages(p.kv, b, start, n_loc, ptab, kFusedThreads);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- scan: TMA -> tcgen05 FP8 MMA -> scores into shared memory ----
    if (warp == 0) {
        scan_tma_loop<DI>(p.kv, ptab, start, limit, ntiles, p.stages, p.box_rows, stages, &tm, full_b, empty_b);
    } else if (warp == 1) {
        if (lane == 0)
            scan_mma_loop<DI>(ntiles, p.stages, stages, smem_u32(qt), full_b, empty_b, tfull, tempty, tmem);
    } else if (warp < 6) {
        float wv[kScanN];
#pragma unroll
        for (int h = 0; h < kScanN; ++h) wv[h] = h < p.hi ? p.w[(int64_t)qi * p.hi + h] : 0.0f;
        scan_epilogue_loop<DI>(ntiles, wv, p.hi, tfull, tempty, tmem, warp & 3, [&](int i, int e_in, uint32_t key) {
            const int e = i * G::kTile + e_in;
            const bool valid = e < n_loc;
            if (valid) keys[e] = key;
            hist_add_warp(hist0, valid ? (key >> 20) : 0xFFFFFFFFu);
        });
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kScanBatch * G::kN);
    }

    // ---- cluster-wide radix select on the shared-memory keys ----
    bool act[2];
    uint32_t rem[2] = {0u, 0u}, b0[2] = {0u, 0u}, b1[2] = {0u, 0u}, T[2] = {0u, 0u};
    #pragma unroll
    for (int tau = 0; tau < 2; ++tau) {
        act[tau] = p.rank[tau] > 0 && (int64_t)p.rank[tau] < limit;
        rem[tau] = (uint32_t)max(p.rank[tau], 0);
    }
    // digit 0 (bits 31..20): the histogram built during the scan
    uint32_t *res = words + 96;  // the first CTA's rank bins of a digit
    {
        const int hoff[2] = {0, 0};
        cluster_rank_bins<4096>(hist0, 4096, full, hoff, act, rem, b0, scratch, res, crank);
    }
    // digits 1 (bits 19..10) and 2 (bits 9..0): each thread takes 4 keys per
    // step (one 16-byte load); most steps hold no key of the threshold bin
    // and cost one ballot
    const int nl = (int)n_loc;
    for (int digit = 1; digit <= 2; ++digit) {
        for (int i = tid; i < 2048; i += kFusedThreads) nh[i] = 0u;
        __syncthreads();
        const int shift = digit == 1 ? 20 : 10;
        uint32_t pre[2];
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) pre[tau] = digit == 1 ? b0[tau] : ((b0[tau] << 10) | b1[tau]);
        // the trip count is the same for every thread (warp-wide ballots inside)
        for (int base4 = 0; base4 < nl; base4 += 4 * kFusedThreads) {
            const int i0 = base4 + 4 * tid;
            // keys has room up to the slice end, a multiple of 4 entries
            const uint4 k4 = i0 < nl ? *reinterpret_cast<const uint4 *>(keys + i0) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
            bool m[2][4];
            bool any = false;
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    m[tau][j] = act[tau] && i0 + j < nl && (kk[j] >> shift) == pre[tau];
                    any |= m[tau][j];
                }
            if (__ballot_sync(0xFFFFFFFFu, any) == 0u) continue;
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (__ballot_sync(0xFFFFFFFFu, m[tau][j]))
                        hist_add_warp(nh + tau * 1024, m[tau][j] ? (kk[j] >> (shift - 10)) & 1023u : 0xFFFFFFFFu);
        }
        __syncthreads();
        const int hoff[2] = {0, 1024};
        uint32_t bin[2] = {0u, 0u};
        cluster_rank_bins<1024>(nh, 2048, full, hoff, act, rem, bin, scratch, res, crank);
        #pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
            if (!act[tau]) continue;
            if (digit == 1) {
                b1[tau] = bin[tau];
            } else {
                T[tau] = (b0[tau] << 20) | (b1[tau] << 10) | bin[tau];
            }
        }
    }

    // ---- ordered emission: counts of every CTA, then this CTA's ids ----
    // Warp w owns the key range [w*R, (w+1)*R) (R a multiple of 32) and walks
    // it 32 consecutive keys at a time (lane = key, conflict-free reads). One
    // pass records, per chunk of 32 keys and per target, the ballot masks of
    // keys above and equal to the threshold (in the TMA ring, free after the
    // scan) and the per-warp counts; the output position of every warp then
    // follows from the counts alone: keys above the threshold are all taken,
    // keys equal to it are taken in entry order up to the remaining rank.
    constexpr int kWarps = kFusedThreads / 32;
    const int R = ((nl + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int cpw = R / 32;
    const int w0 = warp * R, w1 = min(nl, w0 + R);
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t *wgt = words + 64;  // [2 targets][kWarps] keys above the threshold
    uint32_t *weq = words + 80;  // [2 targets][kWarps] keys equal to it
    uint4 *masks = reinterpret_cast<uint4 *>(stages) + (int64_t)warp * cpw;  // [cpw]: gt0, eq0, gt1, eq1
    {
        uint32_t gt0 = 0, eq0 = 0, gt1 = 0, eq1 = 0;
#pragma unroll 4
        for (int c = 0; c < cpw; ++c) {
            const int i = w0 + c * 32 + lane;
            const bool in = i < w1;
            const uint32_t key = in ? keys[i] : 0u;
            const uint32_t mg0 = __ballot_sync(0xFFFFFFFFu, in && act[0] && key > T[0]);
            const uint32_t me0 = __ballot_sync(0xFFFFFFFFu, in && act[0] && key == T[0]);
            const uint32_t mg1 = __ballot_sync(0xFFFFFFFFu, in && act[1] && key > T[1]);
            const uint32_t me1 = __ballot_sync(0xFFFFFFFFu, in && act[1] && key == T[1]);
            if (lane == 0) masks[c] = make_uint4(mg0, me0, mg1, me1);
            gt0 += __popc(mg0);
            eq0 += __popc(me0);
            gt1 += __popc(mg1);
            eq1 += __popc(me1);
        }
        if (lane == 0) {
            wgt[warp] = gt0;
            weq[warp] = eq0;
            wgt[kWarps + warp] = gt1;
            weq[kWarps + warp] = eq1;
        }
    }
    __syncthreads();
    if (tid < 4) {
        const uint32_t *src = (tid & 1) ? weq : wgt;
        uint32_t t = 0;
        for (int ww = 0; ww < kWarps; ++ww) t += src[(tid >> 1) * kWarps + ww];
        cnt[tid] = t;  // [tau][gt, eq]
    }
    cluster_sync_all();
    #pragma unroll
    for (int tau = 0; tau < 2; ++tau) {
        const int32_t r_out = p.rank[tau];
        if (r_out <= 0 || p.out[tau] == nullptr) continue;
        int32_t *out = p.out[tau] + (int64_t)qi * r_out;
        if (crank == 0) {
            const int64_t nsel = min((int64_t)r_out, limit);
            for (int64_t j = nsel + tid; j < r_out; j += kFusedThreads) out[j] = -1;
        }
        if (!act[tau]) {
            for (int64_t i = tid; i < n_loc; i += kFusedThreads) out[start + i] = (int32_t)(start + i);
            continue;
        }
        uint32_t base_gt = 0, base_eq = 0;
        {
            uint32_t g[kFusedClusterMax], e[kFusedClusterMax];  // all remote loads in flight at once
#pragma unroll
            for (int r = 0; r < kFusedClusterMax; ++r) {
                const bool before = (uint32_t)r < crank;
                const uint32_t *pc = cluster_peer(cnt, before ? (uint32_t)r : crank);
                g[r] = before ? pc[2 * tau] : 0u;
                e[r] = before ? pc[2 * tau + 1] : 0u;
            }
#pragma unroll
            for (int r = 0; r < kFusedClusterMax; ++r) {
                base_gt += g[r];
                base_eq += e[r];
            }
        }
        const uint32_t need = rem[tau];
        // equal keys before this warp, and the output position of its first id
        uint32_t er = base_eq, pos = base_gt + min(base_eq, need);
        for (int ww = 0; ww < warp; ++ww) {
            const uint32_t e = weq[tau * kWarps + ww];
            pos += wgt[tau * kWarps + ww] + (need > er ? min(need - er, e) : 0u);
            er += e;
        }
        // 32 chunks at a time, lane l holding chunk c0 + l: the equal keys taken
        // (in entry order, up to the rank left) and the output offsets follow
        // from warp prefix sums, then the warp writes the chunks one by one
        for (int c0 = 0; c0 < cpw; c0 += 32) {
            const int c = c0 + lane;
            const uint4 m4 = c < cpw ? masks[c] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t g = tau ? m4.z : m4.x, e = tau ? m4.w : m4.y;
            const uint32_t ne = (uint32_t)__popc(e);
            uint32_t ie = ne;  // inclusive prefix of the equal keys over the group's chunks
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, ie, o);
                if (lane >= o) ie += y;
            }
            const uint32_t er_c = er + ie - ne;  // equal keys before chunk c
            uint32_t take = 0u;
            if (e != 0u && er_c < need) {
                uint32_t left = min(need - er_c, ne), x = e;
                for (; left > 0u; --left) {  // the lowest `left` equal keys of the chunk
                    take |= x & (0u - x);
                    x &= x - 1u;
                }
            }
            const uint32_t sm = g | take;
            const uint32_t ns = (uint32_t)__popc(sm);
            uint32_t is = ns;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, is, o);
                if (lane >= o) is += y;
            }
            const uint32_t base_c = pos + is - ns;
            const int nj = min(32, cpw - c0);
            for (int j = 0; j < nj; ++j) {
                const uint32_t smj = __shfl_sync(0xFFFFFFFFu, sm, j);
                const uint32_t bj = __shfl_sync(0xFFFFFFFFu, base_c, j);
                if ((smj >> lane) & 1u) {
                    const uint32_t at = bj + __popc(smj & lt_mask);
                    if (at < (uint32_t)r_out) {
                        out[at] = (int32_t)start + w0 + (c0 + j) * 32 + lane;
                    } else {
                        set_error(CSA2_DEVERR_SELECT);
                    }
                }
            }
            pos += __shfl_sync(0xFFFFFFFFu, is, 31);
            er += __shfl_sync(0xFFFFFFFFu, ie, 31);
        }
    }
    cluster_sync_all();  // peers read cnt[] above; keep this CTA's shared memory alive until they are done
}

// ---------------------------------------------------------------------------
// Reindex: (1) k_reindex_score, many CTAs: gather the indexer keys of the
// pool ids (a row per thread, all its loads in flight), score them on the
// CUDA cores (exact for small-integer E4M3 data, like the tensor-core
// path) and write the unique 64-bit keys (score key << 32 | ~id; 0 for an
// empty slot) to the workspace; (2) k_reindex_select, one CTA per query:
// load the pool's keys into shared memory and select the k largest with a
// radix select that starts at the highest bit in which two keys differ;
// output in pool order. With G = true the keys stay in global memory (L2)
// and every pass re-reads them, for key sets larger than shared memory.
// ---------------------------------------------------------------------------
constexpr int kReindexScoreThreads = 128;
constexpr int kReindexSelectThreads = 1024;

// Pool slot j of query qi: its id's indexer key row gathered (all its loads
// in flight before the query is staged by the caller), returned in kv.
template <int DI>
__device__ __forceinline__ int32_t reindex_gather(const ReindexParams &p, int32_t qi, int32_t j, uint4 (&kv)[DI / 16]) {
    const int32_t b = qi / p.q_per_seq;
    int32_t id = (j < p.p) ? p.pool[(int64_t)qi * p.p + j] : -1;
    const int64_t row = id >= 0 ? physical_row(p.kv, b, id) : -1;
    if (id >= 0 && row < 0) {
        set_error(CSA2_DEVERR_BAD_ROW);
        id = -1;
    }
#pragma unroll
    for (int c = 0; c < DI / 16; ++c)
        kv[c] = id >= 0 ? __ldg(reinterpret_cast<const uint4 *>(p.kv.kidx + row * DI) + c) : make_uint4(0u, 0u, 0u, 0u);
    return id;
}

// The query's heads (E4M3 -> f32) and weights into shared memory.
template <int DI, int NT>
__device__ __forceinline__ void reindex_stage_query(const ReindexParams &p, int32_t qi, float *qf, float *wf) {
    for (int i = threadIdx.x; i < p.hi * DI; i += NT)
        qf[i] = e4m3x2_to_float2((uint16_t)p.qidx[(int64_t)qi * p.hi * DI + i]).x;
    if (threadIdx.x < p.hi) wf[threadIdx.x] = p.w[(int64_t)qi * p.hi + threadIdx.x];
}

// The unique 64-bit key of a gathered row (score key << 32 | ~id), 0 for an
// empty slot (a valid key has ~id >= 2^31). CUDA-core products, exact for
// small-integer E4M3 data like the tensor-core path.
template <int DI>
__device__ __forceinline__ unsigned long long reindex_key(const ReindexParams &p, int32_t id, const uint4 (&kv)[DI / 16],
                                                          const float *qf, const float *wf) {
    if (id < 0) return 0ull;
    float dot[kScanN];
#pragma unroll
    for (int h = 0; h < kScanN; ++h) dot[h] = 0.0f;
#pragma unroll
    for (int c = 0; c < DI / 16; ++c) {
        const uint32_t wv[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
        float kf[16];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float2 lo = e4m3x2_to_float2((uint16_t)(wv[t] & 0xFFFFu));
            const float2 hi2 = e4m3x2_to_float2((uint16_t)(wv[t] >> 16));
            kf[t * 4 + 0] = lo.x;
            kf[t * 4 + 1] = lo.y;
            kf[t * 4 + 2] = hi2.x;
            kf[t * 4 + 3] = hi2.y;
        }
#pragma unroll
        for (int h = 0; h < kScanN; ++h) {
            if (h >= p.hi) break;
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                const float4 q4 = *reinterpret_cast<const float4 *>(&qf[h * DI + c * 16 + i]);
                dot[h] = fmaf(q4.x, kf[i], dot[h]);
                dot[h] = fmaf(q4.y, kf[i + 1], dot[h]);
                dot[h] = fmaf(q4.z, kf[i + 2], dot[h]);
                dot[h] = fmaf(q4.w, kf[i + 3], dot[h]);
            }
        }
    }
    float sc = 0.0f;
#pragma unroll
    for (int h = 0; h < kScanN; ++h)
        if (h < p.hi) sc = fmaf(wf[h], fmaxf(dot[h], 0.0f), sc);
    return ((unsigned long long)score_key(sc + 0.0f) << 32) | (unsigned long long)(~(uint32_t)(id + p.id_offset));
}

template <int DI>
__global__ void __launch_bounds__(kReindexScoreThreads) k_reindex_score(ReindexParams p) {
    __shared__ __align__(16) float qf[kScanN * DI];
    __shared__ float wf[kScanN];
    const int32_t qi = blockIdx.y;
    pdl_trigger();
    pdl_wait();
    const int32_t j = blockIdx.x * kReindexScoreThreads + threadIdx.x;
    uint4 kv[DI / 16];
    const int32_t id = reindex_gather<DI>(p, qi, j, kv);  // out before the query is staged
    reindex_stage_query<DI, kReindexScoreThreads>(p, qi, qf, wf);
    __syncthreads();
    if (j >= p.p) return;
    p.k64[(int64_t)qi * p.p + j] = reindex_key<DI>(p, id, kv, qf, wf);
}

// Select the k largest of the m unique 64-bit keys of query qi (0 = empty;
// in shared memory k64 unless G, then read through L2 from src) and write the
// ids they carry in key-array order, padded with -1. nvalid, and_acc and
// or_acc: the count and the AND / OR of the valid keys (made visible to all
// threads by the caller). Block-wide (NT threads, a power of two).
template <bool G, int NT>
__device__ __forceinline__ void select_k64(const unsigned long long *k64, const unsigned long long *src, int32_t m,
                                           int32_t k, int32_t *out, uint32_t nvalid, unsigned long long and_acc,
                                           unsigned long long or_acc, uint32_t *hist, uint32_t *scratch) {
    auto key = [&](int j) -> uint64_t {
        if constexpr (G)
            return __ldcg(src + j);
        else
            return k64[j];
    };
    const uint32_t r = min((uint32_t)k, nvalid);
    uint64_t T = 1ull;  // select keys >= T (every valid key is >= 2^31)
    if (nvalid > (uint32_t)k) {
        // digits of 11 bits from the highest bit in which two keys differ;
        // bits that are equal in every key are skipped (they decide nothing)
        const unsigned long long diff = and_acc ^ or_acc;
        const int hb = 63 - __clzll((long long)diff);
        uint64_t prefix = hb == 63 ? 0ull : (and_acc & ~((1ull << (hb + 1)) - 1ull));
        uint64_t pmask = hb == 63 ? 0ull : ~((1ull << (hb + 1)) - 1ull);
        uint32_t rem = r;
        for (int top = hb; top >= 0;) {
            const int nbits = top + 1 < 11 ? top + 1 : 11;
            const int shift = top + 1 - nbits;
            const int nb = 1 << nbits;
            for (int i = threadIdx.x; i < 2048; i += NT) hist[i] = 0u;
            __syncthreads();
            for (int j = threadIdx.x; j < m; j += NT) {
                const uint64_t v = key(j);
                if ((uint32_t)v >= 0x80000000u && (v & pmask) == prefix)
                    atomicAdd(&hist[(uint32_t)(v >> shift) & (uint32_t)(nb - 1)], 1u);
            }
            __syncthreads();
            uint32_t bin, inbin;
            find_rank_bin<NT, 2048 / NT, false>(hist, nb, rem, scratch, bin, inbin);
            prefix |= (uint64_t)bin << shift;
            pmask |= (uint64_t)(nb - 1) << shift;
            rem = inbin;
            const bool all_taken = hist[bin] == rem;
            __syncthreads();
            if (all_taken) break;
            const uint64_t below = shift > 0 ? (diff & ((1ull << shift) - 1ull)) : 0ull;
            if (below == 0ull) break;
            top = 63 - __clzll((long long)below);
        }
        // the threshold carries the bits every key shares, so that only the
        // resolved digits (and the unresolved low bits of the last bin) decide
        T = prefix | (and_acc & ~diff);
    }
    // ordered emission (key-array order)
    const int per = (m + NT - 1) / NT;
    const int j0 = threadIdx.x * per;
    uint32_t mine = 0;
    for (int j = j0; j < min(m, j0 + per); ++j) {
        const uint64_t v = key(j);
        mine += (uint32_t)v >= 0x80000000u && v >= T;
    }
    uint32_t pos = block_excl_scan<NT>(mine, scratch, nullptr);
    for (int j = j0; j < min(m, j0 + per); ++j) {
        const uint64_t v = key(j);
        if (!((uint32_t)v >= 0x80000000u && v >= T)) continue;
        if (pos < (uint32_t)k) {
            out[pos] = (int32_t)(~(uint32_t)v);
        } else {
            set_error(CSA2_DEVERR_SELECT);
        }
        ++pos;
    }
    for (int j = (int)r + threadIdx.x; j < k; j += NT) out[j] = -1;
}

template <bool G>
__global__ void __launch_bounds__(kReindexSelectThreads, 1) k_reindex_select(ReindexParams p) {
    constexpr int NT = kReindexSelectThreads;
    extern __shared__ uint8_t smem_raw[];
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem_raw);                                 // [2048]
    uint32_t *scratch = hist + 2048;                                                         // [NT/32 + 8]
    unsigned long long *k64 = reinterpret_cast<unsigned long long *>(scratch + NT / 32 + 8);  // [p] (G false)
    __shared__ unsigned long long and_acc, or_acc;
    const int32_t qi = blockIdx.x;
    pdl_trigger();
    if (threadIdx.x == 0) {
        and_acc = ~0ull;
        or_acc = 0ull;
    }
    pdl_wait();
    __syncthreads();
    uint32_t nvalid_t = 0;
    unsigned long long a_loc = ~0ull, o_loc = 0ull;
    const unsigned long long *src = p.k64 + (int64_t)qi * p.p;
    for (int j = threadIdx.x; j < p.p; j += NT) {
        const unsigned long long v = __ldcg(src + j);
        if constexpr (!G) k64[j] = v;
        if ((uint32_t)v >= 0x80000000u) {
            ++nvalid_t;
            a_loc &= v;
            o_loc |= v;
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
    uint32_t nvalid;
    block_excl_scan<NT>(nvalid_t, scratch, &nvalid);  // its barriers also publish k64 and the reductions
    select_k64<G, NT>(k64, src, p.p, p.k, p.topk + (int64_t)qi * p.k, nvalid, and_acc, or_acc, hist, scratch);
}

// ---------------------------------------------------------------------------
// Reindex in one launch: a cluster of ceil(p / 1024) CTAs per query (at most
// 8, the portable cluster size). Thread j of the cluster gathers and scores
// pool slot j as k_reindex_score does and stores its key straight into the
// shared memory of the cluster's first CTA (distributed shared memory); after
// a cluster barrier that CTA selects the k largest with select_k64, as
// k_reindex_select does, with no round trip through global memory and no
// second launch.
// ---------------------------------------------------------------------------
constexpr int kRcThreads = 1024;
constexpr int kRcMaxCluster = 8;

template <int DI>
__global__ void __launch_bounds__(kRcThreads, 1) k_reindex_cluster(ReindexParams p) {
    constexpr int NT = kRcThreads;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem_raw);                                 // [2048]
    uint32_t *scratch = hist + 2048;                                                         // [NT/32 + 8]
    unsigned long long *k64 = reinterpret_cast<unsigned long long *>(scratch + NT / 32 + 8);  // [p], first CTA
    __shared__ __align__(16) float qf[kScanN * DI];
    __shared__ float wf[kScanN];
    __shared__ unsigned long long and_acc, or_acc;
    const uint32_t rank = cluster_rank();
    const int32_t qi = blockIdx.y;
    pdl_trigger();
    if (threadIdx.x == 0) {
        and_acc = ~0ull;
        or_acc = 0ull;
    }
    pdl_wait();
    const int32_t j = (int32_t)rank * NT + threadIdx.x;
    uint4 kv[DI / 16];
    const int32_t id = reindex_gather<DI>(p, qi, j, kv);
    reindex_stage_query<DI, NT>(p, qi, qf, wf);
    __syncthreads();
    if (j < p.p) {
        const unsigned long long v = reindex_key<DI>(p, id, kv, qf, wf);
        const uint32_t addr = cluster_smem_addr(k64 + j, 0);
        asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
    }
    cluster_sync_all();  // release / acquire: the first CTA sees every key
    if (rank != 0) return;
    uint32_t nvalid_t = 0;
    unsigned long long a_loc = ~0ull, o_loc = 0ull;
    for (int i = threadIdx.x; i < p.p; i += NT) {
        const unsigned long long v = k64[i];
        if ((uint32_t)v >= 0x80000000u) {
            ++nvalid_t;
            a_loc &= v;
            o_loc |= v;
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
    uint32_t nvalid;
    block_excl_scan<NT>(nvalid_t, scratch, &nvalid);  // its barriers also publish the reductions
    select_k64<false, NT>(k64, nullptr, p.p, p.k, p.topk + (int64_t)qi * p.k, nvalid, and_acc, or_acc, hist, scratch);
}

}  // namespace csa2
