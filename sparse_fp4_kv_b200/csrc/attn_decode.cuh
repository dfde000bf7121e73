// attn_decode.cuh -- sparse + sliding-window decode attention, persistent
// kernel: one CTA per SM walks a contiguous run of the call's tiles.
//
// DeepSeek V4.1-Flash Cuts KV Cache by 437x (ainewsfeed.tech): paragraph
// "CSA2 assigns each layer one of three static operating modes" (attention
// over the Top-K entries an indexer mode selected) and paragraph
// "V4.1-Flash also uses FP4 quantization" (FP4 long-term KV restored for
// computation at runtime, short-window SWA KV kept at FP8). Each attended
// row is the shared latent vector, used as key and value; per head
//     o_h = sum_j softmax_j(scale * <q_h, v_j>) v_j.
//
// Work list. Query u's attended rows (its selected global entries, then its
// window rows) are cut into tpq tiles of 128 rows, tpq = ceil((k + w_max) /
// 128); the call's T = nq * tpq tiles form one list, query-major. CTA g
// takes tiles [g*per, (g+1)*per) with per = ceil(T / SMs): a run of whole
// queries plus possibly a part of a query at either end. A run of one query inside a CTA is a
// segment; a segment that covers its whole query writes o (bf16, or f32 for
// the partial-output call) directly, the others write an f32 partial (o
// normalised by its own denominators, and its log-sum-exp) that
// k_attn_merge_parts combines. Consecutive tiles of a CTA go through one
// pipeline regardless of segment boundaries.
//
// Warps:
//   * resolver (1 warp): runs up to kResRing tiles ahead: entry ids ->
//     physical rows through the page table (or window ring slots), into a
//     shared-memory ring, and an L2 prefetch of every resolved row;
//   * 16 work warps: gather the next tile's rows into registers with
//     16-byte loads (FP4 codes: four 16-byte pieces of a row per lane, its
//     scale bytes as one 8-byte piece; window rows: eight 16-byte pieces),
//     dequantise chunk by chunk into the f16 tile (exact), run the online
//     softmax (a thread per row) and the segment epilogue;
//   * 1 MMA warp: one elected thread issues S^T = KV * Q^T (tcgen05.mma
//     kind::f16, M = 128 rows, N = H heads) chunk by chunk as chunks are
//     stored, then O^T += V^T * P^T chunk by chunk.
// The f16 tile (128 KiB) is handled in four 128-column chunks, so the
// dequantisation of chunk c of tile t+1 starts as soon as the P*V product
// of tile t on chunk c is done and the tensor pipe runs PV(t) and S(t+1)
// back to back.
#pragma once

#include "attention.cuh"

namespace csa2 {

constexpr int kDecWorkWarps = 16;
constexpr int kDecWorkThreads = kDecWorkWarps * 32;
constexpr int kDecMmaWarp = kDecWorkWarps;
constexpr int kDecResWarp = kDecWorkWarps + 1;
constexpr int kDecThreads = kDecWorkThreads + 64;
constexpr int kResRing = 4;  // resolved tiles in flight

template <int H>
struct DecCfg {
    static constexpr int kKvBytes = kAttnTile * CSA2_D * 2;
    static constexpr int kQBytes = H * CSA2_D * 2;
    static constexpr int kPBytes = kAttnTile * H * 2;
    static constexpr int kPGroup = 16 * H;
    static constexpr uint32_t kPSwizzle = H == 64 ? kSw128 : (H == 32 ? kSw64 : kSw32);
    static constexpr int kColS = 0;
    static constexpr int kColO = H;
    static constexpr uint32_t kTmemCols = H == 64 ? 512u : (H == 32 ? 256u : 128u);
    static constexpr int kMisc = kResRing * kAttnTile * 5 /*rsrc, rkind*/ + kAttnTile * 4 /*valid*/ +
                                 4 * H * 4 /*red*/ + 3 * H * 4 /*m, alpha, l*/ + 256 /*bars, slot, flags*/;
    static constexpr size_t kSmem = 1024 + (size_t)kKvBytes + kQBytes + kPBytes + kMisc;
};

struct DecParams {
    const uint16_t *q;  // bf16 [nq][H][512]
    csa2_kv_desc kv;
    const int32_t *topk;  // [nq][k]
    const uint8_t *swa;
    int64_t swa_seq_stride;
    const int32_t *swa_begin;  // nullable (no window)
    const int32_t *swa_end;
    uint16_t *o;       // bf16 [nq][H][512]
    float *o32;        // f32 [nq][H][512] (partial-output call) or null
    float *lse;        // [nq][H] (nullable unless o32)
    float *o_part;     // f32 [slots][H][512]
    float *lse_part;   // [slots][H]
    int32_t *qslot;    // [nq]: first partial slot of a query split over CTAs (its slots are consecutive)
    float scale_log2;  // softmax scale * log2(e)
    int32_t k, w_max, q_per_seq, nq;
    int32_t tpq;    // tiles per query
    int32_t per;    // tiles per CTA
    int32_t nslots;  // partial slots in the workspace
    // In-kernel merge (queries split over at most kInlineMergeParts CTAs):
    // the last CTA to finish a part of query u merges all of u's parts.
    int32_t inline_merge;
    uint32_t *qcount;  // [nq]: parts of u finished (zeroed before the launch)
};
constexpr int kInlineMergeParts = 2;

// ---- the static work split (host and device) -------------------------------
// CTA g takes tiles [g*per, min((g+1)*per, T)). Its segments are the runs of
// one query inside that range; only its first and its last segment can
// cover part of a query. Partial segments are numbered CTA by CTA (first
// before last); base(g) = the partial segments of CTAs 0..g-1.
struct DecSplit {
    int64_t T;
    int32_t per, tpq;
    __host__ __device__ int64_t lo(int32_t g) const { return (int64_t)g * per; }
    __host__ __device__ int64_t hi(int32_t g) const { return min((int64_t)(g + 1) * per, T); }
    __host__ __device__ int32_t owner(int64_t x) const { return (int32_t)(x / per); }
    __host__ __device__ bool first_partial(int32_t g) const {
        const int64_t a = lo(g), b = hi(g);
        if (b <= a) return false;
        const int64_t u = a / tpq;
        return !(a == u * tpq && b >= (u + 1) * tpq);
    }
    __host__ __device__ bool last_partial(int32_t g) const {
        const int64_t a = lo(g), b = hi(g);
        if (b <= a) return false;
        const int64_t ua = a / tpq, ub = (b - 1) / tpq;
        return ub != ua && b != (ub + 1) * tpq;
    }
    __host__ __device__ int32_t nparts(int32_t g) const {
        return (int32_t)first_partial(g) + (int32_t)last_partial(g);
    }
    // slot of query u's (partial) segment in CTA g, given base(g)
    __host__ __device__ int32_t slot(int32_t g, int64_t u, int32_t base) const {
        return base + ((lo(g) / tpq == u) ? 0 : (int32_t)first_partial(g));
    }
};

// base(g) for every thread of the block (block-wide; blockDim.x <= 1024).
__device__ __forceinline__ int32_t block_part_base(const DecSplit &sp, int32_t g, int32_t *red_word) {
    if (threadIdx.x == 0) *red_word = 0;
    __syncthreads();
    int32_t mine = 0;
    for (int32_t h = threadIdx.x; h < g; h += blockDim.x) mine += sp.nparts(h);
#pragma unroll
    for (int o = 16; o; o >>= 1) mine += __shfl_xor_sync(0xFFFFFFFFu, mine, o);
    if ((threadIdx.x & 31) == 0 && mine) atomicAdd(red_word, mine);
    __syncthreads();
    return *red_word;
}

// One tile's raw rows in registers. Lane l of work warp w holds row 8w + l%8
// of the tile, part m = l / 8: FP4 rows: v[c] = the 16 code bytes 64c + 16m
// (values 128c + 32m .. + 31) for c = 0..3, v[4].xy = scale bytes 8m .. 8m+7
// (the scales of chunk m); window rows: v[2c], v[2c+1] = the 32 E4M3 bytes
// 128c + 32m .. + 31.
struct RawRow {
    uint4 v[8];
    uint32_t kind;  // 0 empty, 1 FP4 entry, 2 window row
};

__device__ __forceinline__ void gather_row(const DecParams &p, const uint8_t *swa_seq, int32_t src, uint32_t kind,
                                           int m, RawRow &raw) {
    raw.kind = kind;
    if (kind == 1) {
        const uint4 *cp = reinterpret_cast<const uint4 *>(p.kv.codes + (int64_t)src * (CSA2_D / 2) + 16 * m);
#pragma unroll
        for (int c = 0; c < 4; ++c) raw.v[c] = __ldg(cp + 4 * c);
        const uint2 sc = __ldg(reinterpret_cast<const uint2 *>(p.kv.scales + (int64_t)src * (CSA2_D / CSA2_BLOCK) + 8 * m));
        raw.v[4] = make_uint4(sc.x, sc.y, 0u, 0u);
    } else if (kind == 2) {
        const uint4 *wp = reinterpret_cast<const uint4 *>(swa_seq + (int64_t)src * CSA2_D + 32 * m);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            raw.v[2 * c] = __ldg(wp + 8 * c);
            raw.v[2 * c + 1] = __ldg(wp + 8 * c + 1);
        }
    }
}

// Dequantise latent chunk c of this lane's row into the f16 tile (K-major,
// 128B swizzle): 32 values, four 16-byte stores. The scale bytes of the
// chunk come from the lane of the same row that loaded chunk c's scales.
// Each quarter warp stores the same piece of eight consecutive rows, which
// the swizzle spreads over the eight 16-byte bank groups.
__device__ __forceinline__ void dequant_chunk(const RawRow &raw, int c, uint8_t *kv_tile) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int m = lane >> 3;
    const int e = warp * 8 + (lane & 7);
    const int src_lane = (lane & 7) | (c << 3);
    const uint32_t slo = __shfl_sync(0xFFFFFFFFu, raw.v[4].x, src_lane);
    const uint32_t shi = __shfl_sync(0xFFFFFFFFu, raw.v[4].y, src_lane);
    uint32_t h[4][4];  // [16-byte piece][f16x2]
    if (raw.kind == 1) {
        const uint32_t sw = (m < 2 ? slo : shi) >> (16 * (m & 1));  // scale bytes of blocks 8c+2m, 8c+2m+1
        const uint32_t sa = sw & 0xFFu, sb = (sw >> 8) & 0xFFu;
        const uint32_t s2a = e4m3x2_to_f16x2((uint16_t)(sa | (sa << 8)));
        const uint32_t s2b = e4m3x2_to_f16x2((uint16_t)(sb | (sb << 8)));
        const uint4 cv = raw.v[c];
        const uint32_t wds[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            e2m1x8_to_f16x8(wds[j], h[j]);
            const uint32_t s2 = j < 2 ? s2a : s2b;
#pragma unroll
            for (int i = 0; i < 4; ++i) h[j][i] = hmul2_u32(h[j][i], s2);
        }
    } else if (raw.kind == 2) {
        const uint4 a = raw.v[2 * c], b = raw.v[2 * c + 1];
        const uint32_t wds[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[j][0] = e4m3x2_to_f16x2((uint16_t)(wds[2 * j] & 0xFFFFu));
            h[j][1] = e4m3x2_to_f16x2((uint16_t)(wds[2 * j] >> 16));
            h[j][2] = e4m3x2_to_f16x2((uint16_t)(wds[2 * j + 1] & 0xFFFFu));
            h[j][3] = e4m3x2_to_f16x2((uint16_t)(wds[2 * j + 1] >> 16));
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j][0] = h[j][1] = h[j][2] = h[j][3] = 0u;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(kv_tile + kv_chunk_off(e, 16 * c + 4 * m + j)) =
            make_uint4(h[j][0], h[j][1], h[j][2], h[j][3]);
}

// One 16-byte piece i of q (bf16 values 8i .. 8i+7 of the query's [H][512]
// rows) converted to f16 into the K-major 128B-swizzled B tile.
// A bf16 magnitude of 65536 or more (0x4780 and up, infinities and NaN
// included) has no finite f16 value: CSA2_DEVERR_Q_RANGE is recorded.
template <int H>
__device__ __forceinline__ void store_q_piece(uint8_t *q_tile, int i, const uint4 &w) {
    const int h = i / (CSA2_D / 8), c64 = i % (CSA2_D / 8);
    const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) bad |= (w4[j] & 0x7FFFu) >= 0x4780u || ((w4[j] >> 16) & 0x7FFFu) >= 0x4780u;
    if (bad) set_error(CSA2_DEVERR_Q_RANGE);
    uint32_t o4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 hh = __floats2half2_rn(__uint_as_float(w4[j] << 16), __uint_as_float(w4[j] & 0xFFFF0000u));
        o4[j] = *reinterpret_cast<const uint32_t *>(&hh);
    }
    *reinterpret_cast<uint4 *>(q_tile + q_chunk_off<H>(h, c64)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
}

// Q of query u into the Q tile by the work threads, four 16-byte pieces per
// thread in flight at a time.
template <int H>
__device__ __forceinline__ void load_q(const DecParams &p, int64_t u, uint8_t *q_tile) {
    constexpr int kPer = H * (CSA2_D / 8) / kDecWorkThreads;  // 16-byte pieces per thread
    constexpr int kBatch = kPer < 4 ? kPer : 4;
    const uint4 *src = reinterpret_cast<const uint4 *>(p.q + u * H * CSA2_D);
#pragma unroll
    for (int t0 = 0; t0 < kPer; t0 += kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int t = 0; t < kBatch; ++t) v[t] = __ldg(src + threadIdx.x + (t0 + t) * kDecWorkThreads);
#pragma unroll
        for (int t = 0; t < kBatch; ++t) store_q_piece<H>(q_tile, threadIdx.x + (t0 + t) * kDecWorkThreads, v[t]);
    }
}

template <int H>
__global__ void __launch_bounds__(kDecThreads, 1) k_attn_decode(DecParams p) {
    using Cfg = DecCfg<H>;
    constexpr int G4 = H >= 32 ? 4 : 2;  // softmax head groups (4 warps each)
    constexpr int HG = H / G4;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *kv_tile = base;
    uint8_t *q_tile = kv_tile + Cfg::kKvBytes;
    uint8_t *p_tile = q_tile + Cfg::kQBytes;
    int32_t *rsrc = reinterpret_cast<int32_t *>(p_tile + Cfg::kPBytes);  // [kResRing][128]
    uint8_t *rkind = reinterpret_cast<uint8_t *>(rsrc + kResRing * kAttnTile);
    int32_t *valid_s = reinterpret_cast<int32_t *>(rkind + kResRing * kAttnTile);
    float *red = reinterpret_cast<float *>(valid_s + kAttnTile);  // [4][H]
    float *m_run = red + 4 * H;
    float *alpha = m_run + H;
    float *l_run = alpha + H;
    uint64_t *bar_kv = reinterpret_cast<uint64_t *>(l_run + H);  // [4]
    uint64_t *bar_pv = bar_kv + 4;                               // [4]
    uint64_t *bar_s = bar_pv + 4;
    uint64_t *bar_p = bar_s + 1;
    uint64_t *res_full = bar_p + 1;            // [kResRing]
    uint64_t *res_empty = res_full + kResRing;  // [kResRing]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(res_empty + kResRing);
    int32_t *rescale_tile = reinterpret_cast<int32_t *>(tmem_slot + 1);  // [4]
    int32_t *part_word = rescale_tile + 4;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const DecSplit sp{(int64_t)p.nq * p.tpq, p.per, p.tpq};
    const int32_t g = blockIdx.x;
    const int64_t x0 = sp.lo(g), x1 = sp.hi(g);
    const int n = (int)max((int64_t)0, x1 - x0);

    pdl_trigger();
    if (warp == kDecResWarp && n > 0) {
        // While the previous kernel finishes: L2 prefetches of what this CTA
        // reads first and no kernel of this library writes -- q of its
        // queries and their sequences' page-table rows. A prefetch only warms
        // L2; every read of them happens after the dependency wait below.
        const int64_t ua = x0 / p.tpq, ub = (x1 - 1) / p.tpq;
        for (int64_t u = ua; u <= ub; ++u) {
            const uint8_t *qb = reinterpret_cast<const uint8_t *>(p.q + u * H * CSA2_D);
            for (int o = lane * 128; o < H * CSA2_D * 2; o += 32 * 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(qb + o));
            if (p.kv.max_pages > 1) {
                const uint8_t *pt = reinterpret_cast<const uint8_t *>(
                    p.kv.page_table + (int64_t)((int32_t)u / p.q_per_seq) * p.kv.max_pages);
                for (int64_t o = lane * 128; o < (int64_t)p.kv.max_pages * 4; o += 32 * 128)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(pt + o));
            }
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        // the work warps arrive once per warp (lane 0, after __syncwarp)
        for (int c = 0; c < 4; ++c) {
            mbar_init(&bar_kv[c], kDecWorkWarps);
            mbar_init(&bar_pv[c], 1);
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_p, kDecWorkWarps);
        for (int r = 0; r < kResRing; ++r) {
            mbar_init(&res_full[r], 32);
            mbar_init(&res_empty[r], kDecWorkWarps);
        }
        rescale_tile[0] = rescale_tile[1] = rescale_tile[2] = rescale_tile[3] = -1;
        fence_mbar_init();
    }
    if (tid < H) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.0f;
    }
    const int32_t part_base = block_part_base(sp, g, part_word);  // its barriers publish the set-up above
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

    if (warp == kDecResWarp) {
        // ---- resolver: rows of tile i into ring slot i % kResRing ----
        int64_t u_cur = -1;
        int32_t b = 0, wb = 0, nw = 0, one_page_pt = -1;
        const bool one_page = p.kv.max_pages == 1;
        const uint8_t *swa_seq = nullptr;
        // query u and tile t of the query advance without divisions
        int64_t u = x0 / p.tpq;
        int32_t t = (int32_t)(x0 - u * p.tpq);
        for (int i = 0; i < n; ++i, ++t) {
            if (t == p.tpq) {
                t = 0;
                ++u;
            }
            const int slot = i % kResRing;
            if (i >= kResRing && !mbar_wait(&res_empty[slot], (uint32_t)((i / kResRing) - 1) & 1u)) break;
            if (u != u_cur) {
                u_cur = u;
                b = (int32_t)u / p.q_per_seq;
                wb = p.swa_begin ? p.swa_begin[u] : 0;
                nw = p.swa_begin ? max(0, p.swa_end[u] - wb) : 0;
                // a window is a run of ring slots: begin in [0, stride), at most
                // min(stride, w_max) rows; anything else is dropped and reported
                if (nw > 0 && (wb < 0 || wb >= p.swa_seq_stride || nw > p.swa_seq_stride || nw > p.w_max)) {
                    if (lane == 0) set_error(CSA2_DEVERR_BAD_ROW);
                    nw = 0;
                }
                one_page_pt = one_page ? p.kv.page_table[b] : -1;
                swa_seq = p.swa ? p.swa + (int64_t)b * p.swa_seq_stride * CSA2_D : nullptr;
            }
            // the tile's entry ids, then their pages, then the rows: every load of
            // a phase is in flight at once
            constexpr int kR = kAttnTile / 32;
            int32_t id[kR];
#pragma unroll
            for (int rr = 0; rr < kR; ++rr) {
                const int64_t j = t * kAttnTile + lane + 32 * rr;
                id[rr] = j < p.k ? p.topk[u * p.k + j] : -1;
            }
            int32_t phys[kR];
#pragma unroll
            for (int rr = 0; rr < kR; ++rr) {
                phys[rr] = -1;
                if (id[rr] >= 0) {
                    if (one_page) {
                        phys[rr] = id[rr] < p.kv.page_size ? one_page_pt : -1;
                    } else {
                        const int64_t pg = id[rr] / p.kv.page_size;
                        phys[rr] = pg < p.kv.max_pages ? p.kv.page_table[(int64_t)b * p.kv.max_pages + pg] : -1;
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < kR; ++rr) {
                const int r = lane + 32 * rr;
                const int64_t j = t * kAttnTile + r;
                int32_t src = 0;
                uint32_t kind = 0;
                if (j < p.k) {
                    if (id[rr] >= 0) {
                        const int64_t row = phys[rr] >= 0 ? (int64_t)phys[rr] * p.kv.page_size + id[rr] % p.kv.page_size
                                                          : -1;
                        if (row >= 0 && row < p.kv.rows_cap) {
                            src = (int32_t)row;
                            kind = 1;
                            const uint8_t *cr = p.kv.codes + row * (CSA2_D / 2);
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(cr));
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(cr + 128));
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.kv.scales + row * (CSA2_D / CSA2_BLOCK)));
                        } else {
                            set_error(CSA2_DEVERR_BAD_ROW);
                        }
                    }
                } else if (j < (int64_t)p.k + nw) {
                    int64_t sl = wb + (j - p.k);  // < 2 * stride
                    if (sl >= p.swa_seq_stride) sl -= p.swa_seq_stride;
                    src = (int32_t)sl;
                    kind = 2;
                    const uint8_t *wr = swa_seq + sl * CSA2_D;
#pragma unroll
                    for (int o = 0; o < CSA2_D; o += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(wr + o));
                }
                rsrc[slot * kAttnTile + r] = src;
                rkind[slot * kAttnTile + r] = (uint8_t)kind;
            }
            mbar_arrive(&res_full[slot]);
        }
    } else if (warp == kDecMmaWarp) {
        // ---- one elected thread issues every tensor-core product ----
        if (lane == 0) {
            const uint32_t kv_addr = smem_u32(kv_tile), q_addr = smem_u32(q_tile), p_addr = smem_u32(p_tile);
            const uint32_t idesc_s = idesc_f16_f32(128, H, 0, 0);
            const uint32_t idesc_o = idesc_f16_f32(128, H, 1, 1);
            const uint64_t a_s = make_sdesc(kv_addr, 16, 1024, kSw128);
            const uint64_t b_s = make_sdesc(q_addr, 16, 1024, kSw128);
            const uint64_t a_o = make_sdesc(kv_addr, 16384, 1024, kSw128);
            const uint64_t b_o = make_sdesc(p_addr, 16, Cfg::kPGroup, Cfg::kPSwizzle);
            bool ok = true;
            int32_t tq = (int32_t)(x0 % p.tpq);  // tile of its query
            for (int i = 0; i < n && ok; ++i, ++tq) {
                if (tq == p.tpq) tq = 0;
                const uint32_t ph = (uint32_t)i & 1u;
                const bool first = i == 0 || tq == 0;
#pragma unroll 1
                for (int c = 0; c < 4 && ok; ++c) {
                    if (!mbar_wait(&bar_kv[c], ph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kb = 2 * c; kb < 2 * c + 2; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16(tmem + Cfg::kColS, a_s + (uint64_t)((kb * 16384 + kk * 32) >> 4),
                                    b_s + (uint64_t)((kb * (H * 128) + kk * 32) >> 4), idesc_s, (kb | kk) ? 1u : 0u);
                }
                if (!ok) break;
                tc_commit(bar_s);
                if (!mbar_wait(bar_p, ph)) break;
                tc_fence_after();
#pragma unroll 1
                for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                    for (int kk = 0; kk < kAttnTile / 16; ++kk)
                        mma_f16(tmem + Cfg::kColO + dc * H, a_o + (uint64_t)((dc * 32768 + kk * 2048) >> 4),
                                b_o + (uint64_t)((kk * 2 * Cfg::kPGroup) >> 4), idesc_o,
                                (!first || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_pv[dc]);
                }
            }
        }
        __syncwarp();
    } else {
        // ---- work warps ----
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int quarter = warp & 3, grp = warp >> 2;
        const bool soft = grp < G4;
        const int m = lane >> 3;
        const int row_e = warp * 8 + (lane & 7);  // this lane's row in the gather / dequantisation
        float l_part[HG];
#pragma unroll
        for (int i = 0; i < HG; ++i) l_part[i] = 0.0f;
        bool ok = true;
        RawRow raw;
        raw.kind = 0;
        // tile 0's rows, then Q of its query
        int64_t u_cur = x0 / p.tpq;
        int32_t tq0 = (int32_t)(x0 - u_cur * p.tpq);  // tile of its query, advanced without divisions
        const uint8_t *swa_seq = p.swa ? p.swa + (int64_t)((int32_t)u_cur / p.q_per_seq) * p.swa_seq_stride * CSA2_D
                                       : nullptr;
        if (n > 0) {
            // Q of the first query does not depend on the resolved rows: its bf16
            // bytes go into the (still unused) KV tile by cp.async first, the first
            // tile's rows are gathered, then each thread converts the pieces it
            // copied into the f16 Q tile
            constexpr int kQPer = H * (CSA2_D / 8) / kDecWorkThreads;
            const uint4 *qsrc = reinterpret_cast<const uint4 *>(p.q + u_cur * H * CSA2_D);
#pragma unroll
            for (int t = 0; t < kQPer; ++t)
                cp_async_16(kv_tile + (size_t)(tid + t * kDecWorkThreads) * 16, qsrc + tid + t * kDecWorkThreads);
            cp_async_commit();
            if (mbar_wait(&res_full[0], 0)) {
                const int32_t src = rsrc[row_e];
                const uint32_t kd = rkind[row_e];
                __syncwarp();
                if (lane == 0) mbar_arrive(&res_empty[0]);
                gather_row(p, swa_seq, src, kd, m, raw);
            } else {
                ok = false;
            }
            cp_async_wait_all();
#pragma unroll
            for (int t = 0; t < kQPer; ++t) {
                const int i = tid + t * kDecWorkThreads;
                const uint4 w = *reinterpret_cast<const uint4 *>(kv_tile + (size_t)i * 16);
                store_q_piece<H>(q_tile, i, w);
            }
            named_bar_sync(kBarWork, kDecWorkThreads);  // the KV tile is free for the first dequantisation
        }
        int64_t u = u_cur;
        int32_t tq = tq0;
        for (int i = 0; i < n; ++i, ++tq) {
            if (tq == p.tpq) {
                tq = 0;
                ++u;
            }
            const int64_t x = x0 + i;
            const bool last = i == n - 1 || tq == p.tpq - 1;
            // 1. dequantise chunk c once the previous tile's P*V on it is done
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (i > 0 && ok && !mbar_wait(&bar_pv[c], (uint32_t)(i - 1) & 1u)) ok = false;
                dequant_chunk(raw, c, kv_tile);
                if (c == 0 && m == 0) valid_s[row_e] = raw.kind != 0u;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_kv[c]);
            }
            // 2. the next tile's rows go in flight under this tile's products
            if (i + 1 < n) {
                const int slot = (i + 1) % kResRing;
                int32_t src = 0;
                uint32_t kd = 0;
                if (ok && mbar_wait(&res_full[slot], (uint32_t)((i + 1) / kResRing) & 1u)) {
                    src = rsrc[slot * kAttnTile + row_e];
                    kd = rkind[slot * kAttnTile + row_e];
                } else {
                    ok = false;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&res_empty[slot]);
                const int64_t un = tq == p.tpq - 1 ? u + 1 : u;
                const uint8_t *sn =
                    p.swa ? p.swa + (int64_t)((int32_t)un / p.q_per_seq) * p.swa_seq_stride * CSA2_D : nullptr;
                gather_row(p, sn, src, kd, m, raw);
            }
            // 3. online softmax: thread = row (TMEM lane), warps 4g..4g+3 take
            //    heads [g*HG, (g+1)*HG)
            if (soft) {
                const bool got = ok && mbar_wait(bar_s, (uint32_t)i & 1u);
                if (!got) ok = false;
                tc_fence_after();
                const int row = quarter * 32 + lane;
                const bool row_valid = valid_s[row] != 0 && got;
                float v[HG];
                load_scores<HG>(lane_addr + Cfg::kColS + grp * HG, p.scale_log2, row_valid, v);
                bool raise = false;
#pragma unroll
                for (int gg = 0; gg < HG / 4; ++gg) {
                    const float4 mm = *reinterpret_cast<const float4 *>(m_run + grp * HG + 4 * gg);
                    raise |= v[4 * gg] > mm.x + kRescaleThreshold;
                    raise |= v[4 * gg + 1] > mm.y + kRescaleThreshold;
                    raise |= v[4 * gg + 2] > mm.z + kRescaleThreshold;
                    raise |= v[4 * gg + 3] > mm.w + kRescaleThreshold;
                }
                raise = named_bar_or(1 + grp, 128, raise);
                if (raise) {
                    float mx[HG];
#pragma unroll
                    for (int j = 0; j < HG; ++j) mx[j] = v[j];
                    warp_transpose_reduce<HG, true>(mx);
                    store_warp_reduced<HG>(red + quarter * H + grp * HG, mx);
                    named_bar_sync(1 + grp, 128);
                    if (quarter == 0 && lane < HG) {
                        const int h = grp * HG + lane;
                        const float mt = fmaxf(fmaxf(red[h], red[H + h]), fmaxf(red[2 * H + h], red[3 * H + h]));
                        const float mo = m_run[h];
                        float a = 1.0f, mn = mo;
                        if (mt > mo + kRescaleThreshold || (mo == -INFINITY && mt > -INFINITY)) {
                            mn = mt;
                            a = (mo == -INFINITY) ? 0.0f : exp2f(mo - mt);
                            if (mo != -INFINITY) rescale_tile[grp] = i;
                        }
                        m_run[h] = mn;
                        alpha[h] = a;
                    }
                    named_bar_sync(1 + grp, 128);
                }
#pragma unroll
                for (int gg = 0; gg < HG / 8; ++gg) {
                    const int h0 = grp * HG + 8 * gg;
                    const float4 ma = *reinterpret_cast<const float4 *>(m_run + h0);
                    const float4 mb = *reinterpret_cast<const float4 *>(m_run + h0 + 4);
                    const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
                    float al[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
                    if (raise) {
                        const float4 aa = *reinterpret_cast<const float4 *>(alpha + h0);
                        const float4 ab = *reinterpret_cast<const float4 *>(alpha + h0 + 4);
                        al[0] = aa.x, al[1] = aa.y, al[2] = aa.z, al[3] = aa.w;
                        al[4] = ab.x, al[5] = ab.y, al[6] = ab.z, al[7] = ab.w;
                    }
                    uint32_t pk[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int j = 8 * gg + 2 * t;
                        const float p0 = (mm[2 * t] == -INFINITY) ? 0.0f : exp2f(v[j] - mm[2 * t]);
                        const float p1 = (mm[2 * t + 1] == -INFINITY) ? 0.0f : exp2f(v[j + 1] - mm[2 * t + 1]);
                        l_part[j] = fmaf(l_part[j], al[2 * t], p0);
                        l_part[j + 1] = fmaf(l_part[j + 1], al[2 * t + 1], p1);
                        const __half2 h2 = __floats2half2_rn(p0, p1);
                        pk[t] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    *reinterpret_cast<uint4 *>(p_tile + p_chunk_off<H>(row, h0 >> 3)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
                // a raise of the running maximum rescales this group's O^T columns
                // (every earlier P*V is complete: this tile's S commit came after)
                if (raise && rescale_tile[grp] == i) {
#pragma unroll 1
                    for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                        for (int c = 0; c < HG; c += 8) {
                            uint32_t r8[8];
                            const uint32_t ta = lane_addr + Cfg::kColO + dc * H + grp * HG + c;
                            tmem_ld8(ta, r8);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                r8[j] = __float_as_uint(__uint_as_float(r8[j]) * alpha[grp * HG + c + j]);
                            tmem_st8(ta, r8);
                        }
                    }
                    tmem_wait_st();
                }
                fence_proxy_async_smem();
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p);

            if (!last) continue;
            // ---- 4. end of a segment: Q of the next one (this tile's S is done,
            //      so the Q tile is free), then o of this one ----
            const bool has_next = i + 1 < n;
            named_bar_sync(kBarWork, kDecWorkThreads);
            if (soft) {
                warp_transpose_reduce<HG, false>(l_part);
                store_warp_reduced<HG>(red + quarter * H + grp * HG, l_part);
            }
            named_bar_sync(kBarWork, kDecWorkThreads);
            if (tid < H) {
                const float l = (red[tid] + red[H + tid]) + (red[2 * H + tid] + red[3 * H + tid]);
                l_run[tid] = l;
                alpha[tid] = l > 0.0f ? 1.0f / l : 0.0f;  // reused as 1 / l
            }
            named_bar_sync(kBarWork, kDecWorkThreads);
            const int64_t seg_start = (i == 0 || x0 > u * p.tpq) ? x0 : u * p.tpq;  // first tile of the segment
            const bool whole = seg_start == u * p.tpq && x == (u + 1) * p.tpq - 1;
            int32_t slot = 0;
            if (!whole) slot = sp.slot(g, u, part_base);
            // o (bf16 or f32) or the f32 partial of this segment: once the last
            // P*V is done the whole KV tile is free; O / l goes there as [h][512]
            // rows (the layout of the destination), then out in four bulk copies
            const bool f32 = !whole || p.o32 != nullptr;
            const int es = f32 ? 4 : 2;
            if (soft) {
                const int d0 = quarter * 32 + lane;
                // the commit of the last chunk follows every product of the tile
                if (ok && !mbar_wait(&bar_pv[3], (uint32_t)i & 1u)) ok = false;
                tc_fence_after();
#pragma unroll 1
                for (int dc = 0; dc < 4; ++dc) {
                    uint32_t vals[HG];
                    const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + Cfg::kColO + dc * H + grp * HG;
                    if (HG == 16) {
                        tmem_ld16(ta, *reinterpret_cast<uint32_t(*)[16]>(&vals[0]));
                    } else {
                        tmem_ld8(ta, *reinterpret_cast<uint32_t(*)[8]>(&vals[0]));
                    }
                    tmem_wait_ld();
                    if (f32) {
#pragma unroll
                        for (int j = 0; j < HG; ++j) {
                            const int h = grp * HG + j;
                            reinterpret_cast<float *>(kv_tile)[h * CSA2_D + dc * 128 + d0] =
                                __uint_as_float(vals[j]) * alpha[h];
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < HG; ++j) {
                            const int h = grp * HG + j;
                            reinterpret_cast<uint16_t *>(kv_tile)[h * CSA2_D + dc * 128 + d0] =
                                f32_to_bf16_bits(__uint_as_float(vals[j]) * alpha[h]);
                        }
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            named_bar_sync(kBarWork, kDecWorkThreads);
            if (warp == 0) {
                uint8_t *dst = whole ? (p.o32 ? reinterpret_cast<uint8_t *>(p.o32 + u * H * CSA2_D)
                                              : reinterpret_cast<uint8_t *>(p.o + u * H * CSA2_D))
                                     : reinterpret_cast<uint8_t *>(p.o_part + (int64_t)slot * H * CSA2_D);
                const uint32_t quarter_bytes = (uint32_t)(H * CSA2_D * es / 4);
                if (lane < 4) {
                    bulk_store(dst + lane * quarter_bytes, kv_tile + lane * quarter_bytes, quarter_bytes);
                    bulk_commit();
                }
                if (!whole && seg_start == u * p.tpq && lane == 0) p.qslot[u] = slot;  // the first part of u
            }
            tc_fence_before();
            if (tid < H) {
                const float l = l_run[tid];
                const float lse = l > 0.0f ? (m_run[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
                if (whole) {
                    if (p.lse) p.lse[u * H + tid] = lse;
                } else {
                    p.lse_part[(int64_t)slot * H + tid] = lse;
                }
                m_run[tid] = -INFINITY;  // the next segment starts afresh
                l_run[tid] = 0.0f;
            }
#pragma unroll
            for (int j = 0; j < HG; ++j) l_part[j] = 0.0f;
            if (p.inline_merge && !whole) {
                // the partial must be visible to the other CTAs of u before this
                // part is counted: bulk copies complete, every store fenced
                if (warp == 0) {
                    bulk_wait_all();
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                __threadfence();
                named_bar_sync(kBarWork, kDecWorkThreads);
                const int32_t np = sp.owner((u + 1) * p.tpq - 1) - sp.owner(u * p.tpq) + 1;
                if (tid == 0) {
                    __threadfence();
                    const uint32_t done = atomicAdd(p.qcount + u, 1u) + 1u;
                    part_word[1] = done == (uint32_t)np ? 1 : 0;
                    __threadfence();
                }
                named_bar_sync(kBarWork, kDecWorkThreads);
                if (part_word[1] != 0 && np <= kInlineMergeParts) {
                    // the last part of u: weights per head, then o = sum_s w_s o_s
                    const int32_t s0 = __ldcg(p.qslot + u);
                    if (s0 < 0 || s0 + np > p.nslots) {
                        if (tid == 0) set_error(CSA2_DEVERR_SELECT);
                    } else {
                        float *wgt = red;  // [H][kInlineMergeParts]
                        if (tid < H) {
                            float ls[kInlineMergeParts], mx = -INFINITY;
#pragma unroll
                            for (int q = 0; q < kInlineMergeParts; ++q) {
                                ls[q] = q < np ? __ldcg(p.lse_part + (int64_t)(s0 + q) * H + tid) : -INFINITY;
                                mx = fmaxf(mx, ls[q]);
                            }
                            float L = 0.0f;
#pragma unroll
                            for (int q = 0; q < kInlineMergeParts; ++q) {
                                ls[q] = (mx == -INFINITY || q >= np) ? 0.0f : expf(ls[q] - mx);
                                L += ls[q];
                            }
                            const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
                            for (int q = 0; q < kInlineMergeParts; ++q) wgt[tid * kInlineMergeParts + q] = ls[q] * inv;
                            if (p.lse) p.lse[u * H + tid] = L > 0.0f ? mx + logf(L) : -INFINITY;
                        }
                        named_bar_sync(kBarWork, kDecWorkThreads);
                        for (int idx = tid; idx < H * (CSA2_D / 4); idx += kDecWorkThreads) {
                            const int h = idx / (CSA2_D / 4), d4 = idx % (CSA2_D / 4);
                            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                            for (int q = 0; q < kInlineMergeParts; ++q) {
                                if (q >= np) break;
                                const float wq = wgt[h * kInlineMergeParts + q];
                                const float4 v = __ldcg(reinterpret_cast<const float4 *>(
                                                            p.o_part + ((int64_t)(s0 + q) * H + h) * CSA2_D) + d4);
                                acc.x = fmaf(wq, v.x, acc.x);
                                acc.y = fmaf(wq, v.y, acc.y);
                                acc.z = fmaf(wq, v.z, acc.z);
                                acc.w = fmaf(wq, v.w, acc.w);
                            }
                            if (p.o32) {
                                *(reinterpret_cast<float4 *>(p.o32 + (u * H + h) * CSA2_D) + d4) = acc;
                            } else {
                                const uint32_t lo = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
                                const uint32_t hi = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
                                *reinterpret_cast<uint2 *>(p.o + (u * H + h) * CSA2_D + d4 * 4) = make_uint2(lo, hi);
                            }
                        }
                    }
                }
            }
            if (has_next) load_q<H>(p, u + 1, q_tile);
            if (warp == 0) bulk_wait_read();  // the KV tile may be overwritten again
            // m_run is reset, the Q tile rewritten and the staging read before any
            // thread starts the next tile (its dequantisation is followed by the
            // fences and arrivals the tensor-core products wait for)
            named_bar_sync(kBarWork, kDecWorkThreads);
        }
    }
    if (warp == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

// Merge the partials of every query that is split over several CTAs:
// o = sum_s exp(lse_s - M) o_s / L, lse = M + log L, M = max_s lse_s,
// L = sum_s exp(lse_s - M). One CTA per (head, query); queries written
// whole by one CTA are skipped. Output bf16 (F32 false) or f32.
constexpr int kMergeThreads = 128;
constexpr int kMergeMaxParts = 64;

template <int H, bool F32>
__global__ void __launch_bounds__(kMergeThreads) k_attn_merge_parts(DecParams p) {
    __shared__ float wsm[kMergeMaxParts + 1];
    __shared__ int32_t slots[kMergeMaxParts];
    pdl_trigger();
    pdl_wait();
    const int h = blockIdx.x;
    const int64_t u = blockIdx.y;
    const DecSplit sp{(int64_t)p.nq * p.tpq, p.per, p.tpq};
    const int32_t g0 = sp.owner(u * p.tpq), g1 = sp.owner((u + 1) * p.tpq - 1);
    const int np = g1 - g0 + 1;
    if (np <= 1) return;  // written whole by one CTA
    if (np > kMergeMaxParts) {
        if (threadIdx.x == 0) set_error(CSA2_DEVERR_SELECT);
        return;
    }
    // the parts' slots are consecutive from the first part's (a slot number
    // outside the workspace is reported, not followed)
    const int32_t s0 = p.qslot[u];
    if (s0 < 0 || s0 + np > p.nslots) {
        if (threadIdx.x == 0) set_error(CSA2_DEVERR_SELECT);
        return;
    }
    if (threadIdx.x < np) slots[threadIdx.x] = s0 + threadIdx.x;
    __syncthreads();
    const int d4 = threadIdx.x;  // 128 threads x 4 values
    constexpr int kEarly = 16;   // parts whose loads go out before the weights are known
    float4 v[kEarly];
#pragma unroll
    for (int s = 0; s < kEarly; ++s)
        v[s] = s < np ? __ldg(reinterpret_cast<const float4 *>(p.o_part + ((int64_t)slots[s] * H + h) * CSA2_D) + d4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x < 32) {
        float M = -INFINITY;
        for (int s = threadIdx.x; s < np; s += 32) M = fmaxf(M, p.lse_part[(int64_t)slots[s] * H + h]);
#pragma unroll
        for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        float L = 0.0f;
        for (int s = threadIdx.x; s < np; s += 32) {
            const float w = (M == -INFINITY) ? 0.0f : expf(p.lse_part[(int64_t)slots[s] * H + h] - M);
            wsm[s] = w;
            L += w;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
        if (threadIdx.x == 0) {
            wsm[kMergeMaxParts] = L;
            if (p.lse) p.lse[u * H + h] = L > 0.0f ? M + logf(L) : -INFINITY;
        }
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kEarly; ++s) {
        if (s < np) {
            const float w = wsm[s];
            acc.x = fmaf(w, v[s].x, acc.x);
            acc.y = fmaf(w, v[s].y, acc.y);
            acc.z = fmaf(w, v[s].z, acc.z);
            acc.w = fmaf(w, v[s].w, acc.w);
        }
    }
    for (int s = kEarly; s < np; ++s) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(p.o_part + ((int64_t)slots[s] * H + h) * CSA2_D) + d4);
        const float w = wsm[s];
        acc.x = fmaf(w, t.x, acc.x);
        acc.y = fmaf(w, t.y, acc.y);
        acc.z = fmaf(w, t.z, acc.z);
        acc.w = fmaf(w, t.w, acc.w);
    }
    const float L = wsm[kMergeMaxParts];
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    if (F32) {
        *(reinterpret_cast<float4 *>(p.o32 + (u * H + h) * CSA2_D) + d4) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    } else {
        uint16_t *dst = p.o + (u * H + h) * CSA2_D + d4 * 4;
        const uint32_t lo = (uint32_t)f32_to_bf16_bits(acc.x * inv) | ((uint32_t)f32_to_bf16_bits(acc.y * inv) << 16);
        const uint32_t hi = (uint32_t)f32_to_bf16_bits(acc.z * inv) | ((uint32_t)f32_to_bf16_bits(acc.w * inv) << 16);
        *reinterpret_cast<uint2 *>(dst) = make_uint2(lo, hi);
    }
}

}  // namespace csa2
