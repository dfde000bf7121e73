// attention.cuh -- sparse + sliding-window decode attention over the FP4
// global KV and the FP8 window KV.
//
// DeepSeek V4.1-Flash Cuts KV Cache by 437x (ainewsfeed.tech): paragraph
// "CSA2 assigns each layer one of three static operating modes" (attention
// over the Top-K entries an indexer mode selected), paragraph "V4.1-Flash
// also uses FP4 quantization" (FP4 long-term KV restored for computation at
// runtime; short-window SWA KV kept at FP8). DeepSeek V4.1 Flash
// Architecture Breakdown (nashnova.com), section "How are cache precision and
// storage arranged?". Each attended row is the shared latent vector and
// serves as both key and value; per head
//     o_h = sum_j softmax_j(scale * <q_h, v_j>) v_j.
//
// Work unit: one query and a split of its attended rows (selected global
// entries followed by its window rows), 128 rows per tile. Per tile:
//   1. all 8 warps dequantise the tile's rows (fetched into registers while
//      the previous tile was on the tensor cores): FP4 codes are widened
//      with cvt.rn.f16x2.e2m1x2 and multiplied by the block scale (exact in
//      f16), window bytes with cvt.rn.f16x2.e4m3x2; the f16 tile lands in
//      shared memory in the 128B-swizzled K-major layout (rows = entries,
//      64-value column blocks 16 KiB apart); then the loads of the next
//      tile are issued.
//   2. one thread issues S^T = KV * Q^T with tcgen05.mma kind::f16
//      (M = 128 rows, N = H heads, K = 512) into TMEM.
//   3. warps 0..3 (one TMEM lane quarter each, a thread per row) read S^T,
//      reduce the per-head tile maximum across the 128 rows (transposed
//      butterfly + shared memory), run the online softmax in base 2, write
//      P^T (f16) into a swizzled M/N-major tile and reduce the per-head sum
//      of the tile's probabilities the same way.
//   4. one thread issues O^T += V^T * P^T (A = the same KV tile read
//      M/N-major, d in four chunks of 128, B = P^T) into TMEM.
// The running maximum is only raised when a tile's maximum exceeds it by
// more than 2^8, so O^T (in TMEM) is rescaled rarely; probabilities stay
// below 2^8 and are exact in range for f16.
// Splits of one query are merged by k_attn_combine with their
// log-sum-exp values.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAttnThreads = 256;
constexpr int kAttnTile = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int H>
struct AttnCfg {
    static constexpr int kKvBytes = kAttnTile * CSA2_D * 2;  // 128 KiB f16 tile
    static constexpr int kQBytes = H * CSA2_D * 2;
    static constexpr int kPBytes = kAttnTile * H * 2;
    static constexpr int kPGroup = 16 * H;  // bytes of 8 rows of P^T
    static constexpr uint32_t kPSwizzle = H == 64 ? kSw128 : (H == 32 ? kSw64 : kSw32);
    static constexpr int kColS = 0;
    static constexpr int kColO = H;
    static constexpr uint32_t kTmemCols = H == 64 ? 512u : (H == 32 ? 256u : 128u);
    static constexpr int kMisc = 8 * 128 * 5 /*resolved rows*/ + 128 * 4 /*valid*/ + 4 * H * 4 /*red*/ +
                                 3 * H * 4 /*m, alpha, l*/ + 64 /*bars, slot, flags*/;
    static constexpr size_t kSmem = 1024 + (size_t)kKvBytes + kQBytes + kPBytes + kMisc;
};

struct AttnParams {
    const uint16_t *q;  // bf16 [nq][H][512]
    csa2_kv_desc kv;
    const int32_t *topk;  // [nq][k]
    const uint8_t *swa;
    int64_t swa_seq_stride;
    const int32_t *swa_begin;
    const int32_t *swa_end;
    uint16_t *o;       // bf16 [nq][H][512] (single split)
    float *lse;        // [nq][H] (nullable)
    float *o_part;     // f32 [nq][S][H][512] (split mode)
    float *lse_part;   // [nq][S][H]
    float scale_log2;  // softmax scale * log2(e)
    int32_t k;
    int32_t q_per_seq;
    int32_t n_splits;
    int32_t tiles_per_split;
};

__device__ __forceinline__ uint32_t kv_chunk_off(int e, int c64) {
    // f16 KV tile: row e, 16-byte chunk c64 (d = 8*c64 .. 8*c64+7)
    return (uint32_t)((c64 >> 3) * 16384 + (e >> 3) * 1024 + (e & 7) * 128 + (((c64 & 7) ^ (e & 7)) << 4));
}

template <int H>
__device__ __forceinline__ uint32_t q_chunk_off(int h, int c64) {
    return (uint32_t)((c64 >> 3) * (H * 128) + (h >> 3) * 1024 + (h & 7) * 128 + (((c64 & 7) ^ (h & 7)) << 4));
}

template <int H>
__device__ __forceinline__ uint32_t p_chunk_off(int e, int c) {
    // P^T tile: row e (entry), 16-byte chunk c (heads 8c .. 8c+7)
    if (H == 64) return (uint32_t)((e >> 3) * 1024 + (e & 7) * 128 + ((c ^ (e & 7)) << 4));
    if (H == 32) return (uint32_t)((e >> 3) * 512 + (e & 7) * 64 + ((c ^ ((e & 7) >> 1)) << 4));
    return (uint32_t)((e >> 3) * 256 + (e & 7) * 32 + ((c ^ ((e & 7) >> 2)) << 4));
}

// Reduce H per-lane values over the 32 lanes of a warp with a transposed
// butterfly: after it, lane l holds the result for heads
//   H = 64: 2l, 2l+1 (v[0], v[1]);  H = 32: l (v[0]);  H = 16: l >> 1 (v[0]).
template <int H, bool kMax>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[H]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 16, n = H; off >= 1; off >>= 1) {
        if (n >= 2) {
            const int half = n / 2;
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int i = 0; i < H / 2; ++i) {
                if (i < half) {
                    const float send = upper ? v[i] : v[i + half];
                    const float keep = upper ? v[i + half] : v[i];
                    const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, off);
                    v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
                }
            }
            n = half;
        } else {
            const float recv = __shfl_xor_sync(0xFFFFFFFFu, v[0], off);
            v[0] = kMax ? fmaxf(v[0], recv) : v[0] + recv;
        }
    }
}

// Write the warp-reduced values of N columns (layout of warp_transpose_reduce)
// to dst[0..N).
template <int N>
__device__ __forceinline__ void store_warp_reduced(float *dst, const float (&v)[N]) {
    const int lane = threadIdx.x & 31;
    if (N == 64) {
        dst[2 * lane] = v[0];
        dst[2 * lane + 1] = v[1];
    } else {
        constexpr int R = N >= 32 ? 1 : 32 / N;  // lanes holding the same column
        if (lane % R == 0) dst[lane / R] = v[0];
    }
}

// ---------------------------------------------------------------------------
// Tile gather: each warp owns 16 rows of the 128-row tile. Lanes 0..15
// resolve the rows' sources in parallel (id -> page table -> physical row,
// or window row), then every lane issues its 16-value slice of all 16 rows
// back to back, so 16 independent loads per lane are in flight. The raw
// bytes stay in registers until the f16 tile buffer is free again, which
// lets the loads of tile t+1 run under the tensor-core work of tile t.
// ---------------------------------------------------------------------------
constexpr int kRowsPerWarp = kAttnTile / (kAttnThreads / 32);  // 16
constexpr int kResolveTiles = 8;  // rows resolved per batch: 8 tiles = 1024 rows

struct TileRaw {
    uint4 v[kRowsPerWarp];  // FP4 row: {codes lo, codes hi, scale byte, 0}; window row: 16 E4M3 bytes
    uint32_t kinds;         // 2 bits per row: 0 empty, 1 FP4 global entry, 2 window row
};

// Resolve the sources of rows [j0, j0 + n) of the query's attended list into
// shared memory: physical FP4 row (kind 1), window buffer row (kind 2) or
// nothing (kind 0). All threads take part; two dependent loads per row, all
// rows in flight together.
__device__ __forceinline__ void resolve_rows(const AttnParams &p, int32_t u, int32_t b, int32_t nw, int32_t wb,
                                             int64_t j0, int n, int32_t *rsrc, uint8_t *rkind) {
    for (int i = threadIdx.x; i < n; i += kAttnThreads) {
        const int64_t j = j0 + i;
        int32_t src = 0;
        uint8_t kind = 0;
        if (j < p.k) {
            const int32_t id = p.topk[(int64_t)u * p.k + j];
            if (id >= 0) {
                const int64_t row = physical_row(p.kv, b, id);
                if (row >= 0) {
                    src = (int32_t)row;
                    kind = 1;
                } else {
                    set_error(CSA2_DEVERR_BAD_ROW);
                }
            }
        } else if (j < (int64_t)p.k + nw) {
            src = (int32_t)(wb + (j - p.k));
            kind = 2;
        }
        rsrc[i] = src;
        rkind[i] = kind;
    }
}

// Issue the loads of one tile's rows (resolved sources at rsrc/rkind + off):
// every lane loads its 16-value slice of the warp's 16 rows back to back.
__device__ __forceinline__ void fetch_tile(const AttnParams &p, int32_t b, const int32_t *rsrc, const uint8_t *rkind,
                                           int off, TileRaw &raw) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int base = off + warp * kRowsPerWarp;
    const int32_t my_src = lane < kRowsPerWarp ? rsrc[base + lane] : 0;
    const uint32_t my_kind = lane < kRowsPerWarp ? rkind[base + lane] : 0u;
    const uint8_t *swa_seq = p.swa ? p.swa + (int64_t)b * p.swa_seq_stride * CSA2_D : nullptr;
    raw.kinds = 0;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const int64_t src = __shfl_sync(0xFFFFFFFFu, my_src, r);
        const uint32_t kd = __shfl_sync(0xFFFFFFFFu, my_kind, r);
        raw.kinds |= kd << (2 * r);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (kd == 1) {
            const uint2 c = __ldg(reinterpret_cast<const uint2 *>(p.kv.codes + src * (CSA2_D / 2)) + lane);
            v = make_uint4(c.x, c.y, (uint32_t)__ldg(p.kv.scales + src * (CSA2_D / CSA2_BLOCK) + lane), 0u);
        } else if (kd == 2) {
            v = __ldg(reinterpret_cast<const uint4 *>(swa_seq + src * CSA2_D) + lane);
        }
        raw.v[r] = v;
    }
}

// Dequantise the fetched rows into the f16 tile (128B-swizzled K-major) and
// record which rows hold data.
__device__ __forceinline__ void store_tile(const TileRaw &raw, uint8_t *kv_tile, int32_t *valid_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const uint32_t kd = (raw.kinds >> (2 * r)) & 3u;
        const uint4 v = raw.v[r];
        uint32_t h0[4] = {0u, 0u, 0u, 0u}, h1[4] = {0u, 0u, 0u, 0u};
        if (kd == 1) {
            const uint32_t s2 = e4m3x2_to_f16x2((uint16_t)(v.z | (v.z << 8)));
            e2m1x8_to_f16x8(v.x, h0);
            e2m1x8_to_f16x8(v.y, h1);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                h0[i] = hmul2_u32(h0[i], s2);
                h1[i] = hmul2_u32(h1[i], s2);
            }
        } else if (kd == 2) {
            h0[0] = e4m3x2_to_f16x2((uint16_t)(v.x & 0xFFFFu));
            h0[1] = e4m3x2_to_f16x2((uint16_t)(v.x >> 16));
            h0[2] = e4m3x2_to_f16x2((uint16_t)(v.y & 0xFFFFu));
            h0[3] = e4m3x2_to_f16x2((uint16_t)(v.y >> 16));
            h1[0] = e4m3x2_to_f16x2((uint16_t)(v.z & 0xFFFFu));
            h1[1] = e4m3x2_to_f16x2((uint16_t)(v.z >> 16));
            h1[2] = e4m3x2_to_f16x2((uint16_t)(v.w & 0xFFFFu));
            h1[3] = e4m3x2_to_f16x2((uint16_t)(v.w >> 16));
        }
        const int e = warp * kRowsPerWarp + r;
        *reinterpret_cast<uint4 *>(kv_tile + kv_chunk_off(e, 2 * lane)) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
        *reinterpret_cast<uint4 *>(kv_tile + kv_chunk_off(e, 2 * lane + 1)) =
            make_uint4(h1[0], h1[1], h1[2], h1[3]);
        if (lane == 0) valid_s[e] = kd != 0u;
    }
}

// NC consecutive S^T columns of this thread's row (TMEM lane), scaled to
// base-2 logits (-inf for an empty row).
template <int NC>
__device__ __forceinline__ void load_scores(uint32_t taddr, float scale_log2, bool valid, float (&s)[NC]) {
    if (NC == 32) {
        uint32_t r[32];
        tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(r));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < NC; ++i) s[i] = valid ? __uint_as_float(r[i]) * scale_log2 : -INFINITY;
    } else if (NC == 16) {
        uint32_t r[16];
        tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < NC; ++i) s[i] = valid ? __uint_as_float(r[i]) * scale_log2 : -INFINITY;
    } else {
        uint32_t r[8];
        tmem_ld8(taddr, *reinterpret_cast<uint32_t(*)[8]>(r));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < NC; ++i) s[i] = valid ? __uint_as_float(r[i]) * scale_log2 : -INFINITY;
    }
}

template <int H>
__global__ void __launch_bounds__(kAttnThreads, 1) k_sparse_attn(AttnParams p) {
    using Cfg = AttnCfg<H>;
    constexpr int HG = H / 2;  // heads per softmax warp group
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *kv_tile = base;
    uint8_t *q_tile = kv_tile + Cfg::kKvBytes;
    uint8_t *p_tile = q_tile + Cfg::kQBytes;
    int32_t *rsrc = reinterpret_cast<int32_t *>(p_tile + Cfg::kPBytes);  // [kResolveTiles * 128]
    uint8_t *rkind = reinterpret_cast<uint8_t *>(rsrc + kResolveTiles * kAttnTile);
    int32_t *valid_s = reinterpret_cast<int32_t *>(rkind + kResolveTiles * kAttnTile);
    float *red = reinterpret_cast<float *>(valid_s + kAttnTile);  // [4][H]
    float *m_run = red + 4 * H;
    float *alpha = m_run + H;
    float *l_run = alpha + H;
    uint64_t *bar_s = reinterpret_cast<uint64_t *>(l_run + H);
    uint64_t *bar_o = bar_s + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_o + 1);
    int32_t *rescale_tile = reinterpret_cast<int32_t *>(tmem_slot + 1);  // [2] (per head group)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t split = blockIdx.x, u = blockIdx.y;
    const int32_t b = u / p.q_per_seq;

    // ---- set-up that reads no global memory, then wait for the previous kernel ----
    pdl_trigger();
    if (warp == 0) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        rescale_tile[0] = rescale_tile[1] = -1;
        fence_mbar_init();
    }
    if (tid < H) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.0f;
    }
    pdl_wait();
    const int32_t wb = p.swa_begin ? p.swa_begin[u] : 0;
    const int32_t nw = p.swa_begin ? max(0, p.swa_end[u] - wb) : 0;
    const int64_t n_total = (int64_t)p.k + nw;
    const int64_t tiles_total = (n_total + kAttnTile - 1) / kAttnTile;
    const int64_t t_begin = (int64_t)split * p.tiles_per_split;
    const int64_t t_end = min(tiles_total, t_begin + p.tiles_per_split);

    // ---- prologue: resolve the first rows, start their loads, stage Q ----------
    if (t_begin < t_end)
        resolve_rows(p, u, b, nw, wb, t_begin * kAttnTile,
                     (int)min((int64_t)kResolveTiles, t_end - t_begin) * kAttnTile, rsrc, rkind);
    __syncthreads();
    TileRaw raw;
    raw.kinds = 0;
    if (t_begin < t_end) fetch_tile(p, b, rsrc, rkind, 0, raw);
    {
        // Q: bf16 -> f16 into the K-major 128B-swizzled B tile; loads in
        // batches of 8 per thread so they are in flight together
        const uint4 *qsrc = reinterpret_cast<const uint4 *>(p.q + (int64_t)u * H * CSA2_D);
        constexpr int kChunks = H * (CSA2_D / 8);
        constexpr int kPer = kChunks / kAttnThreads;  // 16 / 8 / 4 for H = 64 / 32 / 16
        constexpr int kBatch = kPer < 4 ? kPer : 4;
#pragma unroll
        for (int i0 = 0; i0 < kPer; i0 += kBatch) {
            uint4 v[kBatch];
#pragma unroll
            for (int t = 0; t < kBatch; ++t) v[t] = __ldg(qsrc + tid + (i0 + t) * kAttnThreads);
#pragma unroll
            for (int t = 0; t < kBatch; ++t) {
                const int i = tid + (i0 + t) * kAttnThreads;
                const int h = i / (CSA2_D / 8), c64 = i % (CSA2_D / 8);
                const uint32_t w4[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
                uint32_t o4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const __half2 hh =
                        __floats2half2_rn(__uint_as_float(w4[q] << 16), __uint_as_float(w4[q] & 0xFFFF0000u));
                    o4[q] = *reinterpret_cast<const uint32_t *>(&hh);
                }
                *reinterpret_cast<uint4 *>(q_tile + q_chunk_off<H>(h, c64)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t kv_addr = smem_u32(kv_tile), q_addr = smem_u32(q_tile), p_addr = smem_u32(p_tile);
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int quarter = warp & 3, grp = warp >> 2;  // TMEM lane quarter, head group
    float l_part[HG];                                // this row's partial softmax denominators
#pragma unroll
    for (int i = 0; i < HG; ++i) l_part[i] = 0.0f;

    bool ok = true;
    int it = 0;
    for (int64_t tt = t_begin; tt < t_end && ok; ++tt, ++it) {
        // 1. the f16 tile buffer is free (previous P*V done): dequantise this
        //    tile, then put the next tile's loads in flight
        store_tile(raw, kv_tile, valid_s);
        if (tt + 1 < t_end) {
            const int rel = (int)((tt + 1 - t_begin) % kResolveTiles);
            if (rel == 0) {
                // next batch of resolved rows (rare: splits of more than 8 tiles)
                __syncthreads();
                resolve_rows(p, u, b, nw, wb, (tt + 1) * kAttnTile,
                             (int)min((int64_t)kResolveTiles, t_end - (tt + 1)) * kAttnTile, rsrc, rkind);
                __syncthreads();
            }
            fetch_tile(p, b, rsrc, rkind, rel * kAttnTile, raw);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // 2. S^T = KV * Q^T
        if (tid == 0) {
            const uint32_t idesc = idesc_f16_f32(128, H, 0, 0);
#pragma unroll
            for (int kb = 0; kb < CSA2_D / 64; ++kb) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = make_sdesc(kv_addr + kb * 16384 + kk * 32, 16, 1024, kSw128);
                    const uint64_t bd = make_sdesc(q_addr + kb * (H * 128) + kk * 32, 16, 1024, kSw128);
                    mma_f16(tmem + Cfg::kColS, ad, bd, idesc, (kb | kk) ? 1u : 0u);
                }
            }
            tc_commit(bar_s);
        }
        {
            // 3. online softmax: thread = row (TMEM lane), warps 0..3 take heads
            //    [0, H/2), warps 4..7 heads [H/2, H); each group of 4 warps
            //    synchronises on its own named barrier
            const bool got = mbar_wait(bar_s, it & 1);
            tc_fence_after();
            const int row = quarter * 32 + lane;
            const bool row_valid = valid_s[row] != 0 && got;
            const uint32_t s_addr = lane_addr + Cfg::kColS + grp * HG;
            {
                float v[HG];
                load_scores<HG>(s_addr, p.scale_log2, row_valid, v);
                warp_transpose_reduce<HG, true>(v);
                store_warp_reduced<HG>(red + quarter * H + grp * HG, v);
            }
            named_bar_sync(1 + grp, 128);
            if (quarter == 0 && lane < HG) {
                const int h = grp * HG + lane;
                const float mt = fmaxf(fmaxf(red[h], red[H + h]), fmaxf(red[2 * H + h], red[3 * H + h]));
                const float mo = m_run[h];
                float a = 1.0f, mn = mo;
                if (mt > mo + kRescaleThreshold || (mo == -INFINITY && mt > -INFINITY)) {
                    mn = mt;
                    a = (mo == -INFINITY) ? 0.0f : exp2f(mo - mt);
                    if (mo != -INFINITY) rescale_tile[grp] = (int32_t)it;
                }
                m_run[h] = mn;
                alpha[h] = a;
            }
            named_bar_sync(1 + grp, 128);
            // probabilities -> P^T (f16), per-row partial denominators
            {
                float v[HG];
                load_scores<HG>(s_addr, p.scale_log2, row_valid, v);
#pragma unroll
                for (int g = 0; g < HG / 8; ++g) {
                    const float4 ma = *reinterpret_cast<const float4 *>(m_run + grp * HG + 8 * g);
                    const float4 mb = *reinterpret_cast<const float4 *>(m_run + grp * HG + 8 * g + 4);
                    const float4 aa = *reinterpret_cast<const float4 *>(alpha + grp * HG + 8 * g);
                    const float4 ab = *reinterpret_cast<const float4 *>(alpha + grp * HG + 8 * g + 4);
                    const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
                    const float al[8] = {aa.x, aa.y, aa.z, aa.w, ab.x, ab.y, ab.z, ab.w};
                    uint32_t pk[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int i = 8 * g + 2 * t;
                        const float p0 = (mm[2 * t] == -INFINITY) ? 0.0f : exp2f(v[i] - mm[2 * t]);
                        const float p1 = (mm[2 * t + 1] == -INFINITY) ? 0.0f : exp2f(v[i + 1] - mm[2 * t + 1]);
                        l_part[i] = fmaf(l_part[i], al[2 * t], p0);
                        l_part[i + 1] = fmaf(l_part[i + 1], al[2 * t + 1], p1);
                        const __half2 hh = __floats2half2_rn(p0, p1);
                        pk[t] = *reinterpret_cast<const uint32_t *>(&hh);
                    }
                    *reinterpret_cast<uint4 *>(p_tile + p_chunk_off<H>(row, grp * (HG / 8) + g)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            // rare: raise of the running maximum -> rescale this group's O^T columns
            if (rescale_tile[grp] == it) {
#pragma unroll 1
                for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                    for (int c = 0; c < HG; c += 8) {
                        uint32_t r8[8];
                        const uint32_t ta = lane_addr + Cfg::kColO + dc * H + grp * HG + c;
                        tmem_ld8(ta, r8);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            r8[i] = __float_as_uint(__uint_as_float(r8[i]) * alpha[grp * HG + c + i]);
                        tmem_st8(ta, r8);
                    }
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (!got) ok = false;
        }
        ok = __syncthreads_and(ok);
        tc_fence_after();
        // 4. O^T += V^T * P^T
        if (tid == 0 && ok) {
            const uint32_t idesc = idesc_f16_f32(128, H, 1, 1);
#pragma unroll
            for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                for (int kk = 0; kk < kAttnTile / 16; ++kk) {
                    const uint64_t ad = make_sdesc(kv_addr + dc * 32768 + kk * 2048, 16384, 1024, kSw128);
                    const uint64_t bd = make_sdesc(p_addr + kk * 2 * Cfg::kPGroup, 16, Cfg::kPGroup, Cfg::kPSwizzle);
                    mma_f16(tmem + Cfg::kColO + dc * H, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
                }
            }
            tc_commit(bar_o);
        }
        // the next tile overwrites KV / P: wait for this tile's P*V
        if (ok && !mbar_wait(bar_o, it & 1)) ok = false;
        tc_fence_after();
        ok = __syncthreads_and(ok);
    }
    // ---- final denominators: reduce the per-row partials over the 128 rows ----
    __syncthreads();
    warp_transpose_reduce<HG, false>(l_part);
    store_warp_reduced<HG>(red + quarter * H + grp * HG, l_part);
    __syncthreads();
    if (tid < H) {
        const float l = (red[tid] + red[H + tid]) + (red[2 * H + tid] + red[3 * H + tid]);
        l_run[tid] = l;
        alpha[tid] = l > 0.0f ? 1.0f / l : 0.0f;  // reused as 1 / l
    }
    __syncthreads();

    // ---- epilogue: O^T (TMEM) -> o = O / l, staged through the free KV tile
    //      buffer as [h][512] f32 so the global writes are coalesced 16 B ----
    {
        constexpr int HC = H / 2;
        const int half = grp;
        float *stage = reinterpret_cast<float *>(kv_tile);  // [H][512] f32 = H * 2 KiB <= 128 KiB
#pragma unroll 1
        for (int dc = 0; dc < 4; ++dc) {
            const int dd = dc * 128 + quarter * 32 + lane;
            float vals[HC];
            if (it > 0) {
                const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + Cfg::kColO + dc * H + half * HC;
                if (HC == 32) {
                    uint32_t r32[32];
                    tmem_ld32(ta, r32);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < HC; ++i) vals[i] = __uint_as_float(r32[i % 32]);
                } else if (HC == 16) {
                    uint32_t r16[16];
                    tmem_ld16(ta, r16);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < HC; ++i) vals[i] = __uint_as_float(r16[i % 16]);
                } else {
                    uint32_t r8[8];
                    tmem_ld8(ta, r8);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < HC; ++i) vals[i] = __uint_as_float(r8[i % 8]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < HC; ++i) vals[i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < HC; ++i) stage[(half * HC + i) * CSA2_D + dd] = vals[i] * alpha[half * HC + i];
        }
        __syncthreads();
        if (p.n_splits == 1) {
            uint4 *dst = reinterpret_cast<uint4 *>(p.o + (int64_t)u * H * CSA2_D);
            for (int i = tid; i < H * CSA2_D / 8; i += kAttnThreads) {
                const float4 x0 = reinterpret_cast<const float4 *>(stage)[2 * i];
                const float4 x1 = reinterpret_cast<const float4 *>(stage)[2 * i + 1];
                dst[i] = make_uint4((uint32_t)f32_to_bf16_bits(x0.x) | ((uint32_t)f32_to_bf16_bits(x0.y) << 16),
                                    (uint32_t)f32_to_bf16_bits(x0.z) | ((uint32_t)f32_to_bf16_bits(x0.w) << 16),
                                    (uint32_t)f32_to_bf16_bits(x1.x) | ((uint32_t)f32_to_bf16_bits(x1.y) << 16),
                                    (uint32_t)f32_to_bf16_bits(x1.z) | ((uint32_t)f32_to_bf16_bits(x1.w) << 16));
            }
        } else {
            float4 *dst = reinterpret_cast<float4 *>(p.o_part + ((int64_t)u * p.n_splits + split) * H * CSA2_D);
            for (int i = tid; i < H * CSA2_D / 4; i += kAttnThreads) dst[i] = reinterpret_cast<const float4 *>(stage)[i];
        }
        if (tid < H) {
            const float l = l_run[tid];
            const float lse = l > 0.0f ? (m_run[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
            if (p.n_splits == 1) {
                if (p.lse) p.lse[(int64_t)u * H + tid] = lse;
            } else {
                p.lse_part[((int64_t)u * p.n_splits + split) * H + tid] = lse;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

// Merge the splits of each query: o = sum_s exp(lse_s - M) o_s / L,
// lse = M + log L with M = max_s lse_s, L = sum_s exp(lse_s - M).
// One CTA per (query, 4 heads); each thread owns one float4 of a head and
// loads that float4 of every split before combining, so the loads overlap.
constexpr int kCombineThreads = 128;
constexpr int kCombineHeads = 1;  // heads per CTA (128 float4 per head)
constexpr int kCombineBatch = 8;  // split loads in flight per thread

template <int H>
__global__ void __launch_bounds__(kCombineThreads) k_attn_combine(const float *__restrict__ o_part,
                                                                  const float *__restrict__ lse_part,
                                                                  uint16_t *__restrict__ o, float *__restrict__ lse,
                                                                  int32_t n_splits) {
    extern __shared__ float wsm[];  // [n_splits + 1]
    pdl_trigger();
    pdl_wait();
    const int32_t u = blockIdx.y;
    const int h = blockIdx.x;
    const int d4 = threadIdx.x;  // 128 threads x 4 values = 512
    if (threadIdx.x < 32) {
        float M = -INFINITY;
        for (int s = threadIdx.x; s < n_splits; s += 32) M = fmaxf(M, lse_part[((int64_t)u * n_splits + s) * H + h]);
#pragma unroll
        for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        float L = 0.0f;
        for (int s = threadIdx.x; s < n_splits; s += 32) {
            const float ls = lse_part[((int64_t)u * n_splits + s) * H + h];
            const float w = (M == -INFINITY) ? 0.0f : expf(ls - M);
            wsm[s] = w;
            L += w;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
        if (threadIdx.x == 0) {
            wsm[n_splits] = L;
            if (lse) lse[(int64_t)u * H + h] = L > 0.0f ? M + logf(L) : -INFINITY;
        }
    }
    __syncthreads();
    const float *src = o_part + ((int64_t)u * n_splits * H + h) * CSA2_D;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_splits; s0 += kCombineBatch) {
        float4 v[kCombineBatch];
#pragma unroll
        for (int t = 0; t < kCombineBatch; ++t)
            v[t] = (s0 + t < n_splits)
                       ? __ldg(reinterpret_cast<const float4 *>(src + (int64_t)(s0 + t) * H * CSA2_D) + d4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int t = 0; t < kCombineBatch; ++t) {
            if (s0 + t >= n_splits) break;
            const float w = wsm[s0 + t];
            acc.x = fmaf(w, v[t].x, acc.x);
            acc.y = fmaf(w, v[t].y, acc.y);
            acc.z = fmaf(w, v[t].z, acc.z);
            acc.w = fmaf(w, v[t].w, acc.w);
        }
    }
    const float L = wsm[n_splits];
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    uint16_t *dst = o + ((int64_t)u * H + h) * CSA2_D + d4 * 4;
    const uint32_t lo = (uint32_t)f32_to_bf16_bits(acc.x * inv) | ((uint32_t)f32_to_bf16_bits(acc.y * inv) << 16);
    const uint32_t hi = (uint32_t)f32_to_bf16_bits(acc.z * inv) | ((uint32_t)f32_to_bf16_bits(acc.w * inv) << 16);
    *reinterpret_cast<uint2 *>(dst) = make_uint2(lo, hi);
}

}  // namespace csa2
