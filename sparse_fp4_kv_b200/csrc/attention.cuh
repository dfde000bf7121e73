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
//   1. all 8 warps gather the tile: a warp per row, 16 values per lane; FP4
//      codes are widened with cvt.rn.f16x2.e2m1x2 and multiplied by the
//      block scale (exact in f16), window bytes with cvt.rn.f16x2.e4m3x2;
//      the f16 tile lands in shared memory in the 128B-swizzled K-major
//      layout (rows = entries, 64-value column blocks 16 KiB apart).
//   2. one thread issues S^T = KV * Q^T with tcgen05.mma kind::f16
//      (M = 128 rows, N = H heads, K = 512) into TMEM.
//   3. warps 0..3 (one TMEM lane quarter each, a thread per row) read S^T,
//      reduce the per-head tile maximum across the 128 rows (transposed
//      butterfly + shared memory), run the online softmax in base 2 and
//      write P^T (f16) into a swizzled M/N-major tile.
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
    static constexpr int kMisc = 128 * 4 /*valid*/ + 4 * H * 4 /*red*/ + 2 * H * 4 /*m, alpha*/ + H * 4 /*l*/ +
                                 64 /*bars, slot, flags*/;
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

template <int H>
__device__ __forceinline__ void store_warp_reduced(float *dst /*[H]*/, const float (&v)[H]) {
    const int lane = threadIdx.x & 31;
    if (H == 64) {
        dst[2 * lane] = v[0];
        dst[2 * lane + 1] = v[1];
    } else if (H == 32) {
        dst[lane] = v[0];
    } else {
        if ((lane & 1) == 0) dst[lane >> 1] = v[0];
    }
}

// Gather + dequantise one attended row into the f16 tile (whole warp).
__device__ __forceinline__ bool gather_row(const AttnParams &p, int32_t u, int32_t b, int32_t nw, int32_t wb,
                                           int64_t j, int e, uint8_t *kv_tile) {
    const int lane = threadIdx.x & 31;
    uint32_t h0[4] = {0u, 0u, 0u, 0u}, h1[4] = {0u, 0u, 0u, 0u};
    bool valid = false;
    if (j < p.k) {
        const int32_t id = p.topk[(int64_t)u * p.k + j];
        if (id >= 0) {
            const int64_t row = physical_row(p.kv, b, id);
            if (row >= 0) {
                valid = true;
                const uint2 cw = __ldg(reinterpret_cast<const uint2 *>(p.kv.codes + row * (CSA2_D / 2)) + lane);
                const uint32_t s = __ldg(p.kv.scales + row * (CSA2_D / CSA2_BLOCK) + lane);
                const uint32_t s2 = e4m3x2_to_f16x2((uint16_t)(s | (s << 8)));
                e2m1x8_to_f16x8(cw.x, h0);
                e2m1x8_to_f16x8(cw.y, h1);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    h0[i] = hmul2_u32(h0[i], s2);
                    h1[i] = hmul2_u32(h1[i], s2);
                }
            } else if (lane == 0) {
                set_error(CSA2_DEVERR_BAD_ROW);
            }
        }
    } else if (j < (int64_t)p.k + nw) {
        valid = true;
        const int64_t r = (int64_t)b * p.swa_seq_stride + wb + (j - p.k);
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.swa + r * CSA2_D) + lane);
        h0[0] = e4m3x2_to_f16x2((uint16_t)(v.x & 0xFFFFu));
        h0[1] = e4m3x2_to_f16x2((uint16_t)(v.x >> 16));
        h0[2] = e4m3x2_to_f16x2((uint16_t)(v.y & 0xFFFFu));
        h0[3] = e4m3x2_to_f16x2((uint16_t)(v.y >> 16));
        h1[0] = e4m3x2_to_f16x2((uint16_t)(v.z & 0xFFFFu));
        h1[1] = e4m3x2_to_f16x2((uint16_t)(v.z >> 16));
        h1[2] = e4m3x2_to_f16x2((uint16_t)(v.w & 0xFFFFu));
        h1[3] = e4m3x2_to_f16x2((uint16_t)(v.w >> 16));
    }
    *reinterpret_cast<uint4 *>(kv_tile + kv_chunk_off(e, 2 * lane)) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
    *reinterpret_cast<uint4 *>(kv_tile + kv_chunk_off(e, 2 * lane + 1)) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
    return valid;
}

template <int H>
__global__ void __launch_bounds__(kAttnThreads, 1) k_sparse_attn(AttnParams p) {
    using Cfg = AttnCfg<H>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *kv_tile = base;
    uint8_t *q_tile = kv_tile + Cfg::kKvBytes;
    uint8_t *p_tile = q_tile + Cfg::kQBytes;
    int32_t *valid_s = reinterpret_cast<int32_t *>(p_tile + Cfg::kPBytes);
    float *red = reinterpret_cast<float *>(valid_s + kAttnTile);  // [4][H]
    float *m_run = red + 4 * H;
    float *alpha = m_run + H;
    float *l_fin = alpha + H;
    uint64_t *bar_s = reinterpret_cast<uint64_t *>(l_fin + H);
    uint64_t *bar_o = bar_s + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_o + 1);
    int32_t *rescale_tile = reinterpret_cast<int32_t *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t split = blockIdx.x, u = blockIdx.y;
    const int32_t b = u / p.q_per_seq;
    const int32_t wb = p.swa_begin ? p.swa_begin[u] : 0;
    const int32_t nw = p.swa_begin ? max(0, p.swa_end[u] - wb) : 0;
    const int64_t n_total = (int64_t)p.k + nw;
    const int64_t tiles_total = (n_total + kAttnTile - 1) / kAttnTile;
    const int64_t t_begin = (int64_t)split * p.tiles_per_split;
    const int64_t t_end = min(tiles_total, t_begin + p.tiles_per_split);

    // ---- set-up: TMEM, barriers, Q tile (bf16 -> f16, K-major SW128) ----
    if (warp == 0) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        *rescale_tile = -1;
        fence_mbar_init();
    }
    if (tid < H) m_run[tid] = -INFINITY;
    {
        const uint4 *qsrc = reinterpret_cast<const uint4 *>(p.q + (int64_t)u * H * CSA2_D);
        for (int i = tid; i < H * (CSA2_D / 8); i += kAttnThreads) {
            const int h = i / (CSA2_D / 8), c64 = i % (CSA2_D / 8);
            const uint4 v = __ldg(qsrc + i);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            uint32_t o4[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float lo = __uint_as_float(w4[t] << 16), hi = __uint_as_float(w4[t] & 0xFFFF0000u);
                const __half2 hh = __floats2half2_rn(lo, hi);
                o4[t] = *reinterpret_cast<const uint32_t *>(&hh);
            }
            *reinterpret_cast<uint4 *>(q_tile + q_chunk_off<H>(h, c64)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t kv_addr = smem_u32(kv_tile), q_addr = smem_u32(q_tile), p_addr = smem_u32(p_tile);

    float l_part[H];  // per-row partial softmax denominators (warps 0..3)
#pragma unroll
    for (int h = 0; h < H; ++h) l_part[h] = 0.0f;

    bool ok = true;
    int it = 0;
    for (int64_t tt = t_begin; tt < t_end && ok; ++tt, ++it) {
        const int64_t j0 = tt * kAttnTile;
        // 1. gather + dequantise the tile (16 rows per warp)
        for (int r = 0; r < kAttnTile / 8; ++r) {
            const int e = warp * (kAttnTile / 8) + r;
            const bool v = gather_row(p, u, b, nw, wb, j0 + e, e, kv_tile);
            if (lane == 0) valid_s[e] = v ? 1 : 0;
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
        if (warp < 4) {
            // 3. online softmax, one row per thread
            const bool got = mbar_wait(bar_s, it & 1);
            tc_fence_after();
            float s[H];
#pragma unroll
            for (int c = 0; c < H; c += (H >= 32 ? 32 : 16)) {
                if (H >= 32) {
                    uint32_t r32[32];
                    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + Cfg::kColS + c, r32);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c + i] = __uint_as_float(r32[i]);
                } else {
                    uint32_t r16[16];
                    tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + Cfg::kColS + c, r16);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) s[c + i] = __uint_as_float(r16[i]);
                }
            }
            const bool row_valid = valid_s[tid] != 0 && got;
#pragma unroll
            for (int h = 0; h < H; ++h) s[h] = row_valid ? s[h] * p.scale_log2 : -INFINITY;
            float mx[H];
#pragma unroll
            for (int h = 0; h < H; ++h) mx[h] = s[h];
            warp_transpose_reduce<H, true>(mx);
            store_warp_reduced<H>(red + warp * H, mx);
            named_bar_sync(1, 128);
            if (tid < H) {
                const float mt = fmaxf(fmaxf(red[tid], red[H + tid]), fmaxf(red[2 * H + tid], red[3 * H + tid]));
                const float mo = m_run[tid];
                float a = 1.0f, mn = mo;
                if (mt > mo + kRescaleThreshold || (mo == -INFINITY && mt > -INFINITY)) {
                    mn = mt;
                    a = (mo == -INFINITY) ? 0.0f : exp2f(mo - mt);
                    if (mo != -INFINITY) *rescale_tile = (int32_t)it;
                }
                m_run[tid] = mn;
                alpha[tid] = a;
            }
            named_bar_sync(1, 128);
            // probabilities -> P^T (f16), partial denominators
#pragma unroll
            for (int c = 0; c < H / 8; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int h = 8 * c + 2 * t;
                    const float m0 = m_run[h], m1 = m_run[h + 1];
                    const float p0 = (m0 == -INFINITY) ? 0.0f : exp2f(s[h] - m0);
                    const float p1 = (m1 == -INFINITY) ? 0.0f : exp2f(s[h + 1] - m1);
                    l_part[h] = fmaf(l_part[h], alpha[h], p0);
                    l_part[h + 1] = fmaf(l_part[h + 1], alpha[h + 1], p1);
                    const __half2 hh = __floats2half2_rn(p0, p1);
                    pk[t] = *reinterpret_cast<const uint32_t *>(&hh);
                }
                *reinterpret_cast<uint4 *>(p_tile + p_chunk_off<H>(tid, c)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            // rare: raise of the running maximum -> rescale O^T in TMEM
            if (*rescale_tile == it) {
#pragma unroll 1
                for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                    for (int c = 0; c < H; c += 16) {
                        uint32_t r16[16];
                        const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + Cfg::kColO + dc * H + c;
                        tmem_ld16(ta, r16);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) r16[i] = __float_as_uint(__uint_as_float(r16[i]) * alpha[c + i]);
                        tmem_st16(ta, r16);
                    }
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            if (!got) ok = false;
            // 4. O^T += V^T * P^T
            if (tid == 0 && ok) {
                tc_fence_after();
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
        }
        // the next tile overwrites KV / P: wait for this tile's P*V
        if (ok && !mbar_wait(bar_o, it & 1)) ok = false;
        tc_fence_after();
        ok = __syncthreads_and(ok);
    }

    // ---- final denominators ----
    if (warp < 4) {
        warp_transpose_reduce<H, false>(l_part);
        store_warp_reduced<H>(red + warp * H, l_part);
    }
    __syncthreads();
    if (tid < H) l_fin[tid] = (red[tid] + red[H + tid]) + (red[2 * H + tid] + red[3 * H + tid]);
    __syncthreads();

    // ---- epilogue: O^T (TMEM) -> o = O / l ----
    {
        const int quarter = warp & 3, half = warp >> 2;
        constexpr int HC = H / 2;
        const bool single = p.n_splits == 1;
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
            for (int i = 0; i < HC; ++i) {
                const int h = half * HC + i;
                const float l = l_fin[h];
                const float o = l > 0.0f ? vals[i] / l : 0.0f;
                if (single) {
                    p.o[((int64_t)u * H + h) * CSA2_D + dd] = f32_to_bf16_bits(o);
                } else {
                    p.o_part[(((int64_t)u * p.n_splits + split) * H + h) * CSA2_D + dd] = o;
                }
            }
        }
        if (tid < H) {
            const float l = l_fin[tid];
            const float lse = l > 0.0f ? (m_run[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
            if (single) {
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
constexpr int kCombineThreads = 256;
constexpr int kCombineHeads = 4;  // heads per CTA

template <int H>
__global__ void __launch_bounds__(kCombineThreads) k_attn_combine(const float *__restrict__ o_part,
                                                                  const float *__restrict__ lse_part,
                                                                  uint16_t *__restrict__ o, float *__restrict__ lse,
                                                                  int32_t n_splits) {
    extern __shared__ float wsm[];  // [kCombineHeads][n_splits + 1]
    const int32_t u = blockIdx.y;
    const int h0 = blockIdx.x * kCombineHeads;
    if (threadIdx.x < kCombineHeads) {
        const int h = h0 + threadIdx.x;
        float M = -INFINITY;
        for (int s = 0; s < n_splits; ++s) M = fmaxf(M, lse_part[((int64_t)u * n_splits + s) * H + h]);
        float L = 0.0f;
        float *w = wsm + threadIdx.x * (n_splits + 1);
        for (int s = 0; s < n_splits; ++s) {
            const float ls = lse_part[((int64_t)u * n_splits + s) * H + h];
            w[s] = (M == -INFINITY) ? 0.0f : expf(ls - M);
            L += w[s];
        }
        w[n_splits] = L;
        if (lse) lse[(int64_t)u * H + h] = L > 0.0f ? M + logf(L) : -INFINITY;
    }
    __syncthreads();
    // kCombineHeads * 512 outputs, 4 consecutive per thread
    for (int i = threadIdx.x; i < kCombineHeads * CSA2_D / 4; i += kCombineThreads) {
        const int hl = i / (CSA2_D / 4), d4 = i % (CSA2_D / 4);
        const int h = h0 + hl;
        const float *w = wsm + hl * (n_splits + 1);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < n_splits; ++s) {
            if (w[s] == 0.0f) continue;
            const float4 v =
                __ldg(reinterpret_cast<const float4 *>(o_part + (((int64_t)u * n_splits + s) * H + h) * CSA2_D) + d4);
            acc.x = fmaf(w[s], v.x, acc.x);
            acc.y = fmaf(w[s], v.y, acc.y);
            acc.z = fmaf(w[s], v.z, acc.z);
            acc.w = fmaf(w[s], v.w, acc.w);
        }
        const float L = w[n_splits];
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        uint16_t *dst = o + ((int64_t)u * H + h) * CSA2_D + d4 * 4;
        const uint32_t lo = (uint32_t)f32_to_bf16_bits(acc.x * inv) | ((uint32_t)f32_to_bf16_bits(acc.y * inv) << 16);
        const uint32_t hi = (uint32_t)f32_to_bf16_bits(acc.z * inv) | ((uint32_t)f32_to_bf16_bits(acc.w * inv) << 16);
        *reinterpret_cast<uint2 *>(dst) = make_uint2(lo, hi);
    }
}

}  // namespace csa2
