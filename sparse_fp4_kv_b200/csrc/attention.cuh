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
// entries followed by its window rows), 128 rows per tile. The f16 tile is
// handled in four chunks of 128 latent columns (32 KiB each), so the work
// overlaps across chunks and tiles:
//   1. sixteen warps dequantise chunk c of tile t (raw bytes fetched into
//      registers one tile ahead) as soon as the P*V products of tile t-1 on
//      that chunk are done: FP4 codes widened with cvt.rn.f16x2.e2m1x2 and
//      multiplied by the block scale (exact in f16), window bytes widened with
//      cvt.rn.f16x2.e4m3x2, stored in the 128B-swizzled K-major layout;
//   2. one elected thread of a seventeenth warp issues S^T += KV_c * Q_c^T
//      (tcgen05.mma kind::f16, M = 128 rows, N = H heads) for each chunk as
//      soon as every thread has stored it, then commits S; meanwhile the
//      sixteen warps put the loads of tile t+1 in flight;
//   3. the warps (a thread per row, up to four head groups) run the online
//      softmax in base 2 on S^T from TMEM and write P^T (f16). The running
//      maximum is only raised when some score exceeds it by more than 2^8, so
//      the common case needs no tile maximum: one vote per head group decides;
//      a raise takes the full path (tile maximum, rescale of O^T in TMEM);
//   4. the same thread issues O^T += V^T * P^T chunk by chunk (A = the same KV
//      chunk read M/N-major, B = P^T), committing each chunk separately so
//      step 1 of the next tile can reuse it at once.
// Probabilities stay below 2^8 and are exact in range for f16.
// Splits of one query are merged by k_attn_combine with their
// log-sum-exp values.
//
// NVFP4 variant (NV = true, 64 heads): q is rounded to NVFP4 beforehand
// (k_quant_rows_nvfp4). Splits made only of whole tiles of selected entries
// store each tile's raw FP4 codes into a K-major A tile and its E4M3 block
// scales into TMEM as scale factors, and S^T comes from block-scaled FP4
// products (kind::mxf4nvf4) without waiting for the dequantisation, which
// still feeds P*V. The remaining tiles (a partial last entry tile, the
// window) take the path above with the rounded q in f16.
#pragma once

#include "append.cuh"
#include "common.cuh"

namespace csa2 {

constexpr int kAttnWorkWarps = 16;                     // dequantise, softmax, epilogue
constexpr int kAttnWorkThreads = kAttnWorkWarps * 32;
constexpr int kAttnThreads = kAttnWorkThreads + 32;  // + the warp that issues the tensor-core products
constexpr int kMmaWarp = kAttnWorkWarps;
constexpr uint32_t kBarWork = 5;                      // named barrier of the work warps (1..4: head groups)
constexpr int kAttnTile = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int H, bool NV = false>
struct AttnCfg {
    static constexpr int kKvBytes = kAttnTile * CSA2_D * 2;  // 128 KiB f16 tile
    static constexpr int kQBytes = H * CSA2_D * 2;
    // NVFP4 variant: the Q region holds, in splits of selected entries, the
    // raw FP4 codes of the tile and of q (K-major, 128B-swizzled) and the
    // staging of their scale bytes (rows padded to 36 bytes); in window
    // splits it holds the f16 Q tile as above.
    static constexpr int kRawBytes = kAttnTile * CSA2_D / 2;
    static constexpr int kQ4Bytes = H * CSA2_D / 2;
    static constexpr int kStage = 36;
    static constexpr int kStageBytes = kAttnTile * kStage;
    static constexpr int kQStageBytes = H * kStage;
    static constexpr int kNvBytes = kRawBytes + kQ4Bytes + kStageBytes + kQStageBytes;
    static constexpr int kQRegion = NV ? ((kNvBytes > kQBytes ? kNvBytes : kQBytes) + 1023) / 1024 * 1024 : kQBytes;
    static constexpr int kPBytes = kAttnTile * H * 2;
    static constexpr int kPGroup = 16 * H;  // bytes of 8 rows of P^T
    static constexpr uint32_t kPSwizzle = H == 64 ? kSw128 : (H == 32 ? kSw64 : kSw32);
    static constexpr int kColS = 0;
    static constexpr int kColO = H;
    static constexpr int kColSFA = 5 * H;       // NV: scale factors of the tile rows, 4 columns per K step
    static constexpr int kColSFB = 5 * H + 32;  // NV: scale factors of q, H / 32 columns per K step
    static constexpr uint32_t kTmemCols = H == 64 ? 512u : (H == 32 ? 256u : 128u);
    static constexpr int kMisc = 8 * 128 * 5 /*resolved rows*/ + (NV ? 2 : 1) * 128 * 4 /*valid*/ +
                                 4 * H * 4 /*red*/ + 3 * H * 4 /*m, alpha, l*/ + 128 /*bars, slot, flags*/;
    static constexpr size_t kSmem = 1024 + (size_t)kKvBytes + kQRegion + kPBytes + kMisc;
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
    int32_t out_f32;   // write normalised f32 o (o_part, S = 1) instead of bf16 o
    // NVFP4 variant: splits [0, e_splits) take tp_e tiles each of the first
    // e_tiles tiles (selected entries only) with FP4 products for S; the other
    // splits take tiles_per_split tiles each from tile e_tiles on.
    int32_t e_splits, e_tiles, tps_e;
    uint8_t *q4;   // NV: q in NVFP4, codes [nq][H][256] (element i in nibble i & 1 of byte i / 2)
    uint8_t *q4s;  // NV: its E4M3 block scales [nq][H][32]
};

// NVFP4 variant, before the attention kernel: every 16-value block of q
// quantised with the cache's block quantiser, a thread per block.
constexpr int kQuantThreads = 256;
__global__ void __launch_bounds__(kQuantThreads)
    k_quant_rows_nvfp4(const uint16_t *__restrict__ x, int32_t n_blocks, uint8_t *__restrict__ codes,
                       uint8_t *__restrict__ scales) {
    pdl_trigger();
    pdl_wait();
    const int32_t i = blockIdx.x * kQuantThreads + threadIdx.x;
    if (i >= n_blocks) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)i * CSA2_BLOCK);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        f[2 * j] = __uint_as_float(w8[j] << 16);
        f[2 * j + 1] = __uint_as_float(w8[j] & 0xFFFF0000u);
    }
    uint32_t pk[2];
    const uint32_t sc = quantize_block16(f, pk);
    *reinterpret_cast<uint2 *>(codes + (int64_t)i * 8) = make_uint2(pk[0], pk[1]);
    scales[i] = (uint8_t)sc;
}

// NVFP4 variant with fewer than 64 heads: the call runs as a 64-head problem
// (the one shape whose block-scaled products are validated) with q padded by
// zero heads; the padded heads' outputs are dropped. 16-byte pieces, a
// thread each.
__global__ void k_pad_heads(const uint4 *__restrict__ src, int32_t h, int32_t nq, uint4 *__restrict__ dst) {
    pdl_trigger();
    pdl_wait();
    constexpr int kPiecesPerHead = CSA2_D * 2 / 16;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // piece of the padded q
    if (i >= (int64_t)nq * 64 * kPiecesPerHead) return;
    const int64_t u = i / (64 * kPiecesPerHead);
    const int hh = (int)((i / kPiecesPerHead) % 64), c = (int)(i % kPiecesPerHead);
    dst[i] = hh < h ? src[(u * h + hh) * kPiecesPerHead + c] : make_uint4(0u, 0u, 0u, 0u);
}
__global__ void k_unpad_heads(const uint4 *__restrict__ src, const float *__restrict__ lse_src, int32_t h, int32_t nq,
                              uint4 *__restrict__ dst, float *__restrict__ lse_dst) {
    pdl_trigger();
    pdl_wait();
    constexpr int kPiecesPerHead = CSA2_D * 2 / 16;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // piece of the unpadded o
    if (i >= (int64_t)nq * h * kPiecesPerHead) return;
    const int64_t u = i / (h * kPiecesPerHead);
    const int hh = (int)((i / kPiecesPerHead) % h), c = (int)(i % kPiecesPerHead);
    dst[i] = src[(u * 64 + hh) * kPiecesPerHead + c];
    if (lse_dst != nullptr && c == 0) lse_dst[u * h + hh] = lse_src[u * 64 + hh];
}

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
// Tile gather: each work warp owns 8 rows of the 128-row tile. For latent
// chunk c (128 columns) lane l holds columns 128c + 16(l%8) .. +15 of rows
// 4j + l/8 (j = 0, 1), so every lane takes part in every chunk's
// dequantisation. All 8 loads of a lane are issued back to back; the raw
// bytes stay in registers until the chunk's f16 slot is free again, which
// lets the loads of tile t+1 run under the tensor-core work of tile t.
// ---------------------------------------------------------------------------
constexpr int kRowsPerWarp = kAttnTile / kAttnWorkWarps;  // 8
constexpr int kRowGroups = kRowsPerWarp / 4;                // rows of a lane per chunk
constexpr int kResolveTiles = 8;  // rows resolved per batch: 8 tiles = 1024 rows

struct TileRaw {
    uint4 v[4 * kRowGroups];  // [chunk * kRowGroups + j]: FP4 piece {codes lo, codes hi, scale byte, 0};
                              // window piece: 16 E4M3 bytes
    uint32_t kinds;  // 2 bits per j: 0 empty, 1 FP4 global entry, 2 window row
};

// Resolve the sources of rows [j0, j0 + n) (n <= kResolveTiles * 128) of the
// query's attended list into shared memory: physical FP4 row (kind 1), window
// buffer row (kind 2) or nothing (kind 0). The work warps take part; thread t
// takes rows t and t + 512. id_pre (nullable) holds those rows' entry ids
// already loaded; pt0 is the sequence's page when the cache has one page per
// sequence (one_page), so that no row waits for a page-table load.
constexpr int kResolvePerThread = kResolveTiles * kAttnTile / kAttnWorkThreads;  // 2
__device__ __forceinline__ void resolve_rows(const AttnParams &p, int32_t u, int32_t b, int32_t nw, int32_t wb,
                                             int64_t j0, int n, int32_t *rsrc, uint8_t *rkind,
                                             const int32_t (*id_pre)[kResolvePerThread], bool one_page, int64_t pt0) {
#pragma unroll
    for (int r = 0; r < kResolvePerThread; ++r) {
        const int i = threadIdx.x + r * kAttnWorkThreads;
        if (i >= n) break;
        const int64_t j = j0 + i;
        int32_t src = 0;
        uint8_t kind = 0;
        if (j < p.k) {
            const int32_t id = id_pre ? (*id_pre)[r] : p.topk[(int64_t)u * p.k + j];
            if (id >= 0) {
                int64_t row;
                if (one_page) {
                    // physical_row with the one page of the sequence already loaded
                    row = (id < p.kv.page_size && pt0 >= 0) ? pt0 * p.kv.page_size + id : -1;
                    if (row >= p.kv.rows_cap) row = -1;
                } else {
                    row = physical_row(p.kv, b, id);
                }
                if (row >= 0) {
                    src = (int32_t)row;
                    kind = 1;
                } else {
                    set_error(CSA2_DEVERR_BAD_ROW);
                }
            }
        } else if (j < (int64_t)p.k + nw) {
            int64_t slot = wb + (j - p.k);  // < 2 * stride
            if (slot >= p.swa_seq_stride) slot -= p.swa_seq_stride;
            src = (int32_t)slot;
            kind = 2;
        }
        rsrc[i] = src;
        rkind[i] = kind;
    }
}

// Issue the loads of latent chunks [C0, C1) of one tile's rows (resolved
// sources at rsrc/rkind + off).
template <int C0, int C1>
__device__ __forceinline__ void fetch_tile(const AttnParams &p, int32_t b, const int32_t *rsrc, const uint8_t *rkind,
                                           int off, TileRaw &raw) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int piece = lane & 7;
    const uint8_t *swa_seq = p.swa ? p.swa + (int64_t)b * p.swa_seq_stride * CSA2_D : nullptr;
    raw.kinds = 0;
#pragma unroll
    for (int j = 0; j < kRowGroups; ++j) {
        const int r = off + warp * kRowsPerWarp + 4 * j + (lane >> 3);
        const int64_t src = rsrc[r];
        const uint32_t kd = rkind[r];
        raw.kinds |= kd << (2 * j);
#pragma unroll
        for (int c = C0; c < C1; ++c) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (kd == 1) {
                const uint2 cc =
                    __ldg(reinterpret_cast<const uint2 *>(p.kv.codes + src * (CSA2_D / 2) + c * 64 + piece * 8));
                v = make_uint4(cc.x, cc.y, (uint32_t)__ldg(p.kv.scales + src * (CSA2_D / CSA2_BLOCK) + c * 8 + piece),
                               0u);
            } else if (kd == 2) {
                v = __ldg(reinterpret_cast<const uint4 *>(swa_seq + src * CSA2_D + c * 128 + piece * 16));
            }
            raw.v[c * kRowGroups + j] = v;
        }
    }
}

// Dequantise latent chunk c of the fetched rows into the f16 tile
// (128B-swizzled K-major); chunk 0 also records which rows hold data. Lanes
// of pieces 4..7 store their second 16-byte half first, so the eight lanes
// of each store phase hit eight different bank groups.
__device__ __forceinline__ void store_chunk(const TileRaw &raw, int c, uint8_t *kv_tile, int32_t *valid_s,
                                            bool write_valid = true) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int piece = lane & 7;
#pragma unroll
    for (int j = 0; j < kRowGroups; ++j) {
        const uint32_t kd = (raw.kinds >> (2 * j)) & 3u;
        const uint4 v = raw.v[c * kRowGroups + j];
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
        const int e = warp * kRowsPerWarp + 4 * j + (lane >> 3);
        const int c64 = 16 * c + 2 * piece;
        const bool swap = piece >= 4;
        const uint4 first = swap ? make_uint4(h1[0], h1[1], h1[2], h1[3]) : make_uint4(h0[0], h0[1], h0[2], h0[3]);
        const uint4 second = swap ? make_uint4(h0[0], h0[1], h0[2], h0[3]) : make_uint4(h1[0], h1[1], h1[2], h1[3]);
        *reinterpret_cast<uint4 *>(kv_tile + kv_chunk_off(e, c64 + (swap ? 1 : 0))) = first;
        *reinterpret_cast<uint4 *>(kv_tile + kv_chunk_off(e, c64 + (swap ? 0 : 1))) = second;
        if (write_valid && c == 0 && piece == 0) valid_s[e] = kd != 0u;
    }
}

// NVFP4 variant: the raw FP4 codes of the fetched rows (selected entries or
// empty) into the K-major 128B-swizzled A tile of the block-scaled product,
// their scale bytes into the staging rows, and which rows hold data.
template <int STAGE>
__device__ __forceinline__ void store_raw(const TileRaw &raw, uint8_t *raw_tile, uint8_t *stage, int32_t *valid_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int piece = lane & 7;
#pragma unroll
    for (int j = 0; j < kRowGroups; ++j) {
        const uint32_t kd = (raw.kinds >> (2 * j)) & 3u;
        const int e = warp * kRowsPerWarp + 4 * j + (lane >> 3);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 v = raw.v[c * kRowGroups + j];
            const bool fp4 = kd == 1u;
            const int blk = 8 * c + piece;
            const uint32_t off = (uint32_t)((blk >> 4) * 16384 + (e >> 3) * 1024 + (e & 7) * 128 +
                                            ((((blk & 15) >> 1) ^ (e & 7)) << 4) + (blk & 1) * 8);
            *reinterpret_cast<uint2 *>(raw_tile + off) = fp4 ? make_uint2(v.x, v.y) : make_uint2(0u, 0u);
            stage[e * STAGE + blk] = fp4 ? (uint8_t)(v.z & 0xFFu) : (uint8_t)0;
        }
        if (piece == 0) valid_s[e] = kd == 1u;
    }
}

// OR of `pred` over the `n` threads of named barrier `id`.
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0u;
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

template <int H, bool NV>
__global__ void __launch_bounds__(kAttnThreads, 1) k_sparse_attn(AttnParams p) {
    using Cfg = AttnCfg<H, NV>;
    static_assert(!NV || H == 64, "the NVFP4 variant runs its S product at N = 64");
    constexpr int G = H >= 32 ? 4 : 2;  // softmax head groups (4 warps each, a warp per TMEM lane quarter)
    constexpr int HG = H / G;            // heads per group
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *kv_tile = base;
    uint8_t *q_tile = kv_tile + Cfg::kKvBytes;
    uint8_t *p_tile = q_tile + Cfg::kQRegion;
    int32_t *rsrc = reinterpret_cast<int32_t *>(p_tile + Cfg::kPBytes);  // [kResolveTiles * 128]
    uint8_t *rkind = reinterpret_cast<uint8_t *>(rsrc + kResolveTiles * kAttnTile);
    int32_t *valid_s = reinterpret_cast<int32_t *>(rkind + kResolveTiles * kAttnTile);
    float *red = reinterpret_cast<float *>(valid_s + (NV ? 2 : 1) * kAttnTile);  // [4][H]
    float *m_run = red + 4 * H;
    float *alpha = m_run + H;
    float *l_run = alpha + H;
    uint64_t *bar_kv = reinterpret_cast<uint64_t *>(l_run + H);  // [4] chunk c of the tile stored
    uint64_t *bar_pv = bar_kv + 4;                               // [4] P*V of chunk c done
    uint64_t *bar_s = bar_pv + 4;                                // S^T of the tile ready
    uint64_t *bar_p = bar_s + 1;                                 // P^T of the tile written
    uint64_t *bar_raw = bar_p + 1;                               // NV: raw FP4 tile + scale factors stored
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_raw + 1);
    int32_t *rescale_tile = reinterpret_cast<int32_t *>(tmem_slot + 1);  // [4] (per head group)

    uint8_t *raw_tile = q_tile;                 // NV, entry splits
    uint8_t *q4_tile = q_tile + Cfg::kRawBytes;
    uint8_t *stage = q4_tile + Cfg::kQ4Bytes;
    uint8_t *qstage = stage + Cfg::kStageBytes;

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
        for (int c = 0; c < 4; ++c) {
            mbar_init(&bar_kv[c], kAttnWorkThreads);
            mbar_init(&bar_pv[c], 1);
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_p, kAttnWorkThreads);
        if (NV) mbar_init(bar_raw, kAttnWorkThreads);
        rescale_tile[0] = rescale_tile[1] = rescale_tile[2] = rescale_tile[3] = -1;
        fence_mbar_init();
    }
    if (tid < H) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.0f;
    }
    pdl_wait();
    // NV: an entry split (FP4 products for S) or a split from tile e_tiles on
    const bool fp4 = NV && split < p.e_splits;
    const int64_t t_begin = fp4 ? (int64_t)split * p.tps_e
                                : (NV ? (int64_t)p.e_tiles : 0) +
                                      (int64_t)(NV ? split - p.e_splits : split) * p.tiles_per_split;
    // the entry ids of the first resolved rows and, for a cache with one page per
    // sequence, that page go in flight together with the window bounds
    const bool one_page = p.kv.max_pages == 1;
    int64_t pt0 = 0;
    int32_t id_pre[kResolvePerThread];
#pragma unroll
    for (int r = 0; r < kResolvePerThread; ++r) id_pre[r] = -1;
    if (tid < kAttnWorkThreads) {
#pragma unroll
        for (int r = 0; r < kResolvePerThread; ++r) {
            const int64_t j = t_begin * kAttnTile + tid + r * kAttnWorkThreads;
            if (j < p.k) id_pre[r] = p.topk[(int64_t)u * p.k + j];
        }
        if (one_page) pt0 = p.kv.page_table[b];
    }
    const int32_t wb = p.swa_begin ? p.swa_begin[u] : 0;
    int32_t nw = p.swa_begin ? max(0, p.swa_end[u] - wb) : 0;
    // the window is a run of ring slots: begin in [0, stride), at most stride rows
    if (nw > 0 && (wb < 0 || wb >= p.swa_seq_stride || nw > p.swa_seq_stride)) {
        if (tid == 0) set_error(CSA2_DEVERR_BAD_ROW);
        nw = 0;
    }
    const int64_t n_total = (int64_t)p.k + nw;
    const int64_t tiles_total = (n_total + kAttnTile - 1) / kAttnTile;
    const int64_t t_end = fp4 ? min((int64_t)p.e_tiles, t_begin + p.tps_e) : min(tiles_total, t_begin + p.tiles_per_split);
    const int ntiles = (int)max((int64_t)0, t_end - t_begin);

    // ---- prologue: Q loads in flight first, then resolve the first rows and
    //      start their loads, then Q (bf16 -> f16) into the K-major
    //      128B-swizzled B tile ----
    TileRaw raw;
    raw.kinds = 0;
    const bool mma_warp = warp == kMmaWarp;
    if (!mma_warp) {
        const uint4 *qsrc = reinterpret_cast<const uint4 *>(p.q + (int64_t)u * H * CSA2_D);
        constexpr int kChunks = H * (CSA2_D / 8);
        constexpr int kPer = kChunks / kAttnWorkThreads;  // 8 / 4 / 2 for H = 64 / 32 / 16
        uint4 qv[kPer];
        if (NV) {
            // NVFP4 q from the pre-pass: block b = tid + t * threads (codes, scale)
#pragma unroll
            for (int t = 0; t < kPer / 2; ++t) {
                const int bq = tid + t * kAttnWorkThreads;
                const uint2 cc = *reinterpret_cast<const uint2 *>(p.q4 + ((int64_t)u * H * 32 + bq) * 8);
                qv[t] = make_uint4(cc.x, cc.y, (uint32_t)p.q4s[(int64_t)u * H * 32 + bq], 0u);
            }
        } else {
#pragma unroll
            for (int t = 0; t < kPer; ++t) qv[t] = __ldg(qsrc + tid + t * kAttnWorkThreads);
        }
        if (ntiles > 0)
            resolve_rows(p, u, b, nw, wb, t_begin * kAttnTile, min(kResolveTiles, ntiles) * kAttnTile, rsrc, rkind,
                         &id_pre, one_page, pt0);
        named_bar_sync(kBarWork, kAttnWorkThreads);
        if (ntiles > 0) fetch_tile<0, 4>(p, b, rsrc, rkind, 0, raw);
        if constexpr (NV) {
            // q in NVFP4: FP4 codes + scale staging for entry splits, its exact
            // f16 values for window splits
#pragma unroll
            for (int t = 0; t < kPer / 2; ++t) {
                const int bq = tid + t * kAttnWorkThreads;
                const int h = bq >> 5, blk = bq & 31;
                const uint32_t pk[2] = {qv[t].x, qv[t].y};
                const uint32_t sc = qv[t].z;
                if (fp4) {
                    const uint32_t off = (uint32_t)((blk >> 4) * (H * 128) + (h >> 3) * 1024 + (h & 7) * 128 +
                                                    ((((blk & 15) >> 1) ^ (h & 7)) << 4) + (blk & 1) * 8);
                    *reinterpret_cast<uint2 *>(q4_tile + off) = make_uint2(pk[0], pk[1]);
                    qstage[h * Cfg::kStage + blk] = (uint8_t)sc;
                } else {
                    const uint32_t s2 = e4m3x2_to_f16x2((uint16_t)(sc | (sc << 8)));
                    uint32_t h0[4], h1[4];
                    e2m1x8_to_f16x8(pk[0], h0);
                    e2m1x8_to_f16x8(pk[1], h1);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        h0[i] = hmul2_u32(h0[i], s2);
                        h1[i] = hmul2_u32(h1[i], s2);
                    }
                    *reinterpret_cast<uint4 *>(q_tile + q_chunk_off<H>(h, 2 * blk)) =
                        make_uint4(h0[0], h0[1], h0[2], h0[3]);
                    *reinterpret_cast<uint4 *>(q_tile + q_chunk_off<H>(h, 2 * blk + 1)) =
                        make_uint4(h1[0], h1[1], h1[2], h1[3]);
                }
            }
        } else {
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
            const int i = tid + t * kAttnWorkThreads;
            const int h = i / (CSA2_D / 8), c64 = i % (CSA2_D / 8);
            const uint32_t w4[4] = {qv[t].x, qv[t].y, qv[t].z, qv[t].w};
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
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t kv_addr = smem_u32(kv_tile), q_addr = smem_u32(q_tile), p_addr = smem_u32(p_tile);

    {
        const uint32_t idesc_s = idesc_f16_f32(128, H, 0, 0);
        const uint32_t idesc_o = idesc_f16_f32(128, H, 1, 1);
        // base descriptors; an operand offset is added to the start-address
        // field (address / 16, shared memory stays below 2^18 bytes)
        const uint64_t a_s = make_sdesc(kv_addr, 16, 1024, kSw128);
        const uint64_t b_s = make_sdesc(q_addr, 16, 1024, kSw128);
        const uint64_t a_o = make_sdesc(kv_addr, 16384, 1024, kSw128);
        const uint64_t b_o = make_sdesc(p_addr, 16, Cfg::kPGroup, Cfg::kPSwizzle);
        if (mma_warp) {
            // ---- one elected thread issues every tensor-core product ----
            if (NV && fp4 && lane == 0) {
                // S^T = A * B^T with A = the raw FP4 rows, B = q in FP4, one UE4M3
                // scale per 16 values from TMEM, as soon as the rows are stored;
                // the P*V products follow as below, chunk by chunk once each f16
                // chunk is dequantised
                const uint32_t idesc_s4 = idesc_nvf4_f32(128, H);
                const uint64_t a_s4 = make_sdesc(smem_u32(raw_tile), 16, 1024, kSw128);
                const uint64_t b_s4 = make_sdesc(smem_u32(q4_tile), 16, 1024, kSw128);
                bool ok = true;
                for (int it = 0; it < ntiles && ok; ++it) {
                    const uint32_t ph = (uint32_t)it & 1u;
                    if (!mbar_wait(bar_raw, ph)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kb = 0; kb < CSA2_D / 64; ++kb)
                        mma_nvf4(tmem + Cfg::kColS, a_s4 + (uint64_t)(((kb >> 2) * 16384 + (kb & 3) * 32) >> 4),
                                 b_s4 + (uint64_t)(((kb >> 2) * (H * 128) + (kb & 3) * 32) >> 4), idesc_s4,
                                 tmem + Cfg::kColSFA + 4 * kb, tmem + Cfg::kColSFB + (H / 32) * kb, kb > 0 ? 1u : 0u);
                    tc_commit(bar_s);
                    if (!mbar_wait(bar_p, ph)) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int dc = 0; dc < 4; ++dc) {
                        if (!mbar_wait(&bar_kv[dc], ph)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < kAttnTile / 16; ++kk)
                            mma_f16(tmem + Cfg::kColO + dc * H, a_o + (uint64_t)((dc * 32768 + kk * 2048) >> 4),
                                    b_o + (uint64_t)((kk * 2 * Cfg::kPGroup) >> 4), idesc_o,
                                    (it > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&bar_pv[dc]);
                    }
                }
            } else if (lane == 0) {
                bool ok = true;
                for (int it = 0; it < ntiles && ok; ++it) {
                    const uint32_t ph = (uint32_t)it & 1u;
                    // S^T += KV_c * Q_c^T, chunk by chunk as the work warps store them
#pragma unroll 1
                    for (int c = 0; c < 4 && ok; ++c) {
                        if (!mbar_wait(&bar_kv[c], ph)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int kb = 2 * c; kb < 2 * c + 2; ++kb) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_f16(tmem + Cfg::kColS, a_s + (uint64_t)((kb * 16384 + kk * 32) >> 4),
                                        b_s + (uint64_t)((kb * (H * 128) + kk * 32) >> 4), idesc_s,
                                        (kb | kk) ? 1u : 0u);
                        }
                    }
                    if (!ok) break;
                    tc_commit(bar_s);
                    // O^T += V^T * P^T once the softmax has written P^T, chunk by chunk
                    if (!mbar_wait(bar_p, ph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                        for (int kk = 0; kk < kAttnTile / 16; ++kk)
                            mma_f16(tmem + Cfg::kColO + dc * H, a_o + (uint64_t)((dc * 32768 + kk * 2048) >> 4),
                                    b_o + (uint64_t)((kk * 2 * Cfg::kPGroup) >> 4), idesc_o,
                                    (it > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&bar_pv[dc]);
                    }
                }
            }
            __syncwarp();
        } else {
        // ---- work warps: dequantise, fetch ahead, online softmax, epilogue ----
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int quarter = warp & 3, grp = warp >> 2;  // TMEM lane quarter, head group
        const bool soft = grp < G;                       // this warp runs the softmax of group grp
        float l_part[HG];                                // this row's partial softmax denominators
#pragma unroll
        for (int i = 0; i < HG; ++i) l_part[i] = 0.0f;
        bool ok = true;
        if (NV && fp4 && warp < 4) {
            // scale factors of q (B), replicated in every TMEM lane quarter: lane l,
            // column (H / 32) * kb + j holds the four scales of K step kb of head 32 j + l
            const uint32_t *qs = reinterpret_cast<const uint32_t *>(qstage);
            const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + Cfg::kColSFB;
            if constexpr (H == 64) {
                uint32_t r[16];
#pragma unroll
                for (int kb = 0; kb < 8; ++kb)
#pragma unroll
                    for (int j = 0; j < 2; ++j) r[2 * kb + j] = qs[((32 * j + lane) * Cfg::kStage) / 4 + kb];
                tmem_st16(ta, r);
            } else {
                uint32_t r[8];
#pragma unroll
                for (int kb = 0; kb < 8; ++kb) r[kb] = qs[(lane * Cfg::kStage) / 4 + kb];
                tmem_st8(ta, r);
            }
        }
        for (int it = 0; it < ntiles; ++it) {
            const int64_t tt = t_begin + it;
            int32_t *vs = valid_s + ((NV && fp4) ? (it & 1) * kAttnTile : 0);
            if (NV && fp4) {
                // 0. raw FP4 rows and their scale factors for S (the previous tile's S is
                //    complete: this thread waited for it in the softmax)
                store_raw<Cfg::kStage>(raw, raw_tile, stage, vs);
                fence_proxy_async_smem();
                named_bar_sync(kBarWork, kAttnWorkThreads);
                if (warp < 4) {
                    // lane l, column 4 kb + j: the four scales of K step kb of row 32 j + l
                    const uint32_t *st = reinterpret_cast<const uint32_t *>(stage);
                    uint32_t r[32];
#pragma unroll
                    for (int kb = 0; kb < 8; ++kb)
#pragma unroll
                        for (int j = 0; j < 4; ++j) r[4 * kb + j] = st[((32 * j + lane) * Cfg::kStage) / 4 + kb];
                    tmem_st32(tmem + ((uint32_t)(warp * 32) << 16) + Cfg::kColSFA, r);
                    tmem_wait_st();
                }
                tc_fence_before();
                mbar_arrive(bar_raw);
            }
            // 1. dequantise chunk c as soon as the previous tile's P*V on it is done
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (it > 0 && ok && !mbar_wait(&bar_pv[c], (uint32_t)(it - 1) & 1u)) ok = false;
                store_chunk(raw, c, kv_tile, vs, !(NV && fp4));
                fence_proxy_async_smem();
                mbar_arrive(&bar_kv[c]);
            }
            // 2. the next tile's loads go in flight under this tile's products
            const int rel = (it + 1) % kResolveTiles;
            if (tt + 1 < t_end) {
                if (rel == 0) {
                    // next batch of resolved rows (rare: splits of more than 8 tiles)
                    named_bar_sync(kBarWork, kAttnWorkThreads);
                    resolve_rows(p, u, b, nw, wb, (tt + 1) * kAttnTile,
                                 (int)min((int64_t)kResolveTiles, t_end - (tt + 1)) * kAttnTile, rsrc, rkind,
                                 nullptr, one_page, pt0);
                    named_bar_sync(kBarWork, kAttnWorkThreads);
                }
                fetch_tile<0, 4>(p, b, rsrc, rkind, rel * kAttnTile, raw);
            }
            // 3. online softmax: thread = row (TMEM lane), warps 4g..4g+3 take
            //    the heads [g*HG, (g+1)*HG) of group g
            if (soft) {
                const bool got = ok && mbar_wait(bar_s, (uint32_t)it & 1u);
                if (!got) ok = false;
                tc_fence_after();
                const int row = quarter * 32 + lane;
                const bool row_valid = vs[row] != 0 && got;
                const uint32_t s_addr = lane_addr + Cfg::kColS + grp * HG;
                float v[HG];
                load_scores<HG>(s_addr, p.scale_log2, row_valid, v);
                // does any score exceed its head's running maximum by more than 2^8?
                bool raise = false;
                {
#pragma unroll
                    for (int g = 0; g < HG / 4; ++g) {
                        const float4 mm = *reinterpret_cast<const float4 *>(m_run + grp * HG + 4 * g);
                        raise |= v[4 * g] > mm.x + kRescaleThreshold;
                        raise |= v[4 * g + 1] > mm.y + kRescaleThreshold;
                        raise |= v[4 * g + 2] > mm.z + kRescaleThreshold;
                        raise |= v[4 * g + 3] > mm.w + kRescaleThreshold;
                    }
                    raise = named_bar_or(1 + grp, 128, raise);
                    if (raise) {
                        // full path: tile maximum per head, new running maximum
                        float mx[HG];
#pragma unroll
                        for (int i = 0; i < HG; ++i) mx[i] = v[i];
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
                                if (mo != -INFINITY) rescale_tile[grp] = it;
                            }
                            m_run[h] = mn;
                            alpha[h] = a;
                        }
                        named_bar_sync(1 + grp, 128);
                    }
                }
                // probabilities -> P^T (f16), per-row partial denominators
                {
#pragma unroll
                    for (int g = 0; g < HG / 8; ++g) {
                        const int h0 = grp * HG + 8 * g;  // first head of these 8
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
                            const int i = 8 * g + 2 * t;
                            const float p0 = (mm[2 * t] == -INFINITY) ? 0.0f : exp2f(v[i] - mm[2 * t]);
                            const float p1 = (mm[2 * t + 1] == -INFINITY) ? 0.0f : exp2f(v[i + 1] - mm[2 * t + 1]);
                            l_part[i] = fmaf(l_part[i], al[2 * t], p0);
                            l_part[i + 1] = fmaf(l_part[i + 1], al[2 * t + 1], p1);
                            const __half2 h2 = __floats2half2_rn(p0, p1);
                            pk[t] = *reinterpret_cast<const uint32_t *>(&h2);
                        }
                        *reinterpret_cast<uint4 *>(p_tile + p_chunk_off<H>(row, h0 >> 3)) =
                            make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
                // rare: a raise of the running maximum -> rescale this group's
                // O^T columns (every earlier P*V is complete: the S^T commit of
                // this tile came after them)
                if (raise && rescale_tile[grp] == it) {
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
            }
            mbar_arrive(bar_p);
        }
        // ---- final denominators: reduce the per-row partials over the 128 rows
        //      (the last softmax is done; the last tile's P*V may still run) ----
        named_bar_sync(kBarWork, kAttnWorkThreads);
        if (soft) {
            warp_transpose_reduce<HG, false>(l_part);
            store_warp_reduced<HG>(red + quarter * H + grp * HG, l_part);
        }
        named_bar_sync(kBarWork, kAttnWorkThreads);
        if (tid < H) {
            const float l = (red[tid] + red[H + tid]) + (red[2 * H + tid] + red[3 * H + tid]);
            l_run[tid] = l;
            alpha[tid] = l > 0.0f ? 1.0f / l : 0.0f;  // reused as 1 / l
        }
        named_bar_sync(kBarWork, kAttnWorkThreads);

        // ---- epilogue: O^T (TMEM) -> o = O / l written straight from registers,
        //      latent chunk dc as soon as the last tile's P*V on it is done (the
        //      stores of a chunk run under the products of the next ones): a
        //      thread owns latent column d = 128*dc + 32*quarter + lane of its
        //      group's heads, so each store instruction of a warp covers 32
        //      consecutive columns of one head (coalesced) ----
        {
            if (soft) {
                const int d0 = quarter * 32 + lane;
                const bool bf16_out = p.n_splits == 1 && !p.out_f32;
                uint16_t *dst16 = p.o + (int64_t)u * H * CSA2_D;
                float *dst32 = bf16_out ? nullptr : p.o_part + ((int64_t)u * p.n_splits + split) * H * CSA2_D;
#pragma unroll 1
                for (int dc = 0; dc < 4; ++dc) {
                    uint32_t vals[HG];  // raw f32 bits
                    if (ntiles > 0) {
                        if (ok && !mbar_wait(&bar_pv[dc], (uint32_t)(ntiles - 1) & 1u)) ok = false;
                        tc_fence_after();
                        const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + Cfg::kColO + dc * H + grp * HG;
                        if (HG == 16) {
                            tmem_ld16(ta, *reinterpret_cast<uint32_t(*)[16]>(&vals[0]));
                        } else {
                            tmem_ld8(ta, *reinterpret_cast<uint32_t(*)[8]>(&vals[0]));
                        }
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int i = 0; i < HG; ++i) vals[i] = 0u;
                    }
                    if (bf16_out) {
#pragma unroll
                        for (int i = 0; i < HG; ++i) {
                            const int h = grp * HG + i;
                            dst16[(int64_t)h * CSA2_D + dc * 128 + d0] = f32_to_bf16_bits(__uint_as_float(vals[i]) * alpha[h]);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < HG; ++i) {
                            const int h = grp * HG + i;
                            dst32[(int64_t)h * CSA2_D + dc * 128 + d0] = __uint_as_float(vals[i]) * alpha[h];
                        }
                    }
                }
            }
            if (tid < H) {
                const float l = l_run[tid];
                const float lse = l > 0.0f ? (m_run[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
                if (p.n_splits == 1 && !p.out_f32) {
                    if (p.lse) p.lse[(int64_t)u * H + tid] = lse;
                } else {
                    p.lse_part[((int64_t)u * p.n_splits + split) * H + tid] = lse;
                }
            }
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
// One CTA per (query, head); each thread owns one float4 of the head and
// puts the loads of that float4 of the first 16 splits in flight before the
// weights are computed, so the two memory latencies overlap.
constexpr int kCombineThreads = 128;
constexpr int kCombineHeads = 1;   // heads per CTA (128 float4 per head)
constexpr int kCombineBatch = 16;  // split loads in flight per thread

// Partials of query u, part s: o at o_part + u * q_stride + s * s_stride
// (+ h * 512), lse at lse_part + u * lq_stride + s * ls_stride (+ h). Output:
// bf16 o [u][h][512] (F32 = false) or f32 (F32 = true).
struct CombineArgs {
    const float *o_part;
    const float *lse_part;
    int64_t q_stride, s_stride, lq_stride, ls_stride;
    void *o;
    float *lse;
    int32_t n_splits;
};

template <int H, bool F32>
__global__ void __launch_bounds__(kCombineThreads) k_attn_combine(CombineArgs a) {
    extern __shared__ float wsm[];  // [n_splits + 1]
    pdl_trigger();
    pdl_wait();
    const int32_t u = blockIdx.y;
    const int h = blockIdx.x;
    const int d4 = threadIdx.x;  // 128 threads x 4 values = 512
    const int32_t n_splits = a.n_splits;
    const float *src = a.o_part + (int64_t)u * a.q_stride + h * CSA2_D;
    const float *lsrc = a.lse_part + (int64_t)u * a.lq_stride + h;
    float4 v[kCombineBatch];
#pragma unroll
    for (int t = 0; t < kCombineBatch; ++t)
        v[t] = t < n_splits ? __ldg(reinterpret_cast<const float4 *>(src + (int64_t)t * a.s_stride) + d4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x < 32) {
        float M = -INFINITY;
        for (int s = threadIdx.x; s < n_splits; s += 32) M = fmaxf(M, lsrc[(int64_t)s * a.ls_stride]);
#pragma unroll
        for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        float L = 0.0f;
        for (int s = threadIdx.x; s < n_splits; s += 32) {
            const float ls = lsrc[(int64_t)s * a.ls_stride];
            const float w = (M == -INFINITY) ? 0.0f : expf(ls - M);
            wsm[s] = w;
            L += w;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
        if (threadIdx.x == 0) {
            wsm[n_splits] = L;
            if (a.lse) a.lse[(int64_t)u * H + h] = L > 0.0f ? M + logf(L) : -INFINITY;
        }
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_splits; s0 += kCombineBatch) {
        if (s0 > 0) {
#pragma unroll
            for (int t = 0; t < kCombineBatch; ++t)
                v[t] = (s0 + t < n_splits)
                           ? __ldg(reinterpret_cast<const float4 *>(src + (int64_t)(s0 + t) * a.s_stride) + d4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
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
    if (F32) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.o) + ((int64_t)u * H + h) * CSA2_D) + d4;
        *dst = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    } else {
        uint16_t *dst = static_cast<uint16_t *>(a.o) + ((int64_t)u * H + h) * CSA2_D + d4 * 4;
        const uint32_t lo = (uint32_t)f32_to_bf16_bits(acc.x * inv) | ((uint32_t)f32_to_bf16_bits(acc.y * inv) << 16);
        const uint32_t hi = (uint32_t)f32_to_bf16_bits(acc.z * inv) | ((uint32_t)f32_to_bf16_bits(acc.w * inv) << 16);
        *reinterpret_cast<uint2 *>(dst) = make_uint2(lo, hi);
    }
}

}  // namespace csa2
