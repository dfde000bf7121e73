// append.cuh -- FP4 E2M1 quantise + append of new latent KV rows.
//
// DeepSeek V4.1-Flash Cuts KV Cache by 437x (ainewsfeed.tech), paragraph
// "V4.1-Flash also uses FP4 quantization": the long-term global KV is stored
// in FP4; DeepSeek V4.1 Flash Architecture Breakdown (nashnova.com),
// section "How are cache precision and storage arranged?": E2M1 scheme.
// The pages give no scale rule; this kernel uses one E4M3 scale per block of
// 16 values, s = E4M3_RNE_satfinite(amax / 6), codes E2M1_RNE_satfinite of
// x / value(s), ties to the even mantissa, and all-zero codes when value(s)
// is 0.
//
// Layout: one warp per 512-value row. Lane l owns block l (values 16l ..
// 16l+15): it reads 32 contiguous bytes of bf16 input, writes 8 bytes of
// codes and 1 scale byte, so a warp moves 1 KiB in and 288 B out with fully
// coalesced 16-byte loads. HBM-bound: 1312 algorithmic bytes per row.
//
// The E2M1 rounding compares |x| against the seven decision points of the
// grid scaled by value(s) instead of dividing. The products t * value(s)
// are exact in binary32 (at most 3 + 4 significant bits), and for bf16 x
// (8 significant bits) the quotient x / value(s) cannot land within half a
// binary32 ulp of a decision point without being equal to it, so the
// comparison gives the same code as rounding the binary32 quotient.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAppendWarps = 8;

// Quantise one block of 16 values (binary32 copies of bf16 or narrower
// inputs) with the rule above: returns the E4M3 scale byte and writes the 16
// E2M1 codes, element i in nibble i of packed[i / 8].
__device__ __forceinline__ uint32_t quantize_block16(const float (&f)[16], uint32_t (&packed)[2]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));  // fmaxf drops NaN operands
    const uint32_t s = f32_to_e4m3_satfinite(__fdiv_rn(amax, 6.0f));
    const float sv = __half2float(__ushort_as_half((uint16_t)(e4m3x2_to_f16x2((uint16_t)s) & 0xFFFFu)));
    // decision points of the E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}; at an
    // exact midpoint the even-mantissa neighbour wins ('>' keeps the lower
    // point, '>=' takes the upper one)
    const float t1 = 0.25f * sv, t2 = 0.75f * sv, t3 = 1.25f * sv, t4 = 1.75f * sv;
    const float t5 = 2.5f * sv, t6 = 3.5f * sv, t7 = 5.0f * sv;
    packed[0] = packed[1] = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float a = fabsf(f[i]);
        uint32_t c = (uint32_t)(a > t1) + (uint32_t)(a >= t2) + (uint32_t)(a > t3) + (uint32_t)(a >= t4) +
                     (uint32_t)(a > t5) + (uint32_t)(a >= t6) + (uint32_t)(a > t7);
        c |= (__float_as_uint(f[i]) >> 31) << 3;
        if (sv == 0.0f) c = 0u;
        packed[i >> 3] |= c << (4 * (i & 7));
    }
    return s;
}

// A warp walks rows r, r + W, r + 2W, ... (W = warps in the grid). The
// loads of its next row (input values and destination lookup) are issued
// before the current row is quantised and stored, so every warp keeps two
// rows in flight; the grid fills every SM.
__device__ __forceinline__ int64_t append_dest(const csa2_kv_desc &kv, const int32_t *__restrict__ seq,
                                               const int64_t *__restrict__ pos, int64_t r) {
    const int32_t b = seq[r];
    return (b >= 0 && b < kv.batch) ? physical_row(kv, b, pos[r]) : -1;
}

__global__ void __launch_bounds__(kAppendWarps * 32)
    k_append_fp4(const uint16_t *__restrict__ x, int32_t n, const int32_t *__restrict__ seq,
                 const int64_t *__restrict__ pos, csa2_kv_desc kv) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kAppendWarps;
    int64_t r = (int64_t)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    if (r >= n) return;
    uint4 v0 = __ldg(reinterpret_cast<const uint4 *>(x + r * CSA2_D + lane * 16));
    uint4 v1 = __ldg(reinterpret_cast<const uint4 *>(x + r * CSA2_D + lane * 16) + 1);
    int64_t row = append_dest(kv, seq, pos, r);
    for (; r < n; r += stride) {
        // the next row's values and destination go in flight first
        const int64_t rn = r + stride;
        uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
        int64_t row_n = -1;
        if (rn < n) {
            n0 = __ldg(reinterpret_cast<const uint4 *>(x + rn * CSA2_D + lane * 16));
            n1 = __ldg(reinterpret_cast<const uint4 *>(x + rn * CSA2_D + lane * 16) + 1);
            row_n = append_dest(kv, seq, pos, rn);
        }
        if (row < 0) {
            if (lane == 0) set_error(CSA2_DEVERR_BAD_ROW);
        } else {
            const uint32_t wds[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float f[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[2 * i] = __uint_as_float(wds[i] << 16);
                f[2 * i + 1] = __uint_as_float(wds[i] & 0xFFFF0000u);
            }
            uint32_t packed[2];
            const uint32_t s = quantize_block16(f, packed);
            // codes: 8 bytes per lane (256 contiguous bytes per warp); scales: one
            // byte per lane (the row's 32-byte sector in one warp store)
            *reinterpret_cast<uint2 *>(kv.codes + row * (CSA2_D / 2) + lane * 8) = make_uint2(packed[0], packed[1]);
            kv.scales[row * (CSA2_D / CSA2_BLOCK) + lane] = (uint8_t)s;
        }
        v0 = n0;
        v1 = n1;
        row = row_n;
    }
}

// ---------------------------------------------------------------------------
// FP8 appends: the write side of the short-window KV and of the indexer keys
// (DeepSeek V4.1-Flash Cuts KV Cache by 437x, paragraph "V4.1-Flash also uses
// FP4 quantization": the short-window SWA KV is kept at FP8; DeepSeek V4.1
// Flash Architecture Breakdown, section "How are cache precision and storage
// arranged?"). Each bf16 value is converted on its own to E4M3, round to
// nearest even, saturating to +-448, no scale; NaN keeps its sign and becomes
// the E4M3 NaN code 0x7F.
//
// A thread converts 8 consecutive values of a row: one 16-byte load, one
// 8-byte store. Window rows go to ring slot pos % ring_rows of their
// sequence; indexer keys go to the physical row of (seq, pos).
// ---------------------------------------------------------------------------
constexpr int kE4m3Threads = 256;

// Two bf16 values (low half first) -> two E4M3 bytes (low byte first).
__device__ __forceinline__ uint32_t e4m3x2_of_bf16x2(uint32_t w) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
    uint32_t r = out;
    if ((w & 0x7FFFu) > 0x7F80u) r = (r & 0xFF00u) | ((w >> 8) & 0x80u) | 0x7Fu;                     // low NaN
    if (((w >> 16) & 0x7FFFu) > 0x7F80u) r = (r & 0x00FFu) | (((w >> 24) & 0x80u) | 0x7Fu) << 8;  // high NaN
    return r;
}

// mode 0: window rows (width 512) into swa [batch][ring_rows][512];
// mode 1: indexer keys (width kv.di) into kv.kidx at the physical row.
__global__ void __launch_bounds__(kE4m3Threads)
    k_append_e4m3(const uint16_t *__restrict__ x, int32_t n, int32_t width, const int32_t *__restrict__ seq,
                  const int64_t *__restrict__ pos, int32_t mode, uint8_t *__restrict__ swa, int32_t batch,
                  int64_t ring_rows, csa2_kv_desc kv) {
    pdl_trigger();
    pdl_wait();
    const int per_row = width / 8;
    const int64_t t = (int64_t)blockIdx.x * kE4m3Threads + threadIdx.x;
    if (t >= (int64_t)n * per_row) return;
    const int64_t r = t / per_row;
    const int c = (int)(t - r * per_row);
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + r * width) + c);
    const int32_t b = seq[r];
    const int64_t ps = pos[r];
    uint8_t *row = nullptr;
    if (mode == 0) {
        if (b >= 0 && b < batch && ps >= 0) row = swa + ((int64_t)b * ring_rows + ps % ring_rows) * 512;
    } else {
        const int64_t pr = (b >= 0 && b < kv.batch) ? physical_row(kv, b, ps) : -1;
        if (pr >= 0) row = kv.kidx + pr * kv.di;
    }
    if (row == nullptr) {
        if (c == 0) set_error(CSA2_DEVERR_BAD_ROW);
        return;
    }
    const uint32_t lo = e4m3x2_of_bf16x2(v.x) | (e4m3x2_of_bf16x2(v.y) << 16);
    const uint32_t hi = e4m3x2_of_bf16x2(v.z) | (e4m3x2_of_bf16x2(v.w) << 16);
    *reinterpret_cast<uint2 *>(row + c * 8) = make_uint2(lo, hi);
}

}  // namespace csa2
