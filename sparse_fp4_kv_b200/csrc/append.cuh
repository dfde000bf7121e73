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
// Layout: a warp per 512-value row at a time. Lane l owns block l (values 16l ..
// 16l+15): it reads 32 contiguous bytes of bf16 input, writes 8 bytes of
// codes and 1 scale byte, so a warp moves 1 KiB in and 288 B out with fully
// coalesced 16-byte loads. HBM-bound: 1312 algorithmic bytes per row.
//
// The E2M1 rounding is the hardware conversion of the correctly rounded
// binary32 quotient x / value(s) (see quantize_block16).
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAppendWarps = 8;

// Quantise one block of 16 values (binary32 copies of bf16 or narrower
// inputs) with the rule above: returns the E4M3 scale byte and writes the 16
// E2M1 codes, element i in nibble i of packed[i / 8].
// The code of x is the E2M1 rounding (cvt.rn.satfinite.e2m1x2, ties to the
// even mantissa, saturating to 6) of the correctly rounded binary32 quotient
// x / value(s): q0 = x * r with r ~ 1 / value(s) (rcp.approx), the remainder
// x - q0 * value(s) by one fma, and q = q0 + remainder * r by another (the
// fma remainder correction of Markstein's division). For bf16 x a quotient
// that is not exactly a decision point of the grid is at least 2^-9 (relative)
// away from one, far beyond the correction's error, and an exact decision
// point is reproduced exactly, so the codes equal those of the exact quotient.
// NaN inputs give a zero code with their sign, infinite ones the largest
// code with their sign; value(s) = 0 gives all-zero codes.
__device__ __forceinline__ uint32_t e2m1x2_of_f32(float hi, float lo) {
    uint16_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u16.u8 %0, b;\n\t}"
        : "=h"(out)
        : "f"(hi), "f"(lo));
    return out & 0xFFu;
}
// Hardware reciprocal approximation (rcp.approx.f32: within a few ulps).
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
// a / b for a finite a >= 0 and b > 0 with r ~ 1 / b (a few ulps): the
// remainder correction above, which reproduces an exactly representable
// quotient exactly; the scale needs it because amax / 6 can be an exact
// E4M3 rounding midpoint. amax = +inf stays +inf.
__device__ __forceinline__ float quotient_rn(float a, float b, float r) {
    const float q0 = a * r;
    const float q = fmaf(fmaf(-q0, b, a), r, q0);
    return q == q ? q : q0;
}
__device__ __forceinline__ uint32_t quantize_block16(const float (&f)[16], uint32_t (&packed)[2]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));  // fmaxf drops NaN operands
    const uint32_t s = f32_to_e4m3_satfinite(quotient_rn(amax, 6.0f, 1.0f / 6.0f));
    const float sv = __half2float(__ushort_as_half((uint16_t)(e4m3x2_to_f16x2((uint16_t)s) & 0xFFFFu)));
    packed[0] = packed[1] = 0u;
    if (sv == 0.0f) return s;
    const float r = rcp_approx(sv);
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float q0 = f[i] * r;
        const float rem = fmaf(-q0, sv, f[i]);
        const float qq = fmaf(rem, r, q0);
        // an infinite x leaves q0 infinite (it saturates to 6) and a NaN remainder
        q[i] = qq == qq ? qq : (f[i] == f[i] ? q0 : copysignf(0.0f, f[i]));
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) packed[j >> 2] |= e2m1x2_of_f32(q[2 * j + 1], q[2 * j]) << (8 * (j & 3));
    return s;
}

// Eight E2M1 codes from eight binary32 quotients: element i in nibble i.
__device__ __forceinline__ uint32_t e2m1x8_of_f32(const float *q) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}
// Per 16-bit half, the unsigned maximum.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// quantize_block16 on 16 bf16 values as they are loaded (w[i] holds values
// 2i, 2i+1), with the same results in fewer instructions: the block maximum
// is taken on the magnitudes' bit patterns two at a time (their integer order
// is the values' order; 0x7F80 and above mean inf or NaN, which go to the
// general routine), and the quotients of finite values, which can be neither
// infinite nor NaN there, are formed two at a time with the same three
// correctly rounded operations per value.
__device__ __forceinline__ uint32_t quantize_block16_bf16(const uint32_t (&w)[8], uint32_t (&packed)[2]) {
    uint32_t m = w[0] & 0x7FFF7FFFu;
#pragma unroll
    for (int i = 1; i < 8; ++i) m = max_u16x2(m, w[i] & 0x7FFF7FFFu);
    const uint32_t mm = max(m & 0xFFFFu, m >> 16);
    if (mm >= 0x7F80u) {
        float f[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
        return quantize_block16(f, packed);
    }
    const float amax = __uint_as_float(mm << 16);
    const uint32_t s = f32_to_e4m3_satfinite(quotient_rn(amax, 6.0f, 1.0f / 6.0f));
    const float sv = __half2float(__ushort_as_half((uint16_t)(e4m3x2_to_f16x2((uint16_t)s) & 0xFFFFu)));
    packed[0] = packed[1] = 0u;
    if (sv == 0.0f) return s;
    const float r = rcp_approx(sv);
    const float2 r2 = make_float2(r, r), nsv2 = make_float2(-sv, -sv);
    float q[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 x = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
        const float2 q0 = __fmul2_rn(x, r2);
        const float2 rem = __ffma2_rn(q0, nsv2, x);  // x - q0 * value(s), exactly as fma(-q0, sv, x)
        const float2 qq = __ffma2_rn(rem, r2, q0);
        q[2 * i] = qq.x;
        q[2 * i + 1] = qq.y;
    }
    packed[0] = e2m1x8_of_f32(q);
    packed[1] = e2m1x8_of_f32(q + 8);
    return s;
}

// One wave of resident CTAs; warp w of the W warps in the grid takes rows
// w, w + W, w + 2W, ... Two things keep its memory traffic and its
// arithmetic overlapped:
//   * destinations are resolved 32 rows at a time, lane j looking up the
//     physical row of the warp's j-th row of the group (sequence, position,
//     page table: every lane's chain in flight at once), and handed to the
//     quantising lanes by a shuffle, so no row waits for its own lookup;
//   * the bf16 input of kAppendRing - 1 rows is in flight while a row is
//     quantised: a ring of kAppendRing rows in registers, the slot of the row
//     just stored refilled with the row kAppendRing - 1 further on.
// (A grid that loaded a batch of rows, then quantised it, then loaded the
// next spent its time alternately waiting on memory and on instruction
// issue.)
constexpr int kAppendRing = 4;

__device__ __forceinline__ int64_t append_dest(const csa2_kv_desc &kv, const int32_t *__restrict__ seq,
                                               const int64_t *__restrict__ pos, int64_t r) {
    const int32_t b = seq[r];
    return (b >= 0 && b < kv.batch) ? physical_row(kv, b, pos[r]) : -1;
}

__device__ __forceinline__ void append_load_row(const uint16_t *__restrict__ x, int64_t r, int lane, uint4 (&v)[2]) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + r * CSA2_D + lane * 16);
    v[0] = __ldg(src);
    v[1] = __ldg(src + 1);
}

// Quantise one row held as lane l's 16 values (block l) and store it at
// physical row `dest` (< 0: a bad destination, reported and skipped).
__device__ __forceinline__ void append_store_row(const csa2_kv_desc &kv, int64_t dest, int lane, const uint4 (&v)[2]) {
    if (dest < 0) {
        if (lane == 0) set_error(CSA2_DEVERR_BAD_ROW);
        return;
    }
    const uint32_t wds[8] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w};
    uint32_t packed[2];
    const uint32_t s = quantize_block16_bf16(wds, packed);
    // codes: 8 bytes per lane (256 contiguous bytes per warp); scales: one
    // byte per lane (the row's 32-byte sector in one warp store)
    *reinterpret_cast<uint2 *>(kv.codes + dest * (CSA2_D / 2) + lane * 8) = make_uint2(packed[0], packed[1]);
    kv.scales[dest * (CSA2_D / CSA2_BLOCK) + lane] = (uint8_t)s;
}

__global__ void __launch_bounds__(kAppendWarps * 32, 3)
    k_append_fp4(const uint16_t *__restrict__ x, int32_t n, const int32_t *__restrict__ seq,
                 const int64_t *__restrict__ pos, csa2_kv_desc kv) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t W = (int64_t)gridDim.x * kAppendWarps;
    const int64_t w = (int64_t)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    if (w >= n) return;
    const int64_t rows = (n - w + W - 1) / W;  // rows of this warp: w + k * W, k < rows
    for (int64_t g0 = 0; g0 < rows; g0 += 32) {
        const int m = (int)min((int64_t)32, rows - g0);  // rows of this group (warp-uniform)
        const int64_t first = w + g0 * W;                 // row of group index 0
        uint4 v[kAppendRing][2];
#pragma unroll
        for (int s = 0; s < kAppendRing - 1; ++s)
            if (s < m) append_load_row(x, first + s * W, lane, v[s]);
        // lane j: destination of group row j (its lookups overlap the loads above)
        const int64_t dest_j = lane < m ? append_dest(kv, seq, pos, first + lane * W) : -1;
        for (int k0 = 0; k0 < m; k0 += kAppendRing) {
#pragma unroll
            for (int s = 0; s < kAppendRing; ++s) {
                const int k = k0 + s;
                // refill the slot of row k - 1 (stored in the previous step)
                if (k + kAppendRing - 1 < m)
                    append_load_row(x, first + (int64_t)(k + kAppendRing - 1) * W, lane,
                                    v[(s + kAppendRing - 1) % kAppendRing]);
                const int64_t dest = __shfl_sync(0xFFFFFFFFu, dest_j, k & 31);
                if (k < m) append_store_row(kv, dest, lane, v[s]);
            }
        }
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
// A thread converts P x 8 consecutive values of one row: P 16-byte loads in
// flight, one destination lookup, P 8-byte stores. Window rows go to ring
// slot pos % ring_rows of their sequence (P = kE4m3WindowPieces, so a thread
// moves 64 bytes in); indexer keys go to the physical row of (seq, pos)
// (P = 1: keys are short, and more threads keep more of their dependent
// lookups in flight). P divides the pieces of a row (64 for window rows),
// so a thread never spans two rows.
// ---------------------------------------------------------------------------
constexpr int kE4m3Threads = 256;
constexpr int kE4m3WindowPieces = 4;

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
template <int P>
__global__ void __launch_bounds__(kE4m3Threads)
    k_append_e4m3(const uint16_t *__restrict__ x, int32_t n, int32_t width, const int32_t *__restrict__ seq,
                  const int64_t *__restrict__ pos, int32_t mode, uint8_t *__restrict__ swa, int32_t batch,
                  int64_t ring_rows, csa2_kv_desc kv) {
    pdl_trigger();
    pdl_wait();
    const int groups = width / (8 * P);  // threads per row
    const int64_t t = (int64_t)blockIdx.x * kE4m3Threads + threadIdx.x;
    if (t >= (int64_t)n * groups) return;
    const int64_t r = t / groups;
    const int c = (int)(t - r * groups) * P;  // first 8-value piece
    uint4 v[P];
#pragma unroll
    for (int j = 0; j < P; ++j) v[j] = __ldg(reinterpret_cast<const uint4 *>(x + r * width) + c + j);
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
#pragma unroll
    for (int j = 0; j < P; ++j) {
        const uint32_t lo = e4m3x2_of_bf16x2(v[j].x) | (e4m3x2_of_bf16x2(v[j].y) << 16);
        const uint32_t hi = e4m3x2_of_bf16x2(v[j].z) | (e4m3x2_of_bf16x2(v[j].w) << 16);
        *reinterpret_cast<uint2 *>(row + (c + j) * 8) = make_uint2(lo, hi);
    }
}

}  // namespace csa2
