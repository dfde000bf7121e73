/*
 * csa2_oracle.h -- plain CPU oracle for the CSA2 sparse FP4-KV decode path.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library. The product path
 * (the CUDA library under sparse_fp4_kv_b200/) never links, includes or
 * calls it, and this file shares no code, header, table or constant with
 * that path.
 *
 * Sources (web pages on DeepSeek V4.1-Flash; they give no formulas, so the
 * arithmetic below is the plainest reading of what they describe):
 *   [P3] "DeepSeek V4.1-Flash Cuts KV Cache by 437x With New CED and CSA2
 *        Architecture" (ainewsfeed.tech), the paragraphs that begin
 *        "CSA2 tackles storage", "CSA2 assigns each layer one of three
 *        static operating modes" and "V4.1-Flash also uses FP4 quantization".
 *   [P4] "DeepSeek V4.1 Flash Architecture Breakdown: KV Cache Compressed to
 *        1/437 of First Generation" (nashnova.com), sections "How does the
 *        cache compress along three dimensions at once?" and "How are cache
 *        precision and storage arranged?".
 *   [OCP-MX]  OCP Microscaling Formats (MX) v1.0, section 5.3.3 (FP4 E2M1).
 *   [OCP-FP8] OCP 8-bit Floating Point Specification (OFP8) v1.0, E4M3.
 *
 * Every floating-point result is computed in double unless a comment says
 * otherwise. The two quantiser divisions are done in IEEE binary32 because
 * they decide integer codes and the GPU takes the same decision in binary32.
 *
 * Parity pins (what each function is checked against, outside itself) are
 * listed in tests/test_oracle_pins.py. Functions with no pin: none.
 */
#ifndef CSA2_ORACLE_H
#define CSA2_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- number formats ([P4]: E2M1 for the main KV; [OCP-MX]; [OCP-FP8]) --- */

/* Value of a 4-bit E2M1 code (bit 3 sign, bits 2..1 exponent, bit 0 mantissa,
 * exponent bias 1, no infinities or NaN). */
double orc_e2m1_value(uint32_t code);

/* Value of an E4M3 byte (bit 7 sign, bits 6..3 exponent, bits 2..0 mantissa,
 * bias 7, no infinities, 0x7F and 0xFF are NaN). */
double orc_e4m3_value(uint32_t byte);

/* Round a binary32 value to E4M3: nearest, ties to the even mantissa,
 * magnitudes at or above 448 saturate to +-448, NaN gives 0x7F|sign. */
uint32_t orc_e4m3_rne_sat(float x);

/* Round a binary32 value to E2M1: nearest, ties to the even mantissa,
 * magnitudes at or above 6 saturate to +-6. A NaN gives the signed zero code. */
uint32_t orc_e2m1_rne_sat(float y);

/* ---- FP4 block quantiser ([P3] FP4 paragraph; [P4] precision section) ----
 * One block of 16 bf16 values (raw bits) -> 8 packed bytes (element 2i in the
 * low nibble of byte i) and one E4M3 scale byte.
 *   amax = max |x_i| (binary32; NaN elements are ignored)
 *   s    = E4M3_RNE_sat(amax / 6)        (binary32 division)
 *   c_i  = 0 if value(s) == 0, else E2M1_RNE_sat(x_i / value(s)) (binary32) */
void orc_quantize_block16(const uint16_t *x_bf16, uint8_t *packed8, uint8_t *scale);

/* Quantise one row of d values (d a multiple of 16): d/2 code bytes and d/16
 * scale bytes. */
void orc_quantize_row(const uint16_t *x_bf16, int32_t d, uint8_t *codes, uint8_t *scales);

/* Physical cache row of logical entry t of a sequence whose page table row is
 * page_table_seq: page_table_seq[t / page_size] * page_size + t % page_size. */
int64_t orc_physical_row(const int32_t *page_table_seq, int32_t page_size, int64_t t);

/* Append n rows of d bf16 values: row i is quantised and stored at logical
 * position pos[i] of sequence seq[i] (page_table is [batch][max_pages]). */
void orc_append_fp4(const uint16_t *x_bf16, int32_t n, int32_t d,
                    const int32_t *seq, const int64_t *pos,
                    const int32_t *page_table, int32_t max_pages, int32_t page_size,
                    uint8_t *codes, uint8_t *scales);

/* ---- FP8 appends: the write side of the window KV and the indexer keys --
 * [P3] "V4.1-Flash also uses FP4 quantization" (the short-window SWA KV is
 * kept at FP8) and [P4] "How are cache precision and storage arranged?".
 * Each bf16 value becomes E4M3_RNE_sat(value) (no scale); NaN keeps its sign
 * and becomes the E4M3 NaN code 0x7F. */
void orc_e4m3_row(const uint16_t *x_bf16, int32_t width, uint8_t *out);

/* Window rows: row i (512 values) goes to ring slot pos[i] % ring_rows of
 * sequence seq[i] in swa [batch][ring_rows][512]. */
void orc_append_swa_e4m3(const uint16_t *x_bf16, int32_t n, const int32_t *seq, const int64_t *pos,
                         int64_t ring_rows, uint8_t *swa);

/* Indexer keys: row i (di values) goes to the physical row of logical entry
 * pos[i] of sequence seq[i] in kidx [rows][di]. */
void orc_append_kidx_e4m3(const uint16_t *x_bf16, int32_t n, int32_t di, const int32_t *seq,
                          const int64_t *pos, const int32_t *page_table, int32_t max_pages,
                          int32_t page_size, uint8_t *kidx);

/* ---- indexer ([P3] modes paragraph; [P4] three-dimension section) -------
 * score = sum_h w_h * max(0, sum_i q_{h,i} k_i), q and k E4M3, exact in double
 * for the integer-valued data the tests use; -0 is returned as +0. */
double orc_index_score(const uint8_t *q, const float *w, int32_t hi, int32_t di,
                       const uint8_t *k);

/* Exact Top-k of n (score, id) pairs under the order (score descending, id
 * ascending). Writes min(k, n) ids followed by -1 padding up to k; returns the
 * number of real ids. */
int32_t orc_select_topk(const double *score, const int32_t *ids, int64_t n,
                        int32_t k, int32_t *out);

/* Full mode for one query: scores every visible entry t < n_visible of one
 * sequence, returns the Top-k ids and (if p > 0) the Top-p candidate pool.
 * kidx holds di bytes per physical row. scores_out (nullable) receives the
 * n_visible scores in logical order. */
void orc_index_full(const uint8_t *qidx, const float *w, int32_t hi, int32_t di,
                    const uint8_t *kidx, const int32_t *page_table_seq, int32_t page_size,
                    int64_t n_visible, int32_t k, int32_t p,
                    int32_t *topk, int32_t *pool, double *scores_out);

/* Reindex mode for one query: re-scores only the ids of a pool built by a Full
 * layer (entries < 0 are padding) and returns their Top-k. */
void orc_index_reindex(const uint8_t *qidx, const float *w, int32_t hi, int32_t di,
                       const uint8_t *kidx, const int32_t *page_table_seq, int32_t page_size,
                       const int32_t *pool, int32_t p, int32_t k, int32_t *topk);

/* ---- sparse + sliding-window attention ([P3] modes and FP4 paragraphs) ---
 * One query, h heads of width d (bf16 raw bits). Attended set: the dequantised
 * FP4 rows named by topk (ids < 0 skipped) and the nw E4M3 window rows. Each
 * attended row serves as key and value. Per head:
 *   z_j = softmax_scale * <q_h, v_j>,  m = max z,  l = sum exp(z_j - m)
 *   o_h = sum_j exp(z_j - m) v_j / l,  lse_h = m + log l
 * An empty set gives o = 0 and lse = -inf. Output in double. */
void orc_sparse_attn(const uint16_t *q_bf16, int32_t h, int32_t d,
                     const uint8_t *codes, const uint8_t *scales,
                     const int32_t *page_table_seq, int32_t page_size,
                     const int32_t *topk, int32_t k,
                     const uint8_t *swa_rows, int32_t nw,
                     double softmax_scale, double *o, double *lse);

/* Dequantise one FP4 row (d values) to double: value(c_i) * value(s_{i/16}). */
void orc_dequant_row(const uint8_t *codes, const uint8_t *scales, int32_t d, double *out);

#ifdef __cplusplus
}
#endif
#endif
