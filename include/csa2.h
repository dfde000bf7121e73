/*
 * csa2.h -- C ABI of libcsa2.so, the B200 (sm_100a) CSA2 sparse FP4-KV
 * decode path.
 *
 * What the path computes (web pages on DeepSeek V4.1-Flash; they give no
 * formulas, the readings taken are stated per call):
 *   [P3] "DeepSeek V4.1-Flash Cuts KV Cache by 437x With New CED and CSA2
 *        Architecture" (ainewsfeed.tech): paragraphs "CSA2 tackles storage"
 *        (one global KV shared by all layers, cross-layer Top-K reuse),
 *        "CSA2 assigns each layer one of three static operating modes"
 *        (Full / Reindex / Reuse, hierarchical indexer pool) and
 *        "V4.1-Flash also uses FP4 quantization" (FP4 global KV, FP8 SWA KV,
 *        values restored at runtime for computation).
 *   [P4] "DeepSeek V4.1 Flash Architecture Breakdown: KV Cache Compressed to
 *        1/437 of First Generation" (nashnova.com): sections "How does the
 *        cache compress along three dimensions at once?" (three modes, pool
 *        built by the first Full layer) and "How are cache precision and
 *        storage arranged?" (FP4 E2M1 main KV, FP8 sliding-window KV).
 *
 * Conventions for every call:
 *   - Every pointer argument except the descriptor structs themselves is a
 *     DEVICE pointer owned by the caller. The library allocates and frees
 *     nothing, never synchronises, and enqueues all work on `stream`.
 *   - Arguments are checked on the host before any launch; a failed check
 *     returns CSA2_ERR_INVALID_ARG / CSA2_ERR_UNSUPPORTED /
 *     CSA2_ERR_WORKSPACE and launches nothing. A launch failure returns
 *     CSA2_ERR_CUDA. Conditions only the device can see (an id or page
 *     outside the cache, a timed-out wait) skip the offending access and set
 *     a sticky device error word, read and cleared by csa2_device_status().
 *   - Layouts are dense row-major. Device pointers must be 16-byte aligned.
 *   - Entry ids are logical positions within a sequence; -1 marks an empty
 *     slot in every id list.
 *   - Reuse mode is not a call: a Reuse layer passes its source layer's
 *     Top-k list to csa2_sparse_attn_decode.
 *   - Devices: a call runs on the device current on the calling thread.
 *     Kernel attributes (shared-memory limits) are set up once per device,
 *     at the first call on that device that needs the kernel, so one process
 *     may use several devices.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment      */
    CSA2_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d != 512) */
    CSA2_ERR_WORKSPACE = 3,    /* workspace missing or too small            */
    CSA2_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed       */
    CSA2_ERR_DEVICE = 5        /* the device error word was set            */
} csa2_status;

/* Latent width of the global KV (the pages leave it open; this library
 * fixes it at 512) and the FP4 scale block (one E4M3 scale per 16 values). */
#define CSA2_D 512
#define CSA2_BLOCK 16

/*
 * The global KV cache shared by all layers ([P3] "CSA2 tackles storage").
 * One physical row per entry:
 *   codes  [rows_cap][d/2]  FP4 E2M1, two per byte, element 2i in the low
 *                           nibble of byte i                    (256 B/row)
 *   scales [rows_cap][d/16] E4M3 scale of each block of 16 values (32 B/row)
 *   kidx   [rows_cap][di]   E4M3 indexer key, one per entry, shared by all
 *                           indexer heads                    (di = 64 or 128)
 * Logical entry t of sequence b lives in physical row
 *   page_table[b * max_pages + t / page_size] * page_size + t % page_size.
 * A contiguous per-sequence cache is the case max_pages = 1, page_size =
 * per-sequence capacity, page_table[b] = b. page_size must be a multiple of
 * 32, and of 128 when it exceeds 128. seq_len[b] is the number of valid
 * entries of sequence b (device array).
 */
typedef struct {
    uint8_t *codes;
    uint8_t *scales;
    uint8_t *kidx;
    const int32_t *page_table;
    const int32_t *seq_len;
    int64_t rows_cap;
    int32_t d;
    int32_t di;
    int32_t page_size;
    int32_t max_pages;
    int32_t batch;
    int32_t reserved;
} csa2_kv_desc;

/*
 * FP4 quantise + append ([P3] "V4.1-Flash also uses FP4 quantization";
 * [P4] "How are cache precision and storage arranged?": E2M1 main KV).
 * x_bf16 [n][d] bf16 rows. Row i is stored at logical position pos[i] of
 * sequence seq[i] (device arrays). For each block of 16 values:
 *   amax = max|x|;  s = E4M3_RNE_satfinite(amax / 6)   (binary32 division)
 *   c_i  = 0 if value(s) == 0 else E2M1_RNE_satfinite(x_i / value(s))
 * Rounding is to nearest with ties to the even mantissa; a NaN element gives
 * a signed zero code and does not enter amax. Rows whose (seq, pos) falls
 * outside the page table or the cache are skipped and set the device error
 * word. seq_len is not updated (the caller owns it).
 */
csa2_status csa2_append_fp4(const void *x_bf16, int32_t n, const int32_t *seq,
                            const int64_t *pos, const csa2_kv_desc *kv,
                            cudaStream_t stream);

/*
 * FP8 appends, the write side of the short-window KV and of the indexer keys
 * ([P3] "V4.1-Flash also uses FP4 quantization": the short-window SWA KV is
 * kept at FP8; [P4] "How are cache precision and storage arranged?").
 * Every bf16 value is converted on its own to E4M3: round to nearest, ties to
 * the even mantissa, saturating to +-448, no scale; a NaN keeps its sign and
 * becomes the E4M3 NaN code 0x7F.
 *
 * csa2_append_swa_e4m3: x_bf16 [n][512] window rows; row i goes to ring slot
 *   pos[i] % ring_rows of sequence seq[i] in swa [batch][ring_rows][512]
 *   (the buffer csa2_sparse_attn_decode reads with swa_seq_stride =
 *   ring_rows). pos >= 0.
 * csa2_append_kidx_e4m3: x_bf16 [n][kv->di] indexer keys; row i goes to the
 *   physical row of logical entry pos[i] of sequence seq[i] in kv->kidx.
 * seq, pos: device arrays. Rows whose destination falls outside the buffer
 * (bad sequence, negative position, outside the page table or the cache) are
 * skipped and set the device error word. n = 0 is a no-op. x_bf16 16-byte
 * aligned; swa 8-byte aligned.
 */
csa2_status csa2_append_swa_e4m3(const void *x_bf16, int32_t n, const int32_t *seq,
                                 const int64_t *pos, uint8_t *swa, int32_t batch,
                                 int64_t ring_rows, cudaStream_t stream);
csa2_status csa2_append_kidx_e4m3(const void *x_bf16, int32_t n, const int32_t *seq,
                                  const int64_t *pos, const csa2_kv_desc *kv,
                                  cudaStream_t stream);

/*
 * Full-mode indexer ([P3] modes paragraph: a Full layer scores the whole
 * context and keeps its Top-K; [P4]: the first Full layer also builds the
 * candidate pool of the hierarchical indexer).
 * nq queries; query i belongs to sequence i / q_per_seq.
 *   qidx [nq][hi][di] E4M3, w [nq][hi] f32.
 *   q_limit [nq]: number of entries query i may see (entries 0..q_limit-1);
 *   NULL means seq_len of its sequence. n_max >= every such limit.
 * Score of entry t (reading of the pages, which give no formula):
 *   score(t) = sum_h w_h * max(0, <q_h, kidx_t>)    (f32, tensor cores)
 * topk [nq][k]: the k best visible entries under (score desc, id asc);
 * pool [nq][p] (optional, p = 0 and pool = NULL to skip): the p best, the
 * candidate pool a Reindex layer re-scores. Both lists are in ascending id
 * order and padded with -1 when fewer entries are visible; topk is a subset
 * of pool. Scores are exact (hence the ids bit-exact) whenever every
 * partial sum is an integer below 2^24, as with small-integer E4M3 data.
 * Requires 1 <= hi <= 16, di in {64, 128}, 1 <= k <= 8192, 0 <= p <= 8192,
 * k <= p if p > 0 (CSA2_ERR_UNSUPPORTED for larger ranks).
 * ws: at least csa2_index_full_workspace_size(nq, n_max) bytes.
 */
csa2_status csa2_index_full(const uint8_t *qidx, const float *w, int32_t nq,
                            int32_t q_per_seq, int32_t hi, const int32_t *q_limit,
                            int64_t n_max, const csa2_kv_desc *kv, int32_t k, int32_t p,
                            int32_t *topk, int32_t *pool, void *ws, size_t ws_bytes,
                            cudaStream_t stream);

size_t csa2_index_full_workspace_size(int32_t nq, int64_t n_max);

/*
 * Reindex-mode indexer ([P3]: a Reindex layer keeps no cache of its own and
 * filters again what a Full layer produced; [P4]: it scores anew to choose
 * its own Top-K, and deeper layers look only inside the Full layer's pool).
 * pool [nq][p]: ids from a Full layer (-1 entries are padding; any order;
 * no duplicates). Scores the pool ids with this layer's qidx/w as in
 * csa2_index_full and writes their Top-k under (score desc, id asc) to
 * topk [nq][k], in pool order, padded with -1. p <= 16384.
 * ws: at least csa2_index_reindex_workspace_size(nq, p) bytes.
 */
csa2_status csa2_index_reindex(const uint8_t *qidx, const float *w, int32_t nq,
                               int32_t q_per_seq, int32_t hi, const int32_t *pool, int32_t p,
                               const csa2_kv_desc *kv, int32_t k, int32_t *topk, void *ws,
                               size_t ws_bytes, cudaStream_t stream);

size_t csa2_index_reindex_workspace_size(int32_t nq, int32_t p);

/*
 * Sparse + sliding-window decode attention ([P3] modes and FP4 paragraphs:
 * attention over the selected global entries, FP4 values restored for
 * computation; SWA KV kept at FP8).
 *   q_bf16 [nq][h][d] bf16, query i of sequence i / q_per_seq.
 *   topk [nq][k]: global entry ids (-1 = empty); each row is dequantised
 *   (E2M1 code x E4M3 scale, exact in f16) and used as key and value.
 *   Window rows of query i: the swa_end[i] - swa_begin[i] rows
 *   (swa_begin[i] + j) mod swa_seq_stride of the E4M3 buffer
 *   swa + (i / q_per_seq) * swa_seq_stride * d (raw E4M3, no scale; a ring of
 *   swa_seq_stride rows per sequence, as csa2_append_swa_e4m3 writes it),
 *   also key and value. A non-empty window needs 0 <= swa_begin[i] <
 *   swa_seq_stride and swa_end[i] - swa_begin[i] <= min(w_max,
 *   swa_seq_stride); otherwise it is dropped and the device error word set.
 * Per head, over the union S of selected rows and window rows:
 *   o_h = sum_j softmax_j(softmax_scale * <q_h, v_j>) v_j
 * written as bf16 o [nq][h][d]; lse [nq][h] (nullable) gets the natural-log
 * sum of exp of the scaled scores. An empty S gives o = 0, lse = -inf.
 * Arithmetic: q converted to f16 (round to nearest), f16 tensor-core
 * products with f32 accumulation, f32 online softmax, probabilities rounded
 * to f16 for the P*V product. h in {16, 32, 64}. Range of q: a bf16 value of
 * magnitude 65536 or more (or an infinity or NaN) has no finite f16 value;
 * the kernel records CSA2_DEVERR_Q_RANGE and that query's o and lse are
 * undefined (other queries are unaffected). Magnitudes below 2^-14 become
 * f16 subnormals: absolute error at most 2^-25 per element.
 * ws: at least csa2_sparse_attn_workspace_size(nq, h, k, w) bytes, with
 * w = w_max when a window is given and w = 0 when swa_begin is NULL (the
 * split plan follows the rows the call really has; the size is not monotone
 * in w, so size a workspace shared by both kinds of call for both).
 */
csa2_status csa2_sparse_attn_decode(const void *q_bf16, int32_t nq, int32_t q_per_seq,
                                    int32_t h, const csa2_kv_desc *kv, const int32_t *topk,
                                    int32_t k, const uint8_t *swa, int64_t swa_seq_stride,
                                    const int32_t *swa_begin, const int32_t *swa_end,
                                    int32_t w_max, float softmax_scale, void *o_bf16, float *lse,
                                    void *ws, size_t ws_bytes, cudaStream_t stream);

size_t csa2_sparse_attn_workspace_size(int32_t nq, int32_t h, int32_t k, int32_t w_max);

/*
 * The same decode attention for callers that cannot allocate device memory
 * (for example code running where cudaMalloc is not permitted, or a caller
 * that owns no allocator). The paper has no counterpart: it is a library
 * convenience. Arguments, results and errors are those of
 * csa2_sparse_attn_decode, without ws / ws_bytes: the split partials live in
 * a fixed array of CSA2_ATTN_STATIC_SCRATCH_BYTES bytes that the library
 * holds in device global memory (one copy per device), and nothing is
 * allocated by the call.
 * Limit: when csa2_sparse_attn_workspace_size(nq, h, k, w_max) (w_max taken
 * as 0 without a window) exceeds CSA2_ATTN_STATIC_SCRATCH_BYTES the call
 * returns CSA2_ERR_WORKSPACE and launches nothing; use
 * csa2_sparse_attn_decode with a caller-owned workspace instead.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress with that device current); make that first call
 * before any stream capture begins. The address belongs to the device's
 * context: when that context is replaced (cudaDeviceReset, or a context
 * destroyed and created again), the next call looks it up again, so make
 * the first call after such a change outside stream capture as well. No part
 * of the array has to start at zero: each call writes every partial it reads
 * back.
 * Concurrency: all calls on one device share the one array, so two calls
 * whose kernels can overlap (different streams, or different host threads,
 * without ordering between them) race on it and give wrong results. Order
 * such calls on one stream, or use csa2_sparse_attn_decode.
 */
#define CSA2_ATTN_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
csa2_status csa2_sparse_attn_decode_static(const void *q_bf16, int32_t nq, int32_t q_per_seq,
                                           int32_t h, const csa2_kv_desc *kv, const int32_t *topk,
                                           int32_t k, const uint8_t *swa, int64_t swa_seq_stride,
                                           const int32_t *swa_begin, const int32_t *swa_end,
                                           int32_t w_max, float softmax_scale, void *o_bf16,
                                           float *lse, cudaStream_t stream);

/*
 * NVFP4 speed variant of csa2_sparse_attn_decode ([P3] paragraph "V4.1-Flash
 * also uses FP4 quantization": the FP4 values are restored for computation
 * on the chip; here the scores of the selected entries are computed from
 * the FP4 codes directly). Arguments, layouts, workspace rule and errors are
 * those of csa2_sparse_attn_decode, with h in {16, 32, 64} and the workspace
 * sized by csa2_sparse_attn_nvfp4_workspace_size. The block-scaled products
 * run at 64 heads only (their scale-factor layout is established for that
 * width): 16 and 32 heads run as a 64-head call whose q is padded with zero
 * heads in the workspace, and the padded heads' outputs are dropped. What it computes differs
 * in one step: q is first quantised to NVFP4 with the cache's own block
 * quantiser (per 16 values one E4M3 scale = RNE(amax / 6), E2M1 codes RNE
 * of x / scale), and that quantised q (exact in f16) is used for the scores
 * of every row; the values (P * V), the softmax and the probabilities are as
 * in csa2_sparse_attn_decode. Its reference is therefore
 * csa2_sparse_attn_decode's result for the quantised q, within the same
 * tolerance; against the unquantised q it deviates by the effect of the
 * quantisation on the scores.
 * Kernel: tiles made only of selected entries multiply the raw FP4 codes and
 * E4M3 block scales of the cache against the FP4 q with block-scaled
 * tensor-core products (no dequantisation before S); the remaining tiles
 * (a partial last entry tile and the window) take the f16 path.
 */
csa2_status csa2_sparse_attn_decode_nvfp4(const void *q_bf16, int32_t nq, int32_t q_per_seq,
                                          int32_t h, const csa2_kv_desc *kv, const int32_t *topk,
                                          int32_t k, const uint8_t *swa, int64_t swa_seq_stride,
                                          const int32_t *swa_begin, const int32_t *swa_end,
                                          int32_t w_max, float softmax_scale, void *o_bf16,
                                          float *lse, void *ws, size_t ws_bytes,
                                          cudaStream_t stream);

/* Workspace bytes of csa2_sparse_attn_decode_nvfp4 (split partials plus q's
 * FP4 codes and scales; for 16 or 32 heads also the padded q, o and lse);
 * 0 for a head count other than 16, 32, 64. */
size_t csa2_sparse_attn_nvfp4_workspace_size(int32_t nq, int32_t h, int32_t k, int32_t w_max);

/*
 * Building blocks of a long sequence decoded with its entries split across
 * GPUs by entry range (one exchange step per layer; the pages put 1M-token
 * contexts on one sequence: [P3] "CSA2 tackles storage", [P4] "How does the
 * cache compress along three dimensions at once?"). Each rank holds the
 * entries [offset, offset + n_r) of the sequence in its own cache.
 *
 * csa2_score_ids: score the given entry ids (local to kv, -1 = empty) as the
 *   indexer does, into unique 64-bit keys (ordered score key << 32 |
 *   ~(id + id_offset)); empty ids give key 0. ids [nq][m], keys [nq][m]
 *   (8-byte aligned), qidx / w as in csa2_index_full. Requires
 *   kv->di in {64, 128} and 1 <= hi <= 16 (else CSA2_ERR_UNSUPPORTED),
 *   m >= 1 and id_offset >= 0 (else CSA2_ERR_INVALID_ARG); id + id_offset
 *   must stay below 2^31. An id outside the cache gives key 0 and sets
 *   CSA2_DEVERR_BAD_ROW. No workspace.
 * csa2_select_keys: the k largest keys of each query's m keys, written as
 *   the ids they carry (~ of the low 32 bits), in key-array order, padded
 *   with -1; key 0 is empty. Because the id is part of the key, equal scores
 *   are taken in ascending id order. keys [nq][m], ids [nq][k]. Requires
 *   m, k >= 1 (else CSA2_ERR_INVALID_ARG) and m <= 2^20 (else
 *   CSA2_ERR_UNSUPPORTED); up to about 28000 keys are staged in shared
 *   memory, larger sets are re-read from L2 in every radix pass. No
 *   workspace.
 * csa2_sparse_attn_partial: csa2_sparse_attn_decode over this rank's rows,
 *   writing the normalised f32 o [nq][h][512] and lse [nq][h] instead of
 *   bf16 o; lse is required (else CSA2_ERR_INVALID_ARG); the same workspace
 *   rule. A query with no rows gives o = 0 and lse = -inf.
 * csa2_attn_merge: merge g such partials o_parts [g][nq][h][512],
 *   lse_parts [g][nq][h] into bf16 o [nq][h][512] and lse [nq][h]
 *   (nullable): o = sum_r exp(lse_r - M) o_r / sum_r exp(lse_r - M) with
 *   M = max_r lse_r; parts with lse = -inf weigh nothing, and all of them
 *   -inf give o = 0, lse = -inf. Requires h in {16, 32, 64} (else
 *   CSA2_ERR_UNSUPPORTED), g >= 1, o_parts / o_bf16 16-byte aligned (else
 *   CSA2_ERR_INVALID_ARG). No workspace.
 */
csa2_status csa2_score_ids(const uint8_t *qidx, const float *w, int32_t nq, int32_t q_per_seq,
                           int32_t hi, const int32_t *ids, int32_t m, const csa2_kv_desc *kv,
                           int32_t id_offset, unsigned long long *keys, cudaStream_t stream);
csa2_status csa2_select_keys(const unsigned long long *keys, int32_t nq, int32_t m, int32_t k,
                             int32_t *ids, cudaStream_t stream);
csa2_status csa2_sparse_attn_partial(const void *q_bf16, int32_t nq, int32_t q_per_seq, int32_t h,
                                     const csa2_kv_desc *kv, const int32_t *topk, int32_t k,
                                     const uint8_t *swa, int64_t swa_seq_stride,
                                     const int32_t *swa_begin, const int32_t *swa_end,
                                     int32_t w_max, float softmax_scale, float *o_f32, float *lse,
                                     void *ws, size_t ws_bytes, cudaStream_t stream);
csa2_status csa2_attn_merge(const float *o_parts, const float *lse_parts, int32_t g, int32_t nq,
                            int32_t h, void *o_bf16, float *lse, cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the device error word.
 * *code receives 0 when no device-side condition was recorded since the
 * last call, else a bit set of CSA2_DEVERR_* values. Returns CSA2_OK, or
 * CSA2_ERR_DEVICE when *code != 0, or CSA2_ERR_CUDA. */
#define CSA2_DEVERR_BAD_ROW 1u       /* id / page / position outside the cache */
#define CSA2_DEVERR_WAIT_TIMEOUT 2u  /* a bounded barrier wait gave up         */
#define CSA2_DEVERR_SELECT 4u        /* selection produced more ids than asked  */
#define CSA2_DEVERR_Q_RANGE 8u       /* attention q outside f16's finite range  */
csa2_status csa2_device_status(cudaStream_t stream, uint32_t *code);

/*
 * Self-check of the device-side failure detection (no counterpart in the
 * pages). Every barrier wait in the library's kernels is bounded (one second
 * of device time); a wait that runs out records CSA2_DEVERR_WAIT_TIMEOUT,
 * skips the rest of its work and lets the kernel end, so the context stays
 * usable. This call launches one thread that waits, with a limit of
 * limit_us microseconds (1 ... 1000000, else CSA2_ERR_INVALID_ARG), on a
 * barrier that nothing arrives at; afterwards csa2_device_status() reports
 * CSA2_DEVERR_WAIT_TIMEOUT. Nothing else is touched.
 */
csa2_status csa2_check_wait_timeout(uint32_t limit_us, cudaStream_t stream);

const char *csa2_status_string(csa2_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t csa2_version(void);

#ifdef __cplusplus
}
#endif
#endif
