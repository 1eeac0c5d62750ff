/*
 * jssa.h - C ABI of libjssa.so: Joint Subspace Sparse Attention (JSSA) decode and calibration
 * on NVIDIA B200 (sm_100a).
 *
 * Method (JSSA summary, picx.dev, "Theoretical Foundation" and "Methodology" sections 3.1-3.4;
 * JSSA README, "Paper-to-code map" and section 4): per layer and KV head an orthonormal basis
 * M (r x d) is calibrated once as the top-r eigenvectors of the sum of the unit-trace second
 * moments of group-mean queries and of keys (eq. (5)). At each decode step the new key's
 * projection M k is stored as FP8 E4M3 in a scoring cache (section 3.4), every cached token is
 * scored with the projected group-mean query (eq. (1), section 3.1 step 2), the top-B tokens are
 * selected independently per KV head, and attention of every query head runs over its KV head's
 * selected rows, read in place from the paged KV cache (section 3.3).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers owned by the caller, except where stated. The library never
 *   allocates or frees memory and never synchronises a stream (jssa_device_error excepted);
 *   jssa_decode_host creates two streams and a few events per workspace on its first call.
 *   Every call is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 * - bf16 tensors are passed as `const jssa_bf16*` (raw 16-bit storage).
 * - Return value: JSSA_OK (0); a negative JSSA_ERR_* code when the host-side argument check
 *   fails, in which case nothing was launched; or a positive cudaError_t from the launch.
 * - Head mapping: query head i belongs to KV head i / G with G = h_q / h_kv.
 * - Paged KV cache: element (page, slot, head, x) of the K (or V) cache is at
 *   cache[page*kv_page_stride + slot*kv_slot_stride + head*kv_head_stride + x]; strides are in
 *   elements, the head dimension is contiguous. Logical position t of sequence b lives in page
 *   block_table[b*max_pages + t/page_size], slot t%page_size. block_table is int32
 *   [batch, max_pages], seq_lens int32 [batch]. page_size is a power of two.
 * - Scoring cache: uint8 E4M3 codes laid out [num_pages, h_kv, page_size, r] (one contiguous
 *   run of page_size*r bytes per page and KV head), same page numbering as the KV cache.
 * - Basis: float32 [h_kv, r, d], rows orthonormal (output of jssa_compute_basis); the store
 *   and score entry points want it, the scoring cache and the queries q 16-byte aligned
 *   (JSSA_ERR_ALIGN otherwise).
 * - Index sets: int32 idx [batch, h_kv, budget] holds logical positions in ascending order,
 *   padded with -1; int32 count [batch, h_kv] = min(budget, seq_len).
 * - Device-side checks: a page number outside [0, num_pages), a position outside the block
 *   table, or a seq_len above max_pages*page_size is never dereferenced: the row is skipped and
 *   a flag is raised in the library's device error word (jssa_device_error). Kernels never trap.
 * - Supported template shapes: d = 128 with r in {16, 32, 64}, and d = 256 with r = 64 (the
 *   global layer of a hybrid sliding-window / global stack); G <= 8 for attention. A basis of
 *   rank below 16 runs through the r = 16 instance with zero rows appended: their codes are
 *   zero and the scores, hence the selections, are those of the smaller rank.
 * - Multi-head latent attention (one latent "KV head" of 576 dimensions per token: 512 latent +
 *   64 rotary): the store and score entry points take d = 576 and r = 64, the rank of the latent
 *   basis, float32 [1, r, 512], which projects the 512 latent dimensions; the 64 rotary
 *   dimensions pass through unprojected, so a scoring row holds r + 64 = 128 codes (JSSA README,
 *   section 4 notes: the MLA basis is [1, r, kv_lora_rank]; JSSA summary, section 3.4: 64 latent
 *   + 64 RoPE scoring dimensions). The scoring cache is then uint8 [num_pages, 1, page_size, 128].
 */
#ifndef JSSA_H_
#define JSSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JSSA_API __attribute__((visibility("default")))
#else
#define JSSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t jssa_bf16;   /* bfloat16 storage */
typedef void* jssa_stream_t;  /* cudaStream_t */

enum jssa_status {
  JSSA_OK = 0,
  JSSA_ERR_NULL = -1,         /* a required pointer is NULL */
  JSSA_ERR_SHAPE = -2,        /* inconsistent or out-of-range sizes */
  JSSA_ERR_UNSUPPORTED = -3,  /* no kernel instance for (d, r, G) or size beyond the limits */
  JSSA_ERR_ALIGN = -4,        /* a pointer or stride breaks the 16-byte alignment rule */
  JSSA_ERR_WORKSPACE = -5,    /* workspace NULL or smaller than jssa_workspace_size */
  JSSA_ERR_DEVICE = -6,       /* no usable CUDA device / device query failed */
  JSSA_ERR_SCRATCH_LIMIT = -7 /* sizes need more than the allocation-free entry point's scratch */
};

/* Device error flags (bitwise OR), read with jssa_device_error. */
enum jssa_device_flag {
  JSSA_DEVERR_PAGE = 1,       /* block_table or slot_mapping named a page outside [0, num_pages) */
  JSSA_DEVERR_INDEX = 2,      /* an index-set entry outside [0, max_pages*page_size) */
  JSSA_DEVERR_SEQLEN = 4,     /* seq_len < 0 or > max_pages*page_size (clamped) */
  JSSA_DEVERR_SELECT = 8,     /* internal: inconsistent top-B counts (never expected) */
  JSSA_DEVERR_RESCAN = 16,    /* information only: a sampled candidate threshold was too high and
                                 the selection rescanned the sequence (the result is exact) */
  JSSA_DEVERR_TIMEOUT = 32    /* a bounded wait inside a kernel ran out (its results are invalid) */
};

/* Workspace clients for jssa_workspace_size. */
enum jssa_fn {
  JSSA_FN_SCORE_TOPK = 1,
  JSSA_FN_INDEXED_ATTEND = 2,
  JSSA_FN_DENSE_DECODE = 3,
  JSSA_FN_DECODE = 4,
  JSSA_FN_COMPUTE_BASIS = 5,
  JSSA_FN_MLA_ATTEND = 6,
  JSSA_FN_MLA_DECODE = 7,
  JSSA_FN_DECODE_HOST = 8
};

/* Text for a status code (static storage). */
JSSA_API const char* jssa_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
JSSA_API int jssa_version(void);

/*
 * Debug control (the pages have no counterpart): the clock-cycle limit of each wait on the tensor
 * cores inside the tile loop of jssa_mla_attend (default 2e9 cycles, about one second at the
 * boost clock). A wait that runs out raises JSSA_DEVERR_TIMEOUT in the device error word; the
 * CTA then waits, with the default limit, for every tensor-core operation it issued, frees its
 * tensor memory and returns, so the context stays usable and the next call runs normally (its
 * output is invalid only for the call that timed out). cycles <= 0 restores the default. The limit
 * is read when a call is enqueued (a kernel argument): a CUDA graph keeps the limit it was captured
 * with. Returns the previous limit. Process-wide; not synchronised with calls in flight.
 */
JSSA_API long long jssa_set_wait_limit(long long cycles);

/*
 * Bytes of device workspace the entry point `fn` needs for these sizes (written to *bytes; 0
 * means none). max_pages and page_size are the block-table width and page size the call will
 * get (every seq_len is at most max_pages*page_size); budget is the token budget B, except for
 * JSSA_FN_DENSE_DECODE where it carries the call's window (<= 0: full context); the basis
 * ignores it. Score + top-B keeps its candidate keys and positions in the workspace. The
 * split-K attention entry points keep a per-(sequence, KV head) ticket counter at the start of
 * theirs: for jssa_indexed_attend and jssa_dense_decode those counters must be zero when the call
 * starts -- clear the workspace with jssa_workspace_init before its first use and again after it
 * served another entry point or a larger batch*h_kv (the kernels leave the counters at zero on
 * exit). jssa_decode clears its counters itself. Calls that share one workspace must not overlap
 * on the GPU.
 */
JSSA_API int jssa_workspace_size(int fn, int batch, int h_q, int h_kv, int d, int max_pages,
                                 int page_size, int budget, size_t* bytes);

/* Zero `ws_bytes` bytes of workspace on `stream` (cudaMemsetAsync). */
JSSA_API int jssa_workspace_init(void* ws, size_t ws_bytes, jssa_stream_t stream);

/*
 * Calibration, step 1: accumulate uncentred second moments of group-mean queries and of keys.
 * JSSA summary, Theoretical Foundation (the second-moment matrices of eq. (3)) and section 3.2;
 * JSSA README, section 2 (second moments of post-RoPE queries and keys).
 *   gram_q[h] += sum_n qbar_n qbar_n^T,  qbar_n = (1/G) sum_g q[n, h*G+g, :]
 *   gram_k[h] += sum_n k_n k_n^T,        k_n = k[n, h, :]
 * q: bf16 [n, h_q, d], row n at q + n*q_stride_n (elements, >= h_q*d, multiple of 8).
 * k: bf16 [n, h_kv, d], row n at k + n*k_stride_n (elements, >= h_kv*d, multiple of 8).
 * gram_q, gram_k: float64 [h_kv, d, d], accumulated in place (zero them before the first call).
 * d in {128, 256, 512}; n <= 16776960 per call (JSSA_ERR_SHAPE beyond), any G.
 * Products of exact bf16 inputs are summed in fp32 on tensor cores within a tile of samples and
 * added to the float64 totals: for G * d <= 2048 the G^2 products of each sample's query heads
 * (exact), otherwise the group mean formed in fp32 and split exactly into three bf16 planes (the
 * six largest plane products; the rest are below 2^-24 of the result). n may be 0 (no-op).
 */
JSSA_API int jssa_calibrate_accumulate(const jssa_bf16* q, int64_t q_stride_n, const jssa_bf16* k,
                              int64_t k_stride_n, int n, int h_q, int h_kv, int d,
                              double* gram_q, double* gram_k, jssa_stream_t stream);

/*
 * Calibration, step 1, for a multi-head latent layer: the second moments of the head mean of the
 * latent part of the absorbed queries and of the latent part of the cached rows, from which
 * jssa_compute_basis (d = 512) gives the latent basis [1, r, 512]. JSSA README, section 2 (the MLA
 * basis [1, r, kv_lora_rank]; the Gram collection of large latent models) and section 4 notes.
 *   gram_q += sum_n qbar_n qbar_n^T, qbar_n = (1/h_q) sum_i q[n, i, 0:512]
 *   gram_k += sum_n c_n c_n^T,       c_n = kv[n, 0:512]
 * q: bf16 absorbed queries, head i of sample n at q + n*q_stride_n + i*q_stride_head (576 per
 * head, q_stride_head >= 512; strides multiples of 8 elements). kv: bf16 latent rows, row n at
 * kv + n*kv_stride_n (>= 512). gram_q, gram_k: float64 [1, 512, 512], accumulated in place.
 * Same arithmetic and limits as jssa_calibrate_accumulate (the mean-plane form).
 */
JSSA_API int jssa_mla_calibrate_accumulate(const jssa_bf16* q, int64_t q_stride_n,
                                           int64_t q_stride_head, const jssa_bf16* kv,
                                           int64_t kv_stride_n, int n, int h_q, double* gram_q,
                                           double* gram_k, jssa_stream_t stream);

/*
 * Calibration, step 2: M = TopEig_r(gram_q/tr(gram_q) + gram_k/tr(gram_k))^T per KV head.
 * JSSA summary, eq. (5); JSSA README, paper-to-code map (compute_basis) and section 2 (one
 * eigendecomposition per layer and KV head). Cyclic Jacobi in float64 on the device.
 * basis: float32 [h_kv, r, d], rows = eigenvectors of the r largest eigenvalues, descending,
 * each signed so that its largest-magnitude entry is positive (lowest index on ties).
 * eigvals: float64 [h_kv, d] descending, or NULL. ws: >= jssa_workspace_size(JSSA_FN_COMPUTE_BASIS)
 * (h_kv d^2 doubles for the eigenvectors, plus h_kv d (d + 1) for the matrices at d = 256).
 */
JSSA_API int jssa_compute_basis(const double* gram_q, const double* gram_k, int h_kv, int d, int r,
                       float* basis, double* eigvals, void* ws, size_t ws_bytes,
                       jssa_stream_t stream);

/*
 * Store step: scoring code c = e4m3(M_h k) of each given token and KV head.
 * JSSA summary, section 3.4 (K_proj = K M^T kept as an FP8 scoring-only cache); JSSA README,
 * section 4 notes (r bytes per token and KV head). The projection is summed in float64 and
 * rounded once to E4M3 (round to nearest even, saturating to +-448, no scale).
 * k: bf16 [t, h_kv, d] with row stride k_stride_t elements. slot_mapping: int64 [t], flat slot
 * page*page_size + offset, negative = skip. score_cache: see conventions. A latent layer (d 576,
 * r 64) writes e4m3(M_lat k[0:512]) and then e4m3(k[512:576]) (the rotary dimensions, one
 * rounding each).
 */
JSSA_API int jssa_store(const jssa_bf16* k, int64_t k_stride_t, const int64_t* slot_mapping, int t,
               int h_kv, int d, int r, const float* basis, uint8_t* score_cache,
               int64_t num_pages, int page_size, jssa_stream_t stream);

/*
 * Score + top-B: for every sequence b and KV head h, p = M_h qbar (qbar the mean of the G query
 * heads of h), s_t = sum_j dec(c_tj) p_j for every t < seq_len (fp32), and the index set of the
 * min(budget, seq_len) largest s_t, ties to the lower position, written ascending.
 * JSSA summary, eq. (1) and section 3.1 steps 1-2; JSSA README, section 4 (jssa_budget).
 * Three kernels: a per-(sequence, KV head) prep (query projection, p split into two f16 digit
 * vectors with power-of-two weights, and a candidate threshold from a sample of the scores), a
 * streaming scan (codes widened exactly to f16 and multiplied on the tensor cores, fp32
 * accumulation) that keeps only keys at or above the threshold, and an exact per-(sequence,
 * KV head) selection (which rescans when the threshold let through fewer than
 * min(budget, seq_len) keys).
 * q: bf16 [batch, h_q, d] contiguous. ws: >= jssa_workspace_size(JSSA_FN_SCORE_TOPK).
 * Limits (JSSA_ERR_UNSUPPORTED beyond them): max_pages * page_size <= 4194304 positions and
 * batch * h_kv <= 65535.
 */
JSSA_API int jssa_score_topk(const jssa_bf16* q, const float* basis, const uint8_t* score_cache,
                    const int32_t* block_table, int max_pages, const int32_t* seq_lens, int batch,
                    int h_q, int h_kv, int d, int r, int64_t num_pages, int page_size, int budget,
                    int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                    jssa_stream_t stream);

/*
 * Gather-free indexed attention: out[b, i] = softmax(scale * q_i K_S^T) V_S over the positions
 * S = idx[b, i/G, 0:count[b, i/G]], with K and V rows read in place from the paged cache (no
 * staging buffer), split-K over S and an online-softmax merge (last CTA of each (b, h) merges).
 * JSSA summary, section 3.1 step 3 and section 3.3; JSSA README, paper-to-code map.
 * q, out: bf16 [batch, h_q, d] contiguous. count = 0 gives a zero output row.
 */
JSSA_API int jssa_indexed_attend(const jssa_bf16* q, const jssa_bf16* k_cache, const jssa_bf16* v_cache,
                        int64_t kv_page_stride, int64_t kv_slot_stride, int64_t kv_head_stride,
                        const int32_t* block_table, int max_pages, const int32_t* idx,
                        const int32_t* count, int batch, int h_q, int h_kv, int d, int budget,
                        int64_t num_pages, int page_size, float softmax_scale, jssa_bf16* out,
                        void* ws, size_t ws_bytes, jssa_stream_t stream);

/*
 * Dense paged decode attention (the full-KV baseline): out[b, i] = attention of q_i over every
 * position [lo, seq_len) with lo = max(0, seq_len - window) when window > 0, else 0.
 * JSSA README, section 3 (attention microbenchmark against full-KV decode) and section 4 notes
 * (sliding-window layers keep dense attention). Same kernel body as jssa_indexed_attend. Launched
 * with programmatic dependent launch: it may be scheduled while the preceding kernel on `stream`
 * finishes, and reads nothing before that kernel has completed.
 */
JSSA_API int jssa_dense_decode(const jssa_bf16* q, const jssa_bf16* k_cache, const jssa_bf16* v_cache,
                      int64_t kv_page_stride, int64_t kv_slot_stride, int64_t kv_head_stride,
                      const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                      int batch, int h_q, int h_kv, int d, int64_t num_pages, int page_size,
                      int window, float softmax_scale, jssa_bf16* out, void* ws,
                      size_t ws_bytes, jssa_stream_t stream);

/*
 * BF16 scoring-cache ablation (JSSA README, section 4 notes, and JSSA summary, section 3.4: the
 * method keeps the projected keys in FP8; these two entry points keep them in bf16, two bytes per
 * dimension, to measure that choice). jssa_store_bf16 is jssa_store writing bf16(M_h k) (float64
 * dot product, one correct rounding) into score_cache bf16 [num_pages, h_kv, page_size, r];
 * jssa_score_topk_bf16 is jssa_score_topk reading that cache (the scores multiply the bf16 codes
 * by four bf16 digits of p). Only d = 128, r = 32 (JSSA_ERR_UNSUPPORTED otherwise). Same
 * arguments, layouts, workspace and errors as the FP8 entry points.
 */
JSSA_API int jssa_store_bf16(const jssa_bf16* k, int64_t k_stride_t, const int64_t* slot_mapping,
                             int t, int h_kv, int d, int r, const float* basis,
                             jssa_bf16* score_cache, int64_t num_pages, int page_size,
                             jssa_stream_t stream);
JSSA_API int jssa_score_topk_bf16(const jssa_bf16* q, const float* basis,
                                  const jssa_bf16* score_cache, const int32_t* block_table,
                                  int max_pages, const int32_t* seq_lens, int batch, int h_q,
                                  int h_kv, int d, int r, int64_t num_pages, int page_size,
                                  int budget, int32_t* idx, int32_t* count, void* ws,
                                  size_t ws_bytes, jssa_stream_t stream);

/*
 * Multi-head latent attention over selected positions, absorbed form (JSSA summary, section 3.3;
 * JSSA README, paper-to-code map and section 4 notes: one latent row per token, 512 latent + 64
 * rotary dimensions, attended in place):
 *   out[b, i, :] = sum_j softmax_j(softmax_scale * q[b, i] . kv[j]) kv[j, 0:512]
 * over j in the index set of sequence b, i.e. jssa_score_topk run with h_kv = 1, d = 576 and
 * r = 64 on the latent scoring cache (the latent basis [1, 64, 512]; the 64 rotary dimensions
 * pass through).
 * q: bf16 [batch, h_q, 576] absorbed queries (h_q a multiple of 16; budget <= 262144,
 * JSSA_ERR_UNSUPPORTED otherwise). kv_cache: bf16 latent cache,
 * row (page p, slot s) at p*kv_page_stride + s*kv_slot_stride elements (576 contiguous, 16-byte
 * aligned). idx/count: int32 [batch, 1, budget] / [batch, 1] (count clamped to [0, budget]).
 * out: bf16 [batch, h_q, 512], 16-byte aligned. ws: >= jssa_workspace_size(JSSA_FN_MLA_ATTEND,
 * batch, h_q, 1, 576, ...); its split counters must be zero when the call starts
 * (jssa_workspace_init once) and are zero again when it ends. Out-of-range positions and pages
 * are skipped and flagged; a bounded wait on the tensor cores that runs out raises
 * JSSA_DEVERR_TIMEOUT (the output is then invalid).
 */
JSSA_API int jssa_mla_attend(const jssa_bf16* q, const jssa_bf16* kv_cache, int64_t kv_page_stride,
                             int64_t kv_slot_stride, const int32_t* block_table, int max_pages,
                             const int32_t* idx, const int32_t* count, int batch, int h_q,
                             int budget, int64_t num_pages, int page_size, float softmax_scale,
                             jssa_bf16* out, void* ws, size_t ws_bytes, jssa_stream_t stream);

/*
 * One whole decode step of a multi-head latent attention layer: (1) when kv_new is non-NULL,
 * write the new token's latent row (position seq_len-1 of each sequence) into the latent cache
 * and its scoring code (e4m3 of the latent basis applied to the 512 latent dimensions, then the 64
 * rotary dimensions) into the scoring cache; (2) score + top-B over the latent scoring cache
 * (jssa_score_topk with h_kv = 1, d = 576); (3) the latent attention over the selected rows
 * (jssa_mla_attend). The kernels are chained on `stream` with programmatic dependent launch and
 * no host synchronisation. JSSA README, paper-to-code map (JSSA on MLA) and section 4 notes; JSSA
 * summary, sections 3.1 and 3.4.
 * q: bf16 [batch, h_q, 576] absorbed queries (h_q a multiple of 16). kv_new: bf16 [batch, 576]
 * or NULL. kv_cache, strides, idx, count, out: as in jssa_mla_attend. basis: float32 [1, r, 512],
 * r = 64. score_cache: uint8 [num_pages, 1, page_size, r + 64]. ws: >=
 * jssa_workspace_size(JSSA_FN_MLA_DECODE, batch, h_q, 1, 576, max_pages, page_size, budget); no
 * clearing needed (the selection clears the attention's split counters).
 */
JSSA_API int jssa_mla_decode(const jssa_bf16* q, const jssa_bf16* kv_new, jssa_bf16* kv_cache,
                             int64_t kv_page_stride, int64_t kv_slot_stride, uint8_t* score_cache,
                             const float* basis, const int32_t* block_table, int max_pages,
                             const int32_t* seq_lens, int batch, int h_q, int r, int64_t num_pages,
                             int page_size, int budget, float softmax_scale, int32_t* idx,
                             int32_t* count, jssa_bf16* out, void* ws, size_t ws_bytes,
                             jssa_stream_t stream);

/*
 * Gather-then-attend ablation, step 1: copy the selected K and V rows of every (sequence, KV
 * head), in index order, into contiguous staging buffers (JSSA README, "Highlights" and section
 * 3: the gather-free attention is measured against gathering the selected rows first; JSSA
 * summary, section 3.3). Step 2 is jssa_dense_decode over the staging buffers viewed as a paged
 * cache of 16-token pages: page_stride 16*h_kv*d, slot_stride h_kv*d, head_stride d, sequence b
 * on pages b*budget_pad/16 ... (b+1)*budget_pad/16 - 1, seq_lens = lens_out.
 * idx, count: as produced by jssa_score_topk (count clamped to [0, budget]).
 * k_out, v_out: bf16 [batch, budget_pad, h_kv, d], budget_pad = budget rounded up to a multiple
 * of 16, 16-byte aligned, owned by the caller; slots at or past count are left untouched.
 * lens_out: int32 [batch] = count[b, 0] (every head of a sequence has the same count).
 * A position outside the block table or an unusable page is skipped (its staged row is
 * written as zeros) and flagged in the device error word.
 */
JSSA_API int jssa_gather_kv(const jssa_bf16* k_cache, const jssa_bf16* v_cache,
                            int64_t kv_page_stride, int64_t kv_slot_stride, int64_t kv_head_stride,
                            const int32_t* block_table, int max_pages, const int32_t* idx,
                            const int32_t* count, int batch, int h_kv, int d, int budget,
                            int64_t num_pages, int page_size, jssa_bf16* k_out, jssa_bf16* v_out,
                            int32_t* lens_out, jssa_stream_t stream);

/*
 * One whole decode step for one layer: (1) when k_new and v_new are non-NULL, write the new
 * token (position seq_len-1 of each sequence) into the K and V caches and its scoring code into
 * the scoring cache; (2) score + top-B; (3) gather-free indexed attention. The three kernels
 * are chained on `stream` with programmatic dependent launch and no host synchronisation.
 * JSSA summary, section 3.1; JSSA README, paper-to-code map (_sparse_decode_forward).
 * k_new, v_new: bf16 [batch, h_kv, d] contiguous (or both NULL). idx/count: outputs as in
 * jssa_score_topk. ws: >= jssa_workspace_size(JSSA_FN_DECODE); no clearing needed.
 */
JSSA_API int jssa_decode(const jssa_bf16* q, const jssa_bf16* k_new, const jssa_bf16* v_new,
                jssa_bf16* k_cache, jssa_bf16* v_cache, int64_t kv_page_stride,
                int64_t kv_slot_stride, int64_t kv_head_stride, uint8_t* score_cache,
                const float* basis, const int32_t* block_table, int max_pages,
                const int32_t* seq_lens, int batch, int h_q, int h_kv, int d, int r,
                int64_t num_pages, int page_size, int budget, float softmax_scale,
                int32_t* idx, int32_t* count, jssa_bf16* out, void* ws, size_t ws_bytes,
                jssa_stream_t stream);

/*
 * jssa_decode fed from host memory: copies this step's q (bf16 [batch, h_q, d]) and, when
 * non-NULL, k_new and v_new (bf16 [batch, h_kv, d]) from host memory into device staging inside
 * `ws`, runs jssa_decode on `stream` and copies the output back to out_host (bf16
 * [batch, h_q, d]); the caches, basis, page table, lengths and idx / count are device memory as
 * for jssa_decode. The library has no counterpart of this in the pages: it is the host
 * plumbing of a serving loop. Consecutive calls on the same workspace alternate between two
 * staging sets: the uploads of a call run on an internal stream while the previous call's
 * kernels run, and its download on a second internal stream while the next call's kernels run
 * (events order the three streams; use pinned host memory, or the copies are synchronous).
 * Every call returns before its copies complete: out_host holds the step's output, and the host
 * inputs may be rewritten, once the device has been synchronised, or once `stream` has been
 * synchronised after jssa_decode_host_join. The first call on a workspace (per device) creates
 * the two streams and the events, which live until the process exits; make it outside stream
 * capture. Calls sharing one workspace must come from one thread at a time. The state is keyed
 * by the workspace address: before a sequence of calls on memory that an earlier sequence used
 * as its workspace (for instance freed and allocated again), call jssa_decode_host_join on it,
 * which makes the next call order its copies after the work already on its stream.
 * ws: >= jssa_workspace_size(JSSA_FN_DECODE_HOST, batch, h_q, h_kv, d, max_pages, page_size,
 * budget). Errors as jssa_decode (host pointers are not checked for alignment).
 */
JSSA_API int jssa_decode_host(const jssa_bf16* q_host, const jssa_bf16* k_new_host,
                              const jssa_bf16* v_new_host, jssa_bf16* k_cache,
                              jssa_bf16* v_cache, int64_t kv_page_stride, int64_t kv_slot_stride,
                              int64_t kv_head_stride, uint8_t* score_cache, const float* basis,
                              const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                              int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                              int page_size, int budget, float softmax_scale, int32_t* idx,
                              int32_t* count, jssa_bf16* out_host, void* ws, size_t ws_bytes,
                              jssa_stream_t stream);

/*
 * Make `stream` wait for every copy that jssa_decode_host has issued with this workspace (the
 * last output included); the next jssa_decode_host call on it orders its copies after the work
 * then on its `stream`. No-op for a workspace that has not been used by jssa_decode_host.
 */
JSSA_API int jssa_decode_host_join(const void* ws, jssa_stream_t stream);

/* Size of the device scratch array used by jssa_indexed_attend_noalloc (per GPU, bytes). */
#define JSSA_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * Allocation-free indexed attention. The paper has no counterpart to this entry point: it is a
 * library convenience. It computes exactly what jssa_indexed_attend computes, with the same
 * arguments except the workspace, for callers that cannot allocate or pass device memory of
 * their own: an inference runtime that owns all device memory through its own pool and gives
 * plug-ins no allocator, a latency-critical loop that must avoid cudaMalloc (which synchronises
 * the device), or a host program that only links this C ABI and has no allocator.
 * Instead of a workspace, the split-K scratch (ticket counters and fp32 partials) lives in a
 * fixed device array of JSSA_NOALLOC_SCRATCH_BYTES inside the library; every GPU that loads the
 * library holds that array until the process exits. Sizes whose scratch would exceed it return
 * JSSA_ERR_SCRATCH_LIMIT without launching (jssa_workspace_size(JSSA_FN_INDEXED_ATTEND, ...)
 * gives the requirement). The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it with the id of the device's
 * CUDA context; the first call after a cudaDeviceReset (a new context) looks it up again. Make
 * those first calls before any stream capture. The call itself allocates nothing (it clears the ticket counters with
 * cudaMemsetAsync on `stream`, then launches). All calls on a device share the array and it
 * keeps the last call's contents: calls that overlap on the GPU (different streams or threads
 * of the same process) race and must be serialised by the caller.
 */
JSSA_API int jssa_indexed_attend_noalloc(const jssa_bf16* q, const jssa_bf16* k_cache,
                                         const jssa_bf16* v_cache, int64_t kv_page_stride,
                                         int64_t kv_slot_stride, int64_t kv_head_stride,
                                         const int32_t* block_table, int max_pages,
                                         const int32_t* idx, const int32_t* count, int batch,
                                         int h_q, int h_kv, int d, int budget, int64_t num_pages,
                                         int page_size, float softmax_scale, jssa_bf16* out,
                                         jssa_stream_t stream);

/*
 * Read (and with clear != 0, reset) the device error word of the current device. Synchronises
 * `stream` first so that the flags of every kernel enqueued on it are visible.
 */
JSSA_API int jssa_device_error(uint32_t* flags, int clear, jssa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* JSSA_H_ */
