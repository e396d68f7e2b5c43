/*
 * deltakv.h -- C ABI of the B200 (sm_100a) DeltaKV residual KV-cache library.
 *
 * Method: "DeltaKV: Residual-Based KV Cache Compression via Long-Range
 * Similarity" (gist.science summary, section 3 "Metodologia").  A few tokens,
 * picked with a fixed stride, are kept whole as references ("Struttura della
 * Compressione"); every other token stores only a low-dimensional code of its
 * residual against the mean of its k most similar earlier references
 * ("Processo di Compressione", steps 1-4); decode rebuilds tokens from the
 * references and the decoded residual ("Ricostruzione") on demand inside the
 * attention that reads the cache (section 4, "Ottimizza i Kernel").
 *
 * Conventions shared by every entry point:
 *  - The caller owns all memory.  Device pointers are plain CUDA device
 *    addresses on the current device; nothing here allocates device memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  The returned status covers host-side validation and launch
 *    errors only.  Errors the kernels detect (a bounded wait that ran out, an
 *    out-of-range index) are latched in the first 16 bytes of the workspace and
 *    reported by deltakv_device_status().
 *  - Inputs are const and are never written.
 *  - Every device pointer must be 16-byte aligned and innermost dimensions
 *    must be contiguous, else DELTAKV_ERR_ALIGNMENT; nothing is launched on any
 *    error.
 *  - One call processes one layer; a model loops over its layers and passes
 *    each layer's weights and cache.
 *
 * Notation: B sequences, H kv-heads, Hq query heads (G = Hq / H, consecutive
 * query heads share a kv-head), d_h head size, D = 2 d_h, stride s, k
 * references per token, d_c code width, `hidden` MLP width, T tokens.  Token
 * t is a reference iff t mod s == 0; reference slot j is token j s.
 */
#ifndef DELTAKV_H
#define DELTAKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DELTAKV_OK = 0,
    DELTAKV_ERR_INVALID_ARG = 1,    /* NULL, negative or inconsistent argument */
    DELTAKV_ERR_UNSUPPORTED = 2,    /* valid but not built (see deltakv_plan) */
    DELTAKV_ERR_ALIGNMENT = 3,      /* pointer or stride breaks the 16-byte rule */
    DELTAKV_ERR_WORKSPACE = 4,      /* workspace smaller than deltakv_plan said */
    DELTAKV_ERR_CUDA = 5,           /* a CUDA runtime call failed */
    DELTAKV_ERR_DEVICE_TIMEOUT = 6, /* a kernel's bounded wait ran out */
    DELTAKV_ERR_DEVICE_BOUNDS = 7   /* a kernel met an out-of-range index */
} deltakv_status;

/* Element types.  DELTAKV_BF16_CODE4: K, V, queries, weights and reference
 * rows in bfloat16, and every code row quantised to 4 bits ("Efficienza di
 * Memoria", section 5 of the summary: the saving is largest combined with
 * 4-bit quantisation): per compressed token one scale = bf16(max |c| / 7)
 * and signed 4-bit q = clamp(rne(c / scale), -7, 7), the stored code being
 * q * scale.  Needs d_c in {16, 32, 64}, hidden in {128, 256} and a
 * nonlinear act (it runs on the tensor-core compressor and decoder). */
typedef enum { DELTAKV_BF16 = 0, DELTAKV_F32 = 1, DELTAKV_BF16_CODE4 = 2 } deltakv_dtype;

/* Nonlinearity between the two linear layers of the compressor and of the
 * decompressor.  GELU_ERF is x * Phi(x). */
typedef enum {
    DELTAKV_ACT_GELU_ERF = 0,
    DELTAKV_ACT_GELU_TANH = 1,
    DELTAKV_ACT_NONE = 2
} deltakv_act;

/* The problem as the DeltaKV summary states it (section 3): layers,
 * kv-heads, head size, stride, k, code width, MLP width.
 * Supported: d_h in {64, 128}; 1 <= s; 1 <= k <= 8; d_c in {16, 32, 64} or
 * d_c == hidden == 2 d_h with d_h = 64 (identity codec); 32 <= hidden <= 256, hidden a
 * multiple of 32; q_heads a multiple of kv_heads with G <= 8. */
typedef struct {
    int32_t layers;    /* informational: the model holds `layers` caches */
    int32_t batch;     /* B */
    int32_t kv_heads;  /* H */
    int32_t q_heads;   /* Hq */
    int32_t d_h;
    int32_t max_T;     /* token capacity of one cache */
    int32_t stride_s;  /* s */
    int32_t k;
    int32_t d_c;
    int32_t hidden;
    deltakv_dtype dtype; /* element type of K, V, q, weights, stored refs and codes */
    deltakv_act act;
} deltakv_config;

typedef struct deltakv_plan_s* deltakv_plan_t; /* opaque, host memory only */
typedef struct CUstream_st* deltakv_stream_t;  /* same type as cudaStream_t */

/* Packed compressed cache of one layer, offsets in bytes from its base.
 * Four planes, each [B][H][rows][cols] row-major:
 *   ref_k, ref_v : [B][H][n_ref_cap][d_h]  dtype  -- reference rows, stored
 *                  whole (slot j = token j s);
 *   code         : [B][H][n_code_cap][d_c] dtype  -- one row per non-reference
 *                  token, in token order: token t (t mod s != 0) is row
 *                  t - floor(t / s) - 1; with DELTAKV_BF16_CODE4 a row is
 *                  d_c / 2 bytes, element 2i in the low nibble of byte i and
 *                  2i + 1 in its high nibble (two's complement);
 *   idx          : [B][H][n_code_cap][k]   int32  -- its reference slots in
 *                  ascending (distance, slot) order, -1 where fewer than k
 *                  earlier references exist;
 *   code_scale   : [B][H][n_code_cap]      bf16   -- with DELTAKV_BF16_CODE4
 *                  only, each code row's scale (code_scale_offset is 0 and
 *                  the plane absent otherwise).
 * For a cache holding T tokens the first ceil(T/s) reference rows and the
 * first T - ceil(T/s) code/idx rows of each (b, head) are used. */
typedef struct {
    size_t ref_k_offset, ref_v_offset, code_offset, idx_offset;
    size_t total_bytes;
    int64_t n_ref_cap;
    int64_t n_code_cap;
    size_t code_scale_offset;
} deltakv_cache_layout;

/* Validate `cfg`, build a host-side plan, and report the bytes of one layer's
 * packed cache and of the device workspace that compress, decode and
 * reconstruct need (both 256-byte aligned sizes).  No device work.
 * Errors: INVALID_ARG, UNSUPPORTED. */
deltakv_status deltakv_plan(const deltakv_config* cfg, deltakv_plan_t* plan_out,
                            size_t* cache_bytes_per_layer, size_t* workspace_bytes);

deltakv_status deltakv_plan_destroy(deltakv_plan_t plan);

deltakv_status deltakv_get_cache_layout(deltakv_plan_t plan, deltakv_cache_layout* out);

/* Compress one layer ("Processo di Compressione" steps 1-4): for every
 * non-reference token, choose its k nearest earlier references by squared
 * L2 distance over [K_t ; V_t] (ties to the lower slot), subtract their mean,
 * and encode the residual with code = W2 act(W1 r + b1) + b2; write the
 * reference rows, codes and slots into `cache`.
 *   T          : 0 <= T <= max_T tokens (T = 0 launches nothing)
 *   K, V       : device, element (b, h, t, e) at base + b*strides[0] +
 *                h*strides[1] + t*strides[2] + e (strides in elements)
 *   W1 [hidden][D], W2 [d_c][hidden]: device, dtype, row-major
 *   b1 [hidden], b2 [d_c]: device float32 or NULL (zero)
 *   cache      : device, cache_bytes_per_layer bytes (overwritten)
 *   workspace  : device, workspace_bytes bytes, contents scratch. */
deltakv_status deltakv_compress(deltakv_plan_t plan, int32_t T,
                                const void* K, const void* V, const int64_t kv_strides[3],
                                const void* W1, const float* b1,
                                const void* W2, const float* b2,
                                void* cache, void* workspace, size_t workspace_bytes,
                                deltakv_stream_t stream);

/* Streaming compression ("Processo di Compressione" steps 1-4, applied as
 * tokens arrive during decoding): extend a layer's packed cache that holds
 * the compressed tokens [0, T0) to the tokens [0, T1).  New tokens with
 * t mod s == 0 become references; every other new token t searches all
 * references with slot j, j s < t (those appended by this call included)
 * with exact float32 squared distances, keeps the k nearest (ties to the
 * lower slot), and stores its code and slots.  The slots match the exact
 * selection under the same near-tie rule as deltakv_compress's (where two
 * references lie within float32 rounding of the same distance, append and
 * compress may keep different ones); everything else equals compressing
 * [0, T1) in one call.
 *   0 <= T0 <= T1 <= max_T; T0 == T1 returns DELTAKV_OK without launching.
 *   cache      : device, as written by deltakv_compress(T0) or by earlier
 *                appends up to T0 (the caller guarantees it); rows of the
 *                tokens [T0, T1) are written, nothing else changes.
 *   K, V       : device, as for deltakv_compress; only tokens [T0, T1) are
 *                read.
 *   W1, b1, W2, b2, workspace, stream: as for deltakv_compress.
 * Runs on CUDA cores (a few tokens per call): each new token's references
 * are scanned by several CTAs, whose lists one CTA per (token, kv-head)
 * merges before the MLP.  The two kernels are launched with programmatic
 * stream serialisation: they may start while the work before them on the
 * stream is still running, but read nothing until it has completed, so the
 * call is stream-ordered like any other (and can be captured in a CUDA
 * graph).  Errors: as for deltakv_compress. */
deltakv_status deltakv_append(deltakv_plan_t plan, int32_t T0, int32_t T1,
                              const void* K, const void* V, const int64_t kv_strides[3],
                              const void* W1, const float* b1,
                              const void* W2, const float* b2,
                              void* cache, void* workspace, size_t workspace_bytes,
                              deltakv_stream_t stream);

/* Decode attention over one layer's compressed cache ("Ricostruzione" and
 * section 4): for query head hq (kv-head hq / G),
 *   out = sum_t softmax_t(q . K_hat_t / sqrt(d_h)) V_hat_t over the T cached
 * tokens, where reference rows are used as stored and every other token is
 * KV_R + W4 act(W3 code + b3) + b4 (first d_h entries K, last d_h V),
 * rebuilt on the fly and never written out.
 *   T >= 1; q: device [B][Hq][d_h] dtype with element strides
 *   q_strides = {batch, head}; W3 [hidden][d_c], W4 [D][hidden] dtype;
 *   b3 [hidden], b4 [D] float32 or NULL; out: device float32 [B][Hq][d_h]
 *   with element strides out_strides = {batch, head}. */
deltakv_status deltakv_decode_attention(deltakv_plan_t plan, int32_t T,
                                        const void* q, const int64_t q_strides[2],
                                        const void* cache,
                                        const void* W3, const float* b3,
                                        const void* W4, const float* b4,
                                        float* out, const int64_t out_strides[2],
                                        void* workspace, size_t workspace_bytes,
                                        deltakv_stream_t stream);

/* Sparse decode attention (section 4, reconstruction of only the tokens a
 * sparse-attention selector such as OmniKV picks): for query head hq of
 * kv-head h,
 *   out = sum_{t in sel(b, h)} softmax_t(q . K_hat_t / sqrt(d_h)) V_hat_t,
 * rebuilding only the selected tokens (reference rows as stored, the others
 * as KV_R + W4 act(W3 code + b3) + b4) and never writing them out.
 *   tokens : device int32 [B][H][n_sel], token indices in [0, T) chosen by
 *            the caller (any order; a repeated index counts once per
 *            occurrence; an index outside [0, T) is skipped and reported as
 *            DELTAKV_ERR_DEVICE_BOUNDS); n_sel >= 1; caller-owned, read only.
 *   every other argument as for deltakv_decode_attention.
 * Plans that take the tensor-core token loop of deltakv_decode_attention
 * (bf16 codes, hidden 128 or 256, a nonlinear codec), with n_sel at most the
 * plan's reference plus compressed-row capacity, run that loop over the
 * selected tokens' compressed rows (listed per (sequence, kv-head), gathered
 * 128 at a time), with each selected reference counted in the reference
 * combine.  Other plans run CUDA-core kernels in float32, 16 selected tokens
 * per pass of a CTA: the first decompressor layer per token, and the
 * (linear) second layer folded into the query and applied once per CTA to
 * the softmax-weighted sum of its activations.  Neither forms a K_hat/V_hat
 * row. */
deltakv_status deltakv_decode_attention_sparse(deltakv_plan_t plan, int32_t T,
                                               const void* q, const int64_t q_strides[2],
                                               const void* cache,
                                               const void* W3, const float* b3,
                                               const void* W4, const float* b4,
                                               const int32_t* tokens, int32_t n_sel,
                                               float* out, const int64_t out_strides[2],
                                               void* workspace, size_t workspace_bytes,
                                               deltakv_stream_t stream);

/* Rebuild every token of one layer ("Ricostruzione") into dense float32
 * K_out, V_out [B][H][T][d_h] (contiguous).  For tests and debugging; the
 * decode path never materialises these. */
deltakv_status deltakv_reconstruct(deltakv_plan_t plan, int32_t T, const void* cache,
                                   const void* W3, const float* b3,
                                   const void* W4, const float* b4,
                                   float* K_out, float* V_out,
                                   void* workspace, size_t workspace_bytes,
                                   deltakv_stream_t stream);

/* Decode attention for callers that cannot allocate device memory: code
 * running inside a memory budget fixed at start-up, plugins hosted by an
 * engine that owns every allocation, or steps where an allocation could block
 * or fail.  Same computation and arguments as deltakv_decode_attention, minus
 * the workspace: scratch comes from a 16 MiB array that the library holds in
 * device memory (every GPU that loads this part of the library keeps it until
 * the process exits).  The paper has no counterpart to this entry point.
 *  - Only the decode part of the plan's workspace must fit in 16 MiB (the
 *    compress part is not used): the reference-logit and slot-weight tables,
 *    8 G / s bytes per token of capacity and kv-head, plus about 33 KB per
 *    kv-head of partials at G = 4, hidden 256.  One 128k-token sequence with
 *    8 kv-heads fits (about 3.6 MiB); batch 8 at 128k does not.  A plan whose
 *    decode part is larger: DELTAKV_ERR_WORKSPACE, nothing launched.
 *  - Nothing is allocated: no cudaMalloc, no cudaFree, no allocating library
 *    call.  The first call on a device looks up the array's device address
 *    (once per device); make that first call before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents;
 *    the call clears what must start at zero.  Calls that overlap on the GPU
 *    race on the array: order them on one stream.
 *  - Device-side range checks latch into the shared array, which has no
 *    status read-back; use deltakv_decode_attention to diagnose. */
deltakv_status deltakv_decode_attention_noalloc(deltakv_plan_t plan, int32_t T,
                                                const void* q, const int64_t q_strides[2],
                                                const void* cache,
                                                const void* W3, const float* b3,
                                                const void* W4, const float* b4,
                                                float* out, const int64_t out_strides[2],
                                                deltakv_stream_t stream);

/* ---- Paged compressed cache (section 4, "Implementazione: Sparse-vLLM":
 * the memory manager that holds the irregular compressed layout, decoupled
 * from the attention kernels).  The cache of one (sequence, kv-head) is a
 * list of pages, each 128 consecutive blocks of s tokens: 128 reference
 * rows, 128 (s - 1) code rows, their slot rows and (4-bit codes) their
 * scales.  Pages come from a pool shared by the batch; a page table maps
 * logical page l of (sequence b, kv-head h) to a physical page, so sequences
 * of different lengths share one pool and grow a page at a time.
 *
 * Pool layout: five planes (ref_k, ref_v, code, idx, code_scale), each an
 * array of n_pages pages; page p of a plane holds its rows p rows_per_page ..
 * (p + 1) rows_per_page - 1, laid out like the contiguous cache's rows.
 * Token t of a sequence is in logical page t / tokens_per_page; reference
 * slot j in page j / refs_per_page, row j mod refs_per_page; compressed row
 * r (as in the contiguous layout) in page r / codes_per_page, row r mod
 * codes_per_page. */
typedef struct {
    int32_t refs_per_page;    /* 128 */
    int32_t codes_per_page;   /* 128 (s - 1) */
    int32_t tokens_per_page;  /* 128 s */
    int32_t n_pages;
    size_t ref_k_offset, ref_v_offset, code_offset, idx_offset, code_scale_offset;
    size_t pool_bytes;        /* 256-byte aligned */
} deltakv_page_layout;

/* Layout of a pool of n_pages (>= 1) pages for `plan`'s configuration.  No
 * device work.  Errors: INVALID_ARG. */
deltakv_status deltakv_page_pool_layout(deltakv_plan_t plan, int32_t n_pages, deltakv_page_layout* out);

/* Copy the compressed cache of every (sequence, kv-head) of `cache` (the
 * plan's contiguous layout, T tokens per sequence, as deltakv_compress and
 * deltakv_append write it) into its pages of `pool`:
 *   page_table : device int32 [B][H][max_pages]; entries of the logical pages
 *                l < ceil(T / tokens_per_page) name physical pages in
 *                [0, n_pages) (distinct pages are the caller's business; an
 *                entry outside the range is skipped and reported as
 *                DELTAKV_ERR_DEVICE_BOUNDS by deltakv_device_status);
 *   pool       : device, deltakv_page_pool_layout(n_pages).pool_bytes, 16-byte
 *                aligned; the rows of the used pages are written, nothing else.
 *   workspace  : the plan's workspace (its error word only).
 * Errors: INVALID_ARG (T outside [1, max_T], max_pages too small, NULL),
 * ALIGNMENT, WORKSPACE, CUDA. */
deltakv_status deltakv_pages_from_cache(deltakv_plan_t plan, int32_t T, const void* cache,
                                        const int32_t* page_table, int32_t max_pages,
                                        void* pool, int32_t n_pages,
                                        void* workspace, size_t workspace_bytes,
                                        deltakv_stream_t stream);

/* Decode attention over a paged cache whose sequences may differ in length:
 * the same result as deltakv_decode_attention on each sequence b alone with
 * T = seq_lens[b] (up to float32 summation order).
 *   seq_lens  : device int32 [B], 1 <= seq_lens[b] <= max_len (a length out
 *               of range is read as 1 and reported as DEVICE_BOUNDS);
 *   max_len   : host, 1 <= max_len <= max_T, the longest of them;
 *   pool, n_pages, page_table, max_pages: as for deltakv_pages_from_cache,
 *               every logical page l < ceil(seq_lens[b] / tokens_per_page)
 *               of (b, h) mapped (max_pages >= ceil(max_len /
 *               tokens_per_page)); a page index out of range is read as page
 *               0 and reported as DEVICE_BOUNDS;
 *   everything else as for deltakv_decode_attention.
 * The tensor-core token loop splits the flattened (sequence, kv-head, 128-row
 * chunk) list evenly over one CTA per SM, so a long sequence among short ones
 * is shared out like any other work.  Errors: as for
 * deltakv_decode_attention, plus INVALID_ARG for max_len, n_pages or
 * max_pages out of range. */
deltakv_status deltakv_decode_attention_paged(deltakv_plan_t plan, const int32_t* seq_lens, int32_t max_len,
                                              const void* q, const int64_t q_strides[2],
                                              const void* pool, int32_t n_pages,
                                              const int32_t* page_table, int32_t max_pages,
                                              const void* W3, const float* b3,
                                              const void* W4, const float* b4,
                                              float* out, const int64_t out_strides[2],
                                              void* workspace, size_t workspace_bytes,
                                              deltakv_stream_t stream);

/* Synchronise `stream`, read and clear the error word that the kernels latch
 * in `workspace`, and return DELTAKV_OK, DEVICE_TIMEOUT or DEVICE_BOUNDS. */
deltakv_status deltakv_device_status(deltakv_plan_t plan, void* workspace,
                                     deltakv_stream_t stream);

/* Tracing: every call that launches kernels (compress, append, the decode
 * calls, pages_from_cache, reconstruct) opens an NVTX range named after the
 * call for its duration, so a tool that records NVTX ranges shows each
 * call's kernels under its name.  Without such a tool the ranges cost a
 * pointer test each.
 *
 * Benchmark support: per-kernel device time.  While profiling is on for a
 * plan, every kernel its calls launch is bracketed by two CUDA events
 * recorded on the call's own stream (host-side bookkeeping only; the kernels
 * are unchanged).  deltakv_profile_collect waits for the recorded events,
 * writes one entry per kernel that ran (up to n_max) with its launch count
 * and summed time, and forgets the records. */
typedef struct {
    char name[32];
    int32_t launches;
    double total_ms;
} deltakv_kernel_time;

deltakv_status deltakv_set_profiling(deltakv_plan_t plan, int32_t enable);
deltakv_status deltakv_profile_collect(deltakv_plan_t plan, deltakv_kernel_time* out,
                                       int32_t n_max, int32_t* n_out);

/* Static description of a status code. */
const char* deltakv_status_string(deltakv_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t deltakv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DELTAKV_H */
