/*
 * llama_attn.h -- C ABI of the B200 (sm_100a) attention library for the dense
 * Llama 3 / 3.1 decoder: grouped-query causal attention with rotary position
 * embeddings and the cross-document mask, as a prefill over packed sequences
 * and as a single-token decode against a KV cache.
 *
 * What the calls compute (the pages' statement of the method):
 *   - RoPE frequencies theta_k = rope_theta^(-2k/D), k in [0, D/2 - 1]
 *     ("Llama 3.1 Architecture: Dense Scaling to 405B and 128K Context",
 *     "Context Expansion", "High Base Frequency"); base 500,000 for Llama 3
 *     (same subsection; "The Llama 3 Herd of Models", architecture chapter).
 *     The rotation turns adjacent pairs (x_2k, x_2k+1) by p * theta_k
 *     (RoFormer, cited on the first page), p = the token's position.
 *   - Grouped-query attention: query head h reads KV head h / (Hq / Hkv)
 *     ("How Meta's Llama 3.1 405B Architecture Actually Works", GQA
 *     paragraph; 128 query heads over 8 KV heads on the 405B chart).
 *   - Causal attention with the cross-document mask ("The Llama 3 Herd of
 *     Models", architecture chapter): key j is visible to query i iff both are
 *     in the same batch row and the same document and j <= i. Positions
 *     restart at 0 at each document start. Scores are scaled by 1/sqrt(D).
 *   - Decode: the KV cache of GQA ("How Meta's Llama 3.1 405B ...", GQA
 *     paragraph: the KV cache used while decoding) holds keys already rotated
 *     at their positions; the new query is rotated at position len.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers to contiguous memory, owned by
 *     the caller. bf16 tensors are passed as raw 16-bit patterns.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *   - Two forms of the bf16 prefill. The *_ws entry points take every buffer
 *     from the caller (a RoPE table built once by llama_attn_rope_table_build
 *     and a workspace of llama_attn_prefill_workspace_size bytes): they only
 *     enqueue kernels and a 4-byte memset, never allocate and never
 *     synchronise. The convenience entry points (llama_attn_prefill, _ex, _cp,
 *     _rotated, and the fp32 and FP8 calls) keep the table and the workspace
 *     in a library-owned per-device cache instead: the first use of a
 *     (device, theta, D) table, or a request larger than the cached buffers,
 *     allocates device memory and synchronises the device before enqueueing
 *     work; later calls of the same or smaller sizes do neither.
 *   - The decode calls never allocate or synchronise: the caller passes the
 *     workspace and the query's RoPE row is formed inside the kernel.
 *   - Arguments are checked on the host before anything is launched; a
 *     failed check returns a negative status and launches nothing.
 *   - The convenience calls share their per-device caches: calls from several
 *     host threads at once are serialised by a lock, and two calls whose
 *     kernels can overlap on the GPU (different streams, no ordering) must not
 *     both use the cache. Calls with caller-owned memory share nothing.
 *   - No C++ exception crosses this interface.
 */
#ifndef LLAMA_ATTN_H
#define LLAMA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as the CUDA runtime's cudaStream_t. */
typedef struct CUstream_st *cudaStream_t;

/* Raw bf16 bit pattern (1 sign, 8 exponent, 7 mantissa bits). */
typedef uint16_t llama_attn_bf16;

typedef enum {
  LLAMA_ATTN_OK = 0,
  LLAMA_ATTN_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, Hq % Hkv != 0, ... */
  LLAMA_ATTN_ERR_UNSUPPORTED = -2, /* a shape the kernels do not implement (e.g. D != 128 on bf16) */
  LLAMA_ATTN_ERR_WORKSPACE = -3,   /* decode workspace missing or too small */
  LLAMA_ATTN_ERR_CUDA = -4,        /* a CUDA runtime/driver call or a launch failed */
  LLAMA_ATTN_ERR_DEVICE = -5       /* a kernel reported an error word (see get_device_error) */
} llama_attn_status;

/*
 * Prefill, bf16 in / bf16 out, fp32 accumulation (tcgen05 tensor cores).
 *
 *   q   [B, S, Hq,  D]  un-rotated queries
 *   k   [B, S, Hkv, D]  un-rotated keys
 *   v   [B, S, Hkv, D]  values
 *   out [B, S, Hq,  D]  result (must not alias q, k or v)
 *   doc_offsets: NULL (each batch row is one document), or a device int32
 *     array of document starts in flattened B*S token coordinates:
 *     0 = o_0 < o_1 < ... < o_n = B*S, ending with the sentinel B*S; no
 *     document crosses a batch-row boundary. Its length is implicit (it is
 *     read up to the sentinel). A malformed array is detected on the device:
 *     the output is then unspecified and the device error word is set to
 *     LLAMA_ATTN_DEVERR_DOC_OFFSETS.
 *   B, S >= 1; Hq, Hkv >= 1 with Hq % Hkv == 0; D == 128; rope_theta > 0.
 *   Working memory (a rotated copy of k, B*S*Hkv*D bf16, and the per-token
 *   document starts) comes from the library's per-device cache; see
 *   llama_attn_prefill_ws for the form that takes it from the caller.
 */
int llama_attn_prefill(const llama_attn_bf16 *q, const llama_attn_bf16 *k,
                       const llama_attn_bf16 *v, llama_attn_bf16 *out,
                       const int32_t *doc_offsets, int B, int S, int Hq, int Hkv, int D,
                       float rope_theta, cudaStream_t stream);

/*
 * llama_attn_prefill plus the two outputs that link prefill to decode:
 *
 *   lse    [B, S, Hq] float32, or NULL: per query row and head, the natural
 *          log of the softmax denominator over the row's visible keys,
 *          log(sum_j exp(q_i . k_j / sqrt(D))) with rotated q and k. With it,
 *          attention over disjoint key sets can be merged exactly.
 *   kcache, vcache  [B, Hkv, Lmax, D] bf16, or both NULL: the batch is
 *          appended to a decode-layout KV cache, token i of batch row b and KV
 *          head h going to cache row i of (b, h): the key rotated at the
 *          token's document position (position i when doc_offsets is NULL,
 *          which is the form a following llama_attn_decode continues from at
 *          cache_lens[b] = S), the value copied. Rows S .. Lmax-1 are not
 *          touched. Lmax >= S.
 *
 * The attention output equals llama_attn_prefill's. Errors as for
 * llama_attn_prefill; a cache pointer without the other, Lmax < S or a cache
 * not 16-byte aligned returns LLAMA_ATTN_ERR_INVALID_ARG.
 */
int llama_attn_prefill_ex(const llama_attn_bf16 *q, const llama_attn_bf16 *k,
                          const llama_attn_bf16 *v, llama_attn_bf16 *out, float *lse,
                          const int32_t *doc_offsets, int B, int S, int Hq, int Hkv, int D,
                          float rope_theta, llama_attn_bf16 *kcache, llama_attn_bf16 *vcache,
                          int Lmax, cudaStream_t stream);

/*
 * Prefill of query chunks against a whole sequence: the per-GPU step of
 * context parallelism ("Llama 3.1 Architecture: Dense Scaling to 405B and
 * 128K Context", "The 4D Parallelism Execution Strategy", context-parallel
 * bullet: the 128K sequence is split along tokens across GPUs and the KV
 * states are exchanged). Each rank holds some query rows and, after an
 * exchange of keys and values, the whole sequence's k and v; this call
 * computes causal attention of its query rows over that sequence.
 *
 *   q   [B, Sq, Hq, D]  un-rotated queries: local rows [0, q_split) are the
 *                       tokens at global positions q_pos_a .. q_pos_a+q_split-1,
 *                       rows [q_split, Sq) those at q_pos_b .. q_pos_b+Sq-q_split-1
 *   k   [B, Skv, Hkv, D] un-rotated keys of the whole sequence (positions 0..Skv-1)
 *   v   [B, Skv, Hkv, D] values of the whole sequence
 *   out [B, Sq, Hq, D]  result for the local query rows
 *   lse [B, Sq, Hq] float32, or NULL: as for llama_attn_prefill_ex
 *
 * Each batch row is one document (no cross-document mask); the query at global
 * position P sees keys 0..P and is rotated at P. q_split, q_pos_a and q_pos_b
 * are multiples of 128 (the kernel's query tile), 0 <= q_split <= Sq,
 * q_pos_a + q_split <= Skv and q_pos_b + (Sq - q_split) <= Skv; otherwise
 * LLAMA_ATTN_ERR_INVALID_ARG. With Skv = Sq = q_split and q_pos_a = 0 the
 * result equals llama_attn_prefill with doc_offsets NULL. Other errors and the
 * scratch (a rotated copy of the Skv keys) as for llama_attn_prefill.
 */
int llama_attn_prefill_cp(const llama_attn_bf16 *q, const llama_attn_bf16 *k,
                          const llama_attn_bf16 *v, llama_attn_bf16 *out, float *lse, int B,
                          int Sq, int Skv, int Hq, int Hkv, int D, int q_pos_a, int q_split,
                          int q_pos_b, float rope_theta, cudaStream_t stream);

/*
 * Caller-owned RoPE table for the *_ws entry points: rows 0 .. maxpos-1, row
 * p holding (cos(p theta_k), sin(p theta_k)) as two floats for k = 0 ..
 * D/2-1, theta_k = rope_theta^(-2k/D) (the frequencies of "Llama 3.1
 * Architecture ...", "Context Expansion", "High Base Frequency"). The angle
 * p theta_k is formed and reduced in float64 and only cos and sin are rounded
 * to float32 (a float32 product is off by ~4e-3 rad at p ~ 1.3e5).
 *
 * llama_attn_rope_table_size returns the bytes for maxpos rows (0 for
 * maxpos < 1 or D not even in [2, 128]). llama_attn_rope_table_build writes
 * the table into `table` (device, 16-byte aligned, table_bytes >= that size,
 * else LLAMA_ATTN_ERR_WORKSPACE) with one kernel on `stream`. Build it once
 * per (theta, D) and reuse it: for 128K positions and D = 128 it is 64 MiB.
 */
size_t llama_attn_rope_table_size(int maxpos, int D);
int llama_attn_rope_table_build(void *table, size_t table_bytes, int maxpos, int D,
                                float rope_theta, cudaStream_t stream);

/*
 * Bytes of device workspace the bf16 prefill needs with caller-owned memory:
 * a 256-byte work-item counter, the per-token document starts (B*S int32) and
 * the rotated keys (B*S*Hkv*D bf16), each part 256-byte aligned. S is the
 * number of key rows per batch row (Skv for llama_attn_prefill_cp_ws). Returns
 * 0 for invalid sizes (D must be 128).
 */
size_t llama_attn_prefill_workspace_size(int B, int S, int Hkv, int D);

/*
 * llama_attn_prefill_ex with caller-owned memory: the same attention, LSE and
 * optional KV-cache append, with
 *
 *   rope_table, rope_rows  a table from llama_attn_rope_table_build (D = 128,
 *          the base of its build is the rope_theta of the computation), 16-byte
 *          aligned, rope_rows >= S rows (else LLAMA_ATTN_ERR_INVALID_ARG)
 *   workspace, workspace_bytes  device memory, 256-byte aligned, at least
 *          llama_attn_prefill_workspace_size(B, S, Hkv, D) bytes (else
 *          LLAMA_ATTN_ERR_WORKSPACE, before anything is launched); its contents
 *          need no initialisation and are overwritten.
 *
 * The call only enqueues kernels and a 4-byte memset on `stream`: no
 * allocation, no synchronisation. Two calls whose kernels can overlap on the
 * GPU must not share a workspace. Other arguments and errors as for
 * llama_attn_prefill_ex.
 */
int llama_attn_prefill_ws(const llama_attn_bf16 *q, const llama_attn_bf16 *k,
                          const llama_attn_bf16 *v, llama_attn_bf16 *out, float *lse,
                          const int32_t *doc_offsets, int B, int S, int Hq, int Hkv, int D,
                          const void *rope_table, int rope_rows, llama_attn_bf16 *kcache,
                          llama_attn_bf16 *vcache, int Lmax, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream);

/*
 * llama_attn_prefill_cp with caller-owned memory: rope_rows >= Skv, workspace
 * of llama_attn_prefill_workspace_size(B, Skv, Hkv, D) bytes; otherwise as
 * llama_attn_prefill_cp and llama_attn_prefill_ws.
 */
int llama_attn_prefill_cp_ws(const llama_attn_bf16 *q, const llama_attn_bf16 *k,
                             const llama_attn_bf16 *v, llama_attn_bf16 *out, float *lse, int B,
                             int Sq, int Skv, int Hq, int Hkv, int D, int q_pos_a, int q_split,
                             int q_pos_b, const void *rope_table, int rope_rows, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/*
 * Prefill on queries and keys that are already rotated (for example by
 * llama_attn_qkv_fp8_rope): the same attention as llama_attn_prefill_ex
 * without the RoPE step, so no rotated copy of k is made and no RoPE table
 * is read. q [B, S, Hq, D] and k [B, S, Hkv, D] hold the rotated rows; v,
 * out, lse, doc_offsets and the errors as for llama_attn_prefill_ex (no KV
 * cache output). D == 128.
 */
int llama_attn_prefill_rotated(const llama_attn_bf16 *q, const llama_attn_bf16 *k,
                               const llama_attn_bf16 *v, llama_attn_bf16 *out, float *lse,
                               const int32_t *doc_offsets, int B, int S, int Hq, int Hkv, int D,
                               cudaStream_t stream);

/*
 * Per-tensor dynamic E4M3 quantization ("Llama 3.1 Architecture: Dense
 * Scaling to 405B and 128K Context", "FP8 Quantization: Fitting 405B on an
 * 8xH100 Node": E4M3 with values up to 448, X_fp8 = clip(round(X / s_X),
 * -448, 448) with one scale per tensor).
 *
 *   x      [n] bf16 (device, 16-byte aligned), n > 0 and n % 8 == 0
 *   y      [n] E4M3 codes (device, 8-byte aligned): y_i = E4M3(x_i / s),
 *          x_i / s an IEEE float32 division, rounded to nearest-even onto
 *          the E4M3 grid and saturated to +-448
 *   scale  one float (device): s = amax_i |x_i| / 448 in float32, or 1 when
 *          x is all zeros
 * The scale is left on the device, so a following llama_attn_qkv_fp8_rope
 * reads it without a host round trip. NaN inputs give unspecified codes. The
 * library keeps a 4-byte amax in per-device scratch.
 */
int llama_attn_quantize_e4m3(const llama_attn_bf16 *x, int64_t n, uint8_t *y, float *scale,
                             cudaStream_t stream);

/*
 * FP8 QKV projection with RoPE: Y = (s_x * s_w) * (X_fp8 . W_fp8^T) on the
 * tcgen05 tensor cores (E4M3 x E4M3, fp32 accumulation), split into the query,
 * key and value heads, the query and key heads rotated by RoPE at each
 * token's document position, rounded to bf16 (same page and section as
 * llama_attn_quantize_e4m3; the QKV projection is one of the GEMMs it
 * quantizes; RoPE as for llama_attn_prefill).
 *
 *   x    [B*S, d_model] E4M3 codes of the activations (row-major), s_x its scale
 *   w    [N, d_model] E4M3 codes of the weight, N = (Hq + 2 Hkv) * D: rows
 *        0 .. Hq*D-1 are the query heads, then Hkv key heads, then Hkv value
 *        heads (the transpose of the page's K x N weight); s_w its scale
 *   s_x, s_w  device floats (as written by llama_attn_quantize_e4m3)
 *   q    [B, S, Hq, D] bf16 out, rotated; k [B, S, Hkv, D] bf16 out, rotated;
 *   v    [B, S, Hkv, D] bf16 out
 *   doc_offsets: as for llama_attn_prefill (positions restart per document)
 * D == 128 and d_model % 128 == 0 (else LLAMA_ATTN_ERR_UNSUPPORTED); all
 * tensors 16-byte aligned. Outputs must not alias inputs.
 */
int llama_attn_qkv_fp8_rope(const uint8_t *x, const float *s_x, const uint8_t *w, const float *s_w,
                            llama_attn_bf16 *q, llama_attn_bf16 *k, llama_attn_bf16 *v,
                            const int32_t *doc_offsets, int B, int S, int d_model, int Hq, int Hkv,
                            int D, float rope_theta, cudaStream_t stream);

/*
 * Prefill in true fp32 arithmetic on CUDA cores (FFMA, accurate expf), same
 * semantics and layouts as llama_attn_prefill with float tensors.
 * D even, 2 <= D <= 128.
 */
int llama_attn_prefill_f32(const float *q, const float *k, const float *v, float *out,
                           const int32_t *doc_offsets, int B, int S, int Hq, int Hkv, int D,
                           float rope_theta, cudaStream_t stream);

/*
 * Bytes of device workspace llama_attn_decode needs for these sizes (split-KV
 * partial outputs and log-sum-exps). Returns 0 for invalid sizes.
 */
size_t llama_attn_decode_workspace_size(int B, int Hq, int Lmax, int D);

/*
 * Single-token decode against a KV cache, bf16 in / bf16 out, fp32 math.
 *
 *   q          [B, Hq, D]          un-rotated query of the new token
 *   kcache     [B, Hkv, Lmax, D]   keys, row n already rotated at position n
 *   vcache     [B, Hkv, Lmax, D]   values
 *   cache_lens [B] int32, device   valid rows per sequence, 0 <= len <= Lmax
 *   out        [B, Hq, D]
 *   The query of sequence b is rotated at position cache_lens[b] and attends
 *   to cache rows 0 .. cache_lens[b]-1 (the new token's own key/value are the
 *   caller's to append). Rows at or past cache_lens[b] are never used, so they
 *   may hold anything. cache_lens[b] == 0 gives out = 0. A length outside
 *   [0, Lmax] sets LLAMA_ATTN_DEVERR_CACHE_LEN and that sequence's output is 0.
 *   D == 128; Hq % Hkv == 0 and Hq / Hkv <= 16; Lmax >= 1.
 *   workspace: device memory of at least
 *   llama_attn_decode_workspace_size(B, Hq, Lmax, D) bytes, 16-byte aligned,
 *   owned by the caller; its contents need no initialisation.
 *   The (cos, sin) row of position cache_lens[b] is formed in the kernel
 *   (float64 angle), so the call reads no table, allocates nothing and does
 *   not synchronise.
 */
int llama_attn_decode(const llama_attn_bf16 *q, const llama_attn_bf16 *kcache,
                      const llama_attn_bf16 *vcache, const int32_t *cache_lens,
                      llama_attn_bf16 *out, int B, int Hq, int Hkv, int D, int Lmax,
                      float rope_theta, void *workspace, size_t workspace_bytes,
                      cudaStream_t stream);

/*
 * llama_attn_decode against a paged KV cache (block-table indirection, the
 * dynamic KV-cache management named on the fifth page, "Meta's Llama 3 ...",
 * serving paragraph): the cache of every sequence is a list of fixed-size
 * pages in a shared pool.
 *
 *   kpages, vpages  [n_pages, Hkv, page_size, D] bf16: page p holds page_size
 *                   consecutive cache rows of every KV head (keys already
 *                   rotated at their positions)
 *   block_table     [B, max_blocks] int32, device: logical block j of sequence
 *                   b (cache rows j*page_size .. (j+1)*page_size - 1) is page
 *                   block_table[b * max_blocks + j]; entries past the
 *                   sequence's length are never read
 *   cache_lens      [B] int32, device, 0 <= len <= max_blocks * page_size
 *   page_size       a multiple of 64
 * Everything else (q, out, rotation, workspace with Lmax = max_blocks *
 * page_size, errors) is as in llama_attn_decode. A block id outside
 * [0, n_pages) sets LLAMA_ATTN_DEVERR_BLOCK_TABLE and its rows read as zero.
 */
int llama_attn_decode_paged(const llama_attn_bf16 *q, const llama_attn_bf16 *kpages,
                            const llama_attn_bf16 *vpages, const int32_t *block_table,
                            const int32_t *cache_lens, llama_attn_bf16 *out, int B, int Hq,
                            int Hkv, int D, int page_size, int max_blocks, int n_pages,
                            float rope_theta, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/*
 * llama_attn_decode without a caller-supplied workspace and without any
 * device allocation, for callers that cannot allocate device memory: a host
 * whose allocator owns all of device memory, or code running where
 * cudaMalloc is not allowed. Nothing on the pages corresponds to it; it exists
 * only for such callers.
 *
 * Same arguments, layouts, results and error codes as llama_attn_decode, minus
 * the workspace. The split-KV partials live in one fixed 72 MiB device array
 * inside the library, which every device that loads the library holds until
 * the process exits. A request needing more than that
 * (llama_attn_decode_workspace_size(B, Hq, Lmax, D) > 72 MiB, i.e. more than
 * 146,312 slots of B * Hq * ceil(Lmax / 1024)) is rejected with
 * LLAMA_ATTN_ERR_WORKSPACE before anything is launched. The RoPE angle of the
 * query is formed inside the kernel, so no table is allocated either.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and sets a kernel attribute; make that first call
 * outside any stream capture. All calls share the one array and it keeps the
 * last call's contents; nothing in it needs to start at zero, because every
 * partial is written before it is read within a call. Calls whose kernels can
 * overlap on the GPU (different streams, no ordering between them) race on
 * the array: order them, e.g. on one stream. If a call's kernels give up a
 * bounded wait (LLAMA_ATTN_DEVERR_TIMEOUT in the device error word), the
 * output of that call is undefined.
 */
int llama_attn_decode_noalloc(const llama_attn_bf16 *q, const llama_attn_bf16 *kcache,
                              const llama_attn_bf16 *vcache, const int32_t *cache_lens,
                              llama_attn_bf16 *out, int B, int Hq, int Hkv, int D, int Lmax,
                              float rope_theta, cudaStream_t stream);

/* Static, human-readable text for a status code. Never NULL. */
const char *llama_attn_status_string(int status);

/* Device error word bits (kernels OR them in; they never trap). */
#define LLAMA_ATTN_DEVERR_TIMEOUT 0x1     /* a bounded wait on a barrier gave up */
#define LLAMA_ATTN_DEVERR_DOC_OFFSETS 0x2 /* malformed doc_offsets */
#define LLAMA_ATTN_DEVERR_CACHE_LEN 0x4   /* cache_lens[b] outside [0, Lmax] */
#define LLAMA_ATTN_DEVERR_BLOCK_TABLE 0x8 /* a paged-cache block id outside [0, n_pages) */

/*
 * Waits for `stream`, then returns and clears the current device's error word
 * (0 = no error). Returns a negative llama_attn_status if the CUDA calls
 * themselves fail.
 */
int llama_attn_get_device_error(cudaStream_t stream);

/*
 * Benchmark instrumentation (host side, current device only).
 * llama_attn_profile_begin() starts a session: each later prefill, decode or
 * QKV projection call records a CUDA event pair on its stream around its main
 * kernel (prefill: the attention kernel; decode: the split-KV kernel;
 * projection: the FP8 GEMM) and every kernel the library launches is counted. llama_attn_profile_end() waits for the recorded events,
 * writes the summed main-kernel time in milliseconds, the number of timed main
 * kernels and the number of kernels launched, and ends the session. At most
 * 4096 main kernels are timed per session; later ones are counted only.
 * Returns LLAMA_ATTN_OK or a negative status. Any output pointer may be NULL.
 */
int llama_attn_profile_begin(void);
int llama_attn_profile_end(double *main_kernel_ms, int *main_kernels_timed, int *kernels_launched);

/* Library version, as MAJOR * 10000 + MINOR * 100 + PATCH. */
int llama_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_ATTN_H */
