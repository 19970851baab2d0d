/*
 * isoquant.h -- C ABI of the IsoQuant compressed-space attention library
 * (B200 / sm_100a).
 *
 * Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via
 * Fused Compressed-Space Attention" (arXiv 2608.08081), Abstract.  Each K/V
 * head vector (d = 128) is isotropized by a Walsh-Hadamard transform
 * followed by 32 block-diagonal SO(4) rotations (256 stored parameters per
 * head), then quantized to 3-bit scalar codes; attention runs directly on
 * the packed codes, and full-precision KV is never materialised.
 *
 * Conventions fixed by this library where the pages are silent:
 *   R = B * Hn * D: D = diag(signs), Hn = Sylvester Hadamard / sqrt(128)
 *   (natural order), B = 32 SO(4) blocks, block b acting on coordinates
 *   4b..4b+3 as the quaternion (w,x,y,z) by v -> qL (x) v (x) conj(qR).
 *   Per vector: n = ||x||_2 (fp64) stored as fp16 (nearest even, saturating
 *   at 65504); z = sqrt(128) * (R x) / n; code_j = #{k : z_j > t_k} with the
 *   8-level Lloyd-Max levels for N(0,1) rounded to fp16 (ascending, code 0 =
 *   most negative) and t_k the midpoints of adjacent levels.  Ten codes per
 *   32-bit word, code j at bits 3*(j%10) of word j/10, 13 words per vector.
 *   Attention: s_t = scale * (n16_t / sqrt(128)) * <R q, C[code_t]>,
 *   softmax over visible tokens, o = R^-1 sum_t p_t (n16v_t/sqrt(128))
 *   C[codev_t].
 *
 * Memory: every device buffer is owned by the caller, except the per-head
 * parameter block and a 16-byte status word that isoquant_init allocates and
 * isoquant_destroy frees.  No call below allocates, frees or synchronises,
 * except isoquant_init, isoquant_destroy and isoquant_get_status.
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 * default stream); all work is enqueued asynchronously on it.
 * Errors: every call returns an isoquant_status.  Argument errors are found
 * on the host before anything is launched; a failed launch returns
 * ISOQUANT_ERR_CUDA.  Errors the host cannot see (a device index out of
 * range, a bounded device-side wait that expired) set bits in the context's
 * status word, read with isoquant_get_status.
 */
#ifndef ISOQUANT_H
#define ISOQUANT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ISOQUANT_HEAD_DIM 128
#define ISOQUANT_WORDS_PER_VECTOR 13
#define ISOQUANT_PARAMS_PER_HEAD 256

typedef enum {
  ISOQUANT_OK = 0,
  ISOQUANT_ERR_INVALID_ARG = -1,   /* null pointer, bad count or size */
  ISOQUANT_ERR_UNSUPPORTED = -2,   /* head_dim != 128, unknown dtype, page size */
  ISOQUANT_ERR_OUT_OF_RANGE = -3,  /* an index or length outside its buffer */
  ISOQUANT_ERR_WORKSPACE = -4,     /* workspace too small */
  ISOQUANT_ERR_CUDA = -5,          /* a CUDA runtime call failed */
  ISOQUANT_ERR_ALIGNMENT = -6      /* a pointer is not 16-byte aligned */
} isoquant_status;

/* device status bits (isoquant_get_status) */
#define ISOQUANT_DEVERR_WAIT_TIMEOUT 1u   /* a bounded pipeline wait expired */
#define ISOQUANT_DEVERR_PAGE_RANGE 2u     /* page_table entry outside [0, num_pages) */
#define ISOQUANT_DEVERR_SLOT_RANGE 4u     /* slot_mapping entry outside the cache */
#define ISOQUANT_DEVERR_PLAN_MISMATCH 8u  /* attend_combine given another workspace size than
                                             attend_partial: records not merged, zeros written */

typedef enum {
  ISOQUANT_F32 = 0,
  ISOQUANT_BF16 = 1,
  ISOQUANT_F16 = 2
} isoquant_dtype;

typedef struct isoquant_ctx isoquant_ctx;

/* Paged packed KV cache, caller-owned device memory.
 *   codes: uint32 [num_pages][2 (K,V)][num_kv_heads][13][page_size]
 *          (8 or 16 words instead of 13 for contexts of 2 or 4 bits)
 *          (word-major inside a page: word w of every token, then word w+1)
 *   norms: uint16 (fp16 bits) [num_pages][2][num_kv_heads][page_size]
 * Token t of a sequence lives in page page_table[b][t / page_size] at
 * offset t % page_size.  page_size must be 32, 64, 128 or 256; both
 * pointers 16-byte aligned.  Bytes per token and KV head: 2 * (52 + 2). */
typedef struct {
  uint32_t *codes;
  uint16_t *norms;
  int32_t num_pages;
  int32_t page_size;
} isoquant_cache;

/* Create a context for `num_kv_heads` heads on the current CUDA device.
 *   head_dim: must be 128 (RotaryQuant, Abstract: 256 parameters per head
 *             = 32 SO(4) blocks x 2 unit quaternions x 4).
 *   signs:    host int8 [num_kv_heads][128], each +1 or -1 (the D of R).
 *   quats:    host float [num_kv_heads][32][2][4], (w,x,y,z), left then
 *             right quaternion of each block; normalised here in fp64.
 * Allocates the device parameter block (per head: 2 KB fp32 and 4 KB fp64
 * block matrices, 16 B of sign bits) and the status word.  Synchronous.
 * Errors: INVALID_ARG (null, num_kv_heads < 1, a sign not +-1, a zero or
 * non-finite quaternion), UNSUPPORTED (head_dim), CUDA. */
int isoquant_init(isoquant_ctx **out, int num_kv_heads, int head_dim,
                  const int8_t *signs, const float *quats);

/* isoquant_init with another code width (RotaryQuant, Abstract: the KV path
 * is 3-bit; the system quantizes elsewhere at 2, 4 and 8 bits).  bits in
 * {2, 3, 4}: 2^bits fp16-rounded Lloyd-Max levels for N(0,1) with midpoint
 * thresholds, floor(32 / bits) codes per word (16, 10, 8; code j at bits
 * bits * (j % per_word) of word j / per_word) and ceil(128 / per_word)
 * words per vector (8, 13, 16) in the cache's code array instead of 13;
 * everything else as isoquant_init.  A context's width fixes the layout of
 * every cache used with it.  Attention picks its kernel by shape at every
 * width (see isoquant_attend_decode).
 * Errors: as isoquant_init; UNSUPPORTED for another width. */
int isoquant_init_bits(isoquant_ctx **out, int num_kv_heads, int head_dim,
                       const int8_t *signs, const float *quats, int bits);

/* Free the context and its device memory (synchronises the device). */
void isoquant_destroy(isoquant_ctx *ctx);

/* Human-readable text for an isoquant_status. */
const char *isoquant_strerror(int status);

/* The library's own codebook (host only, no device work): the 8 fp16-
 * rounded Lloyd-Max levels for N(0,1), ascending, widened to float, and the
 * 7 decision thresholds (midpoints, exact in float). */
int isoquant_codebook(float levels[8], float thresholds[7]);

/* The codebook of another width: levels[2^bits], thresholds[2^bits - 1].
 * Errors: INVALID_ARG (null), UNSUPPORTED (bits not 2, 3 or 4). */
int isoquant_codebook_bits(int bits, float *levels, float *thresholds);

/* Bytes of the two cache arrays for `num_pages` pages. */
int isoquant_cache_bytes(const isoquant_ctx *ctx, int num_pages, int page_size,
                         size_t *code_bytes, size_t *norm_bytes);

/* Rotate, quantize, pack and append K and V vectors into the paged cache
 * (RotaryQuant, Abstract: each KV vector is isotropized by the
 * Walsh-Hadamard transform and the block-diagonal SO(4) rotations, then
 * scalar-quantized to 3 bits; the quantizer -- per-vector fp16 norm,
 * Lloyd-Max levels, ten codes per word -- is the one stated at the top of
 * this file, where the pages leave it open).
 *   k, v:  device [n_tok][num_kv_heads][128] of `dtype` (F32, BF16, F16),
 *          contiguous, 8-byte aligned.
 *   slot_mapping: device int64 [n_tok], slot = page * page_size + offset;
 *          a negative slot skips that token; a slot beyond the cache sets
 *          ISOQUANT_DEVERR_SLOT_RANGE and is skipped.
 * Writes 13 code words and one fp16 norm per (token, head, K/V).
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA. */
int isoquant_compress_kv(isoquant_ctx *ctx, const isoquant_cache *cache,
                         const void *k, const void *v, int dtype, int n_tok,
                         const int64_t *slot_mapping, void *stream);

/* q_rot = R q for every row (RotaryQuant, Abstract: scores are formed in the
 * rotated space, so the query takes the same R = B Hn D as the keys of its
 * head; <R q, R k> = <q, k> because R is orthogonal).
 *   q:     device [n_rows][num_q_heads][128] of dtype (F32, BF16, F16),
 *          contiguous, 8-byte aligned (16 for F32);
 *   q_rot: device float [n_rows][num_q_heads][128], 16-byte aligned,
 *          caller-owned.
 * Query head h uses the rotation of KV head h / (num_q_heads /
 * num_kv_heads).  Errors: INVALID_ARG (null, n_rows < 0, num_q_heads not a
 * multiple of num_kv_heads), UNSUPPORTED (dtype), ALIGNMENT, CUDA. */
int isoquant_rotate_q(isoquant_ctx *ctx, const void *q, int dtype, int n_rows,
                      int num_q_heads, float *q_rot, void *stream);

/* Workspace bytes isoquant_attend_decode (and the partial/combine pair)
 * needs for this shape with pages of 64 tokens or more: a 256-byte header,
 * then the partial records of (16 + 8 * 128) floats of the kernel the shape
 * runs on.  Below 64 query rows per KV head (nq * num_q_heads /
 * num_kv_heads) that is the mma.sync kernel: a record per CTA plus one per
 * (8-row group, sequence, KV head).  From 64 rows it is a tcgen05 kernel:
 * 8 or 16 records per (CTA or 64/128-row stream, sequence, KV head) slot
 * and its work prefix.  A workspace too small for the tcgen05 plan but
 * large enough for the mma.sync records runs the mma.sync kernel; calls
 * accept any workspace that holds one of the two. */
int isoquant_workspace_size(const isoquant_ctx *ctx, int batch, int nq,
                            int num_q_heads, size_t *bytes);

/* isoquant_workspace_size for a given page size (32, 64, 128 or 256):
 * caches of 32-token pages always run the mma.sync kernel, whose records a
 * long prefill needs more room for.  Errors: INVALID_ARG, UNSUPPORTED. */
int isoquant_workspace_size_paged(const isoquant_ctx *ctx, int batch, int nq,
                                  int num_q_heads, int page_size,
                                  size_t *bytes);

/* Split-context decode attention over the packed cache, then the merge of
 * the splits with R^-1 applied once per output row (RotaryQuant, Abstract:
 * attention on the packed codes in the rotated space).  Two kernel launches,
 * the second a programmatic dependent launch that overlaps the first's tail.
 * The same call serves decode (nq = 1), verification chunks and causal
 * prefill (nq = the prompt length, causal = 1): with 64 or more query rows
 * per KV head, pages of at least 64 tokens and the full workspace, the
 * partial step runs on tcgen05 tensor cores (streams of 64 rows, or of 128
 * rows from 128 rows up), each stream walking only the pages inside its
 * causal horizon; otherwise on the mma.sync kernel (8-row groups), at every
 * code width and page size.
 *   q_rot:      device float [batch][nq][num_q_heads][128] (from rotate_q)
 *   page_table: device int32 [batch][max_pages]
 *   seq_lens:   device int32 [batch]; tokens 0..seq_lens[b]-1 are in the
 *               cache (including the nq query positions' own K/V)
 *   causal:     if nonzero, query position i sees tokens
 *               t <= seq_lens[b] - nq + i; otherwise all seq_lens[b] tokens
 *   scale:      softmax scale; 0 selects 1/sqrt(128)
 *   workspace:  device, >= isoquant_workspace_size bytes, 16-byte aligned;
 *               its contents on entry do not matter; calls whose kernels
 *               overlap on the GPU must not share one workspace
 *   out:        device float [batch][nq][num_q_heads][128]
 * A row that sees no token outputs zeros.  Rows of heads in one GQA group
 * share each KV tile.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE,
 * ALIGNMENT, CUDA. */
int isoquant_attend_decode(isoquant_ctx *ctx, const isoquant_cache *cache,
                           const float *q_rot, int batch, int nq,
                           int num_q_heads, const int32_t *page_table,
                           int max_pages, const int32_t *seq_lens, int causal,
                           float scale, void *workspace, size_t ws_bytes,
                           float *out, void *stream);

/* The preparation half of a decode step in one launch: append the step's new
 * K/V tokens to the cache (as isoquant_compress_kv: k, v device
 * [n_tok][num_kv_heads][128], slot_mapping device int64 [n_tok]) and rotate
 * the queries (as isoquant_rotate_q: q device [n_rows][num_q_heads][128],
 * q_rot device float, same shape).  The two are independent, so one grid
 * does both and their latencies overlap.  k, v and q share `dtype`.  Either
 * half may be empty (n_tok = 0 or n_rows = 0).  Errors: as the two calls. */
int isoquant_decode_prep(isoquant_ctx *ctx, const isoquant_cache *cache,
                         const void *k, const void *v, int n_tok,
                         const int64_t *slot_mapping, const void *q, int dtype,
                         int n_rows, int num_q_heads, float *q_rot,
                         void *stream);

/* Workspace bytes isoquant_decode_step needs: the attention workspace
 * rounded up to 256 bytes, then the rotated queries
 * (batch * nq * num_q_heads * 128 floats). */
int isoquant_step_workspace_size(const isoquant_ctx *ctx, int batch, int nq,
                                 int num_q_heads, size_t *bytes);

/* One whole decode step (RotaryQuant, Abstract: compress the new KV, then
 * attend on the packed codes): isoquant_decode_prep (append + rotate q) and
 * isoquant_attend_decode, three kernel launches chained by programmatic
 * dependent launch.  Arguments as those calls; q is
 * [batch][nq][num_q_heads][128] of `dtype`, seq_lens must already count the
 * appended tokens, and the rotated queries live in the workspace
 * (>= isoquant_step_workspace_size bytes, 16-byte aligned, contents on entry
 * irrelevant).  With batch = 0 it only appends.  Errors: as those calls. */
int isoquant_decode_step(isoquant_ctx *ctx, const isoquant_cache *cache,
                         const void *k, const void *v, int n_tok,
                         const int64_t *slot_mapping, const void *q, int dtype,
                         int batch, int nq, int num_q_heads,
                         const int32_t *page_table, int max_pages,
                         const int32_t *seq_lens, int causal, float scale,
                         void *workspace, size_t ws_bytes, float *out,
                         void *stream);

/* isoquant_attend_decode without a workspace argument, for callers that can
 * neither allocate device memory nor lend the library a buffer (a serving
 * process whose memory pool owns all device memory, or a decode loop that
 * must not risk the device-wide synchronisation of cudaMalloc/cudaFree).
 * The paper has no counterpart to this call; it is a deployment aid.
 * Same arguments and result as isoquant_attend_decode.  The split records
 * live in a 16 MiB array compiled into the library (held by every GPU that
 * loads it until exit); a shape whose minimum workspace exceeds 16 MiB
 * is rejected with ISOQUANT_ERR_WORKSPACE.  The first call on a device looks
 * up the array's device address and must come before any stream capture.
 * Calls share the array: calls whose kernels overlap on the GPU race and
 * must be ordered by the caller.  Allocates and frees nothing. */
int isoquant_attend_decode_static(isoquant_ctx *ctx, const isoquant_cache *cache,
                                  const float *q_rot, int batch, int nq,
                                  int num_q_heads, const int32_t *page_table,
                                  int max_pages, const int32_t *seq_lens,
                                  int causal, float scale, float *out,
                                  void *stream);

/* The two halves of isoquant_attend_decode, for callers that schedule them
 * separately (same arguments): the partial half writes the records to the
 * workspace, the combine half (one warp per output row) merges them, applies
 * R^-1 and writes `out`. */
int isoquant_attend_partial(isoquant_ctx *ctx, const isoquant_cache *cache,
                            const float *q_rot, int batch, int nq,
                            int num_q_heads, const int32_t *page_table,
                            int max_pages, const int32_t *seq_lens, int causal,
                            float scale, void *workspace, size_t ws_bytes,
                            void *stream);
int isoquant_attend_combine(isoquant_ctx *ctx, int batch, int nq,
                            int num_q_heads, const int32_t *seq_lens,
                            int page_size, const void *workspace,
                            size_t ws_bytes, float *out, void *stream);

/* Debug export of the normalised rotated coordinates z that
 * isoquant_compress_kv quantizes: z_j = sqrt(128) * (R x)_j / ||x||_2, the
 * Walsh-Hadamard transform then the SO(4) blocks (RotaryQuant, Abstract),
 * from the same fp32 rotation as the compress kernels' fast path, divided by
 * the fp32 norm (the compress kernel itself compares |y| with t * ||x||
 * rather than forming z), before any fp64 re-check (coordinates within 1e-5
 * of a decision threshold and norms near an fp16 rounding midpoint are
 * redone in fp64 when compressing).
 * Lets a test measure the fp32 error of z against an exact reference.  Not
 * on the decode path.
 *   x: device [n_tok][num_kv_heads][128] of dtype (F32, BF16, F16),
 *      contiguous, 16-byte aligned;
 *   z: device float [n_tok][num_kv_heads][128], 16-byte aligned,
 *      caller-owned; a zero vector exports zeros.
 * Errors: INVALID_ARG, UNSUPPORTED (dtype), ALIGNMENT, CUDA. */
int isoquant_debug_export_z(isoquant_ctx *ctx, const void *x, int dtype,
                            int n_tok, float *z, void *stream);

/* Copy the device status word to *status and clear it (synchronises the
 * stream).  0 means no device-side error since the last call. */
int isoquant_get_status(isoquant_ctx *ctx, uint32_t *status, void *stream);

/* Number of kernels the most recent call on this context launched. */
int isoquant_last_launch_count(const isoquant_ctx *ctx);

/* Self-test of the failure path.  Launches one thread that waits, through
 * the same bounded wait the pipelines use, on a barrier that nothing
 * completes: the wait gives up after limit_ns nanoseconds (1 ns .. 10 s,
 * else ISOQUANT_ERR_INVALID_ARG), sets ISOQUANT_DEVERR_WAIT_TIMEOUT in the
 * status word and the kernel returns; nothing faults and the context stays
 * usable.  elapsed_ns (device, may be NULL) receives the measured wait in
 * nanoseconds.  Asynchronous on stream; read the bit with
 * isoquant_get_status. */
int isoquant_selftest_wait(isoquant_ctx *ctx, uint64_t limit_ns,
                           uint64_t *elapsed_ns, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ISOQUANT_H */
