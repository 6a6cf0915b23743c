/*
 * qvg.h -- C ABI of the B200 (sm_100a) implementation of the Quant VideoGen
 * (QVG) 2-bit KV-cache codec.
 *
 * The method (arXiv:2602.02958, as described by the m.163.com article on
 * Quant VideoGen, sections 三-五, and by gist.science/de, "Technische
 * Zusammenfassung" 2A-2C):
 *   1. semantic-aware smoothing: k-means over the tokens of a block, each
 *      token minus its centroid leaves a small, even residual (section 三);
 *   2. progressive residual quantisation: T such stages, R(0) = X, stage t
 *      gives centroids C(t), uint8 assignments pi(t) and R(t) (section 四);
 *   3. the final residual R(T) is quantised per group of G channels to 2-bit
 *      codes with FP8 E4M3 group scales (section 五);
 *   4. reconstruction runs in reverse: dequantise R(T), then add back the
 *      centroids of stage T, T-1, ..., 1, in one fused kernel (sections 四,
 *      五; "Fused Kernel" in Technische Zusammenfassung 2C);
 *   5. in streaming generation each chunk's k-means starts from the previous
 *      chunk's centroids (streaming centroid cache, section 五).
 *
 * Conventions for every call below:
 *   - "device" pointers are CUDA global-memory pointers on the current
 *     device; the caller owns them and keeps them alive until the work queued
 *     on `stream` has finished.  Only a qvg_cache owns memory.
 *   - Work is queued asynchronously on `stream` (0 = legacy default stream);
 *     a call returns once the work is queued.  Errors found while queueing
 *     (bad arguments, launch failures) are returned.
 *   - Device-side timeouts: every wait of the tensor-core kernel on another
 *     of its warps is bounded (2 s); a wait that runs out records
 *     QVG_ERR_DEVICE_TIMEOUT in the sticky status word of the workspace,
 *     cache or static reserve the call used, the kernel drains and returns,
 *     and that call's outputs are invalid.  The next qvg_quantize,
 *     qvg_append_chunk or qvg_quantize_static on the same workspace, cache or
 *     reserve returns QVG_ERR_DEVICE_TIMEOUT without queueing anything, when
 *     the earlier work has completed by the time of the call (the check never
 *     waits for the GPU: it reads the word only when the stream is idle and
 *     not being captured).  qvg_workspace_status, qvg_cache_status and
 *     qvg_static_status wait for the stream, read the word and clear it.
 *   - Fault injection for tests (host side; unset in normal use): the
 *     environment variable QVG_FAULT_INJECT holds a comma-separated list of
 *       alloc    every device allocation of qvg_cache_create and
 *                qvg_cache_create_adaptive fails (QVG_ERR_NO_MEMORY, nothing
 *                allocated);
 *       stream   the quantising calls (qvg_quantize, qvg_quantize_static,
 *                both appends), qvg_dequantize, qvg_cache_dequantize and
 *                qvg_attention report QVG_ERR_CUDA after queueing, as a
 *                failed launch would (an append then leaves the cache
 *                unchanged);
 *       timeout  the first CTA of the tensor-core assignment withholds one
 *                tile load and its waits give up after 1 ms, so that the
 *                bounded waits run out and record a device-side timeout.
 *   - Nothing is thrown across the ABI; all entry points are thread-compatible
 *     (distinct workspaces/caches may be used from distinct threads).
 *   - Tensor layouts are row-major.  H is the number of independent blocks
 *     in one call (heads, or heads x layers x K/V), N the tokens per block,
 *     d the channels per token (head dimension).
 *   - Supported by the kernels: d = 128; G in {8, 16, 32, 64, 128};
 *     bits = 2; 1 <= K <= 256; 0 <= T <= 8; N < 2^23.  Other values that the method
 *     allows return QVG_ERR_UNSUPPORTED.
 */
#ifndef QVG_H_
#define QVG_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QVG_API __attribute__((visibility("default")))
#else
#define QVG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (cudaStream_t). */
typedef struct CUstream_st* qvg_stream_t;

typedef enum {
    QVG_OK = 0,
    QVG_ERR_INVALID_ARG = 1,         /* argument outside the method's domain */
    QVG_ERR_UNSUPPORTED = 2,         /* allowed by the method, not by these kernels */
    QVG_ERR_NO_MEMORY = 3,           /* a qvg_cache allocation failed */
    QVG_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
    QVG_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device-side wait gave up */
    QVG_ERR_WORKSPACE_TOO_SMALL = 6, /* ws_bytes below qvg_workspace_bytes(...) for one block */
    QVG_ERR_CAPACITY = 7             /* a qvg_cache is full (tokens or chunks) */
} qvg_status;

/* Storage dtype of X, of the centroid tables and of the reconstruction. */
typedef enum { QVG_BF16 = 0, QVG_FP32 = 1 } qvg_dtype;

/* How a group of G residual values is scaled (section 五 of the m.163.com
 * article: INT2 codes with FP8 E4M3 group scales).
 *   QVG_SCALE_ASYM  two E4M3 bytes per group, scale s and zero point m:
 *                   m = E4M3(min), s = E4M3((max - m)/3),
 *                   q = clamp(rint((r - m)/s), 0, 3); value s*q + m.
 *   QVG_SCALE_SYM   one E4M3 byte per group (symmetric signed INT2):
 *                   s = E4M3(max |r|), q = clamp(rint(r/s), -2, 1), stored
 *                   u = q + 2; value s*(u - 2).  With it the closed-form
 *                   compression at K = 256 on a 38,000-token block is 6.97x
 *                   at T = 1, G = 64 (the pages' QVG range 6.94-7.05x,
 *                   section 六) and 5.03x at T = 4, G = 16 (QVG-Pro,
 *                   4.97-5.20x); plain rounding at G = 16 gives the 6.40x the
 *                   pages quote for their round-to-nearest baseline.
 * In both, divides are IEEE fp32, rint and E4M3 round to nearest even (E4M3
 * saturates at 448), and q = 0 when s = 0. */
typedef enum { QVG_SCALE_ASYM = 0, QVG_SCALE_SYM = 1 } qvg_scale_mode;

typedef struct {
    int32_t K;          /* centroids per block and stage (section 七 uses 256, stored as uint8) */
    int32_t T;          /* progressive residual stages (section 四); 0 = plain per-group RTN */
    int32_t group_size; /* G: contiguous channels of one token that share a scale */
    int32_t bits;       /* code width; 2 (INT2) */
    int32_t iters;      /* Lloyd iterations of a cold start (no initial centroids) */
    int32_t warm_iters; /* Lloyd iterations when started from given centroids */
    int32_t scale_mode; /* qvg_scale_mode */
} qvg_config;

/* The packed (compressed) form of H blocks of N tokens.  All DEVICE
 * pointers, caller-owned, written by qvg_quantize, read by qvg_dequantize.
 *   codes     [H][N][d*bits/8]  2-bit codes, channel j of a token at bits
 *                               2*(j%4) of byte j/4 of the token's row
 *   scale     [H][N][d/G]       E4M3 bytes: group step s
 *   zero      [H][N][d/G]       E4M3 bytes: group zero point m (the rounded
 *                               group minimum); value = s*q + m.  Not used
 *                               (may be NULL) with QVG_SCALE_SYM
 *   assign    [T][H][N]         uint8 centroid index of each token per stage
 *   centroids [T][H][K][d]      centroid tables in the storage dtype
 * With T = 0, assign and centroids are not accessed (may be NULL). */
typedef struct {
    uint8_t* codes;
    uint8_t* scale;
    uint8_t* zero;
    uint8_t* assign;
    void* centroids;
} qvg_packed;

/* Human-readable name of a status code (static string). */
QVG_API const char* qvg_status_string(qvg_status s);

/* Library build string, e.g. "qvg-b200 sm_100a". */
QVG_API const char* qvg_version(void);

/* Bytes of the packed form (the storage that section 五 of the m.163.com
 * article lists: INT2 codes, FP8 E4M3 group scales, uint8 assignment vectors,
 * and the centroid tables of every stage): H*N*d*bits/8 + z*H*N*d/G + T*H*N +
 * T*H*K*d*sizeof(S), with z = 2 scale bytes per group (QVG_SCALE_ASYM) or 1
 * (QVG_SCALE_SYM).  This equals bits-per-element x H*N*d/8 with
 * bits-per-element = bits + 8z/G + 8T/d + 8*sizeof(S)*T*K/N.  Returns 0 for
 * invalid arguments.  Host-only, no CUDA call. */
QVG_API size_t qvg_packed_bytes(const qvg_config* cfg, int64_t N, int32_t H, int32_t d,
                        qvg_dtype dtype);

/* Device scratch bytes qvg_quantize needs to process `H` blocks of N tokens
 * in the library's preferred batch: one wave of up to one block per SM, or
 * two waves in flight when H needs more than one wave.  Any ws_bytes >=
 * qvg_workspace_bytes(cfg, N, 1, d, dtype) works (the call then processes
 * fewer blocks at a time, one wave at a time if two do not fit).
 * Returns 0 for invalid arguments.  Host-only apart from reading the SM
 * count of the current device. */
QVG_API size_t qvg_workspace_bytes(const qvg_config* cfg, int64_t N, int32_t H, int32_t d,
                           qvg_dtype dtype);

/* Compress H independent blocks X[H][N][d] (pre-RoPE K, or V, in `dtype`;
 * section 五 caches keys before the rotary embedding) into `out`.
 *   init_centroids: NULL for a cold start, in which every stage's k-means
 *     starts from the first K tokens of its input and runs cfg->iters Lloyd
 *     iterations; or DEVICE [T][H][K][d] tables in `dtype` (e.g. the previous
 *     chunk's final centroids, section 五), with cfg->warm_iters iterations.
 *   Each Lloyd iteration: assign every token to the centroid at the least
 *     squared Euclidean distance (ties to the lowest index), then replace
 *     every non-empty centroid by the mean of its tokens rounded to `dtype`
 *     (an empty one keeps its value).  The stored pi(t) and C(t) are those of
 *     the last iteration.  R(t) = round(R(t-1) - C(t)[pi(t)]).
 *   The last residual is quantised per group g of G channels of a token as
 *     cfg->scale_mode says (qvg_scale_mode above).
 *   workspace: DEVICE scratch of ws_bytes bytes (see qvg_workspace_bytes),
 *     256-byte aligned, not shared with concurrent calls.
 *   Streams: the work is ordered after the work queued on `stream` before
 *     the call, and `stream` waits for all of it at the end.  When two waves
 *     of blocks fit in the workspace, every other wave runs on a second
 *     stream that the library creates once per device, joined to `stream` by
 *     events (a stream capture of `stream` captures both).
 * Errors: INVALID_ARG for NULL pointers (zero may be NULL with
 * QVG_SCALE_SYM), scale_mode not a qvg_scale_mode, K < 1 or K > 256, T < 0, bits != 2,
 * G not dividing d or not a multiple of 4, N < 1, H < 1, N < K on a cold
 * start with T > 0, iters < 1 (or warm_iters < 1 when warm) with T > 0;
 * UNSUPPORTED for d != 128, G outside {8,16,32,64,128}, T > 8, N >= 2^23;
 * WORKSPACE_TOO_SMALL; CUDA; DEVICE_TIMEOUT. */
QVG_API qvg_status qvg_quantize(const qvg_config* cfg, const void* X, qvg_dtype dtype,
                        int64_t N, int32_t H, int32_t d, const void* init_centroids,
                        const qvg_packed* out, void* workspace, size_t ws_bytes,
                        qvg_stream_t stream);

/* Reconstruct Y[H][N][d] (DEVICE, `dtype`, 16-byte aligned) from `packed`
 * (codes and centroids 16-byte aligned) in one fused kernel (the reverse-order
 * reconstruction of the m.163.com article, sections 四 and 五: dequantise the
 * final residual, then add back the centroid of every stage, last stage
 * first; "Fused Kernel" in gist.science/de, Technische Zusammenfassung 2C):
 * y = s*q + m (s*(u - 2) with QVG_SCALE_SYM), then + C(T)[pi_T],
 * + C(T-1)[pi_(T-1)], ..., + C(1)[pi_1], each
 * an fp32 add in that order, then one rounding to `dtype`.  Assignment
 * values >= K are clamped to K-1.  Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
QVG_API qvg_status qvg_dequantize(const qvg_config* cfg, const qvg_packed* packed, qvg_dtype dtype,
                          int64_t N, int32_t H, int32_t d, void* Y, qvg_stream_t stream);

/* Status word of a workspace after the work queued on it has completed
 * (synchronises `stream`): QVG_OK, or QVG_ERR_DEVICE_TIMEOUT if a bounded
 * device-side wait in a kernel gave up (the outputs of that call are then
 * invalid).  Clears the word, after which calls on the workspace proceed. */
QVG_API qvg_status qvg_workspace_status(void* workspace, size_t ws_bytes, qvg_stream_t stream);

/* Tokens whose tensor-core assignment was a near-tie and was decided by
 * the exact fp64 pass, summed over the calls that used this workspace since
 * the last read (synchronises `stream`; resets the count).  -1 on error.
 * No counterpart in the method: a diagnostic of the assignment kernels. */
QVG_API int64_t qvg_workspace_flagged(void* workspace, size_t ws_bytes, qvg_stream_t stream);

/* qvg_quantize without a caller workspace and without any allocation.
 * The method has no counterpart of this call: it is a library-usage variant
 * for callers that must not allocate device memory while they run (a
 * cudaMalloc/cudaFree can synchronise the device and stall every stream,
 * can fail under memory pressure mid-generation, or can find the memory
 * held by another allocator in the process) and have no workspace to lend.
 * The scratch is a 32 MiB reserve in a static __device__ array, one per
 * device, whose address is looked up on the first call on each device.
 * That first call may load the library's device code, so make it before
 * any stream capture begins.
 * The reserve's device address is looked up once per device and kept for
 * the life of the process; after a cudaDeviceReset of a device this entry
 * must not be called on that device again.
 * Arguments, layouts, results and errors are those of qvg_quantize, less
 * the workspace; the same kernels are queued, one wave at a time on
 * `stream`.
 * Limits: the reserve must hold one block's working set, about 120,000
 * tokens per block at bf16 with K = 256, T = 2 (qvg_workspace_bytes with
 * H = 1 gives the exact need); a larger block returns WORKSPACE_TOO_SMALL
 * before anything is queued.  Blocks beyond what one wave holds run in
 * further waves, as in qvg_quantize.
 * Concurrency: every call on a device uses the same reserve, so two calls
 * whose work can overlap on the device (different streams, or threads
 * without ordering between them) race and corrupt each other's results;
 * order them on one stream, or use qvg_quantize with separate workspaces.
 * A device-side timeout is recorded in the reserve's status word, returned
 * by the next call (as for a workspace, see the conventions above) and read
 * and cleared by qvg_static_status. */
QVG_API qvg_status qvg_quantize_static(const qvg_config* cfg, const void* X, qvg_dtype dtype,
                               int64_t N, int32_t H, int32_t d, const void* init_centroids,
                               const qvg_packed* out, qvg_stream_t stream);

/* Status word of the current device's static reserve after the work queued
 * on `stream` has completed (synchronises `stream`): QVG_OK, or
 * QVG_ERR_DEVICE_TIMEOUT if a bounded wait of a qvg_quantize_static call gave
 * up.  Clears the word.  No counterpart in the method (as qvg_quantize_static). */
QVG_API qvg_status qvg_static_status(qvg_stream_t stream);

/* ------------------------------------------------------------------ */
/* Attention over the compressed cache: the consumer of the m.163.com    */
/* article, section 五 (keys are cached before the rotary position       */
/* embedding, which is applied after dequantisation; the fused kernel     */
/* feeds the reconstruction to attention without writing it out;         */
/* gist.science/de, Technische Zusammenfassung 2C, "Fused Kernel").       */
/* ------------------------------------------------------------------ */

/* Bytes of the rotary tables for head dimension d and positions
 * 0 .. max_pos: a 256-byte header, then (cos, sin) of p * theta_i in fp32
 * for every position p and pair i < d/2 (512 bytes a position at d = 128).
 * 0 for unsupported arguments (d != 128, max_pos < 0 or >= 2^24).
 * Host-only. */
QVG_API size_t qvg_rope_tables_bytes(int32_t d, int64_t max_pos);

/* Fill the rotary tables (DEVICE, caller-owned, 16-byte aligned, `bytes`
 * from qvg_rope_tables_bytes) for theta_i = base^(-2i/d), the RoFormer form:
 * channel pair (2i, 2i+1) of a token at position p is turned by p * theta_i.
 * The angles and their cosines and sines are formed in fp64 on the device and
 * rounded once to fp32.  The header's first 4 bytes are the status word of the
 * qvg_attention calls that use the tables (read and cleared by
 * qvg_workspace_status on the tables buffer).  Errors: INVALID_ARG (base
 * <= 1, d != 128, NULL), WORKSPACE_TOO_SMALL, CUDA. */
QVG_API qvg_status qvg_rope_tables(double base, int32_t d, int64_t max_pos, void* tables, size_t bytes,
                           qvg_stream_t stream);

/* Softmax attention of Nq queries per head over a compressed K/V cache of
 * Nk tokens per head, with the reconstruction fused into the K/V load:
 *   O[h] = softmax(rope(Q[h]) rope(K^[h])^T / sqrt(d)) V^[h]
 * K^ and V^ are what qvg_dequantize would write for `k` and `v` (two
 * qvg_quantize outputs of H blocks of Nk tokens with the same cfg; bf16),
 * bit for bit; they are never written to memory.  Cached token i sits at
 * position i; query n at q_pos[n] (positions outside [0, max_pos] of the
 * tables are clamped).  No mask.
 *   Q      DEVICE [H][Nq][d] bf16, before the rotary embedding, 16-byte aligned
 *   q_pos  DEVICE [Nq] int64
 *   tables DEVICE rotary tables (qvg_rope_tables); they must cover Nk - 1
 *   O      DEVICE [H][Nq][d] fp32, 16-byte aligned
 *   workspace, ws_bytes  DEVICE scratch for the partial results of a cache
 *          split over clusters (qvg_attention_workspace_bytes), 16-byte
 *          aligned, caller-owned; NULL (or too small) keeps every split
 *          inside one thread-block cluster
 * The products run on the tensor cores with bf16 operands (the rotated keys
 * and queries and the softmax weights are rounded to bf16) and fp32
 * accumulation; the softmax uses base-2 exponentials in fp32.
 * Errors: INVALID_ARG, UNSUPPORTED (d != 128, ...), CUDA, DEVICE_TIMEOUT (a
 * timeout recorded in the tables' status word by earlier, completed work). */
QVG_API qvg_status qvg_attention(const qvg_config* cfg, const qvg_packed* k, const qvg_packed* v, int64_t Nk,
                         int32_t H, int32_t d, const void* Q, const int64_t* q_pos, int64_t Nq,
                         const void* tables, size_t tables_bytes, float* O, void* workspace, size_t ws_bytes,
                         qvg_stream_t stream);

/* qvg_attention cuts the cache of each head and block of 256 queries into
 * ranges of its tiles of 128 tokens, one CTA (or pair of CTAs, which share
 * the reconstruction of two query blocks) per range, so that the grid fills
 * the SMs.  The ranges are merged by the usual rescaling of partial softmax
 * sums: inside a thread-block cluster (up to 4 ranges, through distributed
 * shared memory), or, with a workspace, over clusters (up to 16 ranges,
 * through the workspace and a second kernel).  Each range rounds its softmax
 * weights to bf16 against its own running maximum, so cuts differ by such
 * roundings (the error bound of qvg_attention holds for every cut).  By
 * default the library picks the cut from the device's cluster occupancy.
 *   qvg_attention_set_split fixes a cluster split for the process (1 .. 8
 *     CTAs, capped at the cache's tile count and 4 for pairs; 0 = automatic
 *     again) and returns the previous setting, or -1 (nothing changed).
 *   qvg_attention_split returns the number of ranges a qvg_attention call
 *     with these sizes and a workspace of ws_bytes would use on the current
 *     device, or -1 for invalid arguments or no device.
 *   qvg_attention_workspace_bytes returns the workspace the preferred cut
 *     needs (0: none), or 0 for invalid arguments.
 * Host-only; none launches work. */
QVG_API int32_t qvg_attention_set_split(int32_t split);
QVG_API int32_t qvg_attention_split(const qvg_config* cfg, int64_t Nk, int32_t H, int64_t Nq, size_t ws_bytes);
QVG_API size_t qvg_attention_workspace_bytes(const qvg_config* cfg, int64_t Nk, int32_t H, int64_t Nq);

/* ------------------------------------------------------------------ */
/* Diagnostics (no counterpart in the method; used by the benchmark).    */
/* ------------------------------------------------------------------ */

/* Turn per-kernel device timing on or off (process-wide).  When on, every
 * kernel launch is bracketed by two CUDA events on its stream. */
QVG_API void qvg_profile_enable(int enable);

/* Zero the launch counters and timing totals. */
QVG_API void qvg_profile_reset(void);

/* Kernel launches issued by this library since the last reset. */
QVG_API int64_t qvg_profile_launches(void);

/* Write a JSON object {"kernel": {"launches": n, "timed": m, "ms": t}, ...}
 * into buf (NUL-terminated).  Synchronises the device if timed launches are
 * pending.  Returns 0, or the needed size if buf is NULL or too small, or -1
 * on a CUDA error. */
QVG_API int qvg_profile_report(char* buf, size_t buf_bytes);

/* ------------------------------------------------------------------ */
/* Streaming cache (section 五, streaming centroid cache).               */
/* A library-owned, append-only compressed KV cache for H blocks (heads). */
/* Each appended chunk is quantised as one block per head; chunk c > 0    */
/* warm-starts every stage's k-means from chunk c-1's final centroids.    */
/* ------------------------------------------------------------------ */
typedef struct qvg_cache qvg_cache;

/* Allocate a cache for up to max_tokens tokens per head in up to max_chunks
 * chunks of at most max_chunk_tokens tokens each (0 = max_tokens): the
 * packed storage, the centroid tables of every chunk, and the k-means
 * workspace of the largest chunk, all device memory on the current device
 * (synchronises the device).  Errors: INVALID_ARG (also max_chunk_tokens < K
 * with T > 0), UNSUPPORTED, NO_MEMORY (nothing is left allocated). */
QVG_API qvg_status qvg_cache_create(const qvg_config* cfg, qvg_dtype dtype, int32_t H, int32_t d,
                            int64_t max_tokens, int32_t max_chunks, int64_t max_chunk_tokens,
                            qvg_cache** out);

/* Compress and append one chunk X_chunk[H][N_chunk][d] (DEVICE, cache dtype).
 * Chunk 0 runs a cold start (needs N_chunk >= K when T > 0) with cfg->iters;
 * later chunks warm-start with cfg->warm_iters.  Allocates nothing and does
 * not wait for the GPU: the workspace was sized at qvg_cache_create.  On an
 * error the cache is unchanged.  Errors: INVALID_ARG, CAPACITY (more tokens
 * or chunks than the cache holds, or N_chunk > max_chunk_tokens), CUDA,
 * DEVICE_TIMEOUT (see the conventions above; qvg_cache_status clears it). */
QVG_API qvg_status qvg_append_chunk(qvg_cache* cache, const void* X_chunk, int64_t N_chunk,
                            qvg_stream_t stream);

/* Status word of the cache's workspace after the work queued on `stream`
 * has completed (synchronises `stream`): QVG_OK, or QVG_ERR_DEVICE_TIMEOUT if
 * a bounded device-side wait of an append gave up (that chunk's packed data
 * is then invalid).  Clears the word. */
QVG_API qvg_status qvg_cache_status(qvg_cache* cache, qvg_stream_t stream);

/* Reconstruct the whole cache into Y[H][tokens][d] (DEVICE, cache dtype), one
 * fused launch over every (chunk, head) block. */
QVG_API qvg_status qvg_cache_dequantize(const qvg_cache* cache, void* Y, qvg_stream_t stream);

QVG_API int64_t qvg_cache_tokens(const qvg_cache* cache);   /* tokens per head so far */
QVG_API int32_t qvg_cache_chunks(const qvg_cache* cache);   /* chunks so far */

/* Packed view of chunk `chunk` (DEVICE pointers into the cache, valid until
 * qvg_cache_destroy; layouts as qvg_packed with H blocks of *n_tokens
 * tokens); *first_token is the chunk's first token index. */
QVG_API qvg_status qvg_cache_chunk_view(const qvg_cache* cache, int32_t chunk, qvg_packed* view,
                                int64_t* first_token, int64_t* n_tokens);

/* Settings chosen chunk by chunk (the m.163.com article, section 九, names
 * adapting the compression parameters to the content as future work; the
 * rule below is this library's).  A ladder of up to four settings (stage
 * count and group size; the other fields of the cache's qvg_config are
 * shared) from the cheapest to the most expensive.  For each chunk the
 * cache first sums, over every block, token and group of probe_group
 * channels, the E4M3 code of the group's range fl32(max - min) (about eight
 * codes per doubling of the range): the statistic S.  The chunk takes the
 * level equal to the number of thresholds (ascending, in sixteenths of a
 * code) that 16 S exceeds per group, i.e. the mean range code.  Centroid
 * reuse: chunk c > 0 starts stage t from chunk c-1's tables when both have
 * that stage (warm_iters iterations), every other stage from its first K
 * tokens (iters); every refresh_every-th chunk (when > 0) starts cold. */
typedef struct {
    int32_t levels;          /* 1 .. 4 */
    int32_t T[4];            /* stages of each level */
    int32_t group_size[4];   /* G of each level */
    int32_t thresholds[3];   /* levels - 1 ascending thresholds, sixteenths of an E4M3 code */
    int32_t probe_group;     /* group size of the statistic */
    int32_t refresh_every;   /* cold start every n-th chunk; 0 = never */
} qvg_adaptive_policy;

/* A cache whose chunks take their settings from `pol` (cfg gives K, bits,
 * iters, warm_iters and scale_mode; its T and group_size are ignored).
 * Storage is sized for the ladder's largest stage count and smallest group.
 * qvg_append_chunk on it waits for `stream` once per chunk (the statistic
 * is read by the host, which picks the level) and returns INVALID_ARG for a
 * chunk with fewer than K tokens that needs a cold stage; the views of
 * qvg_cache_chunk_view use each chunk's own T and G (qvg_cache_chunk_info).
 * Errors as qvg_cache_create, and INVALID_ARG for a bad policy. */
QVG_API qvg_status qvg_cache_create_adaptive(const qvg_config* cfg, const qvg_adaptive_policy* pol,
                                     qvg_dtype dtype, int32_t H, int32_t d, int64_t max_tokens,
                                     int32_t max_chunks, int64_t max_chunk_tokens, qvg_cache** out);

/* Settings of chunk `chunk`: its level in the policy's ladder, stage count,
 * group size and statistic (0, the cache's T and G, and 0 for a cache
 * without a policy).  Any pointer may be NULL.  Errors: INVALID_ARG. */
QVG_API qvg_status qvg_cache_chunk_info(const qvg_cache* cache, int32_t chunk, int32_t* level, int32_t* T,
                                int32_t* G, uint64_t* stat);

/* Bytes of device memory the cache holds (packed storage + workspace). */
QVG_API size_t qvg_cache_device_bytes(const qvg_cache* cache);

QVG_API void qvg_cache_destroy(qvg_cache* cache);

#ifdef __cplusplus
}
#endif
#endif /* QVG_H_ */
