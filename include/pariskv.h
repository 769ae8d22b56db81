/*
 * pariskv.h -- C ABI of libpariskv.so, the B200 (sm_100a) ParisKV KV-cache retrieval path.
 *
 * The method ("Technical Summary: ParisKV", gist.science/paper/2602.07721, Methodology and
 * System-Level Innovations; "ParisKV: Fast and Drift-Robust KV-Cache Retrieval for
 * Long-Context LLMs", ICML 2026 poster abstract): keys are indexed once at prefill and kept
 * fresh as decoding appends new keys; each decode step returns, for every query head, the
 * top-k cached keys found on the GPU from compact metadata (no CPU-side search); the
 * selected full-precision K/V rows, which may live in pinned host memory, feed a sparse
 * decode attention.
 *
 * Conventions for every call:
 *  - Plain pointers and sizes only. A "device pointer" is memory the current CUDA device can
 *    dereference: cudaMalloc'd memory, or pinned host memory allocated with cudaHostAlloc /
 *    registered with cudaHostRegister (UVA makes its host address usable on the device).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Work is
 *    enqueued asynchronously on it; argument errors are reported synchronously and leave
 *    nothing enqueued.
 *  - The caller owns every buffer it passes; no call keeps a caller pointer after it
 *    returns. The library owns the index and its scratch memory.
 *  - An index is bound to the device that was current when it was built, and is not
 *    thread-safe: calls on one index must not overlap.
 *  - Floating point follows IEEE fp32 (no fast-math); search results are deterministic.
 */
#ifndef PARISKV_H_
#define PARISKV_H_

#include <stdint.h>

#if defined(__GNUC__)
#define PARISKV_API __attribute__((visibility("default")))
#else
#define PARISKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PARISKV_OK = 0,
    PARISKV_EINVAL = 1,     /* an argument is invalid; nothing was done */
    PARISKV_ENOMEM = 2,     /* a device allocation failed; nothing was changed */
    PARISKV_ECUDA = 3,      /* a CUDA call or a kernel launch failed (pariskv_last_error()) */
    PARISKV_ECAPACITY = 4,  /* an append would exceed the index capacity; nothing appended */
    PARISKV_ETIMEOUT = 5    /* a bounded device-side wait expired; results are invalid */
} pariskv_status;

enum { PARISKV_F32 = 0, PARISKV_BF16 = 1 };

/* Hyper-parameters and shapes. "Coarse Candidate Generation" and "Candidate Reranking" in
 * the methodology of the technical summary name B, m, rho, the tiered vote weights and the
 * 5-10% candidate fraction. Constraints checked by every call that takes a config:
 *   d == 128, m == 8, B * m == d (the kernels are specialised for d = 128, m = 8);
 *   1 <= rho <= 2^m; 0 <= w_rest <= w_rank1 <= 3, w_rank1 >= 1 (so a score fits 6 bits);
 *   1 <= cand_bp <= 10000; batch, num_kv_heads, group >= 1; capacity >= 0;
 *   dtype is PARISKV_F32 or PARISKV_BF16; levels is one of the PARISKV_LEVELS_* below.
 *
 * Magnitude levels of the 4-bit RSQ codes ("Candidate Reranking", Quantization: 1 sign bit
 * and 3 magnitude bits, "derived from rotation-induced Beta priors"). Each code quantises
 * r_j = |y_j| / max_i |y_i| over its 8-dim subspace of the rotated key:
 *   PARISKV_LEVELS_UNIFORM: mag = min(7, floor(7 r + 1/2)) in IEEE fp32, signed level
 *     vt = +-mag (8 uniform levels over [0, max]);
 *   PARISKV_LEVELS_PRIOR: the 8 Lloyd-Max levels of the law of r under the rotation (a
 *     subspace direction uniform on the sphere, u_j^2 ~ Beta(1/2, 7/2); r has the law of
 *     half-normal ratios), computed by the library once per process;
 *   PARISKV_LEVELS_TABLE: the caller's level_table (8 finite fp32 values,
 *     0 <= c_0 < c_1 < ... < c_7).
 * With a table, mag = the number of i in 1..7 with r_j >= t_i, r_j in IEEE fp32 and t_i the
 * fp32 rounding of the exact midpoint (c_{i-1} + c_i) / 2 (the nearest level), and
 * vt = +-c_mag. Everything else (factor fold, rerank chains) is the same for all three.
 * level_table is ignored unless levels == PARISKV_LEVELS_TABLE. */
enum { PARISKV_LEVELS_UNIFORM = 0, PARISKV_LEVELS_PRIOR = 1, PARISKV_LEVELS_TABLE = 2 };
typedef struct {
    int32_t d;            /* head dimension */
    int32_t B;            /* number of subspaces */
    int32_t m;            /* dimensions per subspace */
    int32_t rho;          /* centroids selected per subspace by each query */
    int32_t w_rank1;      /* vote weight of a query's nearest centroid (default 2) */
    int32_t w_rest;       /* vote weight of its ranks 2..rho (default 1) */
    int32_t cand_bp;      /* candidate fraction in basis points (500 = 5%) */
    int32_t batch;        /* sequences */
    int32_t num_kv_heads; /* KV heads per sequence */
    int32_t group;        /* query heads per KV head (GQA group size) */
    int64_t capacity;     /* maximum tokens per (sequence, KV head) in the index */
    int32_t dtype;        /* element type of keys, queries, values and outputs */
    int32_t levels;       /* magnitude levels of the codes: PARISKV_LEVELS_* (default 0) */
    float level_table[8]; /* the levels when levels == PARISKV_LEVELS_TABLE */
} pariskv_config;

typedef struct pariskv_index pariskv_index;  /* opaque; owns device memory */

/* Fills *cfg with d=128, B=16, m=8, rho=4, w_rank1=2, w_rest=1, cand_bp=500, batch=1,
 * num_kv_heads=1, group=1, capacity=0, dtype=PARISKV_BF16, levels=PARISKV_LEVELS_UNIFORM. */
PARISKV_API pariskv_status pariskv_config_default(pariskv_config* cfg);

/* The 8 magnitude levels PARISKV_LEVELS_PRIOR uses (ascending), into out[0..7]. */
PARISKV_API pariskv_status pariskv_prior_levels(float* out);

/* Builds an index over the first n keys of every (sequence, KV head).
 * Definition: "Normalization and Rotation" and "Coarse Candidate Generation" /
 * "Quantization" / "Calibration" (technical summary, Core Algorithmic Innovations 1-2):
 * each key is l2-normalised and rotated by the SRHT R = H diag(signs) / sqrt(d) shared by
 * keys and queries, then stored as B one-byte bucket ids (the nearest sign centroid of each
 * m-dim subspace), d 4-bit codes (sign bit + 3-bit uniform magnitude level) and B fp32
 * calibration factors ("precomputed during the prefill phase").
 *   srht_signs: host array of d int8 values, each +1 or -1 (copied).
 *   keys:       device pointer, element (s, t, j) at keys[(s * ld_tok + t) * d + j] with
 *               s = sequence * num_kv_heads + kv_head, t < n, j < d; dtype cfg->dtype.
 *   ld_tok:     token slab stride of `keys` (>= n when n > 0).
 *   n:          0 <= n <= cfg->capacity.
 *   out:        receives the new index (NULL on failure).
 * Errors: EINVAL (config, NULL pointer, misaligned keys, n/ld_tok), ENOMEM, ECUDA. */
PARISKV_API pariskv_status pariskv_build_index(const pariskv_config* cfg, const int8_t* srht_signs,
                                   const void* keys, int64_t ld_tok, int64_t n, void* stream,
                                   pariskv_index** out);

/* Appends t new keys to every (sequence, KV head): the decode-time update that keeps the
 * index fresh under distribution drift ("Drift-Robust Analytic Centroids": the centroids
 * are data-independent, so new keys are encoded exactly like prefill keys).
 *   keys: device pointer, element (s, r, j) at keys[(s * ld_tok + r) * d + j], r < t.
 * Errors: EINVAL, ECAPACITY (size + t > capacity; nothing appended), ECUDA. */
PARISKV_API pariskv_status pariskv_append(pariskv_index* index, const void* keys, int64_t ld_tok, int64_t t,
                              void* stream);

/* One decode-step retrieval for every query head ("Two-Stage GPU-Native Retrieval
 * Pipeline"): rotate the query; per subspace select its top-rho centroids (tiered weights
 * w_rank1, w_rest); collision-vote an integer coarse score for every cached key; keep the
 * C = min(n, max(k, ceil(n * cand_bp / 10000))) best-scoring keys (ties to the lower key
 * index); rerank them with the RSQ-IP estimator est = ||q|| * sum_b w_{i,b} <v_{i,b}, q~_b>;
 * return the k best (ties to the lower key index).
 *   q:         device pointer [batch][num_kv_heads * group][d], dtype cfg->dtype; query head
 *              h uses KV head h / group.
 *   k:         1 <= k <= current size.
 *   topk_idx:  device pointer [batch][num_kv_heads * group][k] int32: the selected key
 *              indices in ascending index order.
 *   topk_est:  device pointer with the same shape (fp32 estimates of <k, q>), or NULL.
 * Scratch memory is owned by the index and sized for a full index when it is created; a
 * search allocates only when k exceeds ceil(capacity * cand_bp / 10000) and k is larger than
 * any earlier search's (so run one search with the largest k before capturing a CUDA graph).
 * Errors: EINVAL, ENOMEM, ECUDA, ETIMEOUT. */
PARISKV_API pariskv_status pariskv_search(pariskv_index* index, const void* q, int32_t k, int32_t* topk_idx,
                              float* topk_est, void* stream);

/* Sparse decode attention over the retrieved tokens (Problem Statement: attend to a Top-k
 * subset; System-Level Innovations 1: the selected full-precision K/V rows are fetched by
 * the GPU kernel directly, from HBM or from pinned host memory over UVA, with no memcpy):
 *   out[s][h] = sum_{t in topk[s][h]} softmax_t(scale * <q[s][h], K[s][h/group][t]>) V[..][t]
 *   q:        device pointer [batch][Hq][d]; K, V: device or pinned-host pointers with the
 *             layout of pariskv_build_index's keys (slab stride ld_tok, n valid tokens);
 *   topk_idx: device pointer [batch][Hq][k]; entries outside [0, n) are skipped; the valid
 *             entries of one head are distinct (as pariskv_search returns them: a repeated
 *             index may be attended once or twice depending on the kernel chosen);
 *   out:      device pointer [batch][Hq][d] of element type out_dtype (PARISKV_F32 keeps the
 *             fp32 accumulator precision; PARISKV_BF16 rounds to nearest even).
 * q, K and V have element type cfg->dtype; accumulation is fp32. With K/V in pinned host
 * memory (or fp32) and 1 < group <= 8, the rows the group's query heads selected are merged
 * into one union per (sequence, KV head) and each union row is fetched once for every head
 * that selected it. The split-K partials (and that union's bitmaps) live in a stream-ordered
 * workspace allocated and freed on `stream` from a memory pool the library keeps per device
 * (it keeps its memory mapped between calls; it holds at most the largest workspaces in
 * flight at once).
 * Errors: EINVAL, ENOMEM, ECUDA. */
PARISKV_API pariskv_status pariskv_sparse_attend(const pariskv_config* cfg, const void* q,
                                                 const void* K, const void* V, int64_t ld_tok,
                                                 int64_t n, const int32_t* topk_idx, int32_t k,
                                                 float scale, void* out, int32_t out_dtype,
                                                 void* stream);

/* Allocation-free variant of pariskv_sparse_attend (an addition of this library; the
 * ParisKV pages have no counterpart). Same arguments, layouts and results (up to the
 * summation order of the split-K partials), but the call never allocates: the partials live
 * in a fixed 4 MiB device array inside the library. It is meant for callers that may not
 * touch a device allocator on the decode path: a serving runtime whose memory manager
 * reserves all of HBM up front, a process where stream-ordered memory pools are unavailable
 * or disabled, or a latency-critical loop where an allocation could block.
 *  - The first call on each device looks the array's device address up (once, with that
 *    device current); make that first call before capturing any CUDA graph.
 *  - Every device that loads the library keeps the array until the process exits.
 *  - All calls on a device share the array: calls that can overlap on the GPU (different
 *    streams without ordering) race and must be serialised by the caller. Nothing in it has
 *    to start at zero; each call overwrites what it reads.
 *  - batch * num_kv_heads * group may not exceed 7943 (one split per head); larger
 *    requests are rejected with PARISKV_EINVAL before anything is enqueued.
 * Errors: EINVAL, ECUDA. */
PARISKV_API pariskv_status pariskv_sparse_attend_noalloc(const pariskv_config* cfg,
                                                         const void* q, const void* K,
                                                         const void* V, int64_t ld_tok,
                                                         int64_t n, const int32_t* topk_idx,
                                                         int32_t k, float scale, void* out,
                                                         int32_t out_dtype, void* stream);

/* Index images, for checkpoint and resume (the index is derived from the keys, so an image
 * only saves re-encoding them). An image is a self-describing byte string: a 256-byte header
 * (magic "PARISKV", format version, the pariskv_config, the SRHT signs, the size n and the
 * number of units) followed by the bucket ids and the code records of every unit in the
 * library's storage layout, units * n * (16 + 128) bytes. Images are read only by the same
 * format version.
 *   pariskv_export_bytes: the image size of the index as it is now.
 *   pariskv_export: writes the image of `index` into `buf` (host memory, pinned or pageable,
 *     at least pariskv_export_bytes bytes), after all work queued on `stream`; returns when
 *     the image is complete.
 *   pariskv_import: creates an index on the current device from an image, with capacity
 *     `capacity` (0: the image's size; it must be >= the image's size); returns when `buf` is
 *     no longer needed. The imported index searches and appends exactly like the exported one.
 * Errors: EINVAL (NULL pointers, too small a buffer, a malformed, truncated or foreign image,
 * capacity below the image's size), ENOMEM, ECUDA. The import checks the image's header and
 * sizes on the host before it touches the device. */
PARISKV_API pariskv_status pariskv_export_bytes(const pariskv_index* index, size_t* bytes);
PARISKV_API pariskv_status pariskv_export(pariskv_index* index, void* buf, size_t bytes,
                                          void* stream);
PARISKV_API pariskv_status pariskv_import(const void* buf, size_t bytes, int64_t capacity,
                                          void* stream, pariskv_index** out);

/* Waits for the index's stream work and reports any asynchronous error or expired wait. */
PARISKV_API pariskv_status pariskv_sync(pariskv_index* index, void* stream);

/* Frees the index (NULL is a no-op). Waits for the device first. */
PARISKV_API pariskv_status pariskv_destroy(pariskv_index* index);

/* Current number of indexed tokens per (sequence, KV head); -1 for NULL. */
PARISKV_API int64_t pariskv_size(const pariskv_index* index);

/* Number of kernels the last search / attend call launched (for launch accounting). */
PARISKV_API int32_t pariskv_last_launch_count(void);

PARISKV_API const char* pariskv_status_string(pariskv_status status);

/* Message of the last failure on the calling thread ("" when none). */
PARISKV_API const char* pariskv_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PARISKV_H_ */
