/* pariskv_cache.h -- four-region KV cache for unbounded decoding, on top of pariskv.h.
 *
 * "Technical Summary: ParisKV", System-Level Innovations 2 ("Sliding-Window Update
 * Mechanism"): the KV cache is managed in four regions, Sink (the earliest tokens, kept on
 * the GPU), Local (the most recent tokens, on the GPU), Retrieval (older tokens, offloaded
 * to host memory and found through the ParisKV index) and an Update Buffer for newly
 * generated tokens. When the buffer fills, the oldest Local tokens move to the Retrieval
 * zone and the buffer's tokens become Local, so the retrieval index stays current while
 * recent and early context keep fast, exact access. "ParisKV: Fast and Drift-Robust KV-Cache Retrieval for Long-Context
 * LLMs" (abstract): offloaded K/V is read over UVA for the retrieved tokens only.
 *
 * Readings this library takes where the pages leave details open:
 *  - a token enters Sink while Sink holds fewer than n_sink tokens, otherwise the buffer;
 *  - when the buffer holds n_buffer tokens after an append, the oldest
 *    max(0, local + n_buffer - n_local) Local tokens are evicted to Retrieval (in token
 *    order) and the buffer's tokens are appended to Local;
 *  - prefill of n tokens: the first min(n, n_sink) go to Sink, the last min(rest, n_local)
 *    to Local, the ones in between to Retrieval;
 *  - every decode step attends, for each query head, to all Sink, Local and buffer tokens
 *    plus the top-k Retrieval tokens of a ParisKV search with that step's query
 *    (k = min(k, Retrieval size)); one softmax over the union.
 * Retrieval row r therefore holds token n_sink + r of the sequence (with Sink full).
 *
 * Memory: the Sink, Local and buffer rows of every (sequence, KV head) live in one device
 * pool of n_sink + n_local + n_buffer rows (kept contiguous: Sink, then Local, then buffer);
 * Retrieval K/V live in pinned host memory the library allocates (retrieval_capacity rows
 * per unit), read by the attention over UVA; the index lives in device memory.
 *
 * All calls are stream-ordered on `stream` (a cudaStream_t), like pariskv.h; the cache's
 * region bookkeeping is on the host, so calls on one cache must be made in order from one
 * host thread. Errors as in pariskv.h; a step or prefill that would overflow
 * retrieval_capacity returns PARISKV_ECAPACITY and leaves the cache unchanged. */
#ifndef PARISKV_CACHE_H_
#define PARISKV_CACHE_H_

#include "pariskv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pariskv_cache pariskv_cache;

typedef struct {
    int32_t n_sink;              /* >= 0 */
    int32_t n_local;             /* >= n_buffer */
    int32_t n_buffer;            /* >= 1 */
    int32_t k;                   /* retrieved tokens per query head and step, >= 1 */
    int64_t retrieval_capacity;  /* tokens per (sequence, KV head) in the Retrieval zone */
} pariskv_cache_config;

/* Creates an empty cache: the index of the Retrieval zone (cfg->capacity is ignored and set
 * to cc->retrieval_capacity), the device pool and the pinned host Retrieval K/V. srht_signs
 * as in pariskv_build_index. */
PARISKV_API pariskv_status pariskv_cache_create(const pariskv_config* cfg,
                                                const pariskv_cache_config* cc,
                                                const int8_t* srht_signs, void* stream,
                                                pariskv_cache** out);

/* Prefill: n tokens of K and V, [batch][num_kv_heads][ld_tok][d] of cfg->dtype, device or
 * pinned host pointers. The cache must be empty. */
PARISKV_API pariskv_status pariskv_cache_prefill(pariskv_cache* cache, const void* K,
                                                 const void* V, int64_t ld_tok, int64_t n,
                                                 void* stream);

/* One decode step: appends the new token's key and value (k_new, v_new: device pointers
 * [batch][num_kv_heads][d]), applies the buffer promotion if the buffer is full, searches the
 * Retrieval zone with q (device [batch][Hq][d]) and attends over the union described above;
 * out: device [batch][Hq][d] of out_dtype (PARISKV_F32 or PARISKV_BF16). topk_idx, if not
 * NULL, receives the Retrieval rows used (device [batch][Hq][k]; entries past the
 * Retrieval size are -1). */
PARISKV_API pariskv_status pariskv_cache_step(pariskv_cache* cache, const void* q,
                                              const void* k_new, const void* v_new,
                                              float scale, void* out, int32_t out_dtype,
                                              int32_t* topk_idx, void* stream);

/* Tokens per region, per (sequence, KV head): counts[0..3] = Sink, Local, buffer, Retrieval. */
PARISKV_API pariskv_status pariskv_cache_counts(const pariskv_cache* cache, int64_t* counts);

/* The Retrieval zone's index (owned by the cache; valid until pariskv_cache_destroy). */
PARISKV_API pariskv_index* pariskv_cache_index(pariskv_cache* cache);

PARISKV_API pariskv_status pariskv_cache_destroy(pariskv_cache* cache);

#ifdef __cplusplus
}
#endif

#endif /* PARISKV_CACHE_H_ */
