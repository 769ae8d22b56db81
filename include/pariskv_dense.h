/* pariskv_dense.h -- dense decode attention over every cached token, the full-attention
 * baseline that ParisKV is compared with.
 *
 * "Technical Summary: ParisKV", Key Contributions 3 and Results, and "ParisKV: Fast and
 * Drift-Robust KV-Cache Retrieval for Long-Context LLMs" (abstract) measure ParisKV against
 * full attention (FlashAttention) over the whole KV cache. This call is that baseline on the
 * same data layout, so the retrieval path can be compared with it on one GPU:
 *   out[s][h] = sum_{t < n} softmax_t(scale * <q[s][h], K[s][h/group][t]>) V[s][h/group][t].
 *
 *   cfg:   batch, num_kv_heads, group (1..8) and dtype (PARISKV_BF16 only) are used; the
 *          search fields and capacity are ignored (capacity must still be valid).
 *   q:     device pointer [batch][num_kv_heads * group][d] bf16, 4-byte aligned.
 *   K, V:  device (or pinned host) pointers [batch][num_kv_heads][ld_tok][d] bf16, 16-byte
 *          aligned; tokens [0, n) are attended, 1 <= n <= ld_tok.
 *   out:   device pointer [batch][Hq][d] of out_dtype (PARISKV_F32 or PARISKV_BF16).
 * Accumulation is fp32. Every K/V byte is read once per call (all query heads of a KV head
 * share one pass). The split-K workspace comes from the library's per-device memory pool,
 * stream-ordered on `stream`, like pariskv_sparse_attend. Two kernel launches.
 * Errors: EINVAL (bad config, dtype not bf16, group > 8, n out of range, bad pointers),
 * ENOMEM, ECUDA. */
#ifndef PARISKV_DENSE_H_
#define PARISKV_DENSE_H_

#include "pariskv.h"

#ifdef __cplusplus
extern "C" {
#endif

PARISKV_API pariskv_status pariskv_dense_attend(const pariskv_config* cfg, const void* q,
                                                const void* K, const void* V, int64_t ld_tok,
                                                int64_t n, float scale, void* out,
                                                int32_t out_dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PARISKV_DENSE_H_ */
