/*
 * pariskv_debug.h -- test-only entry points of libpariskv.so.
 *
 * These calls expose the stages of the retrieval path one by one so that each stage can be
 * compared, bit for bit, with an independent reference on identical inputs. They are not
 * part of the product surface; the conventions of pariskv.h (pointer kinds, streams,
 * ownership, errors) apply unchanged. "units" below means batch * num_kv_heads, and
 * Hq = num_kv_heads * group.
 */
#ifndef PARISKV_DEBUG_H_
#define PARISKV_DEBUG_H_

#include "pariskv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Normalise and rotate n rows ("Normalization and Rotation"): x [n][d] of cfg->dtype
 * (device) -> y fp32 [n][d] and norm fp32 [n] (device). */
PARISKV_API pariskv_status pariskv_debug_rotate(const pariskv_config* cfg, const int8_t* srht_signs,
                                    const void* x, int64_t n, float* y, float* norm,
                                    void* stream);

/* pariskv_build_index from already rotated keys: y fp32 [units][ld_tok][d] and knorm fp32
 * [units][ld_tok] (device) replace the normalise-and-rotate step. */
PARISKV_API pariskv_status pariskv_debug_build_index_rotated(const pariskv_config* cfg,
                                                 const int8_t* srht_signs, const float* y,
                                                 const float* knorm, int64_t ld_tok, int64_t n,
                                                 void* stream, pariskv_index** out);

/* pariskv_append from already rotated keys (layouts as above, t rows per unit). */
PARISKV_API pariskv_status pariskv_debug_append_rotated(pariskv_index* index, const float* y,
                                            const float* knorm, int64_t ld_tok, int64_t t,
                                            void* stream);

/* pariskv_search from already rotated queries: qt fp32 [batch][Hq][d], qnorm fp32
 * [batch][Hq] (device). */
PARISKV_API pariskv_status pariskv_debug_search_rotated(pariskv_index* index, const float* qt,
                                            const float* qnorm, int32_t k, int32_t* topk_idx,
                                            float* topk_est, void* stream);

/* Copies the index to host memory in canonical layouts (synchronous):
 *   ids u8 [units][n][B] (bucket id of subspace b), codes u8 [units][n][d] (bit 3 = sign,
 *   bits 0..2 = magnitude level of dim j), factors fp32 [units][n][B]. NULL skips an array. */
PARISKV_API pariskv_status pariskv_debug_export_index(pariskv_index* index, uint8_t* ids, uint8_t* codes,
                                          float* factors);

/* Copies the intermediates of the last search to host memory (synchronous):
 *   lut u8 [units * group][B][256]  vote weight of each centroid, per query head;
 *   scores int32 [units * group][n] coarse score of every key;
 *   ncand: receives C, the candidate count;
 *   cand int32 [units * group][C]   candidate key indices, ascending;
 *   S fp32 [units * group][C]       rerank value sum_b f_b <vt_b, q~_b> of each candidate.
 * Query head (sequence s, head h) is row s * Hq + h. NULL skips an array. */
PARISKV_API pariskv_status pariskv_debug_export_search(pariskv_index* index, uint8_t* lut, int32_t* scores,
                                           int64_t* ncand, int32_t* cand, float* S);

/* Per-stage timing of pariskv_search with CUDA events recorded on the search stream between
 * the kernel launches. enable != 0 turns it on for this index (events are created then). */
PARISKV_API pariskv_status pariskv_debug_profile(pariskv_index* index, int32_t enable);

/* Waits for the last profiled search and writes the device time (ms) of each of its stages
 * to ms[0..*nstages-1]: query prep, vote scan, threshold, compaction, rerank, top-k. ms must
 * hold at least 8 floats. */
PARISKV_API pariskv_status pariskv_debug_stage_ms(pariskv_index* index, float* ms,
                                                  int32_t* nstages);

/* Reads `bytes` from `src` once, with coalesced 16-byte loads spread over every SM, and
 * folds the data into one word that may be written to `sink` (a device pointer to 4 bytes),
 * on `stream`. Timed with CUDA events around the call it measures how fast the device reads
 * that memory: for pinned host memory (mapped into the device address space) this is the
 * PCIe read bandwidth that bounds sparse attention over host K/V. No counterpart on the
 * pages (a measurement aid). src must be 16-byte aligned and bytes a positive multiple of
 * 16. Errors: EINVAL, ECUDA. */
PARISKV_API pariskv_status pariskv_debug_read_stream(const void* src, int64_t bytes,
                                                     uint32_t* sink, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PARISKV_DEBUG_H_ */
