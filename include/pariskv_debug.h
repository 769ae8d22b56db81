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

/* Test hook: the next pariskv_search on this index writes `value` (which must not be a valid
 * key index: negative or >= the index size) into candidate slot `pos` of query head `head`
 * (row s * Hq + h) after the compaction, as a selection bug would. The rerank and the top-k
 * skip the out-of-range record instead of reading it; pariskv_sync then reports ECUDA with
 * the device status ST_BADINDEX, and the results of every other query head are unaffected.
 * One search consumes the hook. pos must be below that search's candidate count C (else
 * the search fails with EINVAL), with one exception that tests the guard bytes (see
 * pariskv_debug_check_guards): with guards on, a slot of the last head that falls in the
 * guard after the candidate buffer is written there. No counterpart on the pages.
 * Errors: EINVAL. */
PARISKV_API pariskv_status pariskv_debug_inject_bad_candidate(pariskv_index* index, int32_t head,
                                                               int64_t pos, int32_t value);

/* Test hook for the bounded device-side wait: the next pariskv_search's top-k arms the
 * barrier of its part's bulk copies for 16 bytes more than the copies deliver, so the barrier
 * never completes (the copies themselves do) and each CTA's wait runs out after about one
 * second; the kernel then records a timeout and finishes, and pariskv_sync returns
 * PARISKV_ETIMEOUT. The hook is consumed by that search. A search whose top-k stages no
 * copies (C > 65,536 candidates, or launch shape 4) refuses it with EINVAL. No counterpart on
 * the pages. Errors: EINVAL. */
PARISKV_API pariskv_status pariskv_debug_inject_wait_timeout(pariskv_index* index);

/* Forces the launch shapes of later searches on this index, for tests that require the same
 * bits from every shape: vote_ctas / rerank_ctas = the number of CTAs of the vote scan and of
 * the rerank (0: automatic; any positive count is valid, work is split over the CTAs), and
 * topk_mode = 1 one 1024-thread CTA per head (C <= 8192), 2 one 256-thread CTA per head
 * (C <= 8192), 3 a cluster of four 1024-thread CTAs holding the values in shared memory
 * (C <= 65536), 4 the same cluster reading them from global memory (any C), 0 automatic. A
 * search whose C does not fit the forced top-k shape fails with EINVAL. No counterpart on the
 * pages. Errors: EINVAL. */
PARISKV_API pariskv_status pariskv_debug_set_launch(pariskv_index* index, int32_t vote_ctas,
                                                    int32_t rerank_ctas, int32_t topk_mode);

/* K/V rows fetched by pariskv_sparse_attend's GQA-group union since the last call, on the
 * current device (synchronises the device, then resets the count). The row-gather attention
 * (K/V in pinned host memory, or fp32) with 1 < group <= 8 merges the group's top-k lists
 * into one union of rows per (sequence, KV head) and fetches each union row once for every
 * query head that selected it; this count is the number of rows it read, so the bytes that
 * crossed PCIe are rows x 2 x 128 x the element size. PARISKV_ATTEND_UNION=0 in the
 * environment turns the union off (each query head then fetches its own rows). A measurement
 * aid with no counterpart on the pages. Errors: EINVAL, ECUDA. */
PARISKV_API pariskv_status pariskv_debug_union_rows(int64_t* rows);

/* Guard bytes: when PARISKV_GUARD=1 is in the environment before the library's first index
 * allocation, every device buffer an index owns is allocated with 256 bytes of a fixed
 * pattern before and after it. This call synchronises the device and checks the guards of
 * every live buffer (buffers freed since the last call were checked when freed); ECUDA names
 * the first overrun seen, with the buffer's size and side. A stand-in for a memory checker,
 * with no counterpart on the pages. Errors: EINVAL (guards off), ECUDA. */
PARISKV_API pariskv_status pariskv_debug_check_guards(void);

/* Reads the 128-byte records of the last search's candidates once, for every query head (the
 * rerank's memory access: sorted random records of a 1 GiB-scale array, 16-byte loads, eight
 * lanes per record), with no arithmetic on them, on `stream`; `sink` (a device pointer to 4
 * bytes) may receive a fold of the data. Timed with CUDA events it measures the gather rate
 * that bounds the rerank, next to the copy rate of MEASURED peaks. No counterpart on the
 * pages (a measurement aid). Errors: EINVAL (no search yet), ECUDA. */
PARISKV_API pariskv_status pariskv_debug_gather_candidates(pariskv_index* index, uint32_t* sink,
                                                           void* stream);

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
