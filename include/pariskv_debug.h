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

/* Timing of pariskv_search with CUDA events recorded on the search stream around its kernel,
 * and the phase trace read by pariskv_debug_search_phases. enable != 0 turns both on for this
 * index (events and the trace buffer are created then). */
PARISKV_API pariskv_status pariskv_debug_profile(pariskv_index* index, int32_t enable);

/* Waits for the last profiled search and writes the device time (ms) of each of its
 * launches to ms[0..*nstages-1]; the search is one kernel, so *nstages is 1. ms must hold at
 * least 8 floats. */
PARISKV_API pariskv_status pariskv_debug_stage_ms(pariskv_index* index, float* ms,
                                                  int32_t* nstages);

/* Bounds every device-side wait of later searches on this index to `cycles` SM clock cycles
 * (0 restores the default of about one second). A wait that runs out makes pariskv_sync
 * return PARISKV_ETIMEOUT, naming the control word it waited on. Used by tests of the
 * timeout path. No counterpart on the pages. Errors: EINVAL. */
PARISKV_API pariskv_status pariskv_debug_set_wait_limit(pariskv_index* index, int64_t cycles);

/* Makes later searches on this index report, per CTA of the search kernel, the item it is
 * working on into `board` (8 int32 per CTA: item number, kind, head or pack-unit, state 1 =
 * claimed, -1 = its wait expired, 2 = done, 3 = exited; then the last checkpoint passed by
 * threads 1, 32, 224 and 0 as 100 x loop iteration + checkpoint), a pinned host buffer the
 * host may read while the kernel runs; NULL turns it off. The board must hold 8 ints for
 * each of 2 x (number of SMs) CTAs. A debugging aid with no counterpart on the pages. Errors: EINVAL. */
PARISKV_API pariskv_status pariskv_debug_set_progress(pariskv_index* index, int32_t* board);

/* Phases of the last profiled search (pariskv_debug_profile on): the search runs as one
 * persistent kernel whose workers take items of several kinds; for each kind -- 0 query
 * prep, 1 vote, 2 compaction, 3 top-k, 4 threshold finalisation, 5 rerank, 6 vote-group
 * waits, 7 rerank-warp waits, 8 whole kernel -- out[3 i] and out[3 i + 1] receive the first
 * start and the last end (microseconds after the kernel's first CTA started; -1 if that
 * kind never ran) and out[3 i + 2] the busy time summed over workers; out[29] receives the
 * number of polls the bounded waits made; out[30], out[31], out[32] and out[35] the top-k
 * items' passes over the rerank values, their selections finished without the in-memory
 * list, and their summed selection and writing times (us). out holds 36 doubles.
 * Synchronises with the search. No counterpart on the pages (a measurement aid). */
PARISKV_API pariskv_status pariskv_debug_search_phases(pariskv_index* index, double* out);

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
