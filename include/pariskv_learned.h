/* pariskv_learned.h -- coarse centroids learned from prefill keys: the comparator of the
 * drift claim.
 *
 * "Technical Summary: ParisKV", Problem Statement 2 ("Decoding Drift"): centroids learned by
 * clustering prefill keys go stale as decoding keys accumulate, and prior methods' recall
 * collapses; Key Contributions 1: the analytic centroids of ParisKV need no learning. These
 * calls let the same index run with learned centroids instead, everything else unchanged, so
 * that the two can be compared under drift:
 *   - per (sequence, KV head) and subspace, 256 unit-norm centroids mu_c in R^8;
 *   - a key's bucket id is argmax_c <y_b, mu_c> (y_b the subspace of the normalised, rotated
 *     key; fp32 FMA chain over the 8 dims; ties to the lower c);
 *   - a query's top-rho centroids are the rho largest <q~_b, mu_c> (same chain; ties to the
 *     lower c), with the usual tiered vote weights.
 * Centroid layout: float [batch][num_kv_heads][16][256][8], 16-byte aligned. */
#ifndef PARISKV_LEARNED_H_
#define PARISKV_LEARNED_H_

#include "pariskv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Spherical k-means on the rotated directions of the first n keys of every (sequence, KV
 * head) (keys as in pariskv_build_index): centroid c starts as the direction of key
 * floor(c n / 256); each of `iters` iterations assigns every key as above and replaces each
 * centroid by the normalised sum of its keys' unit directions (kept when it has none). The
 * sums are accumulated with atomics, so trained values may differ between runs in the last
 * bits. centroids: device pointer (output). Synchronises `stream` before returning.
 * Errors: EINVAL (config, signs, n, iters outside [0, 1000], pointers), ENOMEM, ECUDA. */
PARISKV_API pariskv_status pariskv_train_centroids(const pariskv_config* cfg,
                                                   const int8_t* srht_signs, const void* keys,
                                                   int64_t ld_tok, int64_t n, int32_t iters,
                                                   float* centroids, void* stream);

/* Switches an empty index (size 0, e.g. built with n = 0) to learned centroids: every key
 * appended afterwards is assigned to them, every search ranks them. The table is copied
 * (device or pinned host source). Indexes with learned centroids have no image
 * (pariskv_export returns EINVAL). Errors: EINVAL (index not empty, pointer), ENOMEM, ECUDA. */
PARISKV_API pariskv_status pariskv_set_centroids(pariskv_index* index, const float* centroids,
                                                 void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PARISKV_LEARNED_H_ */
