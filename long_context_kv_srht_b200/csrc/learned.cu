// learned.cu -- centroids learned from prefill keys: the comparator of the drift claim.
//
// "Technical Summary: ParisKV", Problem Statement 2 ("Decoding Drift"): centroids learned by
// clustering prefill keys go stale as decoding keys accumulate, and prior methods' recall
// collapses; Key Contributions 1: ParisKV's analytic centroids need no learning. This file
// learns such centroids so that the two can be compared on the same index: 256 unit-norm
// centroids per (sequence, KV head) and subspace, by spherical k-means (Lloyd iterations) on
// the prefill keys' rotated subspace directions. The index then assigns every key (prefill and
// appended) to the centroid of largest <y_b, mu_c> and every query ranks centroids by
// <q~_b, mu_c> (encode.cu, query.cu); nothing else changes.
//
// Training, per iteration: one warp per key rotates it (the same normalise + SRHT as the
// index), assigns each subspace (lane pairs scan half of the centroids each) and adds the
// subspace's unit direction to its centroid's running sum with atomics; then one thread per
// centroid replaces it by the normalised sum (a centroid that received no key keeps its
// value). The start is the direction of key floor(c n / 256) for centroid c. The atomic sums
// make the trained values depend on the order of additions in the last bits; the assignment
// given fixed centroids is exact and ordered (ties to the lower id).
#include "common.cuh"
#include "internal.hpp"
#include "pariskv_learned.h"
#include "rotate.cuh"

namespace pkv {

namespace {

constexpr int kLWarps = 8;
constexpr int64_t kCentFloats = static_cast<int64_t>(NB) * NC * 8;   // per unit

// This warp's key, rotated: lane pair (2b, 2b+1) ends with subspace b's 8 coordinates in w.
template <typename T>
__device__ __forceinline__ void rotated_subspace(const T* key, const float sg[4], int lane,
                                                 float w[8]) {
    float v[4];
    Elem<T>::load4(key + 4 * lane, v);
    normalize_rotate_warp(v, sg);
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __shfl_xor_sync(0xffffffffu, v[i], 1);
    const bool odd = lane & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w[i] = odd ? o[i] : v[i];
        w[4 + i] = odd ? v[i] : o[i];
    }
}

__device__ __forceinline__ void unit_dir(const float w[8], float u[8]) {
    float n2 = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) n2 = __fmaf_rn(w[j], w[j], n2);
    const float nr = __fsqrt_rn(n2);
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = nr > 0.0f ? __fdiv_rn(w[j], nr) : 0.0f;
}

// centroid c of every (unit, subspace) <- direction of key floor(c n / 256)
template <typename T>
__global__ void __launch_bounds__(kLWarps * 32)
kmeans_init_kernel(const T* __restrict__ keys, int64_t ld_tok, int64_t n,
                   const float* __restrict__ signs, float* __restrict__ cent) {
    const int lane = threadIdx.x & 31;
    const int c = blockIdx.x * kLWarps + (threadIdx.x >> 5);
    const int64_t unit = blockIdx.y;
    if (c >= NC) return;
    float sg[4], w[8], u[8];
    load_signs(signs, sg);
    const int64_t r = static_cast<int64_t>(c) * n / NC;
    rotated_subspace(keys + (unit * ld_tok + r) * D, sg, lane, w);
    unit_dir(w, u);
    if (!(lane & 1)) {
        float* dst = cent + ((unit * NB + (lane >> 1)) * NC + c) * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = u[j];
    }
}

// assignment + accumulation of unit directions into sums [unit][b][c][8]
template <typename T>
__global__ void __launch_bounds__(kLWarps * 32)
kmeans_assign_kernel(const T* __restrict__ keys, int64_t ld_tok, int64_t n,
                     const float* __restrict__ signs, const float* __restrict__ cent,
                     float* __restrict__ sums) {
    const int lane = threadIdx.x & 31;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * kLWarps + (threadIdx.x >> 5);
    const int64_t unit = blockIdx.y;
    if (r >= n) return;
    float sg[4], w[8], u[8];
    load_signs(signs, sg);
    rotated_subspace(keys + (unit * ld_tok + r) * D, sg, lane, w);
    const bool odd = lane & 1;
    const int b = lane >> 1;
    const float* cb = cent + (unit * NB + b) * NC * 8 + (odd ? 128 * 8 : 0);
    float best = -INFINITY;
    int arg = 0;
#pragma unroll 4
    for (int c = 0; c < 128; ++c) {
        float d = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) d = __fmaf_rn(cb[8 * c + j], w[j], d);
        if (d > best) { best = d; arg = c; }
    }
    arg += odd ? 128 : 0;
    const float ob = __shfl_xor_sync(0xffffffffu, best, 1);
    const int oa = __shfl_xor_sync(0xffffffffu, arg, 1);
    if (ob > best || (ob == best && oa < arg)) arg = oa;
    unit_dir(w, u);
    float* dst = sums + ((unit * NB + b) * NC + arg) * 8 + (odd ? 4 : 0);
#pragma unroll
    for (int j = 0; j < 4; ++j) atomicAdd(dst + j, u[(odd ? 4 : 0) + j]);
}

// centroid <- normalised sum (kept when the sum is zero); the sum is cleared
__global__ void __launch_bounds__(256)
kmeans_update_kernel(float* __restrict__ cent, float* __restrict__ sums, int64_t count) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= count) return;
    float* s = sums + i * 8;
    float n2 = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) n2 = __fmaf_rn(s[j], s[j], n2);
    const float nr = __fsqrt_rn(n2);
    if (nr > 0.0f) {
#pragma unroll
        for (int j = 0; j < 8; ++j) cent[i * 8 + j] = __fdiv_rn(s[j], nr);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j] = 0.0f;
}

template <typename T>
cudaError_t train(const pariskv_config* cfg, const float* signs, const void* keys,
                  int64_t ld_tok, int64_t n, int iters, float* cent, float* sums,
                  cudaStream_t st) {
    const int units = cfg->batch * cfg->num_kv_heads;
    const T* k = static_cast<const T*>(keys);
    kmeans_init_kernel<T><<<dim3(NC / kLWarps, units), kLWarps * 32, 0, st>>>(k, ld_tok, n,
                                                                               signs, cent);
    cudaError_t e = cudaGetLastError();
    const int64_t count = static_cast<int64_t>(units) * NB * NC;
    for (int it = 0; it < iters && e == cudaSuccess; ++it) {
        kmeans_assign_kernel<T><<<dim3(static_cast<unsigned>(ceil_div(n, kLWarps)), units),
                                  kLWarps * 32, 0, st>>>(k, ld_tok, n, signs, cent, sums);
        if ((e = cudaGetLastError()) != cudaSuccess) break;
        kmeans_update_kernel<<<static_cast<unsigned>(ceil_div(count, 256)), 256, 0, st>>>(
            cent, sums, count);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

}  // namespace pkv

using namespace pkv;

extern "C" {

pariskv_status pariskv_train_centroids(const pariskv_config* cfg, const int8_t* srht_signs,
                                       const void* keys, int64_t ld_tok, int64_t n,
                                       int32_t iters, float* centroids, void* stream) {
    if (!cfg) return fail(PARISKV_EINVAL, "config is NULL");
    pariskv_status s = validate_config(cfg);
    if (s != PARISKV_OK) return s;
    if (!srht_signs) return fail(PARISKV_EINVAL, "srht_signs is NULL");
    for (int j = 0; j < D; ++j)
        if (srht_signs[j] != 1 && srht_signs[j] != -1)
            return fail(PARISKV_EINVAL, "srht_signs[%d] = %d is not +-1", j, srht_signs[j]);
    if (n < 1 || ld_tok < n) return fail(PARISKV_EINVAL, "need 1 <= n <= ld_tok");
    if (iters < 0 || iters > 1000) return fail(PARISKV_EINVAL, "iters=%d not in [0, 1000]", iters);
    if ((s = check_device_pointer(keys, cfg->dtype == PARISKV_BF16 ? 8 : 16, "keys")) !=
        PARISKV_OK)
        return s;
    if ((s = check_device_pointer(centroids, 16, "centroids")) != PARISKV_OK) return s;
    const int units = cfg->batch * cfg->num_kv_heads;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* scratch = nullptr;   // signs (128) then sums [units][16][256][8]
    const size_t bytes = (D + static_cast<size_t>(units) * kCentFloats) * sizeof(float);
    if (alloc_fault_injected()) return fail(PARISKV_ENOMEM, "training scratch");
    cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&scratch), bytes, st);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(PARISKV_ENOMEM, "training scratch");
    }
    float hs[D];
    for (int j = 0; j < D; ++j) hs[j] = static_cast<float>(srht_signs[j]);
    e = cudaMemcpyAsync(scratch, hs, sizeof(hs), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(scratch + D, 0, bytes - D * sizeof(float), st);
    if (e == cudaSuccess)
        e = cfg->dtype == PARISKV_BF16
                ? train<__nv_bfloat16>(cfg, scratch, keys, ld_tok, n, iters, centroids,
                                       scratch + D, st)
                : train<float>(cfg, scratch, keys, ld_tok, n, iters, centroids, scratch + D, st);
    // hs lives on this stack frame: the copy must finish before returning
    const cudaError_t e2 = cudaStreamSynchronize(st);
    cudaFreeAsync(scratch, st);
    if (e == cudaSuccess) e = e2;
    set_last_launches(1 + 2 * iters);
    if (e != cudaSuccess) return cuda_fail(e, "centroid training");
    return PARISKV_OK;
}

}  // extern "C"
