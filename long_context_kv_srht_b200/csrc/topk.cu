// topk.cu -- final top-k of the reranked candidates.
//
// "Technical Summary: ParisKV", Problem Statement (attention over a Top-k subset of past
// tokens) and Key Contributions 2 (Top-k selection directly on compressed codes); "ParisKV:
// Fast and Drift-Robust KV-Cache Retrieval for Long-Context LLMs" (on-demand top-k fetch).
// The k candidates with the largest rerank value S are kept, ties going to the lower key
// index, and returned in ascending key order with est = ||q|| * S.
//
// Exact selection on the order-preserving 32-bit image u of S (flip all bits of negative
// values, set the sign bit of the others), one 1024-thread CTA per query head:
//  - the head's candidates are read once into shared memory (up to 53248 of them; larger
//    sets are re-read from global memory on every pass) while the block finds min and max u;
//  - range-adaptive radix levels: the current interval [lo, hi] is cut into at most 2048
//    power-of-two-wide bins, a shared histogram is built over the values in the interval,
//    a suffix scan finds the bin holding the k-th largest, and the interval shrinks to that
//    bin. Because the first interval is [min, max] of the data, one level usually settles
//    all but a few values; every level shrinks the interval 2048-fold, so at most three run;
//  - when the interval is a single value T, E = the remaining rank is the number of T-valued
//    candidates to keep (in key order); a ballot pass per warp-contiguous range compacts
//    every candidate above T and the first E equal to T, in ascending key order.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kT = 1024;
constexpr int kWarps = kT / 32;
constexpr int kBins = 2048;
constexpr int64_t kResident = 53248;   // candidates kept in shared memory (208 KB)

__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kT, 1)
topk_kernel(const float* __restrict__ S, const int32_t* __restrict__ cand,
            const float* __restrict__ qnorm, int64_t C, int64_t cmax, int32_t k,
            int32_t* __restrict__ out_idx, float* __restrict__ out_est, int* status) {
    extern __shared__ uint32_t keys[];
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t wa[kWarps], wb[kWarps];
    __shared__ uint32_t wsel0[kWarps], weq0[kWarps];
    __shared__ uint32_t pick[2];

    const int head = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* Sh = S + head * cmax;
    const int32_t* ch = cand + head * cmax;
    const bool res = C <= kResident;

    // 1. load (and keep) the keys; min and max of the head's values
    uint32_t mn = 0xffffffffu, mx = 0u;
    {
        constexpr int U = 8;
        for (int64_t base = 0; base < C; base += static_cast<int64_t>(kT) * U) {
            uint32_t u[U];
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int64_t i = base + j * kT + threadIdx.x;
                u[j] = i < C ? order_key(Sh[i]) : 0u;
            }
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int64_t i = base + j * kT + threadIdx.x;
                if (i < C) {
                    if (res) keys[i] = u[j];
                    mn = min(mn, u[j]);
                    mx = max(mx, u[j]);
                }
            }
        }
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) { wa[warp] = mn; wb[warp] = mx; }
    __syncthreads();
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll 4
    for (int w = 0; w < kWarps; ++w) { lo = min(lo, wa[w]); hi = max(hi, wb[w]); }
    __syncthreads();

    // 2. range-adaptive radix levels
    uint32_t krem = static_cast<uint32_t>(k);
    while (lo != hi) {
        const uint32_t span = hi - lo;
        const int bitlen = 32 - __clz(span);
        const int sh = bitlen > 11 ? bitlen - 11 : 0;   // (span >> sh) < 2048
        hist[threadIdx.x] = 0u;
        hist[threadIdx.x + kT] = 0u;
        __syncthreads();
        for (int64_t i = threadIdx.x; i < C; i += kT) {
            const uint32_t u = res ? keys[i] : order_key(Sh[i]);
            if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
        }
        __syncthreads();
        // suffix counts: thread t owns bins 2t, 2t + 1
        const uint32_t h0 = hist[2 * threadIdx.x], h1 = hist[2 * threadIdx.x + 1];
        uint32_t x = h0 + h1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += y;
        }
        if (lane == 0) wa[warp] = x;   // warp total
        __syncthreads();
        uint32_t later = 0;            // bins of later warps
        for (int w = warp + 1; w < kWarps; ++w) later += wa[w];
        const uint32_t above1 = later + x - (h0 + h1);  // strictly above bin 2t + 1
        const uint32_t above0 = above1 + h1;             // strictly above bin 2t
        if (above1 < krem && krem <= above1 + h1) { pick[0] = 2 * threadIdx.x + 1; pick[1] = above1; }
        if (above0 < krem && krem <= above0 + h0) { pick[0] = 2 * threadIdx.x; pick[1] = above0; }
        __syncthreads();
        const uint32_t b = pick[0];
        krem -= pick[1];
        const uint32_t nlo = lo + (b << sh);
        const uint32_t nhi = nlo + ((1u << sh) - 1u);
        lo = nlo;
        hi = min(hi, nhi);
        __syncthreads();
    }
    const uint32_t T = lo;
    const uint32_t E = krem;   // ties at T to keep, in key order

    // 3. compaction over warp-contiguous ranges, ascending key order
    const int64_t w0 = C * warp / kWarps, w1 = C * (warp + 1) / kWarps;
    uint32_t ngt = 0, neq = 0;
    for (int64_t pbase = w0; pbase < w1; pbase += 32) {
        const int64_t pp = pbase + lane;
        const bool valid = pp < w1;
        const uint32_t u = valid ? (res ? keys[pp] : order_key(Sh[pp])) : 0u;
        ngt += __popc(__ballot_sync(0xffffffffu, valid && u > T));
        neq += __popc(__ballot_sync(0xffffffffu, valid && u == T));
    }
    if (lane == 0) { wa[warp] = ngt; wb[warp] = neq; }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t sel = 0, eqb = 0;
        for (int w = 0; w < kWarps; ++w) {
            wsel0[w] = sel;
            weq0[w] = eqb;
            sel += wa[w] + (eqb >= E ? 0u : min(E - eqb, wb[w]));
            eqb += wb[w];
        }
    }
    __syncthreads();
    uint32_t sel_run = wsel0[warp], eq_run = weq0[warp];
    const float qn = qnorm[head];
    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t pbase = w0; pbase < w1; pbase += 32) {
        const int64_t pp = pbase + lane;
        const bool valid = pp < w1;
        const uint32_t u = valid ? (res ? keys[pp] : order_key(Sh[pp])) : 0u;
        const uint32_t eqm = __ballot_sync(0xffffffffu, valid && u == T);
        const bool take = valid && u == T && (eq_run + __popc(eqm & lt)) < E;
        const bool sel = (valid && u > T) || take;
        const uint32_t selm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const uint32_t r = sel_run + __popc(selm & lt);
            if (r < static_cast<uint32_t>(k)) {
                const int64_t pos = static_cast<int64_t>(head) * k + r;
                out_idx[pos] = ch[pp];
                if (out_est) out_est[pos] = __fmul_rn(qn, Sh[pp]);
            } else {
                atomicExch(status, ST_BADINDEX);
            }
        }
        sel_run += __popc(selm);
        eq_run += __popc(eqm);
    }
}

}  // namespace

cudaError_t launch_topk(const pariskv_index* ix, int64_t C, int32_t k, int32_t* topk_idx,
                        float* topk_est, cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kResident * 4));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int heads = ix->units * ix->cfg.group;
    const size_t smem = static_cast<size_t>(min64(C, kResident)) * 4;
    topk_kernel<<<heads, kT, smem, st>>>(ix->S, ix->cand, ix->qnorm, C, ix->cmax, k, topk_idx,
                                         topk_est, ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
