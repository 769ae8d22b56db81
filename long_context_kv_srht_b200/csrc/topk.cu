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
//  - one bulk copy brings the head's S values into shared memory (up to kResident of them;
//    larger candidate sets are read from global memory on every pass), where they are turned
//    into u in place while the block finds min and max;
//  - range-adaptive radix levels: the current interval [lo, hi] is cut into at most 2048
//    power-of-two-wide bins, a shared histogram is built over the values in the interval, a
//    suffix scan finds the bin holding the k-th largest, and the interval shrinks to that
//    bin. Because the first interval is [min, max] of the data, one level usually settles
//    all but a few values; every level shrinks the interval 2048-fold, so at most three run;
//  - with T the k-th largest value and E the number of T-valued candidates to keep, a ballot
//    pass over warp-contiguous ranges writes every candidate above T and the first E equal to
//    T, in ascending key order (the candidates are stored in key order). est comes from the
//    value image itself; the candidate indices of eight tiles are fetched at once, so a warp
//    waits for global memory a few times rather than once per tile.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kT = 1024;
constexpr int kWarps = kT / 32;
constexpr int kBins = 2048;
constexpr int kResident = 53248;   // candidates kept in shared memory (208 KB)

__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// the inverse map (exact)
__device__ __forceinline__ float value_of(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

template <bool RES>
__global__ void __launch_bounds__(kT, 1)
topk_kernel(const float* __restrict__ S, const int32_t* __restrict__ cand,
            const float* __restrict__ qnorm, int32_t C, int64_t cmax, int32_t k,
            int32_t* __restrict__ out_idx, float* __restrict__ out_est, int* status) {
    extern __shared__ __align__(16) uint32_t keys[];
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t wa[kWarps], wb[kWarps], wsel0[kWarps], weq0[kWarps];
    __shared__ uint32_t pick[2];
    __shared__ __align__(8) uint64_t bar;

    const int head = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* Sh = S + head * cmax;
    const int32_t* ch = cand + head * cmax;
    auto key_at = [&](int i) -> uint32_t { return RES ? keys[i] : order_key(Sh[i]); };

    // 1. S -> shared memory in one bulk copy (16-byte granules; the array is padded)
    if (RES) {
        const uint32_t b = smem_addr(&bar);
        const uint32_t bytes = static_cast<uint32_t>(round_up(C, 4) * 4);
        if (threadIdx.x == 0) {
            mbar_init(b, 1);
            mbar_fence_init();
            mbar_arrive_expect_tx(b, bytes);
            bulk_g2s(smem_addr(keys), Sh, bytes, b);
        }
        __syncthreads();
        mbar_wait(b, 0, status);
    }
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (int i = threadIdx.x; i < C; i += kT) {
        const uint32_t u = RES ? order_key(__uint_as_float(keys[i])) : order_key(Sh[i]);
        if (RES) keys[i] = u;
        mn = min(mn, u);
        mx = max(mx, u);
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) { wa[warp] = mn; wb[warp] = mx; }
    __syncthreads();
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll 8
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
        if (RES) {
            const uint4* k4 = reinterpret_cast<const uint4*>(keys);
            const int C4 = C >> 2;
            for (int i = threadIdx.x; i < C4; i += kT) {
                const uint4 v = k4[i];
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (u[j] >= lo && u[j] <= hi) atomicAdd(&hist[(u[j] - lo) >> sh], 1u);
            }
            for (int i = (C4 << 2) + threadIdx.x; i < C; i += kT) {
                const uint32_t u = keys[i];
                if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
            }
        } else {
            for (int i = threadIdx.x; i < C; i += kT) {
                const uint32_t u = key_at(i);
                if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
            }
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
        if (lane == 0) wa[warp] = x;   // warp totals
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
        lo = nlo;
        const uint64_t bin_hi = static_cast<uint64_t>(nlo) + ((uint64_t{1} << sh) - 1u);
        hi = static_cast<uint32_t>(min(static_cast<uint64_t>(hi), bin_hi));
        __syncthreads();
    }
    const uint32_t T = lo;
    const uint32_t E = krem;   // ties at T to keep, in key order

    // 3. compaction over warp-contiguous ranges, ascending key order
    const int w0 = static_cast<int>(static_cast<int64_t>(C) * warp / kWarps);
    const int w1 = static_cast<int>(static_cast<int64_t>(C) * (warp + 1) / kWarps);
    uint32_t ngt = 0, neq = 0;
    for (int pbase = w0; pbase < w1; pbase += 32) {
        const int pp = pbase + lane;
        const bool valid = pp < w1;
        const uint32_t u = valid ? key_at(pp) : 0u;
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
    // the candidate indices of kBatch tiles are loaded together, so their latencies overlap
    constexpr int kBatch = 8;
    for (int pb = w0; pb < w1; pb += 32 * kBatch) {
        int32_t ci[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int pp = pb + 32 * b + lane;
            ci[b] = pp < w1 ? ch[pp] : 0;
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int pp = pb + 32 * b + lane;
            const bool valid = pp < w1;
            const uint32_t u = valid ? key_at(pp) : 0u;
            const uint32_t eqm = __ballot_sync(0xffffffffu, valid && u == T);
            const bool take = valid && u == T && (eq_run + __popc(eqm & lt)) < E;
            const bool sel = (valid && u > T) || take;
            const uint32_t selm = __ballot_sync(0xffffffffu, sel);
            if (sel) {
                const uint32_t r = sel_run + __popc(selm & lt);
                if (r < static_cast<uint32_t>(k)) {
                    const int64_t pos = static_cast<int64_t>(head) * k + r;
                    out_idx[pos] = ci[b];
                    if (out_est) out_est[pos] = __fmul_rn(qn, value_of(u));
                } else {
                    atomicExch(status, ST_BADINDEX);
                }
            }
            sel_run += __popc(selm);
            eq_run += __popc(eqm);
        }
    }
}

}  // namespace

cudaError_t launch_topk(const pariskv_index* ix, int64_t C, int32_t k, int32_t* topk_idx,
                        float* topk_est, cudaStream_t st) {
    static std::atomic<uint64_t> smem_raised{0};
    if (cudaError_t e = raise_smem_limit(topk_kernel<true>, kResident * 4, smem_raised);
        e != cudaSuccess)
        return e;
    const int heads = ix->units * ix->cfg.group;
    if (C <= kResident) {
        const size_t smem = static_cast<size_t>(round_up(C, 4)) * 4;
        topk_kernel<true><<<heads, kT, smem, st>>>(ix->S, ix->cand, ix->qnorm,
                                                   static_cast<int32_t>(C), ix->cmax, k,
                                                   topk_idx, topk_est, ix->status);
    } else {
        topk_kernel<false><<<heads, kT, 0, st>>>(ix->S, ix->cand, ix->qnorm,
                                                 static_cast<int32_t>(C), ix->cmax, k, topk_idx,
                                                 topk_est, ix->status);
    }
    return cudaGetLastError();
}

}  // namespace pkv
