// topk.cu -- final top-k of the reranked candidates.
//
// "Technical Summary: ParisKV", Problem Statement (attention over a Top-k subset of past
// tokens) and Key Contributions 2 (Top-k selection directly on compressed codes); "ParisKV:
// Fast and Drift-Robust KV-Cache Retrieval for Long-Context LLMs" (on-demand top-k fetch).
// The k candidates with the largest rerank value S are kept, ties going to the lower key
// index, and returned in ascending key order with est = ||q|| * S.
//
// Exact selection on the order-preserving 32-bit image u of S (flip all bits of negative
// values, set the sign bit of the others), by a cluster of four CTAs per query head:
//  - CTA r copies the r-th quarter of the head's S values and candidate indices into shared
//    memory with asynchronous copies, all in flight at once, and turns S into u in place
//    (quarters longer than kSlice stay in global memory and are re-read on every pass);
//  - the first radix level, the top 11 bits of u, was counted by the rerank as it wrote S
//    (per head, SCOPIES copies of a 2048-bin histogram in global memory), so it costs one
//    round of reads here;
//  - then range-adaptive radix levels: the current interval [lo, hi] is cut into at most 2048
//    power-of-two-wide bins, every CTA histograms its quarter, and every CTA sums the four
//    histograms bin by bin over DSMEM and runs the same suffix scan, so all four pick the
//    same bin (the one holding the k-th largest) without further exchange. Histograms
//    alternate between two buffers, so one cluster barrier per level suffices; the 21 bits
//    left after the first level take at most two more levels;
//  - with T the k-th largest value and E the number of T-valued candidates to keep, each
//    thread counts a contiguous run of values, the counts are scanned over the CTA and the
//    cluster, and each thread then writes its run's values above T and its ties at T while
//    fewer than E ties precede them, in ascending key order (the candidates are stored in
//    key order); est comes from u itself.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace cg = cooperative_groups;

namespace {

constexpr int kCL = 4;             // CTAs per query head
constexpr int kT = 1024;
constexpr int kWarps = kT / 32;
constexpr int kBins = 2048;
constexpr int kSlice = 16384;      // values per CTA kept in shared memory (u and index)

template <bool RES>
__global__ void __cluster_dims__(kCL, 1, 1) __launch_bounds__(kT, 1)
topk_kernel(const float* __restrict__ S, const int32_t* __restrict__ cand,
            const float* __restrict__ qnorm, const uint32_t* __restrict__ shist, int32_t C,
            int64_t cmax, int32_t k, int32_t* __restrict__ out_idx, float* __restrict__ out_est,
            int* status) {
    extern __shared__ __align__(16) uint32_t dyn[];
    __shared__ uint32_t hist[2][kBins];
    __shared__ uint32_t wa[kWarps], wb[kWarps];
    __shared__ uint32_t ctot[2];       // this CTA's candidates above T / ties at T
    __shared__ uint32_t pick[2];

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int head = blockIdx.x / kCL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int s0 = static_cast<int>(static_cast<int64_t>(C) * rank / kCL);
    const int s1 = static_cast<int>(static_cast<int64_t>(C) * (rank + 1) / kCL);
    const int L = s1 - s0;
    const float* Sh = S + head * cmax + s0;
    const int32_t* ch = cand + head * cmax + s0;
    uint32_t* keys = dyn;                                   // [kSlice] u
    int32_t* idx = reinterpret_cast<int32_t*>(dyn + kSlice);  // [kSlice] candidate index
    auto key_at = [&](int i) -> uint32_t { return RES ? keys[i] : order_key(Sh[i]); };
    auto idx_at = [&](int i) -> int32_t { return RES ? idx[i] : ch[i]; };
    pdl_wait();
    pdl_launch_dependents();

    // 1. the quarter into shared memory (asynchronous 4-byte copies, all in flight at once);
    //    then u in place and the local min / max
    if (RES) {
        for (int i = threadIdx.x; i < L; i += kT) {
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(keys + i)),
                         "l"(Sh + i) : "memory");
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(idx + i)),
                         "l"(ch + i) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_all;" ::: "memory");
    }
    if (RES)
        for (int i = threadIdx.x; i < L; i += kT)   // each thread converts what it copied
            keys[i] = order_key(__uint_as_float(keys[i]));

    // 2. radix levels. The first (the top SBINS_BITS bits of u) was counted by the rerank;
    //    the following ones are range-adaptive histograms over the cluster. choose() finds,
    //    from each thread's two bins (2t, 2t + 1), the bin holding the krem-th largest value
    //    and narrows [lo, hi] to it; every CTA of the cluster sees the same counts and so
    //    makes the same choice.
    uint32_t krem = static_cast<uint32_t>(k);
    uint32_t lo = 0u, hi = 0xffffffffu;
    auto choose = [&](uint32_t h0, uint32_t h1, int sh) {
        uint32_t x = h0 + h1;   // suffix counts over the bins
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += y;
        }
        if (lane == 0) wa[warp] = x;   // warp totals
        __syncthreads();
        if (warp == 0) {               // exclusive suffix sums of the warp totals
            const uint32_t t = wa[lane];
            uint32_t y = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t z = __shfl_down_sync(0xffffffffu, y, o);
                if (lane + o < 32) y += z;
            }
            wb[lane] = y - t;
        }
        __syncthreads();
        const uint32_t later = wb[warp];                // bins of later warps
        const uint32_t above1 = later + x - (h0 + h1);  // strictly above bin 2t + 1
        const uint32_t above0 = above1 + h1;             // strictly above bin 2t
        if (above1 < krem && krem <= above1 + h1) { pick[0] = 2 * threadIdx.x + 1; pick[1] = above1; }
        if (above0 < krem && krem <= above0 + h0) { pick[0] = 2 * threadIdx.x; pick[1] = above0; }
        __syncthreads();
        const uint32_t b = pick[0];
        krem -= pick[1];
        const uint32_t nlo = lo + (b << sh);
        const uint64_t bin_hi = static_cast<uint64_t>(nlo) + ((uint64_t{1} << sh) - 1u);
        lo = nlo;
        hi = static_cast<uint32_t>(min(static_cast<uint64_t>(hi), bin_hi));
        __syncthreads();   // pick[], wa[] and wb[] are rewritten by the next level
    };
    static_assert(SBINS == kBins, "the first level has one bin pair per thread");
    {
        uint2 v[SCOPIES];
        const uint2* hs = reinterpret_cast<const uint2*>(shist + static_cast<int64_t>(head) * SCOPIES * SBINS);
#pragma unroll
        for (int r = 0; r < SCOPIES; ++r) v[r] = hs[r * (SBINS / 2) + threadIdx.x];
        uint32_t h0 = 0, h1 = 0;
#pragma unroll
        for (int r = 0; r < SCOPIES; ++r) { h0 += v[r].x; h1 += v[r].y; }
        choose(h0, h1, 32 - SBINS_BITS);
    }
    int level = 0;
    while (lo != hi) {
        uint32_t* hb = hist[level & 1];
        const uint32_t span = hi - lo;
        const int bitlen = 32 - __clz(span);
        const int sh = bitlen > 11 ? bitlen - 11 : 0;   // (span >> sh) < 2048
        hb[threadIdx.x] = 0u;
        hb[threadIdx.x + kT] = 0u;
        __syncthreads();
        if (RES && (L & 3) == 0) {
            const uint4* k4 = reinterpret_cast<const uint4*>(keys);
            for (int i = threadIdx.x; i < (L >> 2); i += kT) {
                const uint4 v = k4[i];
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (u[j] >= lo && u[j] <= hi) atomicAdd(&hb[(u[j] - lo) >> sh], 1u);
            }
        } else {
            for (int i = threadIdx.x; i < L; i += kT) {
                const uint32_t u = key_at(i);
                if (u >= lo && u <= hi) atomicAdd(&hb[(u - lo) >> sh], 1u);
            }
        }
        cluster.sync();   // every quarter's histogram is complete
        // thread t sums bins 2t, 2t + 1 over the cluster
        uint32_t h0 = 0, h1 = 0;
#pragma unroll
        for (int q = 0; q < kCL; ++q) {
            const uint2 v = *reinterpret_cast<const uint2*>(cluster.map_shared_rank(hb, q) +
                                                             2 * threadIdx.x);
            h0 += v.x;
            h1 += v.y;
        }
        choose(h0, h1, sh);
        ++level;
    }
    const uint32_t T = lo;
    const uint32_t E = krem;   // ties at T to keep, in key order

    // 3. counts per thread-contiguous run, then offsets over the CTA (block scan) and over
    //    the cluster
    const int a = static_cast<int>(static_cast<int64_t>(L) * threadIdx.x / kT);
    const int b = static_cast<int>(static_cast<int64_t>(L) * (threadIdx.x + 1) / kT);
    uint32_t ngt = 0, neq = 0;
    for (int i = a; i < b; ++i) {
        const uint32_t u = key_at(i);
        ngt += u > T;
        neq += u == T;
    }
    // inclusive warp scans of (gt, eq), then warp totals
    uint32_t xg = ngt, xe = neq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t yg = __shfl_up_sync(0xffffffffu, xg, o);
        const uint32_t ye = __shfl_up_sync(0xffffffffu, xe, o);
        if (lane >= o) { xg += yg; xe += ye; }
    }
    if (lane == 31) { wa[warp] = xg; wb[warp] = xe; }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t g = 0, e = 0;
        for (int w = 0; w < kWarps; ++w) { g += wa[w]; e += wb[w]; }
        ctot[0] = g;
        ctot[1] = e;
    }
    cluster.sync();
    uint32_t gt_run = xg - ngt, eq_run = xe - neq;   // above T / ties before this thread
    for (int q = 0; q < rank; ++q) {
        const uint32_t* r = cluster.map_shared_rank(ctot, q);
        gt_run += r[0];
        eq_run += r[1];
    }
    for (int w = 0; w < warp; ++w) { gt_run += wa[w]; eq_run += wb[w]; }
    cluster.barrier_arrive();          // no remote read of this CTA's memory follows

    // 4. this thread's winners in key order: every value above T, and the ties at T while
    //    fewer than E ties precede them
    const float qn = qnorm[head];
    uint32_t pos = gt_run + min(eq_run, E);
    if (pos + ngt + (E > eq_run ? min(E - eq_run, neq) : 0u) > static_cast<uint32_t>(k)) {
        atomicExch(status, ST_BADINDEX);   // never taken when the counts are consistent
    } else {
        int32_t* oi = out_idx + static_cast<int64_t>(head) * k;
        float* oe = out_est ? out_est + static_cast<int64_t>(head) * k : nullptr;
        for (int i = a; i < b; ++i) {
            const uint32_t u = key_at(i);
            bool take = u > T;
            if (u == T) take = eq_run++ < E;
            if (take) {
                oi[pos] = idx_at(i);
                if (oe) oe[pos] = __fmul_rn(qn, value_of(u));
                ++pos;
            }
        }
    }
    cluster.barrier_wait();
}

}  // namespace

cudaError_t launch_topk(const pariskv_index* ix, int64_t C, int32_t k, int32_t* topk_idx,
                        float* topk_est, cudaStream_t st) {
    constexpr int kDyn = 2 * kSlice * 4;
    static std::atomic<uint64_t> smem_raised{0};
    if (cudaError_t e = raise_smem_limit(topk_kernel<true>, kDyn, smem_raised); e != cudaSuccess)
        return e;
    const int heads = ix->units * ix->cfg.group;
    if (ceil_div(C, kCL) <= kSlice) {
        return launch_pdl(topk_kernel<true>, heads * kCL, kT, kDyn, st, ix->S, ix->cand,
                          ix->qnorm, ix->shist, static_cast<int32_t>(C), ix->cmax, k, topk_idx,
                          topk_est, ix->status);
    } else {
        return launch_pdl(topk_kernel<false>, heads * kCL, kT, 0, st, ix->S, ix->cand,
                          ix->qnorm, ix->shist, static_cast<int32_t>(C), ix->cmax, k, topk_idx,
                          topk_est, ix->status);
    }
}

}  // namespace pkv
