// topk.cu -- final top-k of the reranked candidates.
//
// "Technical Summary: ParisKV", Problem Statement (attention over a Top-k subset of past
// tokens) and Key Contributions 2 (Top-k selection directly on compressed codes); "ParisKV:
// Fast and Drift-Robust KV-Cache Retrieval for Long-Context LLMs" (on-demand top-k fetch).
// The k candidates with the largest rerank value S are kept, ties going to the lower key
// index, and returned in ascending key order with est = ||q|| * S.
//
// Exact selection on the order-preserving 32-bit image u of S (flip all bits of negative
// values, set the sign bit of the others). A head's candidates are split over CL CTAs: one
// CTA when they fit its shared memory (up to 8192) -- 1024 threads when there are no more
// heads than SMs, else 256 threads (with a 4096-value slice when it suffices, so four CTAs
// share an SM and even many heads run in about one wave) -- and otherwise a cluster of four
// 1024-thread CTAs:
//  - CTA r copies the r-th part of the head's S values and candidate indices into shared
//    memory with two bulk asynchronous copies (each a contiguous range, from the 16-byte
//    boundary at or below the part's start) completing on one mbarrier, and turns S into u
//    in place (parts longer than the slice stay in global memory and are re-read on every
//    pass);
//  - the first radix level, the top 11 bits of u, was counted by the rerank as it wrote S
//    (per head, SCOPIES copies of a 2048-bin histogram in global memory), so it costs one
//    round of reads here;
//  - then range-adaptive radix levels: the current interval [lo, hi] is cut into at most 2048
//    power-of-two-wide bins, every CTA histograms its part, and every CTA sums the CL
//    histograms bin by bin (over DSMEM in a cluster) and runs the same suffix scan, so all
//    pick the same bin (the one holding the k-th largest) without further exchange.
//    Histograms alternate between two buffers, so one barrier per level suffices; the 21
//    bits left after the first level take at most two more levels;
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

constexpr int kBins = 2048;
// limit of the wait for the part's bulk copies: far above any copy's latency (microseconds),
// short enough that a lost completion costs the caller about a second, not a hang
constexpr uint64_t kCopyWaitNs = 1000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

template <int CL, int T, int SLICE, bool RES>
__global__ void __launch_bounds__(T, 1)
topk_kernel(const float* __restrict__ S, const int32_t* __restrict__ cand,
            const float* __restrict__ qnorm, const uint32_t* __restrict__ shist, int32_t C,
            int64_t cmax, int32_t k, int32_t* __restrict__ out_idx, float* __restrict__ out_est,
            int* status, uint32_t extra_tx) {
    constexpr int kWarps = T / 32;
    constexpr int BPT = kBins / T;     // bins per thread: thread t owns bins BPT t .. BPT t + BPT - 1
    static_assert(kWarps <= 32 && kBins % T == 0 && (BPT == 2 || BPT == 8), "layout");
    extern __shared__ __align__(16) uint32_t dyn[];
    __shared__ __align__(16) uint32_t hist[2][kBins];
    __shared__ __align__(8) uint64_t lbar;   // completion of the part's bulk copies
    __shared__ uint32_t wa[2][kWarps], wb[kWarps];   // wa: per-level warp totals (two sets)
    __shared__ uint32_t ctot[2];       // this CTA's candidates above T / ties at T
    __shared__ uint32_t pick[2][2];    // per level (two sets): chosen bin, count above it

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = CL > 1 ? static_cast<int>(cluster.block_rank()) : 0;
    const int head = blockIdx.x / CL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int s0 = static_cast<int>(static_cast<int64_t>(C) * rank / CL);
    const int s1 = static_cast<int>(static_cast<int64_t>(C) * (rank + 1) / CL);
    const int L = s1 - s0;
    const float* Sh = S + head * cmax + s0;
    const int32_t* ch = cand + head * cmax + s0;
    // the part is copied from a 16-byte boundary (rows start on one: cmax is a multiple of
    // 32), so it sits `off` = s0 mod 4 words into each buffer
    const int off = RES ? (s0 & 3) : 0;
    uint32_t* keys = dyn + off;                                    // [SLICE] u
    // (a copied range is at most L + 6 words long: buffers of SLICE + 8 words)
    int32_t* idx = reinterpret_cast<int32_t*>(dyn + SLICE + 8) + off;   // [SLICE] candidate index
    auto key_at = [&](int i) -> uint32_t { return RES ? keys[i] : order_key(Sh[i]); };
    auto idx_at = [&](int i) -> int32_t { return RES ? idx[i] : ch[i]; };
    auto sync_all = [&]() {
        if constexpr (CL > 1) cluster.sync();
        else __syncthreads();
    };
    // this thread's BPT bins of a histogram buffer (uint2 / uint4 loads)
    auto load_bins = [&](const uint32_t* hb, uint32_t h[BPT]) {
        if constexpr (BPT == 2) {
            const uint2 v = reinterpret_cast<const uint2*>(hb)[threadIdx.x];
            h[0] = v.x; h[1] = v.y;
        } else {
            const uint4 v = reinterpret_cast<const uint4*>(hb)[2 * threadIdx.x];
            const uint4 w = reinterpret_cast<const uint4*>(hb)[2 * threadIdx.x + 1];
            h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
            h[4] = w.x; h[5] = w.y; h[6] = w.z; h[7] = w.w;
        }
    };
    pdl_wait();
    pdl_launch_dependents();

    // 1. this CTA's part into shared memory: two bulk asynchronous copies (values and
    //    indices, from the 16-byte boundary at or below s0 to the one at or above s1, which
    //    stays inside the row) completing on one mbarrier; then u in place
    if (RES) {
        const uint32_t bar = smem_addr(&lbar);
        const int a0 = s0 & ~3, a1 = (s1 + 3) & ~3;
        const uint32_t bytes = static_cast<uint32_t>(a1 - a0) * 4u;
        if (threadIdx.x == 0) {
            mbar_init(bar, 1);
            mbar_fence_init();
        }
        __syncthreads();
        if (threadIdx.x == 0 && bytes) {
            // (extra_tx, normally 0, is a test hook: bytes no copy delivers, so the barrier
            // never completes and the wait below runs out)
            mbar_arrive_expect_tx(bar, 2 * bytes + extra_tx);
            bulk_g2s(smem_addr(dyn), S + head * cmax + a0, bytes, bar);
            bulk_g2s(smem_addr(dyn + SLICE + 8), cand + head * cmax + a0, bytes, bar);
        }
        if (bytes) {
            // bounded: past kCopyWaitNs of polling the part is treated as lost and the status
            // word records a timeout (never taken while the copies complete)
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bar, 0u)) {
                if (globaltimer_ns() - t0 > kCopyWaitNs) {
                    atomicExch(status, ST_TIMEOUT);
                    break;
                }
            }
        }
        for (int i = threadIdx.x; i < L; i += T)   // each thread converts a strided share
            keys[i] = order_key(__uint_as_float(keys[i]));
    }

    // 2. radix levels. The first (the top SBINS_BITS bits of u) was counted by the rerank;
    //    the following ones are range-adaptive histograms over the head's CTAs. choose()
    //    finds, from each thread's bins, the bin holding the krem-th largest value and
    //    narrows [lo, hi] to it; every CTA sees the same counts and makes the same choice.
    uint32_t krem = static_cast<uint32_t>(k);
    uint32_t lo = 0u, hi = 0xffffffffu;
    // The shared words a level writes (warp totals, the pick) come in two sets used by
    // alternate levels, so no barrier is needed between one level's last read and the next
    // level's first write (the next level's own barriers come first).
    int par = 0;
    auto choose = [&](const uint32_t h[BPT], int sh) {
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < BPT; ++j) mine += h[j];
        uint32_t x = mine;             // suffix counts over the threads' bin ranges
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += y;
        }
        if (lane == 0) wa[par][warp] = x;   // warp totals
        __syncthreads();
        // the warps after this one, summed by every warp for itself
        uint32_t aw = lane < kWarps && lane > warp ? wa[par][lane] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) aw += __shfl_xor_sync(0xffffffffu, aw, o);
        uint32_t above = aw + x - mine;   // strictly above this thread's bins
#pragma unroll
        for (int j = BPT - 1; j >= 0; --j) {
            if (above < krem && krem <= above + h[j]) {
                pick[par][0] = BPT * threadIdx.x + j;
                pick[par][1] = above;
            }
            above += h[j];
        }
        __syncthreads();
        const uint32_t b = pick[par][0];
        krem -= pick[par][1];
        const uint32_t nlo = lo + (b << sh);
        const uint64_t bin_hi = static_cast<uint64_t>(nlo) + ((uint64_t{1} << sh) - 1u);
        lo = nlo;
        hi = static_cast<uint32_t>(min(static_cast<uint64_t>(hi), bin_hi));
        par ^= 1;
    };
    static_assert(SBINS == kBins, "the first level uses the same bins");
    // the first histogram buffer starts at zero (the first choose's barriers order this
    // before the first pass); each later level clears the buffer of the level after it
#pragma unroll
    for (int j = 0; j < BPT; ++j) hist[0][threadIdx.x + T * j] = 0u;
    {
        uint32_t h[BPT] = {}, v[BPT];
        const uint32_t* hs = shist + static_cast<int64_t>(head) * SCOPIES * SBINS;
#pragma unroll
        for (int r = 0; r < SCOPIES; ++r) {
            load_bins(hs + r * SBINS, v);
#pragma unroll
            for (int j = 0; j < BPT; ++j) h[j] += v[j];
        }
        choose(h, 32 - SBINS_BITS);
    }
    int level = 0;
    while (lo != hi) {
        uint32_t* hb = hist[level & 1];
        const uint32_t span = hi - lo;
        const int bitlen = 32 - __clz(span);
        const int sh = bitlen > 11 ? bitlen - 11 : 0;   // (span >> sh) < 2048
        if (RES && off == 0 && (L & 3) == 0) {
            const uint4* k4 = reinterpret_cast<const uint4*>(keys);
            for (int i = threadIdx.x; i < (L >> 2); i += T) {
                const uint4 v = k4[i];
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (u[j] >= lo && u[j] <= hi) atomicAdd(&hb[(u[j] - lo) >> sh], 1u);
            }
        } else {
            for (int i = threadIdx.x; i < L; i += T) {
                const uint32_t u = key_at(i);
                if (u >= lo && u <= hi) atomicAdd(&hb[(u - lo) >> sh], 1u);
            }
        }
        sync_all();   // every part's histogram is complete
        // the other buffer was last read (by every CTA of the head) before this barrier:
        // clear it for the next level
#pragma unroll
        for (int j = 0; j < BPT; ++j) hist[(level + 1) & 1][threadIdx.x + T * j] = 0u;
        uint32_t h[BPT] = {}, v[BPT];
#pragma unroll
        for (int q = 0; q < CL; ++q) {
            load_bins(CL > 1 ? cluster.map_shared_rank(hb, q) : hb, v);
#pragma unroll
            for (int j = 0; j < BPT; ++j) h[j] += v[j];
        }
        choose(h, sh);
        ++level;
    }
    const uint32_t Tv = lo;
    const uint32_t E = krem;   // ties at Tv to keep, in key order

    // 3. counts per thread-contiguous run, then offsets over the CTA (block scan) and over
    //    the head's CTAs
    const int a = static_cast<int>(static_cast<int64_t>(L) * threadIdx.x / T);
    const int b = static_cast<int>(static_cast<int64_t>(L) * (threadIdx.x + 1) / T);
    uint32_t ngt = 0, neq = 0;
    for (int i = a; i < b; ++i) {
        const uint32_t u = key_at(i);
        ngt += u > Tv;
        neq += u == Tv;
    }
    // inclusive warp scans of (gt, eq), then warp totals
    uint32_t xg = ngt, xe = neq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t yg = __shfl_up_sync(0xffffffffu, xg, o);
        const uint32_t ye = __shfl_up_sync(0xffffffffu, xe, o);
        if (lane >= o) { xg += yg; xe += ye; }
    }
    if (lane == 31) { wa[par][warp] = xg; wb[warp] = xe; }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t g = 0, e = 0;
        for (int w = 0; w < kWarps; ++w) { g += wa[par][w]; e += wb[w]; }
        ctot[0] = g;
        ctot[1] = e;
    }
    sync_all();
    uint32_t gt_run = xg - ngt, eq_run = xe - neq;   // above Tv / ties before this thread
    if constexpr (CL > 1) {
        for (int q = 0; q < rank; ++q) {
            const uint32_t* r = cluster.map_shared_rank(ctot, q);
            gt_run += r[0];
            eq_run += r[1];
        }
    }
    for (int w = 0; w < warp; ++w) { gt_run += wa[par][w]; eq_run += wb[w]; }
    if constexpr (CL > 1) cluster.barrier_arrive();   // no remote read of this CTA follows

    // 4. this thread's winners in key order: every value above Tv, and the ties at Tv while
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
            bool take = u > Tv;
            if (u == Tv) take = eq_run++ < E;
            if (take) {
                oi[pos] = idx_at(i);
                if (oe) oe[pos] = __fmul_rn(qn, value_of(u));
                ++pos;
            }
        }
    }
    if constexpr (CL > 1) cluster.barrier_wait();
}

template <int CL, int T, int SLICE, bool RES>
cudaError_t launch_cfg(const pariskv_index* ix, int64_t C, int32_t k, int32_t* topk_idx,
                       float* topk_est, cudaStream_t st) {
    constexpr int kDyn = RES ? 2 * (SLICE + 8) * 4 : 0;
    static std::atomic<uint64_t> smem_raised{0};
    if (kDyn > 0) {   // static + dynamic shared memory can pass the 48 KB default
        cudaError_t e = raise_smem_limit(topk_kernel<CL, T, SLICE, RES>, kDyn, smem_raised);
        if (e != cudaSuccess) return e;
    }
    const int heads = ix->units * ix->cfg.group;
    return launch_pdl_cluster(topk_kernel<CL, T, SLICE, RES>, dim3(heads * CL), dim3(T), kDyn,
                              st, static_cast<unsigned>(CL), ix->S, ix->cand, ix->qnorm,
                              ix->shist, static_cast<int32_t>(C), ix->cmax, k, topk_idx,
                              topk_est, ix->status,
                              static_cast<uint32_t>(ix->inject_wait ? 16 : 0));
}

}  // namespace

bool topk_mode_fits(int mode, int64_t C) {
    return mode == 1 || mode == 2 ? C <= 8192 : mode == 3 ? C <= 4 * 16384 : mode == 4;
}

cudaError_t launch_topk(const pariskv_index* ix, int64_t C, int32_t k, int32_t* topk_idx,
                        float* topk_est, cudaStream_t st) {
    switch (ix->topk_mode) {   // a launch shape forced by the determinism tests
        case 1: return launch_cfg<1, 1024, 8192, true>(ix, C, k, topk_idx, topk_est, st);
        case 2: return launch_cfg<1, 256, 8192, true>(ix, C, k, topk_idx, topk_est, st);
        case 3: return launch_cfg<4, 1024, 16384, true>(ix, C, k, topk_idx, topk_est, st);
        case 4: return launch_cfg<4, 1024, 16384, false>(ix, C, k, topk_idx, topk_est, st);
        default: break;
    }
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int heads = ix->units * ix->cfg.group;
    if (C <= 8192 && heads <= sms)   // at most one head per SM: use all of its threads
        return launch_cfg<1, 1024, 8192, true>(ix, C, k, topk_idx, topk_est, st);
    if (C <= 4096) return launch_cfg<1, 256, 4096, true>(ix, C, k, topk_idx, topk_est, st);
    if (C <= 8192) return launch_cfg<1, 256, 8192, true>(ix, C, k, topk_idx, topk_est, st);
    if (C <= 4 * 16384)
        return launch_cfg<4, 1024, 16384, true>(ix, C, k, topk_idx, topk_est, st);
    return launch_cfg<4, 1024, 16384, false>(ix, C, k, topk_idx, topk_est, st);
}

}  // namespace pkv
