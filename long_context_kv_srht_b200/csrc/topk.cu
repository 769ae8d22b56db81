// topk.cu -- final top-k of the reranked candidates.
//
// "Technical Summary: ParisKV", Problem Statement (attention over a Top-k subset of past
// tokens) and Key Contributions 2 (Top-k selection directly on compressed codes); "ParisKV:
// Fast and Drift-Robust KV-Cache Retrieval for Long-Context LLMs" (on-demand top-k fetch).
// The k candidates with the largest rerank value S are kept, ties going to the lower key
// index, and returned in ascending key order with est = ||q|| * S.
//
// Exact selection on the order-preserving 32-bit image u of S (flip all bits of negative
// values, set the sign bit of the others) by one thread-block cluster of 8 CTAs per query
// head, so that all SMs take part:
//  - CTA r owns the r-th eighth of the head's candidates (contiguous, hence in key order),
//    keeps its u values in shared memory and finds their min and max; the cluster combines
//    them through distributed shared memory (DSMEM);
//  - range-adaptive radix levels: the current interval [lo, hi] is cut into at most 2048
//    power-of-two-wide bins; each CTA builds a shared histogram of its values in the
//    interval; CTA r sums bins [256 r, 256 r + 256) of all eight histograms over DSMEM and
//    publishes the range total; every CTA then reads the deciding range's bins remotely and
//    finds the bin holding the k-th largest by itself (two cluster barriers per level). The
//    interval shrinks 2048-fold per level, so at most three levels run, usually fewer;
//  - with T the k-th largest value and E the number of T-valued candidates to keep, a
//    ballot pass over warp-contiguous ranges writes every candidate above T and the first E
//    equal to T, in ascending key order.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.hpp"

namespace cg = cooperative_groups;

namespace pkv {

namespace {

constexpr int kCL = 8;
constexpr int kT = 256;
constexpr int kWarps = kT / 32;
constexpr int kBins = 2048;
constexpr int kSliceMax = 8192;   // values kept in shared memory per CTA; larger slices re-read
static_assert(kBins / kCL == kT, "each CTA reduces kT bins");

__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __cluster_dims__(kCL, 1, 1) __launch_bounds__(kT)
topk_kernel(const float* __restrict__ S, const int32_t* __restrict__ cand,
            const float* __restrict__ qnorm, int64_t C, int64_t cmax, int32_t k,
            int32_t* __restrict__ out_idx, float* __restrict__ out_est, int* status) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int head = blockIdx.x / kCL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    __shared__ uint32_t keys[kSliceMax];
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t red[kT];
    __shared__ uint32_t tots[kCL], mins[kCL], maxs[kCL], cgt[kCL], ceq[kCL];
    __shared__ uint32_t wa[kWarps], wb[kWarps], wsel0[kWarps], weq0[kWarps];
    __shared__ uint32_t pick[2];

    const int64_t p0 = C * rank / kCL, p1 = C * (rank + 1) / kCL;
    const int len = static_cast<int>(p1 - p0);
    const bool res = len <= kSliceMax;
    const float* Sh = S + head * cmax + p0;
    const int32_t* ch = cand + head * cmax + p0;

    // 1. load the slice, local min / max, cluster-wide min / max
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (int base = 0; base < len; base += 4 * kT) {
        uint32_t u[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = base + j * kT + threadIdx.x;
            u[j] = i < len ? order_key(Sh[i]) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = base + j * kT + threadIdx.x;
            if (i < len) {
                if (res) keys[i] = u[j];
                mn = min(mn, u[j]);
                mx = max(mx, u[j]);
            }
        }
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) { wa[warp] = mn; wb[warp] = mx; }
    __syncthreads();
    if (threadIdx.x < kCL) {
        uint32_t a = 0xffffffffu, b = 0u;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) { a = min(a, wa[w]); b = max(b, wb[w]); }
        *cluster.map_shared_rank(&mins[rank], threadIdx.x) = a;
        *cluster.map_shared_rank(&maxs[rank], threadIdx.x) = b;
    }
    cluster.sync();
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int q = 0; q < kCL; ++q) { lo = min(lo, mins[q]); hi = max(hi, maxs[q]); }

    // 2. range-adaptive radix levels
    uint32_t krem = static_cast<uint32_t>(k);
    while (lo != hi) {
        const uint32_t span = hi - lo;
        const int bitlen = 32 - __clz(span);
        const int sh = bitlen > 11 ? bitlen - 11 : 0;   // (span >> sh) < 2048
#pragma unroll
        for (int j = 0; j < kBins / kT; ++j) hist[j * kT + threadIdx.x] = 0u;
        __syncthreads();
        for (int i = threadIdx.x; i < len; i += kT) {
            const uint32_t u = res ? keys[i] : order_key(Sh[i]);
            if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
        }
        cluster.sync();                                   // all histograms complete
        const int bin = rank * kT + threadIdx.x;
        uint32_t sum = 0;
#pragma unroll
        for (int q = 0; q < kCL; ++q) sum += *cluster.map_shared_rank(&hist[bin], q);
        red[threadIdx.x] = sum;
        const uint32_t wsum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) wa[warp] = wsum;
        __syncthreads();
        if (threadIdx.x < kCL) {
            uint32_t t = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) t += wa[w];
            *cluster.map_shared_rank(&tots[rank], threadIdx.x) = t;
        }
        cluster.sync();                                   // range totals published
        // the range holding the krem-th largest, and the count above it
        uint32_t cum = 0;
        int rs = 0;
        for (int r = kCL - 1; r >= 0; --r) {
            if (cum + tots[r] >= krem) { rs = r; break; }
            cum += tots[r];
        }
        if (warp == 0) {
            // lane l takes bins 8l .. 8l + 7 of range rs (read remotely)
            const uint32_t* rr = cluster.map_shared_rank(&red[0], rs);
            uint32_t v[8], s8 = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { v[j] = rr[8 * lane + j]; s8 += v[j]; }
            uint32_t x = s8;                              // suffix sums over lanes
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
                if (lane + o < 32) x += y;
            }
            uint32_t above = cum + x - s8;                // bins of higher lanes
#pragma unroll
            for (int j = 7; j >= 0; --j) {
                if (above < krem && krem <= above + v[j]) {
                    pick[0] = static_cast<uint32_t>(rs * kT + 8 * lane + j);
                    pick[1] = above;
                }
                above += v[j];
            }
        }
        __syncthreads();
        const uint32_t b = pick[0];
        krem -= pick[1];
        const uint32_t nlo = lo + (b << sh);
        lo = nlo;
        hi = min(hi, nlo + ((1u << sh) - 1u));
    }
    const uint32_t T = lo;
    const uint32_t E = krem;   // ties at T to keep, in key order

    // 3. compaction: counts per warp-contiguous range, then cluster-wide offsets
    const int w0 = len * warp / kWarps, w1 = len * (warp + 1) / kWarps;
    uint32_t ngt = 0, neq = 0;
    for (int pbase = w0; pbase < w1; pbase += 32) {
        const int pp = pbase + lane;
        const bool valid = pp < w1;
        const uint32_t u = valid ? (res ? keys[pp] : order_key(Sh[pp])) : 0u;
        ngt += __popc(__ballot_sync(0xffffffffu, valid && u > T));
        neq += __popc(__ballot_sync(0xffffffffu, valid && u == T));
    }
    if (lane == 0) { wa[warp] = ngt; wb[warp] = neq; }
    __syncthreads();
    if (threadIdx.x < kCL) {
        uint32_t g = 0, e = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) { g += wa[w]; e += wb[w]; }
        *cluster.map_shared_rank(&cgt[rank], threadIdx.x) = g;
        *cluster.map_shared_rank(&ceq[rank], threadIdx.x) = e;
    }
    cluster.sync();
    if (threadIdx.x == 0) {
        uint32_t gb = 0, eb = 0;
        for (int q = 0; q < rank; ++q) { gb += cgt[q]; eb += ceq[q]; }
        uint32_t sel = gb + min(eb, E), eqb = eb;
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
    for (int pbase = w0; pbase < w1; pbase += 32) {
        const int pp = pbase + lane;
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
    const int heads = ix->units * ix->cfg.group;
    topk_kernel<<<heads * kCL, kT, 0, st>>>(ix->S, ix->cand, ix->qnorm, C, ix->cmax, k,
                                            topk_idx, topk_est, ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
