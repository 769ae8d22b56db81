// topk.cu -- final top-k of the reranked candidates.
//
// "Technical Summary: ParisKV", Problem Statement (attention over a Top-k subset of past
// tokens) and Key Contributions 2 (Top-k selection directly on compressed codes); "ParisKV:
// Fast and Drift-Robust KV-Cache Retrieval for Long-Context LLMs" (on-demand top-k fetch).
// The k candidates with the largest rerank value S are kept, ties going to the lower key
// index, and returned in ascending key order with est = ||q|| * S.
//
// Exact radix select on the order-preserving 32-bit image of S (flip all bits of negative
// values, set the sign bit of the others), run by one thread-block cluster of 8 CTAs per
// query head:
//  - each CTA owns 1/8 of the head's candidates (contiguous, so ascending key order);
//  - three levels of 11, 11 and 10 bits: every CTA histograms the digit of its candidates
//    that match the prefix chosen so far (warp-aggregated shared atomics); CTA r sums bins
//    [256 r, 256 r + 256) of all 8 histograms through distributed shared memory; the range
//    totals are exchanged, and the CTA whose range holds the k-th largest finds the digit
//    and broadcasts it with the remaining rank;
//  - the threshold T and the number E of T-valued candidates to keep are then exact; a
//    final pass compacts, in key order, every candidate above T and the first E equal to T.
// Only the candidates' 8 bytes are read (from L2); no global atomics, no extra launches.
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
static_assert(kBins / kCL == kT, "each CTA reduces kT bins");

__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = __reduce_add_sync(0xffffffffu, v);
    if (lane == 0) sh[warp] = v;
    __syncthreads();
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += sh[w];
    __syncthreads();
    return t;
}

__global__ void __cluster_dims__(kCL, 1, 1) __launch_bounds__(kT)
topk_kernel(const float* __restrict__ S, const int32_t* __restrict__ cand,
            const float* __restrict__ qnorm, int64_t C, int64_t cmax, int32_t k,
            int32_t* __restrict__ out_idx, float* __restrict__ out_est, int* status) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int head = blockIdx.x / kCL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t red[kT];
    __shared__ uint32_t tots[kCL];
    __shared__ uint32_t pick[2];          // digit, remaining rank (written by the decider)
    __shared__ uint32_t cgt[kCL], ceq[kCL];
    __shared__ uint32_t wsh[kWarps];
    __shared__ uint32_t wgt[kWarps], weq[kWarps], wsel0[kWarps], weq0[kWarps];

    const int64_t p0 = C * rank / kCL, p1 = C * (rank + 1) / kCL;
    const float* Sh = S + head * cmax;
    const int32_t* ch = cand + head * cmax;
    const int64_t ntile = ceil_div(p1 - p0, kT);

    uint32_t prefix = 0, krem = static_cast<uint32_t>(k);
    int done = 0;
    for (int lvl = 0; lvl < 3; ++lvl) {
        const int bits = lvl < 2 ? 11 : 10;
        const int shift = 32 - done - bits;
        for (int b = threadIdx.x; b < kBins; b += kT) hist[b] = 0;
        __syncthreads();
        for (int64_t t = 0; t < ntile; ++t) {
            const int64_t p = p0 + t * kT + threadIdx.x;
            const bool valid = p < p1;
            const uint32_t u = valid ? order_key(Sh[p]) : 0u;
            const bool match = valid && (done == 0 || (u >> (32 - done)) == prefix);
            const uint32_t digit = (u >> shift) & ((1u << bits) - 1u);
            const uint32_t m = __ballot_sync(0xffffffffu, match);
            if (match) {
                const uint32_t peers = __match_any_sync(m, digit);
                if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
            }
        }
        cluster.sync();
        const int bin = rank * kT + threadIdx.x;
        uint32_t sum = 0;
#pragma unroll
        for (int q = 0; q < kCL; ++q) sum += *cluster.map_shared_rank(&hist[bin], q);
        red[threadIdx.x] = sum;
        const uint32_t tot_r = block_sum(sum, wsh);
        if (threadIdx.x < kCL) *cluster.map_shared_rank(&tots[rank], threadIdx.x) = tot_r;
        cluster.sync();
        if (threadIdx.x == 0) {
            uint32_t cum = 0;
            int rs = 0;
            for (int r = kCL - 1; r >= 0; --r) {
                if (cum + tots[r] >= krem) { rs = r; break; }
                cum += tots[r];
            }
            if (rs == rank) {
                uint32_t c2 = cum, dsel = 0, knew = 1;
                for (int b = kT - 1; b >= 0; --b) {
                    if (c2 + red[b] >= krem) { dsel = rank * kT + b; knew = krem - c2; break; }
                    c2 += red[b];
                }
                for (int q = 0; q < kCL; ++q) {
                    uint32_t* pk = cluster.map_shared_rank(&pick[0], q);
                    pk[0] = dsel;
                    pk[1] = knew;
                }
            }
        }
        cluster.sync();
        prefix = (prefix << bits) | pick[0];
        krem = pick[1];
        done += bits;
    }
    const uint32_t T = prefix;
    const uint32_t E = krem;   // ties at T to keep, in key order

    // per-warp contiguous ranges inside the CTA slice
    const int64_t w0 = p0 + (p1 - p0) * warp / kWarps, w1 = p0 + (p1 - p0) * (warp + 1) / kWarps;
    uint32_t ngt = 0, neq = 0;
    for (int64_t p = w0; p < w1; p += 32) {
        const int64_t pp = p + lane;
        const uint32_t u = pp < w1 ? order_key(Sh[pp]) : 0u;
        ngt += __popc(__ballot_sync(0xffffffffu, pp < w1 && u > T));
        neq += __popc(__ballot_sync(0xffffffffu, pp < w1 && u == T));
    }
    if (lane == 0) { wgt[warp] = ngt; weq[warp] = neq; }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t g = 0, e = 0;
        for (int w = 0; w < kWarps; ++w) { g += wgt[w]; e += weq[w]; }
        for (int q = 0; q < kCL; ++q) {
            *cluster.map_shared_rank(&cgt[rank], q) = g;
            *cluster.map_shared_rank(&ceq[rank], q) = e;
        }
    }
    cluster.sync();
    if (threadIdx.x == 0) {
        uint32_t gb = 0, eb = 0;
        for (int q = 0; q < rank; ++q) { gb += cgt[q]; eb += ceq[q]; }
        // walk the warps in order: candidates and ties before each warp
        uint32_t sel = gb + min(eb, E), eqb = eb;
        for (int w = 0; w < kWarps; ++w) {
            wsel0[w] = sel;
            weq0[w] = eqb;
            const uint32_t take = eqb >= E ? 0u : min(E - eqb, weq[w]);
            sel += wgt[w] + take;
            eqb += weq[w];
        }
    }
    __syncthreads();
    uint32_t sel_run = wsel0[warp], eq_run = weq0[warp];
    const float qn = qnorm[head];
    const unsigned lt = (1u << lane) - 1u;
    for (int64_t p = w0; p < w1; p += 32) {
        const int64_t pp = p + lane;
        const bool valid = pp < w1;
        const float sv = valid ? Sh[pp] : 0.0f;
        const uint32_t u = order_key(sv);
        const uint32_t eqm = __ballot_sync(0xffffffffu, valid && u == T);
        const bool take = valid && u == T && (eq_run + __popc(eqm & lt)) < E;
        const bool sel = (valid && u > T) || take;
        const uint32_t selm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const uint32_t r = sel_run + __popc(selm & lt);
            if (r < static_cast<uint32_t>(k)) {
                const int64_t pos = static_cast<int64_t>(head) * k + r;
                out_idx[pos] = ch[pp];
                if (out_est) out_est[pos] = __fmul_rn(qn, sv);
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
