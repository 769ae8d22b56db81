// select.cu -- candidate pruning: keep the C best coarse scores per query head.
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations 2 ("Coarse
// Candidate Generation"): the integer coarse score prunes the search space to a small
// candidate set (e.g. the top 5-10%). The candidates are the first C keys in the order
// (score descending, key index ascending), C = min(n, max(k, ceil(n * cand_bp / 10000))),
// and they are produced in ascending key order.
//
// Equivalent exact form used here: T = the largest t with #{score >= t} >= C; every key with
// score > T is a candidate, and so are the E = C - #{score > T} lowest-index keys with
// score == T.
//
//  threshold_kernel (one CTA per query head): sums the per-chunk histograms written by the
//    vote scan (warp per chunk, lane per pair of bins), finds T and E with suffix sums and
//    ballots, and writes for every 8192-key chunk how many candidates and how many score-T
//    keys precede it (exclusive scans over chunks).
//  compact_kernel (one CTA per chunk and vote pack): each thread owns 32 consecutive keys
//    (read coalesced and transposed through shared memory). SWAR byte arithmetic tests the
//    four packed scores of a key against the four heads' thresholds at once. A counting pass
//    and one block-wide scan of the per-head counts give every thread where its candidates
//    start and how many of its ties it keeps (all, none, or -- in the one thread where the
//    E-th tie falls -- the first few); the write pass then visits, in key order, only the
//    keys that reach some head's T (a bit mask from the counting pass) and stores them.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kThr = 256;                  // threshold kernel

// Block-wide exclusive scan of a 64-bit value (4 packed 16-bit counters in the compaction,
// none of which overflows because a block's total per counter is at most CHUNK = 8192).
// Returns the exclusive prefix; *total receives the block total. All threads must call it.
template <int NT>
__device__ __forceinline__ uint64_t block_excl_scan_u64(uint64_t v, uint64_t* total,
                                                        uint64_t* sh /* >= NT/32+1 */) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t run = 0;
        for (int w = 0; w < NT / 32; ++w) {
            const uint64_t t = sh[w];
            sh[w] = run;
            run += t;
        }
        sh[NT / 32] = run;
    }
    __syncthreads();
    const uint64_t res = sh[warp] + x - v;
    *total = sh[NT / 32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kThr)
threshold_kernel(const uint32_t* __restrict__ hist, int group, int packs, int64_t nchunks,
                 int64_t C, int32_t* __restrict__ thr, int32_t* __restrict__ cbase) {
    __shared__ uint32_t part[kThr / 32][NBINS];
    __shared__ int32_t sT, sE;
    __shared__ uint64_t scan_sh[kThr / 32 + 1];
    __shared__ uint64_t cnt[kThr];

    const int head = blockIdx.x;
    const int unit = head / group, g = head % group;
    const int64_t up = static_cast<int64_t>(unit) * packs + g / PACK;
    const int h = g % PACK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t* hb = hist + up * nchunks * (PACK * NBINS) + h * NBINS;

    // total histogram: warp w sums chunks w, w + 8, ...; lane l owns bins l and l + 32
    uint32_t a = 0, b = 0;
    for (int64_t c = warp; c < nchunks; c += kThr / 32) {
        a += hb[c * (PACK * NBINS) + lane];
        b += hb[c * (PACK * NBINS) + lane + 32];
    }
    part[warp][lane] = a;
    part[warp][lane + 32] = b;
    __syncthreads();
    if (warp == 0) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int w = 0; w < kThr / 32; ++w) { lo += part[w][lane]; hi += part[w][lane + 32]; }
        // count of scores >= t for t = lane and lane + 32 (suffix sums over the 64 bins)
        uint32_t shi = hi;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, shi, o);
            if (lane + o < 32) shi += y;
        }
        const uint32_t tot_hi = __shfl_sync(0xffffffffu, shi, 0);
        uint32_t slo = lo;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, slo, o);
            if (lane + o < 32) slo += y;
        }
        slo += tot_hi;
        // T = the largest t with #{score >= t} >= C
        const uint32_t mhi = __ballot_sync(0xffffffffu, shi >= C);
        const uint32_t mlo = __ballot_sync(0xffffffffu, slo >= C);
        int T;
        uint32_t ge_T, cnt_T;
        if (mhi) {
            T = 31 - __clz(mhi) + 32;
            ge_T = __shfl_sync(0xffffffffu, shi, T - 32);
            cnt_T = __shfl_sync(0xffffffffu, hi, T - 32);
        } else {
            T = 31 - __clz(mlo);
            ge_T = __shfl_sync(0xffffffffu, slo, T);
            cnt_T = __shfl_sync(0xffffffffu, lo, T);
        }
        if (lane == 0) {
            const int64_t above = static_cast<int64_t>(ge_T) - cnt_T;  // #{score > T}
            sT = T;
            sE = static_cast<int32_t>(C - above);
            thr[head * 4 + 0] = T;
            thr[head * 4 + 1] = sE;
            thr[head * 4 + 2] = static_cast<int32_t>(C);
            thr[head * 4 + 3] = static_cast<int32_t>(above);
        }
    }
    __syncthreads();
    const int T = sT;
    const int64_t E = sE;
    // per chunk: candidates above T and ties at T, then exclusive scans over chunks
    uint64_t run_gt = 0, run_eq = 0;
    for (int64_t base = 0; base < nchunks; base += kThr) {
        for (int i = warp; i < kThr; i += kThr / 32) {
            const int64_t c = base + i;
            uint32_t gt = 0, eq = 0;
            if (c < nchunks) {
                const uint32_t* hc = hb + c * (PACK * NBINS);
                const uint32_t x = hc[lane], y = hc[lane + 32];
                gt = __reduce_add_sync(0xffffffffu, (lane > T ? x : 0u) + (lane + 32 > T ? y : 0u));
                eq = __shfl_sync(0xffffffffu, T < 32 ? x : y, T & 31);
            }
            if (lane == 0) cnt[i] = (static_cast<uint64_t>(eq) << 32) | gt;
        }
        __syncthreads();
        const int64_t c = base + threadIdx.x;
        uint64_t total;
        const uint64_t mine = cnt[threadIdx.x];
        const uint64_t pre = block_excl_scan_u64<kThr>(mine, &total, scan_sh);
        if (c < nchunks) {
            const int64_t gt_before = run_gt + (pre & 0xffffffffu);
            const int64_t eq_before = run_eq + (pre >> 32);
            cbase[(static_cast<int64_t>(head) * nchunks + c) * 2 + 0] =
                static_cast<int32_t>(gt_before + min64(eq_before, E));
            cbase[(static_cast<int64_t>(head) * nchunks + c) * 2 + 1] =
                static_cast<int32_t>(eq_before);
        }
        run_gt += total & 0xffffffffu;
        run_eq += total >> 32;
    }
}

constexpr int kCW = 8;                          // compaction: warps per block
constexpr int kCThr = 32 * kCW;
constexpr int kKeys = CHUNK / kCThr;            // 32 consecutive keys per thread
static_assert(kKeys == 32, "one 32-key run per thread");

// Bytes 0,1 / 2,3 of a word spread into the 16-bit lanes of a 32-bit word.
__device__ __forceinline__ uint64_t spread_bytes(uint32_t x) {
    return (static_cast<uint64_t>(prmt_i<0x5352u>(x, 0u)) << 32) | prmt_i<0x5150u>(x, 0u);
}

// Block-wide exclusive scan of two 64-bit values at once (4 packed 16-bit counters each,
// none of which overflows: a block's total per counter is at most CHUNK = 8192).
__device__ __forceinline__ void block_excl_scan2(uint64_t& a, uint64_t& b,
                                                 uint64_t (*sh)[2] /* [kCW + 1][2] */) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = a, y = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t xo = __shfl_up_sync(0xffffffffu, x, o);
        const uint64_t yo = __shfl_up_sync(0xffffffffu, y, o);
        if (lane >= o) { x += xo; y += yo; }
    }
    if (lane == 31) { sh[warp][0] = x; sh[warp][1] = y; }
    __syncthreads();
    uint64_t bx = 0, by = 0;
    for (int w = 0; w < warp; ++w) { bx += sh[w][0]; by += sh[w][1]; }
    a = bx + x - a;
    b = by + y - b;
}

__global__ void __launch_bounds__(kCThr)
compact_kernel(const uint32_t* __restrict__ scores, const int32_t* __restrict__ thr,
               const int32_t* __restrict__ cbase, int32_t* __restrict__ cand, int64_t n,
               int64_t cap_pad, int group, int packs, int64_t nchunks, int64_t cmax,
               int* status) {
    __shared__ uint32_t tr[kCW][32 * 33];
    __shared__ uint64_t scan_sh[kCW + 1][2];
    const int64_t c = blockIdx.x;
    const int64_t up = blockIdx.y;
    const int unit = static_cast<int>(up / packs), p = static_cast<int>(up % packs);
    const int hp = min(PACK, group - p * PACK);
    const int head0 = unit * group + p * PACK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t kw = c * CHUNK + static_cast<int64_t>(warp) * (32 * kKeys);  // warp's first key
    const int64_t k0 = kw + static_cast<int64_t>(lane) * kKeys;                // thread's first key
    const int nv = static_cast<int>(max64(0, min64(kKeys, n - k0)));          // its valid keys

    // coalesced load of the warp's 1024 packed scores, transposed so that lane l then reads
    // keys 32 l .. 32 l + 31 (row stride 33 words: both directions are conflict-free)
    {
        const uint32_t* src = scores + up * cap_pad + kw + lane;
        const int nw = static_cast<int>(max64(0, min64(32 * kKeys, n - kw)));
#pragma unroll 8
        for (int t = 0; t < kKeys; ++t)
            tr[warp][t * 33 + lane] = (32 * t + lane < nw) ? src[32 * t] : 0u;
        __syncwarp();
    }
    const uint32_t* s = &tr[warp][lane * 33];

    // Per-head thresholds packed one per byte. A head outside the pack gets T = 127, which
    // no score (< 64) reaches. Byte h of (s + gt_add) has bit 7 set iff score_h > T_h, and
    // of (s + ge_add) iff score_h >= T_h; bytes never carry (score + 128 <= 191).
    uint32_t gt_add = 0, ge_add = 0;
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        const int T = h < hp ? thr[(head0 + h) * 4 + 0] : 127;
        gt_add |= static_cast<uint32_t>(127 - T) << (8 * h);
        ge_add |= static_cast<uint32_t>(128 - T) << (8 * h);
    }
    // counting pass: keys above T and ties, per head in byte counters (at most 32 each),
    // and the mask of keys that reach T for some head (the only ones the write pass visits)
    uint32_t gcnt = 0, ecnt = 0, reach = 0;
#pragma unroll 8
    for (int j = 0; j < kKeys; ++j) {
        const uint32_t m = j < nv ? 0x01010101u : 0u;
        const uint32_t g = ((s[j] + gt_add) >> 7) & m;
        const uint32_t ge = ((s[j] + ge_add) >> 7) & m;
        gcnt += g;
        ecnt += ge ^ g;
        reach |= (ge != 0u ? 1u : 0u) << j;
    }
    uint64_t gb = spread_bytes(gcnt), eb = spread_bytes(ecnt);
    block_excl_scan2(gb, eb, scan_sh);   // keys above T / ties in this chunk before this thread

    // where this thread's candidates start, and how many of its ties it keeps: the chunk
    // keeps the first B = max(0, E - ties before the chunk) of its ties, in key order
    int32_t* out[PACK];
    uint32_t run[PACK], budget[PACK];
    uint32_t all_ties = 0, partial = 0;
    const int32_t C = thr[head0 * 4 + 2];
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        out[h] = cand + static_cast<int64_t>(head0 + min(h, hp - 1)) * cmax;
        run[h] = 0;
        budget[h] = 0;
        if (h >= hp) continue;
        const int64_t hb = (static_cast<int64_t>(head0 + h) * nchunks + c) * 2;
        const int64_t E = thr[(head0 + h) * 4 + 1];
        const int64_t B = max64(0, E - cbase[hb + 1]);
        const int64_t gbefore = (gb >> (16 * h)) & 0xffffu, ebefore = (eb >> (16 * h)) & 0xffffu;
        const int64_t mine_g = (gcnt >> (8 * h)) & 0xffu, mine_e = (ecnt >> (8 * h)) & 0xffu;
        const int64_t take = min64(max64(B - ebefore, 0), mine_e);
        const int64_t start = cbase[hb + 0] + gbefore + min64(B, ebefore);
        if (start + mine_g + take > C) {   // never taken when the histograms are consistent
            atomicExch(status, ST_BADINDEX);
            return;
        }
        run[h] = static_cast<uint32_t>(start);
        budget[h] = static_cast<uint32_t>(take);
        if (take == mine_e) all_ties |= 1u << (8 * h);
        else if (take > 0) partial |= 1u << (8 * h);
    }

    // write pass over the keys that reach T, in key order
    while (reach) {
        const int j = __ffs(reach) - 1;
        reach &= reach - 1u;
        const uint32_t sv = s[j];
        const uint32_t g = (sv + gt_add) >> 7 & 0x01010101u;
        const uint32_t e = ((sv + ge_add) >> 7 & 0x01010101u) ^ g;
        uint32_t sel = g | (e & all_ties);
        if (partial) {                       // the one thread per head where the E-th tie falls
#pragma unroll
            for (int h = 0; h < PACK; ++h) {
                if (((partial & e) >> (8 * h)) & 1u) {
                    if (budget[h] > 0) { sel |= 1u << (8 * h); --budget[h]; }
                }
            }
        }
        const int32_t key = static_cast<int32_t>(k0 + j);
#pragma unroll
        for (int h = 0; h < PACK; ++h) {
            const uint32_t b = (sel >> (8 * h)) & 1u;
            if (b) out[h][run[h]] = key;
            run[h] += b;
        }
    }
}

}  // namespace

cudaError_t launch_threshold(const pariskv_index* ix, int64_t C, cudaStream_t st) {
    const int64_t nchunks = ceil_div(ix->n, CHUNK);
    const int heads = ix->units * ix->cfg.group;
    threshold_kernel<<<heads, kThr, 0, st>>>(ix->hist, ix->cfg.group, ix->packs, nchunks, C,
                                             ix->thr, ix->cbase);
    return cudaGetLastError();
}

cudaError_t launch_compact(const pariskv_index* ix, cudaStream_t st) {
    const int64_t nchunks = ceil_div(ix->n, CHUNK);
    dim3 grid(static_cast<unsigned>(nchunks), static_cast<unsigned>(ix->units * ix->packs));
    compact_kernel<<<grid, kCThr, 0, st>>>(ix->scores, ix->thr, ix->cbase, ix->cand, ix->n,
                                          ix->cap_pad, ix->cfg.group, ix->packs, nchunks,
                                          ix->cmax, ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
