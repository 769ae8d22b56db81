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
//    vote scan, finds T and E, and writes for every 8192-key chunk how many candidates and
//    how many score-T keys precede it (exclusive scans over chunks).
//  compact_kernel (one CTA per chunk and vote pack): each thread owns 32 consecutive keys;
//    two block-wide scans (tie counts, then candidate counts, four heads packed in 16-bit
//    lanes of a 64-bit word) give every candidate its output position.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kThr = 256;

// Block-wide exclusive scan of a 64-bit value (4 packed 16-bit counters; no lane overflows
// because a block's total per counter is at most CHUNK = 8192). Returns the exclusive
// prefix; *total receives the block total. All threads must call it.
__device__ __forceinline__ uint64_t block_excl_scan_u64(uint64_t v, uint64_t* total,
                                                        uint64_t* sh /* >= 9 entries */) {
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
        for (int w = 0; w < kThr / 32; ++w) {
            const uint64_t t = sh[w];
            sh[w] = run;
            run += t;
        }
        sh[kThr / 32] = run;
    }
    __syncthreads();
    const uint64_t res = sh[warp] + x - v;
    *total = sh[kThr / 32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kThr)
threshold_kernel(const uint32_t* __restrict__ hist, int group, int packs, int64_t nchunks,
                 int64_t C, int32_t* __restrict__ thr, int32_t* __restrict__ cbase) {
    __shared__ uint32_t part[4][NBINS];
    __shared__ uint32_t tot[NBINS];
    __shared__ int32_t sT, sE;
    __shared__ uint64_t scan_sh[kThr / 32 + 1];

    const int head = blockIdx.x;
    const int unit = head / group, g = head % group;
    const int64_t up = static_cast<int64_t>(unit) * packs + g / PACK;
    const int h = g % PACK;
    const uint32_t* hb = hist + up * nchunks * (PACK * NBINS) + h * NBINS;

    {
        const int bin = threadIdx.x & (NBINS - 1), p = threadIdx.x / NBINS;
        uint32_t s = 0;
        for (int64_t c = p; c < nchunks; c += 4) s += hb[c * (PACK * NBINS) + bin];
        part[p][bin] = s;
    }
    __syncthreads();
    if (threadIdx.x < NBINS)
        tot[threadIdx.x] = part[0][threadIdx.x] + part[1][threadIdx.x] + part[2][threadIdx.x] +
                           part[3][threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t cum = 0;
        int T = 0;
        for (int t = NBINS - 1; t >= 0; --t) {
            if (cum + tot[t] >= C) { T = t; break; }
            cum += tot[t];
        }
        sT = T;
        sE = static_cast<int32_t>(C - cum);
        thr[head * 4 + 0] = T;
        thr[head * 4 + 1] = sE;
        thr[head * 4 + 2] = static_cast<int32_t>(C);
        thr[head * 4 + 3] = static_cast<int32_t>(cum);
    }
    __syncthreads();
    const int T = sT;
    const int64_t E = sE;
    uint64_t run_gt = 0, run_eq = 0;
    for (int64_t base = 0; base < nchunks; base += kThr) {
        const int64_t c = base + threadIdx.x;
        uint32_t gt = 0, eq = 0;
        if (c < nchunks) {
            const uint32_t* hc = hb + c * (PACK * NBINS);
            for (int t = T + 1; t < NBINS; ++t) gt += hc[t];
            eq = hc[T];
        }
        // two 32-bit counters packed in one 64-bit scan word (totals <= 2^31)
        uint64_t total;
        const uint64_t pre = block_excl_scan_u64((static_cast<uint64_t>(eq) << 32) | gt, &total,
                                                 scan_sh);
        if (c < nchunks) {
            const int64_t gt_before = run_gt + (pre & 0xffffffffu);
            const int64_t eq_before = run_eq + (pre >> 32);
            const int64_t sel_before = gt_before + min(eq_before, E);
            cbase[(static_cast<int64_t>(head) * nchunks + c) * 2 + 0] =
                static_cast<int32_t>(sel_before);
            cbase[(static_cast<int64_t>(head) * nchunks + c) * 2 + 1] =
                static_cast<int32_t>(eq_before);
        }
        run_gt += total & 0xffffffffu;
        run_eq += total >> 32;
    }
}

__global__ void __launch_bounds__(kThr)
compact_kernel(const uint32_t* __restrict__ scores, const int32_t* __restrict__ thr,
               const int32_t* __restrict__ cbase, int32_t* __restrict__ cand, int64_t n,
               int64_t cap_pad, int group, int packs, int64_t nchunks, int64_t cmax,
               int* status) {
    __shared__ uint64_t scan_sh[kThr / 32 + 1];
    const int64_t c = blockIdx.x;
    const int64_t up = blockIdx.y;
    const int unit = static_cast<int>(up / packs), p = static_cast<int>(up % packs);
    const int hp = min(PACK, group - p * PACK);
    const int64_t k0 = c * CHUNK, k1 = min(n, k0 + CHUNK);
    const int64_t my0 = k0 + static_cast<int64_t>(threadIdx.x) * 32;

    int T[PACK], E[PACK], head[PACK], sel_base[PACK], eq_base[PACK];
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        head[h] = unit * group + p * PACK + min(h, hp - 1);
        T[h] = thr[head[h] * 4 + 0];
        E[h] = thr[head[h] * 4 + 1];
        sel_base[h] = cbase[(static_cast<int64_t>(head[h]) * nchunks + c) * 2 + 0];
        eq_base[h] = cbase[(static_cast<int64_t>(head[h]) * nchunks + c) * 2 + 1];
    }

    uint32_t s[32];
    const uint32_t* src = scores + up * cap_pad + my0;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        if (my0 + j < k1) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + j);
            s[j] = v.x; s[j + 1] = v.y; s[j + 2] = v.z; s[j + 3] = v.w;
        } else {
            s[j] = s[j + 1] = s[j + 2] = s[j + 3] = 0;
        }
    }
    const int nvalid = static_cast<int>(max64(0, min64(32, k1 - my0)));

    uint32_t gt[PACK], eq[PACK];
    uint64_t eq_pack = 0;
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        gt[h] = eq[h] = 0;
        if (h < hp) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int sh = (s[j] >> (8 * h)) & 0xff;
                gt[h] += (j < nvalid && sh > T[h]) ? 1u : 0u;
                eq[h] += (j < nvalid && sh == T[h]) ? 1u : 0u;
            }
        }
        eq_pack |= static_cast<uint64_t>(eq[h]) << (16 * h);
    }
    uint64_t tot;
    const uint64_t eq_pre = block_excl_scan_u64(eq_pack, &tot, scan_sh);
    uint32_t take_eq[PACK];
    uint64_t sel_pack = 0;
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        const int64_t before = eq_base[h] + static_cast<int64_t>((eq_pre >> (16 * h)) & 0xffff);
        const int64_t room = max64(0, E[h] - before);
        take_eq[h] = static_cast<uint32_t>(min64(room, eq[h]));
        sel_pack |= static_cast<uint64_t>(gt[h] + take_eq[h]) << (16 * h);
    }
    const uint64_t sel_pre = block_excl_scan_u64(sel_pack, &tot, scan_sh);
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        if (h >= hp) continue;
        int64_t pos = sel_base[h] + static_cast<int64_t>((sel_pre >> (16 * h)) & 0xffff);
        uint32_t eq_left = take_eq[h];
        int32_t* out = cand + static_cast<int64_t>(head[h]) * cmax;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int sh = (s[j] >> (8 * h)) & 0xff;
            bool sel = j < nvalid && sh > T[h];
            if (j < nvalid && sh == T[h] && eq_left > 0) { sel = true; --eq_left; }
            if (sel) {
                if (pos < thr[head[h] * 4 + 2]) out[pos] = static_cast<int32_t>(my0 + j);
                else atomicExch(status, ST_BADINDEX);
                ++pos;
            }
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
    compact_kernel<<<grid, kThr, 0, st>>>(ix->scores, ix->thr, ix->cbase, ix->cand, ix->n,
                                          ix->cap_pad, ix->cfg.group, ix->packs, nchunks,
                                          ix->cmax, ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
