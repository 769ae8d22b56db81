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
//    vote scan (all loads in flight at once), finds T and E with suffix sums and ballots, and
//    writes for every 8192-key chunk how many candidates and how many score-T keys precede
//    it (one thread per chunk reads its 64 bins with vector loads; exclusive scans over
//    chunks).
//  compact_kernel (one CTA per chunk and vote pack, seven per SM so that the million-token
//    search's 1024 CTAs run in one wave): each thread owns 64 consecutive keys, read
//    coalesced and transposed through shared memory in two halves of 32 (the first half
//    before the wait for the threshold kernel, the second once the first is consumed; a
//    single 64-key buffer would allow only six CTAs per SM). SWAR byte arithmetic tests the
//    four packed scores of a key against the four heads' thresholds at once, and the test
//    bits are sliced into 32-bit masks per head (above T, at T) over the thread's keys.
//    POPC gives the counts; one block-wide scan of them gives every thread where its
//    candidates start and how many of its ties it keeps (all, none, or -- in the one thread
//    where the E-th tie falls -- the first few); the set bits are then written in key order.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kThr = 256;                  // threshold kernel

// Block-wide exclusive scan of a 64-bit value (4 packed 16-bit counters in the compaction,
// none of which overflows because a block's total per counter is at most CHUNK).
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
    __shared__ uint32_t part[kThr / NBINS][NBINS];
    __shared__ int32_t sT, sE;
    __shared__ uint64_t scan_sh[kThr / 32 + 1];

    const int head = blockIdx.x;
    const int unit = head / group, g = head % group;
    const int64_t up = static_cast<int64_t>(unit) * packs + g / PACK;
    const int h = g % PACK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t* hb = hist + up * nchunks * (PACK * NBINS) + h * NBINS;
    pdl_wait();
    pdl_launch_dependents();

    // total histogram: thread t sums bin t % 64 over chunks t / 64, t / 64 + 4, ... (the
    // loads are independent, so they are all in flight together)
    {
        constexpr int kRows = kThr / NBINS;
        const int bin = threadIdx.x % NBINS, r0 = threadIdx.x / NBINS;
        uint32_t a = 0;
#pragma unroll 32
        for (int64_t c = r0; c < nchunks; c += kRows) a += hb[c * (PACK * NBINS) + bin];
        part[r0][bin] = a;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int r = 0; r < kThr / NBINS; ++r) { lo += part[r][lane]; hi += part[r][lane + 32]; }
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
    // per chunk (one per thread, its 64 bins in 16 vector loads): keys above T and ties at T,
    // then exclusive scans over chunks
    uint64_t run_gt = 0, run_eq = 0;
    for (int64_t base = 0; base < nchunks; base += kThr) {
        const int64_t c = base + threadIdx.x;
        uint32_t gt = 0, eq = 0;
        if (c < nchunks) {
            const uint4* hc = reinterpret_cast<const uint4*>(hb + c * (PACK * NBINS));
            uint4 v[NBINS / 4];
#pragma unroll
            for (int i = 0; i < NBINS / 4; ++i) v[i] = hc[i];
#pragma unroll
            for (int i = 0; i < NBINS / 4; ++i) {
                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int bin = 4 * i + j;
                    gt += bin > T ? w[j] : 0u;
                    eq += bin == T ? w[j] : 0u;
                }
            }
        }
        const uint64_t mine = (static_cast<uint64_t>(eq) << 32) | gt;
        uint64_t total;
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

constexpr int kKeys = 64;                       // consecutive keys per thread
constexpr int kWords = kKeys / 32;              // 32-bit key masks per head and kind
constexpr int kCW = CHUNK / (32 * kKeys);       // compaction: warps per block (one chunk)
constexpr int kCThr = 32 * kCW;
constexpr int kRow = 33;                        // transposed row stride (conflict-free)
static_assert(kCW * 32 * kKeys == CHUNK, "one chunk per block");

// Block-wide exclusive scan of two 64-bit values at once (4 packed 16-bit counters each,
// none of which overflows: a block's total per counter is at most CHUNK).
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

__global__ void __launch_bounds__(kCThr, 7)
compact_kernel(const uint32_t* __restrict__ scores, const int32_t* __restrict__ thr,
               const int32_t* __restrict__ cbase, int32_t* __restrict__ cand, int64_t n,
               int64_t cap_pad, int group, int packs, int64_t nchunks, int64_t cmax,
               uint32_t* __restrict__ shist, int* status) {
    __shared__ uint32_t tr[kCW][32 * kRow];   // one half (32 keys per lane) at a time
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

    // half w of the warp's keys (32 per lane: lane l's keys kKeys l + 32 w .. + 31) into the
    // transposition buffer: copy t moves lane t's 32 keys, 128 contiguous bytes, so every
    // warp instruction is one coalesced line; lane l then reads row l (stride 33 words:
    // conflict-free both ways). Keys at or past n read as 0 (zero fill, src-size 0); their
    // address stays inside the padded capacity.
    auto load_half = [&](int w) {
        const uint32_t* src = scores + up * cap_pad + kw + 32 * w + lane;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int64_t key = kw + static_cast<int64_t>(kKeys) * t + 32 * w + lane;
            const uint32_t dst = smem_addr(&tr[warp][t * kRow + lane]);
            const uint32_t bytes = key < n ? 4u : 0u;
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst),
                         "l"(src + kKeys * t), "r"(bytes) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // the first half is loaded before the wait for the threshold kernel (the scores were
    // written two kernels back); the second once the first has been consumed
    load_half(0);
    const uint32_t* s = &tr[warp][lane * kRow];
    pdl_wait();
    pdl_launch_dependents();
    // the rerank that follows counts its values per head into shist: start it at zero
    // (the pack's CTAs share the work: CTA c clears words c * kCThr + t, stepping by all)
    for (int64_t i = c * kCThr + threadIdx.x; i < static_cast<int64_t>(hp) * SCOPIES * SBINS;
         i += nchunks * kCThr)
        shist[static_cast<int64_t>(head0) * SCOPIES * SBINS + i] = 0u;

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
    // Bit-sliced tests: for mask word w, word q of G (GE) holds, in byte h, bit i = key
    // 32 w + 8 q + i has score_h > T_h (>= T_h). Then per head and word a 32-bit key mask.
    uint32_t gm[PACK][kWords], em[PACK][kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w) {
        if (w > 0) {
            __syncwarp();            // every lane has read the previous half
            load_half(w);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        uint32_t G[4], GE[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t a = 0, b = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t sv = s[8 * q + i];
                a |= (((sv + gt_add) >> 7) & 0x01010101u) << i;
                b |= (((sv + ge_add) >> 7) & 0x01010101u) << i;
            }
            G[q] = a;
            GE[q] = b;
        }
        const int vw = nv - 32 * w;                         // valid keys in this word
        const uint32_t vbits = vw >= 32 ? 0xffffffffu : (vw <= 0 ? 0u : ((1u << vw) - 1u));
#define PKV_HEAD_MASK(W, H)                                                              \
    (prmt_i<0x5410u>(prmt_i<((4u + (H)) << 4) | (H)>(W[0], W[1]),                      \
                     prmt_i<((4u + (H)) << 4) | (H)>(W[2], W[3])))
        gm[0][w] = PKV_HEAD_MASK(G, 0) & vbits;  em[0][w] = PKV_HEAD_MASK(GE, 0) & vbits & ~gm[0][w];
        gm[1][w] = PKV_HEAD_MASK(G, 1) & vbits;  em[1][w] = PKV_HEAD_MASK(GE, 1) & vbits & ~gm[1][w];
        gm[2][w] = PKV_HEAD_MASK(G, 2) & vbits;  em[2][w] = PKV_HEAD_MASK(GE, 2) & vbits & ~gm[2][w];
        gm[3][w] = PKV_HEAD_MASK(G, 3) & vbits;  em[3][w] = PKV_HEAD_MASK(GE, 3) & vbits & ~gm[3][w];
#undef PKV_HEAD_MASK
    }
    uint64_t gb = 0, eb = 0;
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        uint32_t ng = 0, ne = 0;
#pragma unroll
        for (int w = 0; w < kWords; ++w) { ng += __popc(gm[h][w]); ne += __popc(em[h][w]); }
        gb |= static_cast<uint64_t>(ng) << (16 * h);
        eb |= static_cast<uint64_t>(ne) << (16 * h);
    }
    block_excl_scan2(gb, eb, scan_sh);   // keys above T / ties in this chunk before this thread

    // Per head: where this thread's candidates start, and which of its ties it keeps: the
    // chunk keeps the first B = max(0, E - ties before the chunk) of its ties, in key order.
    // Then its candidates are written in key order.
    const int32_t C = thr[head0 * 4 + 2];
    const int32_t kbase = static_cast<int32_t>(k0);
#pragma unroll
    for (int h = 0; h < PACK; ++h) {
        if (h >= hp) break;
        const int64_t hb = (static_cast<int64_t>(head0 + h) * nchunks + c) * 2;
        const int32_t E = thr[(head0 + h) * 4 + 1];
        const int32_t B = max(0, E - cbase[hb + 1]);
        const int32_t gbefore = static_cast<int32_t>((gb >> (16 * h)) & 0xffffu);
        const int32_t ebefore = static_cast<int32_t>((eb >> (16 * h)) & 0xffffu);
        uint32_t sel[kWords];
        int mine_e = 0, nsel = 0;
#pragma unroll
        for (int w = 0; w < kWords; ++w) mine_e += __popc(em[h][w]);
        const int take = min(max(B - ebefore, 0), mine_e);
#pragma unroll
        for (int w = 0; w < kWords; ++w) sel[w] = gm[h][w] | (take == mine_e ? em[h][w] : 0u);
        if (take != mine_e) {                 // the one thread where the E-th tie falls
            int left = take;
#pragma unroll
            for (int w = 0; w < kWords; ++w) {
                uint32_t m = em[h][w];
                for (; left > 0 && m; --left) {
                    const uint32_t low = m & (0u - m);
                    sel[w] |= low;
                    m ^= low;
                }
            }
        }
#pragma unroll
        for (int w = 0; w < kWords; ++w) nsel += __popc(sel[w]);
        const int32_t start = cbase[hb + 0] + gbefore + min(B, ebefore);
        if (!pkv_check(start >= 0, status)) continue;   // (checked build)
        if (start + nsel > C) {               // never taken when the histograms are consistent
            atomicExch(status, ST_BADINDEX);
            continue;
        }
        int32_t* out = cand + static_cast<int64_t>(head0 + h) * cmax + start;
#pragma unroll
        for (int w = 0; w < kWords; ++w) {
            uint32_t m = sel[w];
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1u;
                *out++ = kbase + 32 * w + j;
            }
        }
    }
}

}  // namespace

static __global__ void poke_kernel(int32_t* dst, int32_t value) { *dst = value; }

cudaError_t launch_poke(int32_t* dst, int32_t value, cudaStream_t st) {
    poke_kernel<<<1, 1, 0, st>>>(dst, value);
    return cudaGetLastError();
}

cudaError_t launch_threshold(const pariskv_index* ix, int64_t C, cudaStream_t st) {
    const int64_t nchunks = ceil_div(ix->n, CHUNK);
    const int heads = ix->units * ix->cfg.group;
    return launch_pdl(threshold_kernel, heads, kThr, 0, st, ix->hist, ix->cfg.group, ix->packs,
                      nchunks, C, ix->thr, ix->cbase);
}

cudaError_t launch_compact(const pariskv_index* ix, cudaStream_t st) {
    const int64_t nchunks = ceil_div(ix->n, CHUNK);
    dim3 grid(static_cast<unsigned>(nchunks), static_cast<unsigned>(ix->units * ix->packs));
    return launch_pdl(compact_kernel, grid, kCThr, 0, st, ix->scores, ix->thr, ix->cbase,
                      ix->cand, ix->n, ix->cap_pad, ix->cfg.group, ix->packs, nchunks, ix->cmax,
                      ix->shist, ix->status);
}

}  // namespace pkv
