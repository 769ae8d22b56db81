// vote.cu -- collision-vote scan: every cached key gets an integer coarse score.
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations 2 ("Coarse
// Candidate Generation"): keys whose bucket in a subspace is one of the query's top-rho
// centroids receive that centroid's tiered vote; votes are summed over the B subspaces into
// an integer coarse score, score_i = sum_b W_b[id_{i,b}].
//
// This is the N-proportional part of the decode step: 16 bytes of bucket ids per key are
// streamed once per KV head and scored for all query heads of its GQA group at once.
//
// Design (sm_100a, HBM-bound):
//  - A producer warp streams id tiles (1024 keys = 16 KB) with cp.async.bulk into a 4-stage
//    shared-memory ring guarded by mbarriers (no multicast); 16 consumer warps score them.
//  - Lane L of a consumer warp scores key (tile base + L). The 32-bit table entry packs the
//    vote weights of up to four query heads (one byte each; a byte sum never exceeds 48), so
//    one lookup per (key, subspace) serves the whole pack of heads.
//  - Conflict-free lookups: the table holds two copies of every subspace's 256 entries, and
//    subspace b / copy k owns shared-memory bank 2b + k (entry c of it at row c, 256-byte
//    rows). Because the encoder stores subspace b of key i at byte (b - i) mod 16, at step t
//    lane L reads subspace (t + L) mod 16 from byte t of its own 16 bytes; the 32 lanes then
//    touch 32 distinct banks. One PRMT builds the address (row = id byte, column from a
//    per-lane constant), one LDS reads the entry, one add accumulates.
//  - Histograms of the packed scores (64 bins per query head) are built in the upper half of
//    the same rows, one private counter column per lane (so no intra-warp conflicts), and
//    flushed once per 8192-key chunk with a warp reduction. The candidate threshold and the
//    per-chunk offsets of the selection are computed from them without rereading scores.
//  - The packed scores (4 bytes per key) are written for the compaction pass; they are
//    small enough to stay in L2.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kStageKeys = 1024;
constexpr int kStageBytes = kStageKeys * 16;
constexpr int kStages = 4;
constexpr int kTableBytes = 256 * 256;
constexpr int kSmemBytes = kTableBytes + kStages * kStageBytes + 2 * kStages * 8;
static_assert(CHUNK % kStageKeys == 0, "chunks hold whole stages");

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" :: "r"(kConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ uint32_t tab_ld(const uint8_t* tab, uint32_t off) {
    return *reinterpret_cast<const uint32_t*>(tab + off);
}
__device__ __forceinline__ void tab_inc(uint8_t* tab, uint32_t off) {
    atomicAdd(reinterpret_cast<uint32_t*>(tab + off), 1u);
}

__global__ void __launch_bounds__(kThreads, 1)
vote_kernel(const uint8_t* __restrict__ ids, const uint32_t* __restrict__ lut,
            uint32_t* __restrict__ scores, uint32_t* __restrict__ hist, int64_t n,
            int64_t cap_pad, int packs, int group, int64_t nchunks, int64_t items,
            int* status) {
    // Shared memory: [table + histograms: 256 rows x 256 B][ring of kStages id tiles][bars].
    // Only 16-byte alignment is needed (bulk-copy destinations, 16-byte id loads); a row
    // start need not sit on bank 0 because every row keeps the same bank permutation.
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* tab = smem;
    const uint8_t* ringp = smem + kTableBytes;
    const uint32_t ring = smem_addr(ringp);
    const uint32_t full_bar = ring + kStages * kStageBytes;
    const uint32_t empty_bar = full_bar + kStages * 8;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i0 = items * blockIdx.x / gridDim.x;
    const int64_t i1 = items * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar + 8 * s, 1);
            mbar_init(empty_bar + 8 * s, kConsumerWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int64_t item = i0; item < i1; ++item) {
                const int64_t up = item / nchunks, c = item % nchunks;
                const int64_t unit = up / packs;
                const int64_t k0 = c * CHUNK, k1 = min64(n, k0 + CHUNK);
                for (int64_t s0 = k0; s0 < k1; s0 += kStageKeys, ++it) {
                    const int slot = it % kStages;
                    if (it >= kStages)
                        mbar_wait(empty_bar + 8 * slot, ((it / kStages) + 1) & 1, status);
                    const int64_t nk = round_up(min64(kStageKeys, k1 - s0), 32);
                    const uint32_t bytes = static_cast<uint32_t>(nk * 16);
                    mbar_arrive_expect_tx(full_bar + 8 * slot, bytes);
                    bulk_g2s(ring + slot * kStageBytes, ids + (unit * cap_pad + s0) * 16, bytes,
                             full_bar + 8 * slot);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------------- consumers
    // Per-lane address parts: at step t lane L reads subspace (t + L) mod 16 (see the
    // encoder's byte rotation), whose copy (L >> 4) owns bank column 2 * subspace + copy.
    uint32_t col[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) col[t] = 4u * (2u * ((t + lane) & 15) + (lane >> 4));
    const uint32_t hcol = 128u + 4u * lane;

    for (int r = warp; r < 256; r += kConsumerWarps)
        *reinterpret_cast<uint32_t*>(tab + r * 256 + hcol) = 0u;

    int64_t cur_up = -1;
    uint32_t it = 0;
    for (int64_t item = i0; item < i1; ++item) {
        const int64_t up = item / nchunks, c = item % nchunks;
        const int hp = min(PACK, group - static_cast<int>(up % packs) * PACK);
        if (up != cur_up) {
            consumer_sync();
            // row c, column 2b + k holds W_b[c] (copies k = 0, 1)
            const uint32_t* lsrc = lut + up * (NB * NC);
            const int b = lane >> 1;
            for (int r = warp; r < NC; r += kConsumerWarps)
                *reinterpret_cast<uint32_t*>(tab + r * 256 + 4 * lane) = __ldg(lsrc + b * NC + r);
            consumer_sync();
            cur_up = up;
        }
        const int64_t k0 = c * CHUNK, k1 = min64(n, k0 + CHUNK);
        for (int64_t s0 = k0; s0 < k1; s0 += kStageKeys, ++it) {
            const int slot = it % kStages;
            mbar_wait(full_bar + 8 * slot, (it / kStages) & 1, status);
            const int nkeys = static_cast<int>(min64(kStageKeys, k1 - s0));
            const uint8_t* stage = ringp + slot * kStageBytes + lane * 16;
            uint32_t* sc_out = scores + up * cap_pad + s0;
            for (int tile = warp; tile * 32 < nkeys; tile += kConsumerWarps) {
                const uint4 idv = *reinterpret_cast<const uint4*>(stage + tile * 512);
                const uint32_t wd[4] = {idv.x, idv.y, idv.z, idv.w};
                uint32_t v[16];
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    v[t] = tab_ld(tab, prmt(wd[t >> 2], col[t], 0x5504u | ((t & 3u) << 4)));
                uint32_t acc = 0;
#pragma unroll
                for (int t = 0; t < 16; ++t) acc += v[t];
                const int kk = tile * 32 + lane;
                if (kk < nkeys) {
                    sc_out[kk] = acc;
                    const uint32_t sc = acc + 0xC0804000u;  // byte h -> 64 h + score_h
                    if (hp == PACK) {
#pragma unroll
                        for (int h = 0; h < PACK; ++h)
                            tab_inc(tab, prmt(sc, hcol, 0x5504u | (static_cast<uint32_t>(h) << 4)));
                    } else {
                        for (int h = 0; h < hp; ++h)
                            tab_inc(tab, prmt(sc, hcol, 0x5504u | (static_cast<uint32_t>(h) << 4)));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar + 8 * slot);
        }
        // flush this chunk's histograms: row 64 h + s, one counter per lane
        consumer_sync();
        uint32_t* hout = hist + (up * nchunks + c) * (PACK * NBINS);
        for (int r = warp; r < PACK * NBINS; r += kConsumerWarps) {
            uint32_t* a = reinterpret_cast<uint32_t*>(tab + r * 256 + hcol);
            const uint32_t tot = __reduce_add_sync(0xffffffffu, *a);
            *a = 0u;
            if (lane == 0) hout[r] = tot;
        }
        consumer_sync();
    }
}

}  // namespace

cudaError_t launch_vote(const pariskv_index* ix, cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(vote_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    if (ix->n <= 0) return cudaSuccess;
    const int64_t nchunks = ceil_div(ix->n, CHUNK);
    const int64_t items = static_cast<int64_t>(ix->units) * ix->packs * nchunks;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = static_cast<int>(min64(items, sms));
    vote_kernel<<<grid, kThreads, kSmemBytes, st>>>(ix->ids, ix->lut, ix->scores, ix->hist,
                                                   ix->n, ix->cap_pad, ix->packs,
                                                   ix->cfg.group, nchunks, items, ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
