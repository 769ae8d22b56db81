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
constexpr int kSmemBytes = kTableBytes + kStages * kStageBytes + 2 * kStages * 8 + 1024;
static_assert(CHUNK % kStageKeys == 0, "chunks hold whole stages");

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" :: "r"(kConsumerWarps * 32) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
vote_kernel(const uint8_t* __restrict__ ids, const uint32_t* __restrict__ lut,
            uint32_t* __restrict__ scores, uint32_t* __restrict__ hist, int64_t n,
            int64_t cap_pad, int packs, int group, int64_t nchunks, int64_t items,
            int* status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (the table rows must not straddle the alignment assumptions)
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t tab = smem_addr(smem);
    const uint32_t ring = tab + kTableBytes;
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
                const int64_t k0 = c * CHUNK, k1 = min(n, k0 + CHUNK);
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
    uint32_t col[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) col[t] = 4u * (2u * ((t + lane) & 15) + (lane >> 4));
    const uint32_t hcol = 128u + 4u * lane;

    // zero the histogram half of every row
    for (int r = warp; r < 256; r += kConsumerWarps)
        asm volatile("st.shared.u32 [%0], %1;" :: "r"(tab + r * 256 + hcol), "r"(0u) : "memory");

    int64_t cur_up = -1;
    uint32_t it = 0;
    for (int64_t item = i0; item < i1; ++item) {
        const int64_t up = item / nchunks, c = item % nchunks;
        const int hp = min(PACK, group - static_cast<int>(up % packs) * PACK);
        if (up != cur_up) {
            consumer_sync();
            // table: column 2b + k of row c holds W_b[c] (both copies k = 0, 1)
            const uint32_t* lsrc = lut + up * (NB * NC);
            const int b = lane >> 1;
            for (int r = warp; r < NC; r += kConsumerWarps) {
                const uint32_t v = __ldg(lsrc + b * NC + r);
                asm volatile("st.shared.u32 [%0], %1;" :: "r"(tab + r * 256 + 4 * lane), "r"(v)
                             : "memory");
            }
            consumer_sync();
            cur_up = up;
        }
        const int64_t k0 = c * CHUNK, k1 = min(n, k0 + CHUNK);
        uint32_t* sc_out = scores + up * cap_pad;
        for (int64_t s0 = k0; s0 < k1; s0 += kStageKeys, ++it) {
            const int slot = it % kStages;
            mbar_wait(full_bar + 8 * slot, (it / kStages) & 1, status);
            const int ntiles = static_cast<int>(ceil_div(min64(kStageKeys, k1 - s0), 32));
            const uint32_t sbase = ring + slot * kStageBytes + lane * 16;
            for (int tile = warp; tile < ntiles; tile += kConsumerWarps) {
                const uint4 idv = lds_u128(sbase + tile * 512);
                const uint32_t wd[4] = {idv.x, idv.y, idv.z, idv.w};
                uint32_t acc = 0;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const uint32_t a = prmt(wd[t >> 2], col[t], 0x5504u | ((t & 3u) << 4));
                    acc += lds_u32(tab + a);
                }
                const int64_t key = s0 + tile * 32 + lane;
                if (key < k1) {
                    sc_out[key] = acc;
                    const uint32_t sc = acc + 0xC0804000u;  // byte h -> 64 h + score_h
                    for (int h = 0; h < hp; ++h)
                        red_shared_add(tab + prmt(sc, hcol, 0x5504u | (static_cast<uint32_t>(h) << 4)), 1u);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar + 8 * slot);
        }
        // flush this chunk's histograms: row 64 h + s, one counter per lane
        consumer_sync();
        uint32_t* hout = hist + (up * nchunks + c) * (PACK * NBINS);
        for (int r = warp; r < PACK * NBINS; r += kConsumerWarps) {
            const uint32_t a = tab + r * 256 + hcol;
            const uint32_t v = lds_u32(a);
            const uint32_t tot = __reduce_add_sync(0xffffffffu, v);
            asm volatile("st.shared.u32 [%0], %1;" :: "r"(a), "r"(0u) : "memory");
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
