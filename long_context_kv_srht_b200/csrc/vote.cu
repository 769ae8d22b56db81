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
// Design (sm_100a; measured bound: the L1/shared-memory pipe, about 84 % busy, with DRAM at
// a third of its bandwidth):
//  - Lane L scores keys L and L + 32 of a 64-key warp-tile, reading their ids with two
//    128-bit non-allocating loads (each a fully coalesced 512-byte warp access); the next
//    tile's ids are loaded while the current one is scored. Measured on B200, staging the ids
//    in shared memory costs more than it hides, because every staged byte is read again
//    through the same pipe: a per-warp ring of 1 KB tiles filled by TMA bulk copies
//    (cp.async.bulk on per-slot mbarriers) ran 51 us against 46 us, the same ring filled by
//    16-byte cp.async 50 us, and a CTA-wide bulk-copy ring refilled only once all warps had
//    released a stage stayed far below HBM bandwidth.
//  - The 32-bit table entry packs the vote weights of up to four query heads (one byte each;
//    a byte sum never exceeds 48), so one lookup per (key, subspace) serves the whole pack.
//  - Conflict-free lookups: the table holds two copies of every subspace's 256 entries, and
//    subspace b / copy k owns shared-memory bank 2b + k (entry c of it at row c, 256-byte
//    rows). Because the encoder stores subspace b of key i at byte (b - i / 2) mod 16, and
//    keys L and L + 32 of a tile share (i / 2) mod 16 = L / 2, at step t lane L reads
//    subspace (t + L / 2) mod 16 from byte t of both its keys, in copy L mod 2; the 32 lanes
//    then touch 32 distinct banks. One PRMT builds the address (row = id byte, column from a
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

constexpr int kWarps = 16;                   // two CTAs per SM: 32 scoring warps
constexpr int kThreads = 32 * kWarps;
constexpr int kTileKeys = 64;                // a warp-tile: two keys per lane
constexpr int kTableBytes = 256 * 256;
constexpr int kSmemBytes = kTableBytes;
constexpr int kTilesPerChunk = CHUNK / kTileKeys;
static_assert(kTilesPerChunk % kWarps == 0, "whole tiles per warp and chunk");

__device__ __forceinline__ uint32_t tab_ld(const uint8_t* tab, uint32_t off) {
    return *reinterpret_cast<const uint32_t*>(tab + off);
}

// The ids of keys L and L + 32 of a 64-key tile (lane L): two 128-bit non-allocating loads,
// each a fully coalesced 512-byte warp access.
__device__ __forceinline__ u32x8 ldg_ids(const uint8_t* p) {
    u32x8 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]) : "l"(p));
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7]) : "l"(p + 512));
    return v;
}

// Table entry of step t: byte0 <- column (byte t % 3 of colp[t / 3]), byte1 <- id byte t % 4,
// bytes 2, 3 <- the zero top byte of colp[t / 3].
template <int T>
__device__ __forceinline__ uint32_t look(const uint8_t* tab, const uint32_t* wd,
                                         const uint32_t* colp) {
    constexpr uint32_t sel = 0x7700u | ((T & 3u) << 4) | (4u + (T % 3));
    return tab_ld(tab, prmt_i<sel>(wd[T >> 2], colp[T / 3]));
}

// Packed coarse score of one key: the sum of its 16 table entries (byte h = query head h).
__device__ __forceinline__ uint32_t score_key(const uint8_t* tab, const uint32_t* wd,
                                              const uint32_t* colp) {
    const uint32_t v0 = look<0>(tab, wd, colp), v1 = look<1>(tab, wd, colp);
    const uint32_t v2 = look<2>(tab, wd, colp), v3 = look<3>(tab, wd, colp);
    const uint32_t v4 = look<4>(tab, wd, colp), v5 = look<5>(tab, wd, colp);
    const uint32_t v6 = look<6>(tab, wd, colp), v7 = look<7>(tab, wd, colp);
    const uint32_t v8 = look<8>(tab, wd, colp), v9 = look<9>(tab, wd, colp);
    const uint32_t v10 = look<10>(tab, wd, colp), v11 = look<11>(tab, wd, colp);
    const uint32_t v12 = look<12>(tab, wd, colp), v13 = look<13>(tab, wd, colp);
    const uint32_t v14 = look<14>(tab, wd, colp), v15 = look<15>(tab, wd, colp);
    const uint32_t a = v0 + v1 + v2, b = v3 + v4 + v5, c = v6 + v7 + v8, d = v9 + v10 + v11;
    const uint32_t e = v12 + v13 + v14;
    return (a + b + c) + (d + e + v15);
}

template <int H>
__device__ __forceinline__ void hist_inc(uint8_t* tab, uint32_t sc, uint32_t hcol) {
    atomicAdd(reinterpret_cast<uint32_t*>(tab + prmt_i<0x5504u | (H << 4)>(sc, hcol)), 1u);
}

__global__ void __launch_bounds__(kThreads, 2)
vote_kernel(const uint8_t* __restrict__ ids, const uint32_t* __restrict__ lut,
            uint32_t* __restrict__ scores, uint32_t* __restrict__ hist, int64_t n,
            int64_t cap_pad, int packs, int group, int64_t nchunks, int64_t items,
            int* status) {
    // Shared memory: table + histograms, 256 rows x 256 B (see the file comment).
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* tab = smem;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i0 = items * blockIdx.x / gridDim.x;
    const int64_t i1 = items * (blockIdx.x + 1) / gridDim.x;

    // Per-lane address parts: at step t lane L reads subspace (t + L / 2) mod 16 of both its
    // keys (the encoder rotates key i's bytes by (i / 2) mod 16), in copy L mod 2, which owns
    // bank column 2 * subspace + copy. Three columns per register with a zero top byte, so
    // one PRMT builds an address.
    uint32_t colp[6];
#pragma unroll
    for (int r = 0; r < 6; ++r) {
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int t = 3 * r + j;
            if (t < 16) w |= (4u * (2u * ((t + (lane >> 1)) & 15) + (lane & 1))) << (8 * j);
        }
        colp[r] = w;
    }
    const uint32_t hcol = 128u + 4u * lane;
    for (int r = warp; r < 256; r += kWarps)
        *reinterpret_cast<uint32_t*>(tab + r * 256 + hcol) = 0u;

    // warp w scores tiles w, w + kWarps, ... of each chunk; the next tile's ids are loaded
    // while the current tile is scored. Item -> ids address: the divisions run once per item.
    auto item_ids = [&](int64_t item) -> const uint8_t* {
        const int64_t up = item / nchunks, c = item - (item / nchunks) * nchunks;
        const int64_t unit = up / packs;
        return ids + (unit * cap_pad + c * CHUNK) * 16 + lane * 16;
    };
    constexpr int kTileBytes = kTileKeys * 16;
    int64_t cur_up = -1;
    u32x8 nxt;
    const uint8_t* base = i0 < i1 ? item_ids(i0) : ids;
    if (i0 < i1) nxt = ldg_ids(base + warp * kTileBytes);
    // the ids were written before the query kernel; its table is read only after the wait
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t item = i0; item < i1; ++item) {
        const int64_t up = item / nchunks, c = item - up * nchunks;
        const int hp = min(PACK, group - static_cast<int>(up % packs) * PACK);
        const uint8_t* next_base = item + 1 < i1 ? item_ids(item + 1) : base;
        if (up != cur_up) {
            __syncthreads();
            // row c, column 2b + k holds W_b[c] (copies k = 0, 1)
            // (all of a warp's loads are issued before its stores: one round trip)
            const uint32_t* lsrc = lut + up * (NB * NC) + (lane >> 1) * NC + warp;
            uint32_t v[NC / kWarps];
#pragma unroll
            for (int i = 0; i < NC / kWarps; ++i) v[i] = __ldg(lsrc + kWarps * i);
#pragma unroll
            for (int i = 0; i < NC / kWarps; ++i)
                *reinterpret_cast<uint32_t*>(tab + (warp + kWarps * i) * 256 + 4 * lane) = v[i];
            __syncthreads();
            cur_up = up;
        }
        const int64_t k0 = c * CHUNK;
        const int nkeys = static_cast<int>(min64(n - k0, CHUNK));
        uint32_t* sc_out = scores + up * cap_pad + k0;
#pragma unroll 1
        for (int tl = warp; tl < kTilesPerChunk; tl += kWarps) {
            const u32x8 cur = nxt;
            // prefetch: the next tile of this chunk, else this warp's first of the next item
            // (tiles past the last key read padding inside the capacity, never beyond it)
            if (tl + kWarps < kTilesPerChunk) nxt = ldg_ids(base + (tl + kWarps) * kTileBytes);
            else if (item + 1 < i1) nxt = ldg_ids(next_base + warp * kTileBytes);
        if (tl * kTileKeys >= nkeys) continue;
            uint32_t acc[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) acc[j] = score_key(tab, cur.w + 4 * j, colp);
            const int kk = tl * kTileKeys + lane;    // keys kk and kk + 32
#pragma unroll
            for (int j = 0; j < 2; ++j)
                if (kk + 32 * j < nkeys) sc_out[kk + 32 * j] = acc[j];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                // (checked build) every packed score byte is below 64: a larger one would
                // count into the next head's histogram rows
                if (kk + 32 * j < nkeys && pkv_check((acc[j] & 0xC0C0C0C0u) == 0u, status)) {
                    const uint32_t sc = acc[j] + 0xC0804000u;  // byte h -> 64 h + score_h
                    hist_inc<0>(tab, sc, hcol);
                    if (hp > 1) hist_inc<1>(tab, sc, hcol);
                    if (hp > 2) hist_inc<2>(tab, sc, hcol);
                    if (hp > 3) hist_inc<3>(tab, sc, hcol);
                }
            }
        }
        // flush this chunk's histograms: row 64 h + s, one counter per lane
        __syncthreads();
        uint32_t* hout = hist + (up * nchunks + c) * (PACK * NBINS);
        {
            constexpr int kRows = PACK * NBINS / kWarps;   // rows warp, warp + kWarps, ...
            uint32_t v[kRows];
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                uint32_t* a = reinterpret_cast<uint32_t*>(tab + (warp + kWarps * i) * 256 + hcol);
                v[i] = *a;
                *a = 0u;
            }
#pragma unroll
            for (int i = 0; i < kRows; ++i) v[i] = __reduce_add_sync(0xffffffffu, v[i]);
            if (lane == 0)
#pragma unroll
                for (int i = 0; i < kRows; ++i) hout[warp + kWarps * i] = v[i];
        }
        __syncthreads();
        base = next_base;
    }
}

}  // namespace

cudaError_t launch_vote(const pariskv_index* ix, cudaStream_t st) {
    static std::atomic<uint64_t> smem_raised{0};
    if (cudaError_t e = raise_smem_limit(vote_kernel, kSmemBytes, smem_raised); e != cudaSuccess) return e;
    if (ix->n <= 0) return cudaSuccess;
    const int64_t nchunks = ceil_div(ix->n, CHUNK);
    const int64_t items = static_cast<int64_t>(ix->units) * ix->packs * nchunks;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = static_cast<int>(min64(items, ix->vote_ctas > 0 ? ix->vote_ctas : 2LL * sms));
    return launch_pdl(vote_kernel, grid, kThreads, kSmemBytes, st, ix->ids, ix->lut, ix->scores,
                      ix->hist, ix->n, ix->cap_pad, ix->packs, ix->cfg.group, nchunks, items,
                      ix->status);
}

}  // namespace pkv
