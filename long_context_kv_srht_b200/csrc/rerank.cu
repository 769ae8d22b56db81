// rerank.cu -- RSQ-IP rerank of the candidates from their compact codes.
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations 2 ("Candidate
// Reranking (RSQ-IP)", "Estimation"): <k, q> is estimated as ||q|| sum_b w_{i,b} <v_{i,b},
// q~_b> without touching the full-precision key. With the folded per-(key, subspace)
// factor f_{i,b} written at encode time, the value ranked here is
//     S_i = sum_b f_{i,b} p_{i,b},    p_{i,b} = sum_j vt_{i,b,j} q~_{b,j},
// where vt are the signed integer magnitude levels. Both sums are fp32 FMA chains in
// ascending order (p over j from 0.0f, then S over b from 0.0f), the order of the reference
// definition, so S is bit-reproducible; est = ||q|| S.
//
// Memory: the candidates' 128-byte records sit at random places in a 1 GiB array, and HBM
// only delivers its bandwidth with far more bytes in flight than registers can hold. So the
// records are gathered with asynchronous global->shared copies (cp.async, 16 bytes per lane;
// eight lanes move one record, so one warp instruction moves four whole records): the kernel
// is persistent (kCtasPerSm CTAs per SM), every warp owns a ring of kSlots stages of 64
// records, and a stage is refilled as soon as it has been scored. Piece c of the record in
// stage row r is stored at 16-byte position c ^ (r mod 8), so that eight lanes reading the
// same piece of eight different records touch all 32 banks once.
//
// Each value is also counted, by the top bits of its order-preserving image, into a per-head
// histogram, which is the top-k's first radix level: lanes holding the same bin are grouped
// with a warp match and one of them adds the group's count, into one of SCOPIES copies chosen
// by the warp. (One global reduction per value piled onto the few hot bins and doubled the
// kernel's time; with the match, eight copies measured no faster than one.)
//
// Scoring: each lane scores two records of a stage (rows lane and lane + 32, whose chains
// interleave). The warp's current query head has its rotated query in shared memory as
// (subspace 2t, subspace 2t + 1) fp32 pairs, each read once by broadcast for both records; a
// lane walks the 8 subspace pairs in order, two p chains advancing together in Blackwell's
// packed fp32x2 FMA (each half an ordinary IEEE fp32 FMA), and extends each record's S chain
// after every pair. Decoding is exact integer arithmetic: the stored offset-binary nibbles
// u = vt + 8 are split into even and odd dims with two masks, a PRMT places u in the
// mantissa of 2^23, and one packed subtraction of 2^23 + 8 gives vt exactly as fp32.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kWarps = 4;               // every warp gathers and scores
constexpr int kCtasPerSm = 3;           // persistent CTAs per SM
constexpr int kThr = 32 * kWarps;
constexpr int kSlots = 2;               // stages in flight per warp
constexpr int kPerLane = 2;             // records scored per lane and stage
constexpr int kStageRecs = 32 * kPerLane;
constexpr int kStageBytes = kStageRecs * REC;
constexpr int kQBytes = D * 4;          // one head's rotated query
constexpr int kWarpBytes = kSlots * kStageBytes + kQBytes;
constexpr int kSmem = kWarps * kWarpBytes;
static_assert(kWarpBytes % 128 == 0, "warp areas stay 128-byte aligned");

__device__ __forceinline__ uint32_t piece_at(int row, int c) {
    return static_cast<uint32_t>(row * REC + ((c ^ (row & 7)) << 4));
}

template <int K>
__device__ __forceinline__ uint64_t level_pair(uint32_t xa, uint32_t xb) {
    // byte K of each word into the mantissa of 2^23: 2^23 + u exactly; minus (2^23 + 8) = vt
    const uint64_t kOff = pack2(-8388616.0f, -8388616.0f);
    return add2(pack2u(prmt_i<0x7650u + K>(xa, 0x4B000000u), prmt_i<0x7650u + K>(xb, 0x4B000000u)),
                kOff);
}

// table levels: nibble u (byte K of each word) -> dec[u], a 16-entry table in shared memory
template <int K>
__device__ __forceinline__ uint64_t table_pair(uint32_t xa, uint32_t xb, const float* dec) {
    return pack2(dec[(xa >> (8 * K)) & 15u], dec[(xb >> (8 * K)) & 15u]);
}

// p chains of the subspace pair (a, b) from their code words, with the query pairs
// q[j] = (q~_{a,j}, q~_{b,j}) for j = 0..7.
template <bool TABLE>
__device__ __forceinline__ float2 pair_dots(uint32_t wa, uint32_t wb, const uint64_t q[8],
                                            const float* dec) {
    const uint32_t ea = wa & 0x0F0F0F0Fu, oa = (wa >> 4) & 0x0F0F0F0Fu;  // dims 0,2,4,6 | 1,3,5,7
    const uint32_t eb = wb & 0x0F0F0F0Fu, ob = (wb >> 4) & 0x0F0F0F0Fu;
    uint64_t p = pack2(0.0f, 0.0f);
    if constexpr (TABLE) {
        p = fma2(table_pair<0>(ea, eb, dec), q[0], p);
        p = fma2(table_pair<0>(oa, ob, dec), q[1], p);
        p = fma2(table_pair<1>(ea, eb, dec), q[2], p);
        p = fma2(table_pair<1>(oa, ob, dec), q[3], p);
        p = fma2(table_pair<2>(ea, eb, dec), q[4], p);
        p = fma2(table_pair<2>(oa, ob, dec), q[5], p);
        p = fma2(table_pair<3>(ea, eb, dec), q[6], p);
        p = fma2(table_pair<3>(oa, ob, dec), q[7], p);
    } else {
        p = fma2(level_pair<0>(ea, eb), q[0], p);
        p = fma2(level_pair<0>(oa, ob), q[1], p);
        p = fma2(level_pair<1>(ea, eb), q[2], p);
        p = fma2(level_pair<1>(oa, ob), q[3], p);
        p = fma2(level_pair<2>(ea, eb), q[4], p);
        p = fma2(level_pair<2>(oa, ob), q[5], p);
        p = fma2(level_pair<3>(ea, eb), q[6], p);
        p = fma2(level_pair<3>(oa, ob), q[7], p);
    }
    return unpack2(p);
}

__device__ __forceinline__ void load_qpairs(const uint64_t* qp, uint64_t q[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const ulonglong2 v = reinterpret_cast<const ulonglong2*>(qp)[i];
        q[2 * i] = v.x;
        q[2 * i + 1] = v.y;
    }
}

// S of the kPerLane records in stage rows row0 + 32 u; qp = the head's 64 query pairs (pair
// t at qp + 8 t). Each query pair is read once for all the lane's records; every record
// keeps its own p and S chains in the defined order.
template <bool TABLE>
__device__ __forceinline__ void score_records(const uint8_t* st, int row0, const uint64_t* qp,
                                              const float* dec, float S[kPerLane]) {
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) S[u] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {   // chunk c: subspaces 4c..4c+3
        uint4 cw[kPerLane], fw[kPerLane];
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            cw[u] = *reinterpret_cast<const uint4*>(st + piece_at(row0 + 32 * u, 2 * c));
            fw[u] = *reinterpret_cast<const uint4*>(st + piece_at(row0 + 32 * u, 2 * c + 1));
        }
        uint64_t q[8];
        load_qpairs(qp + 16 * c, q);
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const float2 pa = pair_dots<TABLE>(cw[u].x, cw[u].y, q, dec);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].x), pa.x, S[u]);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].y), pa.y, S[u]);
        }
        load_qpairs(qp + 16 * c + 8, q);
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const float2 pb = pair_dots<TABLE>(cw[u].z, cw[u].w, q, dec);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].z), pb.x, S[u]);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].w), pb.y, S[u]);
        }
    }
}

// Stages head h's rotated query into the warp's pair table: entry 8 t + j holds
// (q~[16 t + j], q~[16 t + 8 + j]).
__device__ __forceinline__ void stage_query(const float* __restrict__ qt, int64_t h,
                                            float2* qs, int lane) {
    const float* qh = qt + h * D;
#pragma unroll
    for (int e = lane; e < 64; e += 32) {
        const int t = e >> 3, j = e & 7;
        qs[e] = make_float2(qh[16 * t + j], qh[16 * t + 8 + j]);
    }
    __syncwarp();
}

// Work is cut into items of kItem consecutive candidates of one query head; warp g of the
// grid takes items g, g + W, g + 2 W, ... (W warps in all), so within a stage the head, its
// unit's record base and its rotated query are the same for every lane.
constexpr int kItem = 256;
constexpr uint32_t kNoRec = 0xffffffffu;

struct StreamPos {
    int64_t it;            // item
    int s, nst;            // stage within the item, stages in the item
    int head, c0, cend;    // query head, first candidate, one past the item's last
    const uint8_t* ubase;  // records of the head's unit
};

template <bool TABLE>
__global__ void __launch_bounds__(kThr, kCtasPerSm)
rerank_kernel(const uint8_t* __restrict__ rec, const int32_t* __restrict__ cand,
              const float* __restrict__ qt, float* __restrict__ S, int32_t C, int64_t cmax,
              int64_t cap_pad, int64_t n, int group, int iph, int64_t items,
              uint32_t* __restrict__ shist, int* status, const float* __restrict__ lvt) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ float dec[16];   // table levels: code nibble -> signed level
    if constexpr (TABLE) {
        // the index's level table is written when the index is created, never by a search
        if (threadIdx.x < 16) dec[threadIdx.x] = lvt[16 + threadIdx.x];
        __syncthreads();
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = smem + warp * kWarpBytes;
    float2* qs = reinterpret_cast<float2*>(ring + kSlots * kStageBytes);
    const uint64_t* qp = reinterpret_cast<const uint64_t*>(qs);
    const int64_t W = static_cast<int64_t>(gridDim.x) * kWarps;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarps + warp;

    auto start_item = [&](StreamPos& p) {
        if (p.it >= items) return;
        p.head = static_cast<int>(p.it / iph);
        p.c0 = static_cast<int>(p.it - static_cast<int64_t>(p.head) * iph) * kItem;
        p.cend = min(C, p.c0 + kItem);
        p.nst = (p.cend - p.c0 + kStageRecs - 1) / kStageRecs;
        p.s = 0;
        p.ubase = rec + static_cast<int64_t>(p.head / group) * cap_pad * REC;
    };
    auto advance = [&](StreamPos& p) {
        if (++p.s == p.nst) {
            p.it += W;
            start_item(p);
        }
    };
    // candidate indices of this lane's records (rows lane, lane + 32) in the stage at p,
    // loaded one stage ahead of their use so the loads overlap the scoring of a stage
    struct Idx { uint32_t v[kPerLane]; };
    auto load_idx = [&](const StreamPos& p) -> Idx {
        Idx r;
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const int c = p.c0 + kStageRecs * p.s + 32 * u + lane;
            r.v[u] = (p.it < items && c < p.cend) ? static_cast<uint32_t>(cand[p.head * cmax + c])
                                                  : kNoRec;
        }
        return r;
    };
    // stage refill: for copy instruction j, lanes 8g..8g+7 move the 8 16-byte pieces of
    // record 4j + g (whose index lane (4j + g) mod 32 holds)
    auto issue = [&](int slot, const StreamPos& p, Idx idx) {
        if (p.it < items) {
#pragma unroll
            for (int u = 0; u < kPerLane; ++u) {
                if (idx.v[u] != kNoRec && idx.v[u] >= static_cast<uint64_t>(n)) {
                    atomicExch(status, ST_BADINDEX);  // never taken when the selection is consistent
                    idx.v[u] = kNoRec;
                }
            }
            uint8_t* dst0 = ring + slot * kStageBytes;
            const int piece = lane & 7, sub = lane >> 3;
#pragma unroll
            for (int j = 0; j < kStageRecs / 4; ++j) {
                const int rr = 4 * j + sub;
                const uint32_t ri = __shfl_sync(0xffffffffu, idx.v[j / 8], rr & 31);
                if (ri != kNoRec) {
                    const uint32_t dst = smem_addr(dst0 + piece_at(rr, piece));
                    const uint8_t* src = p.ubase + static_cast<uint64_t>(ri) * REC + piece * 16;
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src)
                                 : "memory");
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    pdl_wait();
    pdl_launch_dependents();
    StreamPos iss{gw, 0, 0, 0, 0, 0, rec}, sc{gw, 0, 0, 0, 0, 0, rec};
    start_item(iss);
    start_item(sc);
    // prologue: fill the ring
    Idx pend = load_idx(iss);
    for (int g = 0; g < kSlots; ++g) {
        issue(g, iss, pend);
        if (iss.it < items) advance(iss);
        pend = load_idx(iss);
    }

    int staged = -1;   // head whose query is in qs
#pragma unroll 1
    for (int g = 0; sc.it < items; ++g) {
        const int slot = g % kSlots;
        // the oldest committed group is this stage's; each lane waits for its own pieces and
        // the warp barrier makes every lane's pieces visible
        asm volatile("cp.async.wait_group %0;" :: "n"(kSlots - 1) : "memory");
        __syncwarp();
        if (sc.head != staged) {
            stage_query(qt, sc.head, qs, lane);
            staged = sc.head;
        }
        const uint8_t* st = ring + slot * kStageBytes;
        float sv[kPerLane];
        score_records<TABLE>(st, lane, qp, dec, sv);
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const int c = sc.c0 + kStageRecs * sc.s + 32 * u + lane;
            const bool ok = c < sc.cend;
            if (ok) S[sc.head * cmax + c] = sv[u];
            // the top-k's first radix level: count the values by their top order-key bits,
            // one global reduction per distinct bin in the warp (values cluster in few bins)
            const uint32_t bin = ok ? order_key(sv[u]) >> (32 - SBINS_BITS) : 0xffffffffu;
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (ok && lane == __ffs(peers) - 1)
                atomicAdd(&shist[(static_cast<int64_t>(sc.head) * SCOPIES + (gw & (SCOPIES - 1))) *
                                     SBINS + bin],
                          static_cast<uint32_t>(__popc(peers)));
        }
        __syncwarp();                        // every lane has read the slot and the query
        issue(slot, iss, pend);
        if (iss.it < items) advance(iss);
        pend = load_idx(iss);
        advance(sc);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // no copy in flight at exit
}

}  // namespace

cudaError_t launch_rerank(const pariskv_index* ix, int64_t C, cudaStream_t st) {
    if (C <= 0) return cudaSuccess;
    static std::atomic<uint64_t> smem_raised{0}, smem_raised_t{0};
    const bool table = ix->cfg.levels != PARISKV_LEVELS_UNIFORM;
    if (cudaError_t e = table ? raise_smem_limit(rerank_kernel<true>, kSmem, smem_raised_t)
                              : raise_smem_limit(rerank_kernel<false>, kSmem, smem_raised);
        e != cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int heads = ix->units * ix->cfg.group;
    const int iph = static_cast<int>(ceil_div(C, kItem));
    const int64_t items = static_cast<int64_t>(heads) * iph;
    const int grid =
        static_cast<int>(max64(1, min64(int64_t{kCtasPerSm} * sms, ceil_div(items, kWarps))));
    return launch_pdl(table ? rerank_kernel<true> : rerank_kernel<false>, grid, kThr, kSmem, st,
                      ix->rec, ix->cand, ix->qt, ix->S, static_cast<int32_t>(C), ix->cmax,
                      ix->cap_pad, ix->n, ix->cfg.group, iph, items, ix->shist, ix->status,
                      static_cast<const float*>(ix->lvt));
}

}  // namespace pkv
