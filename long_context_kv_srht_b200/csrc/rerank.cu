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
// after every pair. Decoding is exact integer arithmetic on the code words of the two
// subspaces, which one shared-memory load leaves in a register pair: one LOP3 per half puts
// the offset-binary nibble u = vt + 8 of a dimension into the mantissa of 2^23 (scaled by a
// power of 16 that the staged query undoes exactly), and one packed subtraction gives vt as
// fp32. (Placing the nibbles with PRMT into two single registers needed about one register
// move per value to form the pair, 20 % more instructions per record.)
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
constexpr int kQBytes = 2 * D * 4;      // one head's rotated query, plain and scaled pairs
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

// Scaled decode (uniform levels): the code words of subspaces a and b form one 64-bit value
// w = {wa, wb} (a register pair as loaded), and dim j's nibble u sits at bits 4 j of each
// half. For j <= 4, (w & (15 << 4 j)) | bits(2^23) holds 2^23 + u 16^j in both halves;
// dims 5..7 take the same from w >> 16 with j - 4. Subtracting 2^23 + 8 16^e (e = j or
// j - 4) leaves vt 16^e exactly, and the query pair of dim j is staged as q~ 16^-e, so each
// FMA of the chain gets the exact product vt q~ and rounds exactly as fma(vt, q~, p) does.
// The scaling is exact while no query component is a nonzero value below 2^-100 (checked
// when the query is staged; such a query takes the unscaled path).
// The mask and the exponent bits live in registers (opaque to the compiler's constant
// folding), and each half is one LOP3 (w & m) | e writing straight into the pair that the
// packed subtraction reads, so no register moves are needed to form the pair.
__device__ __forceinline__ uint64_t opaque64(uint64_t v) {
    uint64_t r;
    asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t lev_scaled(uint64_t w, int sh, uint64_t kc) {
    const uint64_t m = opaque64(0x0000000F0000000Full << sh);
    const uint64_t e = opaque64(0x4B0000004B000000ull);
    uint64_t r;
    asm("{\n .reg .b32 wl, wh, ml, mh, el, eh, rl, rh;\n mov.b64 {wl, wh}, %1;\n mov.b64 {ml, mh}, %2;\n"
        " mov.b64 {el, eh}, %3;\n lop3.b32 rl, wl, ml, el, 0xEA;\n lop3.b32 rh, wh, mh, eh, 0xEA;\n"
        " mov.b64 %0, {rl, rh};\n}" : "=l"(r) : "l"(w), "l"(m), "l"(e));
    return add2(r, kc);
}
__device__ __forceinline__ float2 pair_dots_scaled(uint64_t w, const uint64_t q[8],
                                                   const uint64_t kc[5]) {
    uint64_t p = 0;   // (0.0f, 0.0f)
    p = fma2(lev_scaled(w, 0, kc[0]), q[0], p);
    p = fma2(lev_scaled(w, 4, kc[1]), q[1], p);
    p = fma2(lev_scaled(w, 8, kc[2]), q[2], p);
    p = fma2(lev_scaled(w, 12, kc[3]), q[3], p);
    p = fma2(lev_scaled(w, 16, kc[4]), q[4], p);
    const uint64_t v = w >> 16;
    p = fma2(lev_scaled(v, 4, kc[1]), q[5], p);
    p = fma2(lev_scaled(v, 8, kc[2]), q[6], p);
    p = fma2(lev_scaled(v, 12, kc[3]), q[7], p);
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
// t at qp + 8 t), qs_scaled the same pairs scaled for the scaled decode. Each query pair is
// read once for all the lane's records; every record keeps its own p and S chains in the
// defined order.
template <bool TABLE, bool SCALED>
__device__ __forceinline__ void score_records(const uint8_t* st, int row0, const uint64_t* qp,
                                              const float* dec, float S[kPerLane]) {
    const uint64_t kc[5] = {pack2(-8388616.0f, -8388616.0f), pack2(-8388736.0f, -8388736.0f),
                            pack2(-8390656.0f, -8390656.0f), pack2(-8421376.0f, -8421376.0f),
                            pack2(-8912896.0f, -8912896.0f)};   // -(2^23 + 8 16^e)
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) S[u] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {   // chunk c: subspaces 4c..4c+3
        ulonglong2 cw[kPerLane];
        uint4 fw[kPerLane];
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            cw[u] = *reinterpret_cast<const ulonglong2*>(st + piece_at(row0 + 32 * u, 2 * c));
            fw[u] = *reinterpret_cast<const uint4*>(st + piece_at(row0 + 32 * u, 2 * c + 1));
        }
        uint64_t q[8];
        load_qpairs(qp + 16 * c, q);
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const float2 pa =
                SCALED ? pair_dots_scaled(cw[u].x, q, kc)
                       : pair_dots<TABLE>(static_cast<uint32_t>(cw[u].x),
                                          static_cast<uint32_t>(cw[u].x >> 32), q, dec);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].x), pa.x, S[u]);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].y), pa.y, S[u]);
        }
        load_qpairs(qp + 16 * c + 8, q);
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const float2 pb =
                SCALED ? pair_dots_scaled(cw[u].y, q, kc)
                       : pair_dots<TABLE>(static_cast<uint32_t>(cw[u].y),
                                          static_cast<uint32_t>(cw[u].y >> 32), q, dec);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].z), pb.x, S[u]);
            S[u] = __fmaf_rn(__uint_as_float(fw[u].w), pb.y, S[u]);
        }
    }
}

// Stages head h's rotated query into the warp's pair tables: entry 8 t + j of qs holds
// (q~[16 t + j], q~[16 t + 8 + j]) and of qss the same pair times 16^-e (e = j for j <= 4,
// else j - 4) for the scaled decode. Returns whether the scaling is exact for this query.
__device__ __forceinline__ bool stage_query(const float* __restrict__ qt, int64_t h, float2* qs,
                                            float2* qss, int lane) {
    const float* qh = qt + h * D;
    bool tiny = false;
#pragma unroll
    for (int e = lane; e < 64; e += 32) {
        const int t = e >> 3, j = e & 7;
        const float a = qh[16 * t + j], b = qh[16 * t + 8 + j];
        qs[e] = make_float2(a, b);
        const float sc = j == 0 ? 1.0f : j == 1 || j == 5 ? 0.0625f : j == 2 || j == 6 ? 0.00390625f
                       : j == 3 || j == 7 ? 0.000244140625f : 1.52587890625e-05f;   // 16^-e
        qss[e] = make_float2(__fmul_rn(a, sc), __fmul_rn(b, sc));
        tiny |= (a != 0.0f && fabsf(a) < 7.8886091e-31f) || (b != 0.0f && fabsf(b) < 7.8886091e-31f);
    }
    const bool ok = !__any_sync(0xffffffffu, tiny);   // 7.8886091e-31 = 2^-100
    __syncwarp();
    return ok;
}

// Work is cut into stages of kStageRecs consecutive candidates of one query head, numbered
// head by head; warp g of the grid (W warps in all) takes the contiguous run of stages
// [total g / W, total (g + 1) / W), so every warp has the same number of stages to within
// one, and within a stage the head, its unit's record base and its rotated query are the
// same for every lane.
constexpr uint32_t kNoRec = 0xffffffffu;

struct StreamPos {
    int64_t t;             // stage (over all heads)
    int head, c0, cend;    // query head, first candidate, one past the stage's last
    const uint8_t* ubase;  // records of the head's unit
};

template <bool TABLE>
__global__ void __launch_bounds__(kThr, kCtasPerSm)
rerank_kernel(const uint8_t* __restrict__ rec, const int32_t* __restrict__ cand,
              const float* __restrict__ qt, float* __restrict__ S, int32_t C, int64_t cmax,
              int64_t cap_pad, int64_t n, int group, int64_t total,
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
    float2* qss = qs + 64;
    const uint64_t* qp = reinterpret_cast<const uint64_t*>(qs);
    const uint64_t* qps = reinterpret_cast<const uint64_t*>(qss);
    const int64_t W = static_cast<int64_t>(gridDim.x) * kWarps;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarps + warp;

    const int64_t nst = (C + kStageRecs - 1) / kStageRecs;   // stages per head
    const int64_t t_end = total * (gw + 1) / W;
    auto start_at = [&](StreamPos& p, int64_t t) {
        p.t = t;
        p.head = static_cast<int>(t / nst);
        p.c0 = static_cast<int>(t - p.head * nst) * kStageRecs;
        p.cend = min(C, p.c0 + kStageRecs);
        p.ubase = rec + static_cast<int64_t>(p.head / group) * cap_pad * REC;
    };
    auto advance = [&](StreamPos& p) {
        ++p.t;
        p.c0 += kStageRecs;
        if (p.c0 >= C) {
            ++p.head;
            p.c0 = 0;
            p.ubase = rec + static_cast<int64_t>(p.head / group) * cap_pad * REC;
        }
        p.cend = min(C, p.c0 + kStageRecs);
    };
    // candidate indices of this lane's records (rows lane, lane + 32) in the stage at p,
    // loaded one stage ahead of their use so the loads overlap the scoring of a stage
    struct Idx { uint32_t v[kPerLane]; };
    auto load_idx = [&](const StreamPos& p) -> Idx {
        Idx r;
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const int c = p.c0 + 32 * u + lane;
            r.v[u] = (p.t < t_end && c < p.cend) ? static_cast<uint32_t>(cand[p.head * cmax + c])
                                                 : kNoRec;
        }
        return r;
    };
    // stage refill: for copy instruction j, lanes 8g..8g+7 move the 8 16-byte pieces of
    // record 4j + g (whose index lane (4j + g) mod 32 holds)
    auto issue = [&](int slot, const StreamPos& p, Idx idx) {
        if (p.t < t_end) {
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
    StreamPos iss, sc;
    start_at(iss, total * gw / W);
    start_at(sc, total * gw / W);
    // prologue: fill the ring
    Idx pend = load_idx(iss);
    for (int g = 0; g < kSlots; ++g) {
        issue(g, iss, pend);
        if (iss.t < t_end) advance(iss);
        pend = load_idx(iss);
    }

    int staged = -1;       // head whose query is in qs
    bool scaled = false;   // its scaled pairs are exact
#pragma unroll 1
    for (int g = 0; sc.t < t_end; ++g) {
        const int slot = g % kSlots;
        // the oldest committed group is this stage's; each lane waits for its own pieces and
        // the warp barrier makes every lane's pieces visible
        asm volatile("cp.async.wait_group %0;" :: "n"(kSlots - 1) : "memory");
        __syncwarp();
        if (sc.head != staged) {
            scaled = stage_query(qt, sc.head, qs, qss, lane);
            staged = sc.head;
        }
        const uint8_t* st = ring + slot * kStageBytes;
        float sv[kPerLane];
        if (!TABLE && scaled) score_records<false, true>(st, lane, qps, dec, sv);
        else score_records<TABLE, false>(st, lane, qp, dec, sv);
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
            const int c = sc.c0 + 32 * u + lane;
            const bool ok = c < sc.cend && pkv_check(c < cmax, status);   // (checked build)
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
        if (iss.t < t_end) advance(iss);
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
    const int64_t total = static_cast<int64_t>(heads) * ceil_div(C, kStageRecs);
    const int grid = ix->rerank_ctas > 0   // (a launch shape forced by the determinism tests)
                         ? ix->rerank_ctas
                         : static_cast<int>(max64(1, min64(int64_t{kCtasPerSm} * sms,
                                                           ceil_div(total, kWarps))));
    return launch_pdl(table ? rerank_kernel<true> : rerank_kernel<false>, grid, kThr, kSmem, st,
                      ix->rec, ix->cand, ix->qt, ix->S, static_cast<int32_t>(C), ix->cmax,
                      ix->cap_pad, ix->n, ix->cfg.group, total, ix->shist, ix->status,
                      static_cast<const float*>(ix->lvt));
}

}  // namespace pkv
