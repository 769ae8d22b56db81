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
// eight lanes move one record, so a warp instruction moves four whole records): the kernel
// is persistent (two CTAs per SM), every warp owns a ring of kSlots stages of 16 records in
// shared memory (128 KB per SM), and a stage is refilled as soon as it has been scored. The
// candidate indices of the refill are loaded while the stage is scored. (Measured on B200:
// one 128-byte cp.async.bulk per record was several times slower than this.)
//
// Scoring: four lanes cooperate on a record, and each group of four scores two records at
// once so that their dependency chains interleave; lane p owns subspaces 4p..4p+3 (one 32-byte
// chunk: 4 code words + 4 factors) and keeps its 32 rotated-query coordinates in registers
// as fp32 pairs. Decoding is exact integer arithmetic: 8 sign-magnitude nibbles become offset
// nibbles u = vt + 8 with five SWAR instructions, a PRMT places u in the mantissa of 2^23 and
// one packed subtraction of 2^23 + 8 gives vt exactly as fp32. Two subspaces advance
// together in Blackwell's packed fp32x2 FMA (each half an ordinary IEEE fp32 FMA); the S
// chain then runs across the four lanes in order, lane p continuing lane p - 1's sum.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kWarps = 8;               // two persistent CTAs per SM; every warp gathers and scores
constexpr int kThr = 32 * kWarps;
constexpr int kSlots = 4;               // stages in flight per warp
constexpr int kStageRecs = 16;          // records per stage: two per four-lane group
constexpr int kStageBytes = kStageRecs * REC;
constexpr int kSmem = kWarps * kSlots * kStageBytes;

__device__ __forceinline__ uint32_t offset_nibbles(uint32_t w) {
    const uint32_t s = (w >> 3) & 0x11111111u;       // sign bit of each nibble as 0/1
    const uint32_t sm = s * 7u;                        // 7 in every negative nibble
    const uint32_t x = (w & 0x77777777u) ^ sm;         // mag, or 7 - mag when negative
    return x + (0x88888888u - sm);                     // + 8 (positive) or + 1 (negative)
}

template <int K>
__device__ __forceinline__ uint64_t level_pair(uint32_t xa, uint32_t xb) {
    // byte K of each word into the mantissa of 2^23: 2^23 + u exactly; minus (2^23 + 8) = vt
    const uint64_t kOff = pack2(-8388616.0f, -8388616.0f);
    return add2(pack2u(prmt_i<0x7650u + K>(xa, 0x4B000000u), prmt_i<0x7650u + K>(xb, 0x4B000000u)),
                kOff);
}

// p chains of the subspace pair (a, b): codes wa, wb; q pairs q[j] = (q~_{a,j}, q~_{b,j}).
__device__ __forceinline__ float2 pair_dots(uint32_t wa, uint32_t wb, const uint64_t q[8]) {
    const uint32_t ua = offset_nibbles(wa), ub = offset_nibbles(wb);
    const uint32_t ea = ua & 0x0F0F0F0Fu, oa = (ua >> 4) & 0x0F0F0F0Fu;   // dims 0, 2, 4, 6
    const uint32_t eb = ub & 0x0F0F0F0Fu, ob = (ub >> 4) & 0x0F0F0F0Fu;   // dims 1, 3, 5, 7
    uint64_t p = pack2(0.0f, 0.0f);
    p = fma2(level_pair<0>(ea, eb), q[0], p);
    p = fma2(level_pair<0>(oa, ob), q[1], p);
    p = fma2(level_pair<1>(ea, eb), q[2], p);
    p = fma2(level_pair<1>(oa, ob), q[3], p);
    p = fma2(level_pair<2>(ea, eb), q[4], p);
    p = fma2(level_pair<2>(oa, ob), q[5], p);
    p = fma2(level_pair<3>(ea, eb), q[6], p);
    p = fma2(level_pair<3>(oa, ob), q[7], p);
    return unpack2(p);
}

__device__ __forceinline__ void load_q(const float* __restrict__ qt, int64_t head, int p,
                                       uint64_t qa[8], uint64_t qb[8]) {
    const float* qh = qt + head * D + 32 * p;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        qa[j] = pack2(qh[j], qh[8 + j]);
        qb[j] = pack2(qh[16 + j], qh[24 + j]);
    }
}

__global__ void __launch_bounds__(kThr, 2)
rerank_kernel(const uint8_t* __restrict__ rec, const int32_t* __restrict__ cand,
              const float* __restrict__ qt, float* __restrict__ S, int64_t C, int64_t cmax,
              int64_t cap_pad, int64_t n, int group, int64_t total, int* status) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = lane & 3;            // part: subspaces 4p..4p+3
    const int slot_rec = lane >> 2;    // four-lane group: scores records slot_rec, slot_rec + 8
    uint8_t* ring = smem + warp * kSlots * kStageBytes;

    // this CTA's slice of the flattened (head, candidate) sequence, cut in 32-record stages;
    // the warp takes CTA stages warp, warp + kWarps, warp + 2 kWarps, ...
    const int64_t r0 = total * blockIdx.x / gridDim.x, r1 = total * (blockIdx.x + 1) / gridDim.x;
    const int64_t nstage = ceil_div(r1 - r0, kStageRecs);

    // stage refill: lane l < 16 holds the record number of the stage's l-th record; for copy
    // instruction j, lanes 8g..8g+7 move the 8 16-byte pieces of record 4j + g
    auto issue = [&](int slot, int64_t ridx, bool valid) {
        uint8_t* dst0 = ring + slot * kStageBytes;
        const int piece = lane & 7, sub = lane >> 3;
#pragma unroll
        for (int j = 0; j < kStageRecs / 4; ++j) {
            const int rr = 4 * j + sub;
            const int64_t ri = __shfl_sync(0xffffffffu, ridx, rr);
            const bool v = __shfl_sync(0xffffffffu, valid, rr);
            if (v) {
                const uint32_t dst = smem_addr(dst0 + rr * REC + piece * 16);
                const uint8_t* src = rec + ri * REC + piece * 16;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src)
                             : "memory");
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // (head, candidate) positions advance incrementally: one division at the start, then
    // an add and at most one wrap per step when C >= 32 (several for tiny candidate sets)
    auto wrap = [&](int64_t& h, int64_t& c) {
        while (c >= C) { c -= C; ++h; }
    };
    // record number of the stage's lane-th record, with its bounds check
    auto locate = [&](int64_t sh, int64_t sc, bool& valid) -> int64_t {
        if (!valid) return 0;
        int64_t head = sh, c = sc + lane;
        wrap(head, c);
        const int64_t i = cand[head * cmax + c];
        if (i < 0 || i >= n) {  // never taken when the selection is consistent
            atomicExch(status, ST_BADINDEX);
            valid = false;
            return 0;
        }
        const int64_t unit = static_cast<uint32_t>(head) / static_cast<uint32_t>(group);
        return unit * cap_pad + i;
    };
    constexpr int64_t kStep = static_cast<int64_t>(kWarps) * kStageRecs;
    const int64_t first = r0 + static_cast<int64_t>(warp) * kStageRecs;
    int64_t ih = first / C, ic = first - ih * C;    // issue stream: stage start (head, cand)
    int64_t hh = ih, hc = ic;                       // scoring stream

    // prologue: fill the ring
    for (int g = 0; g < kSlots; ++g) {
        const int64_t cs = warp + static_cast<int64_t>(kWarps) * g;
        const int64_t rs = r0 + cs * kStageRecs;
        bool valid = cs < nstage && lane < kStageRecs && rs + lane < r1;
        const int64_t ri = locate(ih, ic, valid);
        issue(g, ri, valid);
        ic += kStep;
        wrap(ih, ic);
    }

    int64_t cur_head = -1;
    uint64_t qa[8], qb[8];
#pragma unroll 1
    for (int64_t g = 0;; ++g) {
        const int64_t cs = warp + static_cast<int64_t>(kWarps) * g;
        if (cs >= nstage) break;
        const int slot = static_cast<int>(g % kSlots);
        // indices of the stage that will refill this slot (their load overlaps the scoring)
        const int64_t cs_next = cs + static_cast<int64_t>(kWarps) * kSlots;
        const int64_t rs_next = r0 + cs_next * kStageRecs;
        bool valid_next = cs_next < nstage && lane < kStageRecs && rs_next + lane < r1;
        const int64_t ri_next = locate(ih, ic, valid_next);
        ic += kStep;
        wrap(ih, ic);

        // the oldest committed group is this stage's; each lane waits for its own pieces and
        // the warp barrier makes every lane's pieces visible
        asm volatile("cp.async.wait_group %0;" :: "n"(kSlots - 1) : "memory");
        __syncwarp();
        const uint8_t* st = ring + slot * kStageBytes;
        const int64_t rs = r0 + cs * kStageRecs;
        // group slot_rec scores records slot_rec and slot_rec + 8 of the stage together
        bool ok[2];
        int64_t head[2], cc[2];
        uint4 w0[2], w1[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int rr = slot_rec + 8 * u;
            ok[u] = rs + rr < r1;
            head[u] = hh;
            cc[u] = hc + rr;
            wrap(head[u], cc[u]);
            w0[u] = *reinterpret_cast<const uint4*>(st + rr * REC + 32 * p);
            w1[u] = *reinterpret_cast<const uint4*>(st + rr * REC + 32 * p + 16);
        }
        float s[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (ok[u] && head[u] != cur_head) {
                load_q(qt, head[u], p, qa, qb);
                cur_head = head[u];
            }
            const float2 pa = pair_dots(w0[u].x, w0[u].y, qa);
            const float2 pb = pair_dots(w0[u].z, w0[u].w, qb);
            const float f0 = __uint_as_float(w1[u].x), f1 = __uint_as_float(w1[u].y);
            const float f2 = __uint_as_float(w1[u].z), f3 = __uint_as_float(w1[u].w);
            float t = 0.0f;
#pragma unroll
            for (int step = 0; step < 4; ++step) {
                const float prev = __shfl_up_sync(0xffffffffu, t, 1, 4);
                if (p == step) {
                    float x = step == 0 ? 0.0f : prev;
                    x = __fmaf_rn(f0, pa.x, x);
                    x = __fmaf_rn(f1, pa.y, x);
                    x = __fmaf_rn(f2, pb.x, x);
                    x = __fmaf_rn(f3, pb.y, x);
                    t = x;
                }
            }
            s[u] = t;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
            if (p == 3 && ok[u]) S[head[u] * cmax + cc[u]] = s[u];
        hc += kStep;
        wrap(hh, hc);
        __syncwarp();                        // every lane has read the slot before its refill
        issue(slot, ri_next, valid_next);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // no copy in flight at exit
}

}  // namespace

cudaError_t launch_rerank(const pariskv_index* ix, int64_t C, cudaStream_t st) {
    if (C <= 0) return cudaSuccess;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(rerank_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int heads = ix->units * ix->cfg.group;
    const int64_t total = static_cast<int64_t>(heads) * C;
    const int64_t stages = ceil_div(total, kStageRecs);
    const int grid = static_cast<int>(max64(1, min64(2LL * sms, ceil_div(stages, kWarps))));
    rerank_kernel<<<grid, kThr, kSmem, st>>>(ix->rec, ix->cand, ix->qt, ix->S, C, ix->cmax,
                                             ix->cap_pad, ix->n, ix->cfg.group, total,
                                             ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
