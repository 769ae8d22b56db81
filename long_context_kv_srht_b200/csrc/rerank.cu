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
// Four lanes cooperate on a candidate. Lane p of the group owns subspaces 4p..4p+3 and
// fetches exactly their 32-byte chunk of the candidate's 128-byte record (4 code words + 4
// factors) with one 256-bit non-allocating load, so a warp instruction reads 8 whole records
// and only the candidates' codes cross HBM. The lane keeps its 32 rotated-query coordinates
// in registers as fp32 pairs. Decoding is exact integer arithmetic:
//  - 8 sign-magnitude nibbles of a subspace become offset nibbles u = vt + 8 with five SWAR
//    instructions (u = (mag ^ 7s) + 8 - 7s per nibble; no nibble carries);
//  - a PRMT places u in the mantissa of 2^23, and one packed subtraction of 2^23 + 8 gives
//    vt exactly as fp32.
// Two subspaces advance together in Blackwell's packed fp32x2 FMA (each lane of the pair an
// ordinary IEEE fp32 FMA). The S chain then runs across the four lanes in order: lane p
// continues the running sum of lane p - 1 through its four subspaces.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kThr = 256;
constexpr int kPerPass = kThr / 4;  // candidates per block and pass
constexpr int kUnroll = 2;          // candidates in flight per lane group

__device__ __forceinline__ uint32_t offset_nibbles(uint32_t w) {
    const uint32_t s = (w >> 3) & 0x11111111u;       // sign bit of each nibble as 0/1
    const uint32_t sm = s * 7u;                        // 7 in every negative nibble
    const uint32_t x = (w & 0x77777777u) ^ sm;         // mag, or 7 - mag when negative
    return x + (0x88888888u - sm);                     // + 8 (positive) or + 1 (negative)
}

// p chains of the subspace pair (a, b): codes wa, wb; q pairs q[j] = (q~_{a,j}, q~_{b,j}).
__device__ __forceinline__ float2 pair_dots(uint32_t wa, uint32_t wb, const uint64_t q[8]) {
    const uint64_t kOff = pack2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
    const uint32_t ua = offset_nibbles(wa), ub = offset_nibbles(wb);
    const uint32_t ea = ua & 0x0F0F0F0Fu, oa = (ua >> 4) & 0x0F0F0F0Fu;
    const uint32_t eb = ub & 0x0F0F0F0Fu, ob = (ub >> 4) & 0x0F0F0F0Fu;
    uint64_t p = pack2(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        const uint32_t sel = 0x7650u + (j >> 1);
        uint64_t v = add2(pack2u(prmt(ea, 0x4B000000u, sel), prmt(eb, 0x4B000000u, sel)), kOff);
        p = fma2(v, q[j], p);
        v = add2(pack2u(prmt(oa, 0x4B000000u, sel), prmt(ob, 0x4B000000u, sel)), kOff);
        p = fma2(v, q[j + 1], p);
    }
    return unpack2(p);
}

__global__ void __launch_bounds__(kThr)
rerank_kernel(const uint8_t* __restrict__ rec, const int32_t* __restrict__ cand,
              const float* __restrict__ qt, float* __restrict__ S, int64_t C, int64_t cmax,
              int64_t cap_pad, int64_t n, int group, int* status) {
    const int head = blockIdx.y;
    const int64_t unit = head / group;
    const int lane = threadIdx.x & 31;
    const int p = lane & 3;             // part: subspaces 4p..4p+3
    const int slot = threadIdx.x >> 2;  // candidate slot in the pass

    uint64_t qa[8], qb[8];
    {
        const float* qh = qt + static_cast<int64_t>(head) * D + 32 * p;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            qa[j] = pack2(qh[j], qh[8 + j]);
            qb[j] = pack2(qh[16 + j], qh[24 + j]);
        }
    }
    const int64_t per = round_up(ceil_div(C, gridDim.x), kPerPass * kUnroll);
    const int64_t c0 = per * blockIdx.x, c1 = min64(C, c0 + per);
    const int32_t* ch = cand + head * cmax;
    float* Sh = S + head * cmax;
    const uint8_t* rbase = rec + unit * cap_pad * REC + 32 * p;

    for (int64_t cb = c0; cb < c1; cb += kPerPass * kUnroll) {
        u32x8 r[kUnroll];
        bool ok[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t c = cb + u * kPerPass + slot;
            ok[u] = c < c1;
            const int64_t i = ok[u] ? ch[c] : 0;
            if (ok[u] && (i < 0 || i >= n)) {  // never taken when the selection is consistent
                atomicExch(status, ST_BADINDEX);
                ok[u] = false;
            }
            if (ok[u]) r[u] = ldg_stream_u256(rbase + i * REC);
            else
#pragma unroll
                for (int w = 0; w < 8; ++w) r[u].w[w] = 0u;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const float2 pa = pair_dots(r[u].w[0], r[u].w[1], qa);
            const float2 pb = pair_dots(r[u].w[2], r[u].w[3], qb);
            const float f0 = __uint_as_float(r[u].w[4]), f1 = __uint_as_float(r[u].w[5]);
            const float f2 = __uint_as_float(r[u].w[6]), f3 = __uint_as_float(r[u].w[7]);
            float s = 0.0f;
#pragma unroll
            for (int step = 0; step < 4; ++step) {
                const float prev = __shfl_up_sync(0xffffffffu, s, 1, 4);
                if (p == step) {
                    float t = step == 0 ? 0.0f : prev;
                    t = __fmaf_rn(f0, pa.x, t);
                    t = __fmaf_rn(f1, pa.y, t);
                    t = __fmaf_rn(f2, pb.x, t);
                    t = __fmaf_rn(f3, pb.y, t);
                    s = t;
                }
            }
            if (p == 3 && ok[u]) Sh[cb + u * kPerPass + slot] = s;
        }
    }
}

}  // namespace

cudaError_t launch_rerank(const pariskv_index* ix, int64_t C, cudaStream_t st) {
    if (C <= 0) return cudaSuccess;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int heads = ix->units * ix->cfg.group;
    const int64_t want = ceil_div(8LL * sms, heads);
    const int64_t most = ceil_div(C, kPerPass * kUnroll);
    dim3 grid(static_cast<unsigned>(max64(1, min64(want, most))), static_cast<unsigned>(heads));
    rerank_kernel<<<grid, kThr, 0, st>>>(ix->rec, ix->cand, ix->qt, ix->S, C, ix->cmax,
                                         ix->cap_pad, ix->n, ix->cfg.group, ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
