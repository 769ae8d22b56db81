// rerank.cu -- RSQ-IP rerank of the candidates from their compact codes.
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations 2 ("Candidate
// Reranking (RSQ-IP)", "Estimation"): <k, q> is estimated as ||q|| sum_b w_{i,b} <v_{i,b},
// q~_b> without touching the full-precision key. With the folded per-(key, subspace)
// factor f_{i,b} written at encode time, the value ranked here is
//     S_i = sum_b f_{i,b} p_{i,b},    p_{i,b} = sum_j vt_{i,b,j} q~_{b,j},
// where vt are the signed integer magnitude levels. Both sums are fp32 FMA chains in
// ascending order (p over j from 0.0f, then S over b from 0.0f), the same order as the
// reference definition, so S is bit-reproducible; est = ||q|| S.
//
// One thread per candidate. The thread streams the candidate's 128-byte record (64 B of
// codes, 16 fp32 factors) with eight 16-byte non-allocating loads, so only the candidates'
// codes cross HBM. Decoding is exact integer arithmetic:
//  - 8 sign-magnitude nibbles of a subspace become offset nibbles u = vt + 8 with five SWAR
//    instructions (u = (mag ^ 7s) + 8 - 7s per nibble; no nibble carries);
//  - a PRMT places u in the mantissa of 2^23, and one packed subtraction of 2^23 + 8 gives
//    vt exactly as fp32.
// Subspaces are processed in pairs with Blackwell's packed fp32x2 FMA/ADD: the two p chains
// of a pair advance together in one instruction, each lane an ordinary IEEE fp32 FMA.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kThr = 256;

__device__ __forceinline__ uint32_t offset_nibbles(uint32_t w) {
    const uint32_t s = (w >> 3) & 0x11111111u;       // sign bit of each nibble as 0/1
    const uint32_t sm = s * 7u;                        // 7 in every negative nibble
    const uint32_t x = (w & 0x77777777u) ^ sm;         // mag, or 7 - mag when negative
    return x + (0x88888888u - sm);                     // + 8 (positive) or + 1 (negative)
}

__global__ void __launch_bounds__(kThr)
rerank_kernel(const uint8_t* __restrict__ rec, const int32_t* __restrict__ cand,
              const float* __restrict__ qt, float* __restrict__ S, int64_t C, int64_t cmax,
              int64_t cap_pad, int64_t n, int group, int* status) {
    __shared__ __align__(16) float qp[8][8][2];  // (subspace pair, dim, member of pair)
    const int head = blockIdx.y;
    const int64_t unit = head / group;
    if (threadIdx.x < D) {
        const int dim = threadIdx.x;
        const int b = dim >> 3, j = dim & 7;
        qp[b >> 1][j][b & 1] = qt[static_cast<int64_t>(head) * D + dim];
    }
    __syncthreads();

    const int64_t c = static_cast<int64_t>(blockIdx.x) * kThr + threadIdx.x;
    if (c >= C) return;
    const int64_t i = cand[head * cmax + c];
    if (i < 0 || i >= n) {  // never taken when the selection is consistent
        atomicExch(status, ST_BADINDEX);
        S[head * cmax + c] = -INFINITY;
        return;
    }
    const uint8_t* r = rec + (unit * cap_pad + i) * REC;
    uint32_t code[16];
    float fac[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = ldg_stream_u128(r + 16 * q);
        code[4 * q] = v.x; code[4 * q + 1] = v.y; code[4 * q + 2] = v.z; code[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = ldg_stream_u128(r + 64 + 16 * q);
        fac[4 * q] = __uint_as_float(v.x); fac[4 * q + 1] = __uint_as_float(v.y);
        fac[4 * q + 2] = __uint_as_float(v.z); fac[4 * q + 3] = __uint_as_float(v.w);
    }

    const uint64_t kOff = pack2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
    const uint32_t qbase = smem_addr(&qp[0][0][0]);
    float s = 0.0f;
#pragma unroll
    for (int bp = 0; bp < 8; ++bp) {
        const uint32_t u0 = offset_nibbles(code[2 * bp]);
        const uint32_t u1 = offset_nibbles(code[2 * bp + 1]);
        const uint32_t e0 = u0 & 0x0F0F0F0Fu, o0 = (u0 >> 4) & 0x0F0F0F0Fu;
        const uint32_t e1 = u1 & 0x0F0F0F0Fu, o1 = (u1 >> 4) & 0x0F0F0F0Fu;
        uint64_t p = pack2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const uint4 qq = lds_u128(qbase + (bp * 16 + j * 2) * 4);  // dims j, j+1 of the pair
            const uint32_t sel = 0x7650u + (j >> 1);
            // dim j (even nibble)
            uint64_t v = add2(pack2u(prmt(e0, 0x4B000000u, sel), prmt(e1, 0x4B000000u, sel)), kOff);
            p = fma2(v, pack2u(qq.x, qq.y), p);
            // dim j + 1 (odd nibble)
            v = add2(pack2u(prmt(o0, 0x4B000000u, sel), prmt(o1, 0x4B000000u, sel)), kOff);
            p = fma2(v, pack2u(qq.z, qq.w), p);
        }
        const float2 pb = unpack2(p);
        s = __fmaf_rn(fac[2 * bp], pb.x, s);
        s = __fmaf_rn(fac[2 * bp + 1], pb.y, s);
    }
    S[head * cmax + c] = s;
}

}  // namespace

cudaError_t launch_rerank(const pariskv_index* ix, int64_t C, cudaStream_t st) {
    if (C <= 0) return cudaSuccess;
    dim3 grid(static_cast<unsigned>(ceil_div(C, kThr)),
              static_cast<unsigned>(ix->units * ix->cfg.group));
    rerank_kernel<<<grid, kThr, 0, st>>>(ix->rec, ix->cand, ix->qt, ix->S, C, ix->cmax,
                                         ix->cap_pad, ix->n, ix->cfg.group, ix->status);
    return cudaGetLastError();
}

}  // namespace pkv
