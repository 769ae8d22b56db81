// rotate.cuh -- warp-level normalise + SRHT rotation of one d = 128 vector.
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations 1 ("Normalization
// and Rotation"): keys and queries are l2-normalised and rotated by one shared random
// orthogonal rotation implemented as an SRHT, y = H diag(s) x / (||x|| sqrt(d)), with H the
// Sylvester-ordered Walsh-Hadamard matrix.
//
// Register layout: lane L holds dims 4L .. 4L+3. The fast Walsh-Hadamard transform does the
// butterflies on dim bits 0-1 inside the lane and those on dim bits 2-6 with xor-shuffles
// over lane bits 0-4, so the whole transform is 7 butterfly stages with no shared memory.
#pragma once

#include "common.cuh"

namespace pkv {

// v: the lane's 4 input values (any scale). On return v holds the lane's 4 rotated,
// unit-norm coordinates and the function returns ||x|| (0 for a zero vector, which rotates
// to 0). sg: the lane's 4 SRHT signs (+-1.0f).
__device__ __forceinline__ float normalize_rotate_warp(float v[4], const float sg[4]) {
    const int lane = threadIdx.x & 31;
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) ss = __fmaf_rn(v[i], v[i], ss);
    ss = warp_sum(ss);
    const float nrm = __fsqrt_rn(ss);
    if (nrm == 0.0f) {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = 0.0f;
        return 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __fdiv_rn(v[i], nrm) * sg[i];
    // dim bit 0
    float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    // dim bit 1
    v[0] = a0 + a2; v[1] = a1 + a3; v[2] = a0 - a2; v[3] = a1 - a3;
    // dim bits 2..6 = lane bits 0..4
#pragma unroll
    for (int msk = 1; msk < 32; msk <<= 1) {
        const bool hi = (lane & msk) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, v[i], msk);
            v[i] = hi ? (o - v[i]) : (v[i] + o);
        }
    }
    const float inv_sqrt_d = 0.088388347648318440550f;  // 1/sqrt(128)
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] *= inv_sqrt_d;
    return nrm;
}

__device__ __forceinline__ void load_signs(const float* signs, float sg[4]) {
    const int lane = threadIdx.x & 31;
    float4 s = *reinterpret_cast<const float4*>(signs + 4 * lane);
    sg[0] = s.x; sg[1] = s.y; sg[2] = s.z; sg[3] = s.w;
}

}  // namespace pkv
