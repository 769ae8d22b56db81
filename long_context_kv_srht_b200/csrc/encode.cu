// encode.cu -- rotate-and-encode kernel: keys -> bucket ids, 4-bit RSQ codes, calibration
// factors. Used at prefill (pariskv_build_index) and for every appended decode key
// (pariskv_append).
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations:
//  - 1 "Analytic Centroids": each m-dim subspace direction of the rotated key is assigned to
//    the nearest sign centroid (+-1/sqrt(m)); with equal-norm centroids that is the sign
//    pattern, stored as one byte per subspace (bit j = dim j is negative).
//  - 2 "Quantization": one 4-bit code per dim, a sign bit and a 3-bit magnitude; the
//    magnitude is the nearest of 8 uniform levels over [0, max_j |y_j|] of its subspace:
//    mag = min(7, floor(7|y| / max + 1/2)) in IEEE fp32, in that order; or, with a level
//    table (levels derived from the rotation prior, or the caller's), the nearest table level
//    to |y| / max (see encode_subspace_table).
//  - 2 "Calibration": the per-(key, subspace) factor precomputed at prefill,
//    f = ||k|| * sum_j y_j^2 / sum_j vt_j y_j  (vt the signed integer levels), which folds
//    w_{i,b} = ||k|| ||y_b|| / <u_b, v_b> and the normalisation of v_b into one number so
//    that f * <vt_b, q~_b> = w_{i,b} <v_b, q~_b>. Both sums are fp32 FMA chains over j
//    ascending; f = 0 when the denominator is 0 (an all-zero subspace).
//
// One warp per key. Lane 2b holds dims 8b..8b+3 and lane 2b+1 dims 8b+4..8b+7, so one lane
// pair owns subspace b; after one shuffle each lane of the pair has all 8 coordinates and
// the even lane writes the id byte, the 32-bit code word and the factor.
//
// HBM layout written here (per unit = (sequence, KV head), per key i):
//  ids: 16 bytes at (unit * cap_pad + i) * 16; subspace b is stored at byte (b - i / 2) mod
//       16. The rotation lets the vote scan (one lane per pair of keys) read, at each step,
//       32 different subspaces across a warp and so hit 32 different shared-memory banks.
//  rec: 128 bytes at (unit * cap_pad + i) * 128, four 32-byte chunks; chunk p serves
//       subspaces 4p..4p+3: its first 16 bytes are their code words (subspace b's 8 codes in
//       one 32-bit word, dim j in nibble j), its last 16 bytes their factors f_b. A code is
//       stored in offset binary, u = vt + 8 in [1, 15], which the rerank turns into fp32 with
//       two integer operations. Nothing is lost: the code's sign bit is the sign of y_j, which
//       is bit j of the bucket id (for a zero level it is only there).
#include "common.cuh"
#include "internal.hpp"
#include "rotate.cuh"

namespace pkv {

namespace {

constexpr int kEncWarps = 8;

// Encodes one subspace from its 8 rotated coordinates w[0..7] (dim order) and the key norm.
__device__ __forceinline__ void encode_subspace(const float w[8], float knorm, uint32_t& id,
                                                uint32_t& code, float& factor) {
    id = 0;
    float mx = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        id |= (w[j] < 0.0f ? 1u : 0u) << j;
        mx = fmaxf(mx, fabsf(w[j]));
    }
    code = 0;
    float n2 = 0.0f, dot = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int q = 0;
        if (mx != 0.0f) {
            float t = __fmul_rn(7.0f, fabsf(w[j]));
            t = __fdiv_rn(t, mx);
            t = __fadd_rn(t, 0.5f);
            q = min(static_cast<int>(floorf(t)), 7);
        }
        const bool sgn = w[j] < 0.0f;
        const int lv = sgn ? -q : q;                               // signed level vt
        code |= static_cast<uint32_t>(lv + 8) << (4 * j);           // offset binary
        const float vt = sgn ? -static_cast<float>(q) : static_cast<float>(q);
        n2 = __fmaf_rn(w[j], w[j], n2);
        dot = __fmaf_rn(vt, w[j], dot);
    }
    const float num = __fmul_rn(knorm, n2);
    factor = (dot == 0.0f) ? 0.0f : __fdiv_rn(num, dot);
}

// The same with table levels (lv[0..7] ascending, th[i] = fp32 midpoint of lv[i-1], lv[i]):
// r = |y| / max in IEEE fp32, mag = #{i in 1..7 : r >= th[i]}, vt = +-lv[mag]; the code
// nibble is 8 + mag for y >= 0 and 7 - mag for y < 0, so that every (sign, magnitude) pair has
// its own nibble (with a table the level of magnitude 0 is not zero).
__device__ __forceinline__ void encode_subspace_table(const float w[8], float knorm,
                                                      const float lv[8], const float th[8],
                                                      uint32_t& id, uint32_t& code,
                                                      float& factor) {
    id = 0;
    float mx = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        id |= (w[j] < 0.0f ? 1u : 0u) << j;
        mx = fmaxf(mx, fabsf(w[j]));
    }
    code = 0;
    float n2 = 0.0f, dot = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int q = 0;
        float c = lv[0];
        if (mx != 0.0f) {
            const float r = __fdiv_rn(fabsf(w[j]), mx);
#pragma unroll
            for (int i = 1; i < 8; ++i)
                if (r >= th[i]) {
                    q = i;
                    c = lv[i];
                }
        }
        const bool sgn = w[j] < 0.0f;
        code |= static_cast<uint32_t>(sgn ? 7 - q : 8 + q) << (4 * j);
        const float vt = sgn ? -c : c;
        n2 = __fmaf_rn(w[j], w[j], n2);
        dot = __fmaf_rn(vt, w[j], dot);
    }
    const float num = __fmul_rn(knorm, n2);
    factor = (dot == 0.0f) ? 0.0f : __fdiv_rn(num, dot);
}

// Learned centroids (the comparator of the drift claim): the id of subspace b is the
// centroid c of largest <y_b, mu_c> (fp32 FMA chain over the 8 dims, ties to the lower c).
// Lanes 2b and 2b+1 both hold y_b; they scan centroids 0..127 and 128..255 and combine.
__device__ __forceinline__ uint32_t learned_id(const float w[8], const float* __restrict__ cb,
                                               bool odd) {
    const float* c0 = cb + (odd ? 128 * 8 : 0);
    float best = -INFINITY;
    int arg = 0;
#pragma unroll 4
    for (int c = 0; c < 128; ++c) {
        const float4 lo = __ldg(reinterpret_cast<const float4*>(c0 + 8 * c));
        const float4 hi = __ldg(reinterpret_cast<const float4*>(c0 + 8 * c + 4));
        float d = 0.0f;
        d = __fmaf_rn(lo.x, w[0], d); d = __fmaf_rn(lo.y, w[1], d);
        d = __fmaf_rn(lo.z, w[2], d); d = __fmaf_rn(lo.w, w[3], d);
        d = __fmaf_rn(hi.x, w[4], d); d = __fmaf_rn(hi.y, w[5], d);
        d = __fmaf_rn(hi.z, w[6], d); d = __fmaf_rn(hi.w, w[7], d);
        if (d > best) { best = d; arg = c; }
    }
    arg += odd ? 128 : 0;
    const float ob = __shfl_xor_sync(0xffffffffu, best, 1);
    const int oa = __shfl_xor_sync(0xffffffffu, arg, 1);
    if (ob > best || (ob == best && oa < arg)) arg = oa;
    return static_cast<uint32_t>(arg);
}

template <typename T, bool ROTATED, bool TABLE>
__global__ void __launch_bounds__(kEncWarps * 32)
encode_kernel(const T* __restrict__ src, const float* __restrict__ knorm_in, int64_t ld_tok,
              int64_t t, const float* __restrict__ signs, uint8_t* __restrict__ ids,
              uint8_t* __restrict__ rec, int64_t cap_pad, int64_t pos0,
              const float* __restrict__ lvt, const float* __restrict__ cent) {
    const int lane = threadIdx.x & 31;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * kEncWarps + (threadIdx.x >> 5);
    const int64_t unit = blockIdx.y;
    if (r >= t) return;
    const int64_t row = unit * ld_tok + r;

    float v[4];
    float knorm;
    if constexpr (ROTATED) {
        Elem<float>::load4(reinterpret_cast<const float*>(src) + row * D + 4 * lane, v);
        knorm = knorm_in[row];
    } else {
        float sg[4];
        load_signs(signs, sg);
        Elem<T>::load4(src + row * D + 4 * lane, v);
        knorm = normalize_rotate_warp(v, sg);
    }

    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __shfl_xor_sync(0xffffffffu, v[i], 1);
    float w[8];
    const bool odd = lane & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w[i] = odd ? o[i] : v[i];
        w[4 + i] = odd ? v[i] : o[i];
    }
    uint32_t id, code;
    float f;
    if constexpr (TABLE) {
        float lv[8], th[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            lv[i] = __ldg(lvt + i);
            th[i] = __ldg(lvt + 8 + i);
        }
        encode_subspace_table(w, knorm, lv, th, id, code, f);
    } else {
        encode_subspace(w, knorm, id, code, f);
    }
    if (cent)   // learned centroids replace the sign-pattern id (codes unchanged)
        id = learned_id(w, cent + (unit * NB + (lane >> 1)) * NC * 8, odd);

    if (!odd) {
        const int b = lane >> 1;
        const int64_t key = pos0 + r;
        const int64_t slot = unit * cap_pad + key;
        ids[slot * 16 + ((b - (key >> 1)) & 15)] = static_cast<uint8_t>(id);
        uint8_t* rr = rec + slot * REC + 32 * (b >> 2) + 4 * (b & 3);
        *reinterpret_cast<uint32_t*>(rr) = code;
        *reinterpret_cast<float*>(rr + 16) = f;
    }
}

template <typename T>
__global__ void __launch_bounds__(kEncWarps * 32)
rotate_kernel(const T* __restrict__ x, int64_t n, const float* __restrict__ signs,
              float* __restrict__ y, float* __restrict__ norm) {
    const int lane = threadIdx.x & 31;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * kEncWarps + (threadIdx.x >> 5);
    if (r >= n) return;
    float v[4], sg[4];
    load_signs(signs, sg);
    Elem<T>::load4(x + r * D + 4 * lane, v);
    const float nr = normalize_rotate_warp(v, sg);
    *reinterpret_cast<float4*>(y + r * D + 4 * lane) = make_float4(v[0], v[1], v[2], v[3]);
    if (lane == 0) norm[r] = nr;
}

}  // namespace

template <bool TABLE>
static void launch_encode_t(const pariskv_index* ix, const void* keys, const float* knorm,
                            int64_t ld_tok, int64_t t, int64_t pos0, bool rotated,
                            cudaStream_t st) {
    dim3 grid(static_cast<unsigned>(ceil_div(t, kEncWarps)), static_cast<unsigned>(ix->units));
    dim3 block(kEncWarps * 32);
    if (rotated) {
        encode_kernel<float, true, TABLE><<<grid, block, 0, st>>>(
            static_cast<const float*>(keys), knorm, ld_tok, t, ix->signs, ix->ids, ix->rec,
            ix->cap_pad, pos0, ix->lvt, ix->cent);
    } else if (ix->cfg.dtype == PARISKV_BF16) {
        encode_kernel<__nv_bfloat16, false, TABLE><<<grid, block, 0, st>>>(
            static_cast<const __nv_bfloat16*>(keys), nullptr, ld_tok, t, ix->signs, ix->ids,
            ix->rec, ix->cap_pad, pos0, ix->lvt, ix->cent);
    } else {
        encode_kernel<float, false, TABLE><<<grid, block, 0, st>>>(
            static_cast<const float*>(keys), nullptr, ld_tok, t, ix->signs, ix->ids, ix->rec,
            ix->cap_pad, pos0, ix->lvt, ix->cent);
    }
}

cudaError_t launch_encode(const pariskv_index* ix, const void* keys, const float* knorm,
                          int64_t ld_tok, int64_t t, int64_t pos0, bool rotated,
                          cudaStream_t st) {
    if (t <= 0) return cudaSuccess;
    if (ix->cfg.levels == PARISKV_LEVELS_UNIFORM)
        launch_encode_t<false>(ix, keys, knorm, ld_tok, t, pos0, rotated, st);
    else
        launch_encode_t<true>(ix, keys, knorm, ld_tok, t, pos0, rotated, st);
    return cudaGetLastError();
}

cudaError_t launch_rotate(const pariskv_config* cfg, const float* signs, const void* x,
                          int64_t n, float* y, float* norm, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    dim3 grid(static_cast<unsigned>(ceil_div(n, kEncWarps)));
    if (cfg->dtype == PARISKV_BF16)
        rotate_kernel<__nv_bfloat16><<<grid, kEncWarps * 32, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), n, signs, y, norm);
    else
        rotate_kernel<float><<<grid, kEncWarps * 32, 0, st>>>(static_cast<const float*>(x), n,
                                                              signs, y, norm);
    return cudaGetLastError();
}

}  // namespace pkv
