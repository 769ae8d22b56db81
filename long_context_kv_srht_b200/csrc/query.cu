// query.cu -- query-side top-rho centroid selection and vote lookup table.
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations 2 ("Coarse
// Candidate Generation"): for a query, each subspace selects the top-rho centroids most
// similar to the rotated query subspace, and keys in those buckets receive tiered votes.
//
// With sign centroids c (entries +-1/sqrt(m)), <q~_b, c> sqrt(m) = sum_j |q~_j| - 2 pen(c),
// where pen(c) sums |q~_j| over the dims j in which c's sign pattern differs from the
// query's own pattern c1. Ranking by (pen ascending, centroid id ascending) therefore ranks
// by similarity with ties to the lower id; pen is an fp32 sum over j ascending. The first
// rho centroids get vote weights w_rank1 (rank 1) and w_rest (ranks 2..rho); all others 0.
//
// One CTA per query head. Warp 0 rotates the query; then each of the 16 warps ranks the 256
// centroids of one subspace, 8 per lane, as 64-bit keys (pen bits << 32 | id): rho rounds
// of a warp-wide minimum for small rho, an all-pairs rank count for large rho.
//
// Output table layout: u8 [unit * packs + pack][b][c][4]; byte (g mod 4) of each 32-bit
// entry is query head g's weight, so one 32-bit lookup in the vote scan serves the four
// query heads of a pack.
#include "common.cuh"
#include "internal.hpp"
#include "rotate.cuh"

namespace pkv {

namespace {

constexpr int kQWarps = NB;   // one warp per subspace

template <typename T, bool ROTATED>
__global__ void __launch_bounds__(32 * kQWarps)
query_prep_kernel(const T* __restrict__ q, const float* __restrict__ qt_in,
                  const float* __restrict__ qn_in, const float* __restrict__ signs, int group,
                  int packs, int rho, int w1, int wr, float* __restrict__ qt_out,
                  float* __restrict__ qn_out, uint8_t* __restrict__ lut8,
                  const float* __restrict__ cent) {
    __shared__ float sq[D];
    const int head = blockIdx.x;  // unit * group + g
    const int unit = head / group, g = head % group;
    const int pack = g / PACK, slot = g % PACK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_launch_dependents();

    if (warp == 0) {
        float v[4];
        float nr;
        if constexpr (ROTATED) {
            Elem<float>::load4(qt_in + static_cast<int64_t>(head) * D + 4 * lane, v);
            nr = qn_in[head];
        } else {
            float sg[4];
            load_signs(signs, sg);
            Elem<T>::load4(q + static_cast<int64_t>(head) * D + 4 * lane, v);
            nr = normalize_rotate_warp(v, sg);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) sq[4 * lane + i] = v[i];
        *reinterpret_cast<float4*>(qt_out + static_cast<int64_t>(head) * D + 4 * lane) =
            make_float4(v[0], v[1], v[2], v[3]);
        if (lane == 0) qn_out[head] = nr;
    }
    __syncthreads();

    for (int b = warp; b < NB; b += kQWarps) {
        float a[8];
        uint32_t c1 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float x = sq[8 * b + j];
            a[j] = fabsf(x);
            c1 |= (x < 0.0f ? 1u : 0u) << j;
        }
        unsigned long long key[8];
        if (cent) {
            // learned centroids (the drift claim's comparator): rank by <mu_c, q~_b>
            // (fp32 FMA chain over j ascending) descending, ties to the lower id
            const float* cb = cent + (static_cast<int64_t>(unit) * NB + b) * NC * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t c = static_cast<uint32_t>(lane + 32 * i);
                float sim = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) sim = __fmaf_rn(cb[c * 8 + j], sq[8 * b + j], sim);
                key[i] = (static_cast<unsigned long long>(~order_key(sim)) << 32) | c;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t c = static_cast<uint32_t>(lane + 32 * i);
                const uint32_t diff = c ^ c1;
                float pen = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if ((diff >> j) & 1u) pen = __fadd_rn(pen, a[j]);
                key[i] = (static_cast<unsigned long long>(__float_as_uint(pen)) << 32) | c;
            }
        }
        uint32_t wgt[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) wgt[i] = 0;
        if (rho <= 32) {
            uint32_t taken = 0;
            for (int r = 0; r < rho; ++r) {
                unsigned long long best = ~0ull;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (!((taken >> i) & 1u) && key[i] < best) best = key[i];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
                    best = other < best ? other : best;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (key[i] == best) {
                        taken |= 1u << i;
                        wgt[i] = r == 0 ? w1 : wr;
                    }
            }
        } else {
            uint32_t rank[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) rank[i] = 0;
            for (int src = 0; src < 32; ++src) {
#pragma unroll
                for (int ii = 0; ii < 8; ++ii) {
                    const unsigned long long other = __shfl_sync(0xffffffffu, key[ii], src);
#pragma unroll
                    for (int i = 0; i < 8; ++i) rank[i] += other < key[i] ? 1u : 0u;
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                wgt[i] = rank[i] == 0 ? w1 : (rank[i] < static_cast<uint32_t>(rho) ? wr : 0u);
        }
        uint8_t* out = lut8 + ((static_cast<int64_t>(unit) * packs + pack) * NB + b) * NC * 4;
#pragma unroll
        for (int i = 0; i < 8; ++i) out[(lane + 32 * i) * 4 + slot] = static_cast<uint8_t>(wgt[i]);
    }
}

}  // namespace

cudaError_t launch_query_prep(const pariskv_index* ix, const void* q, const float* qt_in,
                              const float* qn_in, bool rotated, cudaStream_t st) {
    const auto& c = ix->cfg;
    const int heads = ix->units * c.group;
    uint8_t* lut8 = reinterpret_cast<uint8_t*>(ix->lut);
    if (rotated)
        return launch_pdl(query_prep_kernel<float, true>, heads, 32 * kQWarps, 0, st, nullptr, qt_in,
                          qn_in, ix->signs, c.group, ix->packs, c.rho, c.w_rank1, c.w_rest,
                          ix->qt, ix->qnorm, lut8, static_cast<const float*>(ix->cent));
    else if (c.dtype == PARISKV_BF16)
        return launch_pdl(query_prep_kernel<__nv_bfloat16, false>, heads, 32 * kQWarps, 0, st,
                          static_cast<const __nv_bfloat16*>(q), nullptr, nullptr, ix->signs,
                          c.group, ix->packs, c.rho, c.w_rank1, c.w_rest, ix->qt, ix->qnorm,
                          lut8, static_cast<const float*>(ix->cent));
    else
        return launch_pdl(query_prep_kernel<float, false>, heads, 32 * kQWarps, 0, st,
                          static_cast<const float*>(q), nullptr, nullptr, ix->signs, c.group,
                          ix->packs, c.rho, c.w_rank1, c.w_rest, ix->qt, ix->qnorm, lut8,
                          static_cast<const float*>(ix->cent));
}

}  // namespace pkv
