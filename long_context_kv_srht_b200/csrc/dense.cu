// dense.cu -- dense decode attention over every cached token: the full-attention baseline
// that "Technical Summary: ParisKV" (Key Contributions 3, Results) and "ParisKV: Fast and
// Drift-Robust KV-Cache Retrieval for Long-Context LLMs" (abstract) compare ParisKV against
// (FlashAttention-style full attention, with K/V resident in HBM):
//     o_h = sum_{t < n} softmax_t(scale * <q_h, K_t>) V_t,   K/V of KV head h / group.
//
// Decode attention is a stream over K and V (512 bytes per token per KV head in bf16) with
// little arithmetic per byte, so it is bound by HBM bandwidth; the design goal is to read
// every K/V byte exactly once and to spend few instructions per token:
//  - one CTA serves all `group` (<= 8) query heads of a KV head (GQA), so a K/V tile is read
//    from HBM once per KV head, not once per query head;
//  - split-K over the token axis: CTA (split, unit) streams whole 64-token tiles of its unit,
//    two CTAs per SM, one wave;
//  - tiles are staged in shared memory by a 3-stage cp.async ring (16-byte copies; a tile's K
//    and V rows are contiguous in HBM), the 16-byte chunks of each row XOR-swizzled by the row
//    index so the 8x8 matrix loads below are bank-conflict-free;
//  - both products run on the tensor cores with mma.sync (m16n8k16, bf16 in, fp32
//    accumulate), each warp taking 16 tokens of a tile: S^T = K Q^T puts the 16 tokens in M
//    and the query heads in N (8 columns: every head of the group); O^T += V^T P^T puts 16
//    output dims in M (8 tiles for 128) and the heads in N, so a lane's softmax state and its
//    output accumulators belong to the same two heads and the rescaling needs no shuffles;
//  - P enters the second product as bf16 hi + lo parts (two MMAs), so the weights keep about
//    16 significant bits (q, K and V are bf16 and exact); the C fragment of P becomes the B
//    fragment by an 8x8 register transpose (movmatrix);
//  - online softmax per 16-token block in base 2 (scale * log2(e) applied to S in fp32);
//  - the 4 warps merge in shared memory and each head's split partial (128 accumulators, max,
//    denominator) goes to the workspace format of the sparse attention, whose log-sum-exp
//    combine kernel finishes the job.
#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kDW = 4;                        // warps per CTA, 16 tokens each per tile
constexpr int kTile = 16 * kDW;               // tokens per stage
constexpr int kStages = 3;
constexpr int kRowB = D * 2;                  // bytes per bf16 row
constexpr int kTileB = kTile * kRowB;         // 16 KiB per tensor and stage
constexpr int kSmem = 2 * kStages * kTileB;
constexpr int kHeadsN = 8;                    // N of the MMAs: query heads per KV head
constexpr int kLoadsPerThread = 2 * kTile * (kRowB / 16) / (kDW * 32);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
static_assert(kDW * kHeadsN * kAttendPart * sizeof(float) <= static_cast<size_t>(kSmem),
              "the merge scratch must fit in the stage buffers");
static_assert(kLoadsPerThread * kDW * 32 == 2 * kTile * (kRowB / 16), "whole tiles per pass");

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t r[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t r[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// d += a * b (m16n8k16, bf16 inputs, fp32 accumulators)
__device__ __forceinline__ void mma_bf16(float d[4], const uint32_t a[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fragment of an 8x8 b16 matrix -> fragment of its transpose
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ uint32_t bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 bf2_f(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__global__ void __launch_bounds__(kDW * 32, 2)
dense_attend_kernel(const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ K,
                    const uint8_t* __restrict__ V, int64_t ld_tok, int64_t n, float scale,
                    int group, int nsplit, float* __restrict__ work) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* sK = smem;
    uint8_t* sV = smem + kStages * kTileB;
    const int64_t u = blockIdx.y;
    const int split = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;     // fragment row / column pair of this lane

    const int64_t tiles = ceil_div(n, kTile);
    const int64_t tb0 = tiles * split / nsplit;
    const int64_t ntile = tiles * (split + 1) / nsplit - tb0;
    const uint8_t* Kb = K + u * ld_tok * kRowB;
    const uint8_t* Vb = V + u * ld_tok * kRowB;

    // stage a tile: 2 tensors x 64 rows x 16 chunks of 16 bytes; rows past n are zero-filled
    // (and masked below)
    auto load_tile = [&](int64_t tile, int stage) {
        const int64_t t0 = (tb0 + tile) * kTile;
#pragma unroll
        for (int j = 0; j < kLoadsPerThread; ++j) {
            const int id = tid + kDW * 32 * j;
            const int tensor = id / (kTile * 16), row = (id >> 4) & (kTile - 1), c = id & 15;
            const int64_t tok = t0 + row;
            const bool ok = tok < n;
            const uint8_t* src = (tensor ? Vb : Kb) + (ok ? tok : 0) * kRowB + c * 16;
            const uint32_t dst = smem_addr((tensor ? sV : sK) + stage * kTileB + row * kRowB +
                                           ((c ^ (row & 7)) << 4));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                         :: "r"(dst), "l"(src), "r"(ok ? 16 : 0) : "memory");
        }
    };
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < ntile) load_tile(s, s);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }

    // B fragments of Q^T (k = dims, n = heads): head g, dims 16s + 2t (+1) and 16s + 8 + 2t
    // (+1); heads past the group are zero
    uint32_t qb[8][2];
    {
        const uint32_t* qh = reinterpret_cast<const uint32_t*>(q + (u * group + g) * D);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            qb[s][0] = g < group ? qh[8 * s + t] : 0u;
            qb[s][1] = g < group ? qh[8 * s + 4 + t] : 0u;
        }
    }
    const float qs = scale * kLog2e;

    // this lane's state: heads 2t and 2t+1 (base-2 max, denominator); O^T accumulators of
    // dim tile i: (dim 16i+g, heads 2t, 2t+1), (dim 16i+g+8, heads 2t, 2t+1)
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;

    // ldmatrix row addresses: lane = 8 * matrix + row
    const int mi = lane >> 3, j8 = lane & 7;
    const int krow = 16 * warp + j8 + 8 * (mi & 1);     // K as A (rows = tokens, k = dims)
    const int kc = mi >> 1;
    const int vrow = 16 * warp + j8 + 8 * (mi >> 1);    // V^T as A (rows = dims, k = tokens)
    const int vc = mi & 1;

    for (int64_t it = 0; it < ntile; ++it) {
        asm volatile("cp.async.wait_group %0;" :: "n"(kStages - 2) : "memory");
        __syncthreads();   // tile `it` is visible; every warp is done with tile it - 1
        if (it + kStages - 1 < ntile) load_tile(it + kStages - 1, (it + kStages - 1) % kStages);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const int st = static_cast<int>(it % kStages);
        const uint32_t kbase = smem_addr(sK + st * kTileB + krow * kRowB);
        const uint32_t vbase = smem_addr(sV + st * kTileB + vrow * kRowB);

        // S^T: 16 tokens x 8 heads
        float sacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            uint32_t a[4];
            ldsm_x4(kbase + (((2 * s + kc) ^ (krow & 7)) << 4), a);
            mma_bf16(sacc, a, qb[s][0], qb[s][1]);
        }
        // sacc[0..1]: token g, heads 2t, 2t+1; sacc[2..3]: token g+8
        const int64_t tok = (tb0 + it) * kTile + 16 * warp + g;
        float s0 = sacc[0] * qs, s1 = sacc[1] * qs, s2 = sacc[2] * qs, s3 = sacc[3] * qs;
        if (tok >= n) s0 = s1 = -INFINITY;
        if (tok + 8 >= n) s2 = s3 = -INFINITY;
        float b0 = fmaxf(s0, s2), b1 = fmaxf(s1, s3);
#pragma unroll
        for (int x = 4; x < 32; x <<= 1) {
            b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, x));
            b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, x));
        }
        const float n0 = fmaxf(m0, b0), n1 = fmaxf(m1, b1);
        const float c0 = n0 == -INFINITY ? 1.0f : exp2f(m0 - n0);
        const float c1 = n1 == -INFINITY ? 1.0f : exp2f(m1 - n1);
        const float p0 = n0 == -INFINITY ? 0.0f : exp2f(s0 - n0);
        const float p2 = n0 == -INFINITY ? 0.0f : exp2f(s2 - n0);
        const float p1 = n1 == -INFINITY ? 0.0f : exp2f(s1 - n1);
        const float p3 = n1 == -INFINITY ? 0.0f : exp2f(s3 - n1);
        float r0 = p0 + p2, r1 = p1 + p3;
#pragma unroll
        for (int x = 4; x < 32; x <<= 1) {
            r0 += __shfl_xor_sync(0xffffffffu, r0, x);
            r1 += __shfl_xor_sync(0xffffffffu, r1, x);
        }
        l0 = l0 * c0 + r0;
        l1 = l1 * c1 + r1;
        m0 = n0;
        m1 = n1;
        if (!__all_sync(0xffffffffu, c0 == 1.0f && c1 == 1.0f)) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                o[i][0] *= c0; o[i][1] *= c1; o[i][2] *= c0; o[i][3] *= c1;
            }
        }
        // P^T as B fragments (k = tokens, n = heads): bf16 hi and lo parts
        const uint32_t h01 = bf2(p0, p1), h23 = bf2(p2, p3);
        const float2 f01 = bf2_f(h01), f23 = bf2_f(h23);
        const uint32_t l01 = bf2(p0 - f01.x, p1 - f01.y), l23 = bf2(p2 - f23.x, p3 - f23.y);
        const uint32_t bh0 = movm_t(h01), bh1 = movm_t(h23);
        const uint32_t bl0 = movm_t(l01), bl1 = movm_t(l23);
        // O^T += V^T P^T over the 8 tiles of 16 output dims
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t a[4];
            ldsm_x4_t(vbase + (((2 * i + vc) ^ (vrow & 7)) << 4), a);
            mma_bf16(o[i], a, bh0, bh1);
            mma_bf16(o[i], a, bl0, bl1);
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();   // the stage buffers become the merge scratch

    // per-warp partials -> scratch [warp][head][kAttendPart]
    float* sc = reinterpret_cast<float*>(smem);
    {
        float* w0 = sc + (warp * kHeadsN + 2 * t) * kAttendPart;
        float* w1 = w0 + kAttendPart;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            w0[16 * i + g] = o[i][0];
            w1[16 * i + g] = o[i][1];
            w0[16 * i + g + 8] = o[i][2];
            w1[16 * i + g + 8] = o[i][3];
        }
        if (g == 0) {
            w0[D] = m0; w0[D + 1] = l0;
            w1[D] = m1; w1[D + 1] = l1;
        }
    }
    __syncthreads();
    for (int h = warp; h < group; h += kDW) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDW; ++w) M = fmaxf(M, sc[(w * kHeadsN + h) * kAttendPart + D]);
        float den = 0.0f, a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < kDW; ++w) {
            const float* src = sc + (w * kHeadsN + h) * kAttendPart;
            const float f = src[D] == -INFINITY ? 0.0f : exp2f(src[D] - M);
            den += src[D + 1] * f;
            const float4 v = *reinterpret_cast<const float4*>(src + 4 * lane);
            a[0] += v.x * f; a[1] += v.y * f; a[2] += v.z * f; a[3] += v.w * f;
        }
        float* out = work + ((u * group + h) * nsplit + split) * kAttendPart;
        *reinterpret_cast<float4*>(out + 4 * lane) = make_float4(a[0], a[1], a[2], a[3]);
        if (lane == 0) {
            out[D] = M == -INFINITY ? M : M * kLn2;   // natural-log units, as the combine expects
            out[D + 1] = den;
        }
    }
}

}  // namespace

int dense_splits(int units, int64_t n, int num_sms) {
    // one wave of two CTAs per SM, every split at least one tile
    const int64_t want = ceil_div(2LL * num_sms, units);
    return static_cast<int>(max64(1, min64(want, ceil_div(n, kTile))));
}

cudaError_t launch_dense_partial(const pariskv_config* cfg, const void* q, const void* K,
                                 const void* V, int64_t ld_tok, int64_t n, float scale,
                                 float* work, int nsplit, cudaStream_t st) {
    if (cfg->group > kHeadsN) return cudaErrorInvalidValue;
    static std::atomic<uint64_t> done{0};
    cudaError_t e = raise_smem_limit(dense_attend_kernel, kSmem, done);
    if (e != cudaSuccess) return e;
    const int units = cfg->batch * cfg->num_kv_heads;
    dense_attend_kernel<<<dim3(nsplit, units), kDW * 32, kSmem, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(K),
        static_cast<const uint8_t*>(V), ld_tok, n, scale, cfg->group, nsplit, work);
    return cudaGetLastError();
}

}  // namespace pkv
