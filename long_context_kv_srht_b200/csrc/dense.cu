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
//
// The same kernel in gather mode is the sparse attention over the retrieved tokens when K/V
// are in device memory ("Technical Summary: ParisKV", Problem Statement: attend to the Top-k
// subset): CTA (split, query head) streams the rows named by that head's top-k indices
// through the same ring (the gathered rows are whole 256-byte lines), and the MMAs use one
// column of N (the head itself).
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
constexpr int kMaxGatherTiles = 16;           // gather mode: tiles per CTA (indices in smem)
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

struct MmaAttendArgs {
    const __nv_bfloat16* q;     // [heads][128]
    const uint8_t* K;           // [units][ld_tok][128] bf16
    const uint8_t* V;
    int64_t ld_tok, n;          // rows [0, n) exist
    const int32_t* idx;         // gather mode: row j of head h at idx[h * k_stride + j]
    int32_t k, k_stride;        // gather mode: indices per head
    float scale;
    int group;
    int nsplit, split_base, split_total;
    float* work;                // partials [heads][split_total][kAttendPart]
};

// kGather = false: CTA (split, unit) over rows [0, n) for all `group` heads of the unit.
// kGather = true: CTA (split, head) over the rows its k indices name (outside [0, n): skipped).
template <bool kGather>
__global__ void __launch_bounds__(kDW * 32, 2)
attend_mma_kernel(const MmaAttendArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint8_t s_ok[kStages][kTile];   // gather mode: row holds a valid token
    __shared__ int32_t s_idx[kGather ? kMaxGatherTiles * kTile : 1];  // gather: this CTA's rows
    uint8_t* sK = smem;
    uint8_t* sV = smem + kStages * kTileB;
    const int split = blockIdx.x;
    const int64_t head0 = kGather ? static_cast<int64_t>(blockIdx.y) : 0;
    const int64_t u = kGather ? head0 / a.group : static_cast<int64_t>(blockIdx.y);
    const int ncols = kGather ? 1 : a.group;  // N columns in use
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;     // fragment row / column pair of this lane
    const int64_t n = a.n;
    const int64_t len = kGather ? a.k : n;     // positions to attend
    const int32_t* hidx = kGather ? a.idx + head0 * a.k_stride : nullptr;

    const int64_t tiles = ceil_div(len, kTile);
    const int64_t tb0 = tiles * split / a.nsplit;
    const int64_t ntile = tiles * (split + 1) / a.nsplit - tb0;
    const uint8_t* Kb = a.K + u * a.ld_tok * kRowB;
    const uint8_t* Vb = a.V + u * a.ld_tok * kRowB;
    if (kGather) {
        // the CTA's indices, once, coalesced (the host keeps ntile <= kMaxGatherTiles); -1
        // past the end
        const int64_t p0 = tb0 * kTile;
        for (int i = tid; i < ntile * kTile; i += kDW * 32)
            s_idx[i] = p0 + i < len ? hidx[p0 + i] : -1;
        __syncthreads();
    }

    // stage a tile: 2 tensors x 64 rows x 16 chunks of 16 bytes; missing rows are
    // zero-filled (and masked below)
    auto load_tile = [&](int64_t tile, int stage) {
        const int64_t t0 = (tb0 + tile) * kTile;
#pragma unroll
        for (int j = 0; j < kLoadsPerThread; ++j) {
            const int id = tid + kDW * 32 * j;
            const int tensor = id / (kTile * 16), row = (id >> 4) & (kTile - 1), c = id & 15;
            const int64_t pos = t0 + row;
            int64_t tok = pos;
            bool ok = pos < len;
            if (kGather) {
                tok = s_idx[(tile * kTile) + row];
                ok = tok >= 0 && tok < n;
                if (tensor == 0 && c == 0) s_ok[stage][row] = ok;
            }
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

    // B fragments of Q^T (k = dims, n = heads): column g, dims 16s + 2t (+1) and
    // 16s + 8 + 2t (+1); unused columns are zero
    uint32_t qb[8][2];
    {
        const int64_t qhead = kGather ? head0 : u * a.group + g;
        const uint32_t* qh = reinterpret_cast<const uint32_t*>(a.q + qhead * D);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            qb[s][0] = g < ncols ? qh[8 * s + t] : 0u;
            qb[s][1] = g < ncols ? qh[8 * s + 4 + t] : 0u;
        }
    }
    const float qs = a.scale * kLog2e;

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
        float s0 = sacc[0] * qs, s1 = sacc[1] * qs, s2 = sacc[2] * qs, s3 = sacc[3] * qs;
        bool ok_a, ok_b;
        if (kGather) {
            ok_a = s_ok[st][16 * warp + g];
            ok_b = s_ok[st][16 * warp + g + 8];
        } else {
            const int64_t tok = (tb0 + it) * kTile + 16 * warp + g;
            ok_a = tok < n;
            ok_b = tok + 8 < n;
        }
        if (!ok_a) s0 = s1 = -INFINITY;
        if (!ok_b) s2 = s3 = -INFINITY;
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
    for (int h = warp; h < ncols; h += kDW) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDW; ++w) M = fmaxf(M, sc[(w * kHeadsN + h) * kAttendPart + D]);
        float den = 0.0f, r[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < kDW; ++w) {
            const float* src = sc + (w * kHeadsN + h) * kAttendPart;
            const float f = src[D] == -INFINITY ? 0.0f : exp2f(src[D] - M);
            den += src[D + 1] * f;
            const float4 v = *reinterpret_cast<const float4*>(src + 4 * lane);
            r[0] += v.x * f; r[1] += v.y * f; r[2] += v.z * f; r[3] += v.w * f;
        }
        const int64_t head = kGather ? head0 : u * a.group + h;
        float* out = a.work + (head * a.split_total + a.split_base + split) * kAttendPart;
        *reinterpret_cast<float4*>(out + 4 * lane) = make_float4(r[0], r[1], r[2], r[3]);
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

int gather_splits(int heads, int32_t k, int num_sms) {
    // about two waves of two CTAs per SM, every split at least one tile and at most
    // kMaxGatherTiles
    const int64_t tiles = ceil_div(k, kTile);
    const int64_t want = max64(ceil_div(4LL * num_sms, heads), ceil_div(tiles, kMaxGatherTiles));
    return static_cast<int>(max64(1, min64(want, tiles)));
}

int gather_min_splits(int32_t k) { return static_cast<int>(ceil_div(ceil_div(k, kTile), kMaxGatherTiles)); }

template <bool kGather>
static cudaError_t launch_mma(const MmaAttendArgs& a, dim3 grid, cudaStream_t st) {
    static std::atomic<uint64_t> done{0};
    cudaError_t e = raise_smem_limit(attend_mma_kernel<kGather>, kSmem, done);
    if (e != cudaSuccess) return e;
    attend_mma_kernel<kGather><<<grid, kDW * 32, kSmem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dense_partial(const pariskv_config* cfg, const void* q, const void* K,
                                 const void* V, int64_t ld_tok, int64_t n, float scale,
                                 float* work, int nsplit, int split_base, int split_total,
                                 cudaStream_t st) {
    if (cfg->group > kHeadsN) return cudaErrorInvalidValue;
    MmaAttendArgs a{static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(K),
                    static_cast<const uint8_t*>(V), ld_tok, n, nullptr, 0, 0, scale,
                    cfg->group, nsplit, split_base, split_total, work};
    return launch_mma<false>(a, dim3(nsplit, cfg->batch * cfg->num_kv_heads), st);
}

cudaError_t launch_gather_partial(const pariskv_config* cfg, const void* q, const void* K,
                                  const void* V, int64_t ld_tok, int64_t n, const int32_t* idx,
                                  int32_t k, int32_t k_stride, float scale, float* work,
                                  int nsplit, int split_base, int split_total, cudaStream_t st) {
    if (nsplit < gather_min_splits(k)) return cudaErrorInvalidValue;   // s_idx holds 16 tiles
    MmaAttendArgs a{static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(K),
                    static_cast<const uint8_t*>(V), ld_tok, n, idx, k, k_stride, scale,
                    cfg->group, nsplit, split_base, split_total, work};
    const int heads = cfg->batch * cfg->num_kv_heads * cfg->group;
    return launch_mma<true>(a, dim3(nsplit, heads), st);
}

}  // namespace pkv
