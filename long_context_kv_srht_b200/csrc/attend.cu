// attend.cu -- sparse decode attention over the retrieved top-k tokens.
//
// "Technical Summary: ParisKV", Problem Statement (attend only to a Top-k subset of past
// tokens) and System-Level Innovations 1 (Unified Virtual Addressing offloading: the GPU
// kernel fetches only the selected full-precision K/V rows, from HBM or directly from pinned
// host memory, without memcpy or CPU scheduling):
//     o_h = sum_{t in topk_h} softmax_t(scale * <q_h, K_t>) V_t,   K/V of KV head h / group.
//
// Split-K: CTA (split, head) processes a contiguous slice of the head's k indices; each of
// its 8 warps walks every 8th token of the slice, a lane holding 4 of the 128 dims, and
// keeps an online-softmax state (running max, denominator, 4 accumulators). A warp fetches
// its token indices 64 at a time and pipelines the row reads: the K/V rows of the next four
// tokens are requested before the current four enter the softmax, so reads stay in flight
// while the warp computes (this matters for K/V in host memory, where a read crosses PCIe:
// measured on B200, random 256-byte row reads of pinned host memory reach about 39 GB/s and
// sorted ones about 51 GB/s; the top-k indices are sorted). The warps are merged in shared
// memory and the CTA writes (128 accumulators, max, denominator) to the workspace; a second
// kernel merges the splits with the log-sum-exp rule and writes the output in the input
// dtype.
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kMaxScratchDevices = 64;

constexpr int kAW = 8;            // warps per CTA
constexpr int kUnroll = 4;        // tokens in flight per warp
// floats per partial: 128 accumulators, then max and denominator, padded to a multiple of 4
// so that every partial (and its accumulators) starts on a 16-byte boundary
constexpr int kPart = kAttendPart;
constexpr int kMax = D, kDen = D + 1;
static_assert((kPart * sizeof(float)) % 16 == 0, "partials must stay 16-byte aligned");

template <typename T> __device__ __forceinline__ void store4(T* p, const float v[4]);
template <> __device__ __forceinline__ void store4<float>(float* p, const float v[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, const float v[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

// Online-softmax update of one token: the warp's dot product, then the running state.
__device__ __forceinline__ void softmax_step(const float qv[4], const float kv[4],
                                             const float vv[4], float scale, float& mx,
                                             float& den, float acc[4]) {
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) s = __fmaf_rn(qv[i], kv[i], s);
    s = warp_sum(s) * scale;
    const float mn = fmaxf(mx, s);
    const float corr = expf(mx - mn);
    const float p = expf(s - mn);
    den = den * corr + p;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = acc[i] * corr + p * vv[i];
    mx = mn;
}

template <typename T>
__global__ void __launch_bounds__(kAW * 32)
attend_partial_kernel(const T* __restrict__ q, const T* __restrict__ K, const T* __restrict__ V,
                      int64_t ld_tok, int64_t n, const int32_t* __restrict__ topk, int32_t k,
                      int32_t k_stride, float scale, int group, int nsplit, int split_base,
                      int split_total, float* __restrict__ work) {
    __shared__ __align__(16) float sm[kAW][kPart];
    const int head = blockIdx.y, split = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t unit = head / group;
    const int64_t t0 = static_cast<int64_t>(k) * split / nsplit;
    const int64_t t1 = static_cast<int64_t>(k) * (split + 1) / nsplit;

    float qv[4];
    Elem<T>::load4(q + static_cast<int64_t>(head) * D + 4 * lane, qv);
    const T* Kb = K + unit * ld_tok * D + 4 * lane;
    const T* Vb = V + unit * ld_tok * D + 4 * lane;
    const int32_t* idx = topk + static_cast<int64_t>(head) * k_stride;

    float mx = -INFINITY, den = 0.0f, acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    // this warp's tokens: t0 + warp, t0 + warp + kAW, ...; their indices are fetched 64 at a
    // time (two per lane) and broadcast by shuffles
    const int64_t mine = t1 - t0 > warp ? (t1 - t0 - warp + kAW - 1) / kAW : 0;
    for (int64_t b0 = 0; b0 < mine; b0 += 64) {
        const int cnt = static_cast<int>(min64(64, mine - b0));
        int32_t ir[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 32 * h + lane;
            const int32_t row = j < cnt ? idx[t0 + warp + (b0 + j) * kAW] : -1;
            // rows outside [0, n) are skipped (the caller's indices are not trusted)
            ir[h] = (row >= 0 && row < n) ? row : -1;
        }
        auto row_of = [&](int j) -> int32_t {
            const int32_t a = __shfl_sync(0xffffffffu, ir[0], j & 31);
            const int32_t b = __shfl_sync(0xffffffffu, ir[1], j & 31);
            return j < cnt ? (j < 32 ? a : b) : -1;
        };
        // two register stages of kUnroll tokens: the next stage's K/V rows are requested
        // before the current stage's tokens enter the softmax
        float kv[2][kUnroll][4], vv[2][kUnroll][4];
        int32_t rw[2][kUnroll];
        auto load_stage = [&](int buf, int j0) {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int32_t row = row_of(j0 + u);
                rw[buf][u] = row;
                if (row >= 0) {
                    Elem<T>::load4(Kb + static_cast<int64_t>(row) * D, kv[buf][u]);
                    Elem<T>::load4(Vb + static_cast<int64_t>(row) * D, vv[buf][u]);
                }
            }
        };
        load_stage(0, 0);
        for (int j0 = 0; j0 < cnt; j0 += 2 * kUnroll) {
            if (j0 + kUnroll < cnt) load_stage(1, j0 + kUnroll);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (rw[0][u] >= 0) softmax_step(qv, kv[0][u], vv[0][u], scale, mx, den, acc);
            if (j0 + kUnroll >= cnt) break;
            if (j0 + 2 * kUnroll < cnt) load_stage(0, j0 + 2 * kUnroll);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (rw[1][u] >= 0) softmax_step(qv, kv[1][u], vv[1][u], scale, mx, den, acc);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sm[warp][4 * lane + i] = acc[i];
    if (lane == 0) { sm[warp][kMax] = mx; sm[warp][kDen] = den; }
    __syncthreads();
    if (warp == 0) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAW; ++w) M = fmaxf(M, sm[w][kMax]);
        float dsum = 0.0f, a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < kAW; ++w) {
            const float f = sm[w][kMax] == -INFINITY ? 0.0f : expf(sm[w][kMax] - M);
            dsum += sm[w][kDen] * f;
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] += sm[w][4 * lane + i] * f;
        }
        float* out = work + (static_cast<int64_t>(head) * split_total + split_base + split) * kPart;
        *reinterpret_cast<float4*>(out + 4 * lane) = make_float4(a[0], a[1], a[2], a[3]);
        if (lane == 0) { out[kMax] = M; out[kDen] = dsum; }
    }
}

// Log-sum-exp merge of one head's splits, one warp per head. Lane s (mod 32) reads split s's
// max and denominator, so the global maximum and every split's weight take one round of
// loads; the accumulators are then summed split by split, the weight broadcast by a
// shuffle, with the float4 loads of eight splits in flight at a time.
template <typename T>
__global__ void __launch_bounds__(32)
attend_combine_kernel(const float* __restrict__ work, int nsplit, T* __restrict__ out) {
    const int head = blockIdx.x, lane = threadIdx.x;
    const float* w = work + static_cast<int64_t>(head) * nsplit * kPart;
    float M = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, w[s * kPart + kMax]);
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
    float den = 0.0f, a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int s0 = 0; s0 < nsplit; s0 += 32) {
        const int s = s0 + lane;
        const float ms = s < nsplit ? w[s * kPart + kMax] : -INFINITY;
        const float f = ms == -INFINITY ? 0.0f : expf(ms - M);
        if (s < nsplit) den += w[s * kPart + kDen] * f;
        const int cnt = min(32, nsplit - s0);
#pragma unroll 8
        for (int j = 0; j < cnt; ++j) {
            const float fj = __shfl_sync(0xffffffffu, f, j);
            const float4 v = *reinterpret_cast<const float4*>(w + (s0 + j) * kPart + 4 * lane);
            a[0] += v.x * fj; a[1] += v.y * fj; a[2] += v.z * fj; a[3] += v.w * fj;
        }
    }
    den = warp_sum(den);
    const float inv = den > 0.0f ? 1.0f / den : 0.0f;
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = a[i] * inv;
    store4<T>(out + static_cast<int64_t>(head) * D + 4 * lane, o);
}

// ---------------------------------------------------------------------------------------
// GQA-group union: the G query heads of a KV head often select the same rows; each union row
// is fetched once (over PCIe when K/V live in pinned host memory) and scored for every head
// that selected it.
// ---------------------------------------------------------------------------------------
constexpr int kUnionT = 256;      // threads of a union-building CTA
constexpr int kUnionBlocks = 32;  // union-building CTAs per unit

__device__ unsigned long long g_union_rows;   // union rows fetched, summed until read

// bit (row mod 32) of word row / 32 of head's bitmap, for every valid index of the head
__global__ void __launch_bounds__(256)
union_mark_kernel(const int32_t* __restrict__ topk, int32_t k, int64_t n, int64_t nw,
                  uint32_t* __restrict__ bits) {
    const int64_t head = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= k) return;
    const int32_t r = topk[head * k + i];
    if (r < 0 || r >= n) return;   // skipped like the per-head kernel skips them
    atomicOr(bits + head * nw + (r >> 5), 1u << (r & 31));
}

// The union of the group's bitmaps, scanned into the ascending union row list with each row's
// membership mask (bit g = query head g of the group selected it), over kUnionBlocks CTAs per
// unit: union_count_kernel counts each block's rows, union_write_kernel offsets a block by the
// counts of the unit's earlier blocks and writes its rows in order.
__device__ __forceinline__ void union_block_range(int64_t nw, int b, int64_t* w0, int64_t* w1,
                                                  int64_t* per) {
    const int64_t wb = (nw + kUnionBlocks - 1) / kUnionBlocks;   // words per block
    const int64_t b0 = min64(nw, wb * b), b1 = min64(nw, b0 + wb);
    *per = (b1 - b0 + kUnionT - 1) / kUnionT;                      // words per thread
    *w0 = min64(b1, b0 + *per * threadIdx.x);
    *w1 = min64(b1, *w0 + *per);
}

__device__ __forceinline__ uint32_t union_block_scan(uint32_t c, uint32_t* total,
                                                     uint32_t* wsum /* [kUnionT / 32] */) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kUnionT / 32; ++i) {
        before += i < warp ? wsum[i] : 0u;
        tot += wsum[i];
    }
    *total = tot;
    return before + x - c;
}

__global__ void __launch_bounds__(kUnionT)
union_count_kernel(const uint32_t* __restrict__ bits, int G, int64_t nw,
                   uint32_t* __restrict__ bcount) {
    __shared__ uint32_t wsum[kUnionT / 32];
    const int64_t unit = blockIdx.y;
    const uint32_t* b = bits + unit * G * nw;
    int64_t w0, w1, per;
    union_block_range(nw, blockIdx.x, &w0, &w1, &per);
    uint32_t c = 0;
    for (int64_t w = w0; w < w1; ++w) {
        uint32_t u = 0;
        for (int g = 0; g < G; ++g) u |= b[g * nw + w];
        c += __popc(u);
    }
    uint32_t total;
    union_block_scan(c, &total, wsum);
    if (threadIdx.x == 0) bcount[unit * kUnionBlocks + blockIdx.x] = total;
}

__global__ void __launch_bounds__(kUnionT)
union_write_kernel(const uint32_t* __restrict__ bits, int G, int64_t nw, int64_t cap,
                   const uint32_t* __restrict__ bcount, int32_t* __restrict__ rows,
                   uint8_t* __restrict__ masks, int32_t* __restrict__ count) {
    __shared__ uint32_t wsum[kUnionT / 32];
    __shared__ uint32_t sbase;
    const int64_t unit = blockIdx.y;
    const uint32_t* b = bits + unit * G * nw;
    if (threadIdx.x < 32) {   // the unit's rows in the blocks before this one
        uint32_t x = 0;
        for (int i = threadIdx.x; i < blockIdx.x; i += 32) x += bcount[unit * kUnionBlocks + i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (threadIdx.x == 0) sbase = x;
    }
    int64_t w0, w1, per;
    union_block_range(nw, blockIdx.x, &w0, &w1, &per);
    uint32_t c = 0;
    for (int64_t w = w0; w < w1; ++w) {
        uint32_t u = 0;
        for (int g = 0; g < G; ++g) u |= b[g * nw + w];
        c += __popc(u);
    }
    uint32_t total;
    const uint32_t before = union_block_scan(c, &total, wsum);   // (its barrier orders sbase)
    int64_t pos = unit * cap + sbase + before;
    for (int64_t w = w0; w < w1; ++w) {
        uint32_t bg[8], u = 0;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            bg[g] = g < G ? b[g * nw + w] : 0u;
            u |= bg[g];
        }
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1u;
            uint32_t m = 0;
#pragma unroll
            for (int g = 0; g < 8; ++g) m |= ((bg[g] >> bit) & 1u) << g;
            rows[pos] = static_cast<int32_t>(32 * w + bit);
            masks[pos] = static_cast<uint8_t>(m);
            ++pos;
        }
    }
    if (blockIdx.x == kUnionBlocks - 1 && threadIdx.x == 0) {
        const uint32_t all = sbase + total;
        count[unit] = static_cast<int32_t>(all);
        atomicAdd(&g_union_rows, static_cast<unsigned long long>(all));
    }
}

// Split-K partials over a unit's union rows: CTA (split, unit) takes a contiguous slice of
// the union; each warp walks every 8th row of it, a lane holding 4 of the 128 dims, with the
// row fetches pipelined as in attend_partial_kernel, and keeps one online-softmax state per
// query head of the group (GM >= G, a compile-time bound so the states stay in registers).
// Each head's partial goes where the per-head kernel would put it, so the same merge follows.
template <typename T, int GM>
__global__ void __launch_bounds__(kAW * 32)
attend_union_kernel(const T* __restrict__ q, const T* __restrict__ K, const T* __restrict__ V,
                    int64_t ld_tok, const int32_t* __restrict__ rows,
                    const uint8_t* __restrict__ masks, const int32_t* __restrict__ count,
                    int64_t cap, float scale, int G, int nsplit, int split_base,
                    int split_total, float* __restrict__ work) {
    __shared__ __align__(16) float sm[kAW][kPart];
    const int64_t unit = blockIdx.y;
    const int split = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t u = count[unit];
    const int64_t t0 = u * split / nsplit, t1 = u * (split + 1) / nsplit;
    float qv[GM][4], mx[GM], den[GM], acc[GM][4];
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        if (g < G) Elem<T>::load4(q + (unit * G + g) * D + 4 * lane, qv[g]);
        mx[g] = -INFINITY;
        den[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[g][i] = 0.0f;
    }
    const T* Kb = K + unit * ld_tok * D + 4 * lane;
    const T* Vb = V + unit * ld_tok * D + 4 * lane;
    const int32_t* ur = rows + unit * cap;
    const uint8_t* um = masks + unit * cap;
    const int64_t mine = t1 - t0 > warp ? (t1 - t0 - warp + kAW - 1) / kAW : 0;
    for (int64_t b0 = 0; b0 < mine; b0 += 64) {
        const int cnt = static_cast<int>(min64(64, mine - b0));
        int32_t ir[2];
        uint32_t im[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 32 * h + lane;
            const int64_t t = t0 + warp + (b0 + j) * kAW;
            ir[h] = j < cnt ? ur[t] : -1;
            im[h] = j < cnt ? um[t] : 0u;
        }
        auto row_of = [&](int j) -> int32_t {
            const int32_t a = __shfl_sync(0xffffffffu, ir[0], j & 31);
            const int32_t b = __shfl_sync(0xffffffffu, ir[1], j & 31);
            return j < cnt ? (j < 32 ? a : b) : -1;
        };
        auto mask_of = [&](int j) -> uint32_t {
            const uint32_t a = __shfl_sync(0xffffffffu, im[0], j & 31);
            const uint32_t b = __shfl_sync(0xffffffffu, im[1], j & 31);
            return j < cnt ? (j < 32 ? a : b) : 0u;
        };
        float kv[2][kUnroll][4], vv[2][kUnroll][4];
        uint32_t mw[2][kUnroll];
        auto load_stage = [&](int buf, int j0) {
#pragma unroll
            for (int e = 0; e < kUnroll; ++e) {
                const int32_t row = row_of(j0 + e);
                mw[buf][e] = row >= 0 ? mask_of(j0 + e) : 0u;
                if (row >= 0) {
                    Elem<T>::load4(Kb + static_cast<int64_t>(row) * D, kv[buf][e]);
                    Elem<T>::load4(Vb + static_cast<int64_t>(row) * D, vv[buf][e]);
                }
            }
        };
        auto consume = [&](int buf) {
#pragma unroll
            for (int e = 0; e < kUnroll; ++e)
#pragma unroll
                for (int g = 0; g < GM; ++g)
                    if ((mw[buf][e] >> g) & 1u)
                        softmax_step(qv[g], kv[buf][e], vv[buf][e], scale, mx[g], den[g], acc[g]);
        };
        load_stage(0, 0);
        for (int j0 = 0; j0 < cnt; j0 += 2 * kUnroll) {
            if (j0 + kUnroll < cnt) load_stage(1, j0 + kUnroll);
            consume(0);
            if (j0 + kUnroll >= cnt) break;
            if (j0 + 2 * kUnroll < cnt) load_stage(0, j0 + 2 * kUnroll);
            consume(1);
        }
    }
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        if (g >= G) break;
#pragma unroll
        for (int i = 0; i < 4; ++i) sm[warp][4 * lane + i] = acc[g][i];
        if (lane == 0) { sm[warp][kMax] = mx[g]; sm[warp][kDen] = den[g]; }
        __syncthreads();
        if (warp == 0) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kAW; ++w) M = fmaxf(M, sm[w][kMax]);
            float dsum = 0.0f, a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int w = 0; w < kAW; ++w) {
                const float f = sm[w][kMax] == -INFINITY ? 0.0f : expf(sm[w][kMax] - M);
                dsum += sm[w][kDen] * f;
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] += sm[w][4 * lane + i] * f;
            }
            float* out = work + ((unit * G + g) * split_total + split_base + split) * kPart;
            *reinterpret_cast<float4*>(out + 4 * lane) = make_float4(a[0], a[1], a[2], a[3]);
            if (lane == 0) { out[kMax] = M; out[kDen] = dsum; }
        }
        __syncthreads();
    }
}

// Fixed workspace of the allocation-free attention entry point: split-K partials in a
// file-scope device array, so a call needs no allocator. Every device that loads the library
// holds these 4 MiB until the process exits; all calls on a device share them.
static __device__ __align__(256) float g_attend_scratch[kAttendScratchFloats];

std::mutex g_scratch_mu;
float* g_scratch_addr[kMaxScratchDevices] = {};

// One pass over `n16` 16-byte words, four independent loads in flight per thread.
__global__ void __launch_bounds__(256)
read_stream_kernel(const uint4* __restrict__ p, int64_t n16, uint32_t* __restrict__ sink) {
    uint32_t acc = 0;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = p[i], b = p[i + stride], c = p[i + 2 * stride], d = p[i + 3 * stride];
        acc ^= a.x ^ b.y ^ c.z ^ d.w;
    }
    for (; i < n16; i += stride) acc ^= p[i].x;
    if (acc == 0x9E3779B9u) *sink = acc;   // keeps the loads; almost never stores
}

// The rerank's memory access alone: every (query head, candidate) pair's 128-byte record is
// read with 16-byte loads (eight lanes per record, four records per warp instruction, eight
// instructions in flight per lane) and folded into one word; no arithmetic on the data.
// Warps take groups of 32 candidates of one head in turn.
__global__ void __launch_bounds__(256)
gather_candidates_kernel(const uint8_t* __restrict__ rec, int64_t cap_pad,
                         const int32_t* __restrict__ cand, int64_t cmax, int32_t C, int group,
                         int64_t heads, int64_t n, uint32_t* __restrict__ sink) {
    const int lane = threadIdx.x & 31;
    const int64_t gpr = (C + 31) / 32;                        // groups per head
    const int64_t groups = heads * gpr;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    uint32_t acc = 0;
    for (int64_t gi = w0; gi < groups; gi += nw) {
        const int64_t h = gi / gpr, j0 = (gi - h * gpr) * 32;
        const uint8_t* base = rec + (h / group) * cap_pad * 128;
        const int64_t j = j0 + lane;
        const int32_t idx = j < C ? cand[h * cmax + j] : -1;
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int32_t r = __shfl_sync(0xffffffffu, idx, 4 * i + (lane >> 3));
            v[i] = (r >= 0 && r < n)
                       ? __ldcs(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(r) * 128) +
                                (lane & 7))
                       : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc ^= v[i].x ^ v[i].y ^ v[i].z ^ v[i].w;
    }
    if (acc == 0x9E3779B9u) *sink = acc;   // keeps the loads; almost never stores
}

}  // namespace

cudaError_t launch_gather_candidates(const uint8_t* rec, int64_t cap_pad, const int32_t* cand,
                                     int64_t cmax, int32_t C, int group, int64_t heads,
                                     int64_t n, uint32_t* sink, cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    gather_candidates_kernel<<<4 * sms, 256, 0, st>>>(rec, cap_pad, cand, cmax, C, group, heads, n,
                                                      sink);
    return cudaGetLastError();
}

cudaError_t launch_read_stream(const void* src, int64_t bytes, uint32_t* sink,
                               cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    read_stream_kernel<<<4 * sms, 256, 0, st>>>(static_cast<const uint4*>(src), bytes / 16,
                                                 sink);
    return cudaGetLastError();
}

cudaError_t attend_static_scratch(float** ptr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        // the array's host-side name is only a stand-in; its device address comes from the
        // runtime, once per device, with that device current
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attend_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = static_cast<float*>(p);
    }
    *ptr = g_scratch_addr[dev];
    return cudaSuccess;
}

int attend_splits(int heads, int32_t k, int num_sms, bool mma) {
    if (mma) return gather_splits(heads, k, num_sms);
    // one wave: two 8-warp CTAs per SM
    const int want = static_cast<int>(2LL * num_sms / heads);
    const int most = static_cast<int>(ceil_div(k, 64));
    return max(1, min(want, most));
}

size_t attend_workspace_floats(int heads, int nsplit) {
    return static_cast<size_t>(heads) * nsplit * kPart;
}

bool attend_uses_mma(const pariskv_config* cfg, bool kv_device) {
    return kv_device && cfg->dtype == PARISKV_BF16;
}

cudaError_t launch_attend_partial(const pariskv_config* cfg, const void* q, const void* K,
                                  const void* V, int64_t ld_tok, int64_t n,
                                  const int32_t* idx, int32_t k, int32_t k_stride, float scale,
                                  float* work, int nsplit, int split_base, int split_total,
                                  bool mma, cudaStream_t st) {
    if (mma)
        return launch_gather_partial(cfg, q, K, V, ld_tok, n, idx, k, k_stride, scale, work,
                                     nsplit, split_base, split_total, st);
    const int heads = cfg->batch * cfg->num_kv_heads * cfg->group;
    dim3 grid(nsplit, heads);
    if (cfg->dtype == PARISKV_BF16) {
        using T = __nv_bfloat16;
        attend_partial_kernel<T><<<grid, kAW * 32, 0, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(K), static_cast<const T*>(V),
            ld_tok, n, idx, k, k_stride, scale, cfg->group, nsplit, split_base, split_total,
            work);
    } else {
        attend_partial_kernel<float><<<grid, kAW * 32, 0, st>>>(
            static_cast<const float*>(q), static_cast<const float*>(K),
            static_cast<const float*>(V), ld_tok, n, idx, k, k_stride, scale, cfg->group, nsplit,
            split_base, split_total, work);
    }
    return cudaGetLastError();
}

cudaError_t launch_attend_combine(int heads, const float* work, int split_total, void* out,
                                  int32_t out_dtype, cudaStream_t st) {
    if (out_dtype == PARISKV_BF16)
        attend_combine_kernel<__nv_bfloat16><<<heads, 32, 0, st>>>(
            work, split_total, static_cast<__nv_bfloat16*>(out));
    else
        attend_combine_kernel<float><<<heads, 32, 0, st>>>(work, split_total,
                                                           static_cast<float*>(out));
    return cudaGetLastError();
}

// The union scratch: group bitmaps [units][G][ceil(n / 32)] words, then the union rows
// [units][G k] (int32), their masks [units][G k] (u8) and the counts [units]. Used for
// 1 < group <= 8 while the bitmaps stay within kUnionBitmapBytes, unless the environment has
// PARISKV_ATTEND_UNION=0.
constexpr size_t kUnionBitmapBytes = size_t(256) << 20;

static size_t union_bitmap_words(const pariskv_config* cfg, int64_t n) {
    return static_cast<size_t>(cfg->batch) * cfg->num_kv_heads * cfg->group *
           static_cast<size_t>((n + 31) / 32);
}

size_t union_workspace_bytes(const pariskv_config* cfg, int64_t n, int32_t k) {
    const char* env = getenv("PARISKV_ATTEND_UNION");
    if (env && env[0] == '0') return 0;
    if (cfg->group < 2 || cfg->group > 8) return 0;
    const size_t words = union_bitmap_words(cfg, n);
    if (words * 4 > kUnionBitmapBytes) return 0;
    const size_t units = static_cast<size_t>(cfg->batch) * cfg->num_kv_heads;
    const size_t cap = static_cast<size_t>(cfg->group) * k;
    const size_t b = words * 4 + units * cap * 4 + round_up(units * cap, 16) + units * 4 +
                     units * kUnionBlocks * 4;
    return round_up(b, 256);
}

int union_splits(int units, int group, int32_t k, int num_sms) {
    // one wave of one CTA per SM (the kernel keeps G softmax states and two register stages
    // of rows per lane: one 8-warp CTA fills an SM's registers)
    const int want = static_cast<int>(static_cast<int64_t>(num_sms) / units);
    const int most = static_cast<int>(ceil_div(static_cast<int64_t>(group) * k, 64));
    return max(1, min(want, most));
}

cudaError_t launch_union_build(const pariskv_config* cfg, int64_t n, const int32_t* topk,
                               int32_t k, void* scratch, cudaStream_t st, UnionLists* out) {
    const int G = cfg->group;
    const int units = cfg->batch * cfg->num_kv_heads;
    const int64_t nw = (n + 31) / 32, cap = static_cast<int64_t>(G) * k;
    const size_t words = union_bitmap_words(cfg, n);
    uint32_t* bits = static_cast<uint32_t*>(scratch);
    out->cap = cap;
    out->rows = reinterpret_cast<int32_t*>(bits + words);
    out->masks = reinterpret_cast<uint8_t*>(out->rows + static_cast<size_t>(units) * cap);
    out->count = reinterpret_cast<int32_t*>(out->masks +
                                            round_up(static_cast<size_t>(units) * cap, 16));
    cudaError_t e = cudaMemsetAsync(bits, 0, words * 4, st);
    if (e != cudaSuccess) return e;
    union_mark_kernel<<<dim3(static_cast<unsigned>(ceil_div(k, 256)), units * G), 256, 0, st>>>(
        topk, k, n, nw, bits);
    uint32_t* bcount = reinterpret_cast<uint32_t*>(out->count + units);
    union_count_kernel<<<dim3(kUnionBlocks, units), kUnionT, 0, st>>>(bits, G, nw, bcount);
    union_write_kernel<<<dim3(kUnionBlocks, units), kUnionT, 0, st>>>(bits, G, nw, cap, bcount,
                                                                      out->rows, out->masks,
                                                                      out->count);
    return cudaGetLastError();
}

cudaError_t launch_union_partial(const pariskv_config* cfg, const void* q, const void* K,
                                 const void* V, int64_t ld_tok, int64_t n, const int32_t* topk,
                                 int32_t k, float scale, float* work, int nsplit,
                                 int split_base, int split_total, void* scratch,
                                 cudaStream_t st) {
    const int G = cfg->group;
    const int units = cfg->batch * cfg->num_kv_heads;
    UnionLists ul;
    cudaError_t e = launch_union_build(cfg, n, topk, k, scratch, st, &ul);
    if (e != cudaSuccess) return e;
    const int32_t* rows = ul.rows;
    const uint8_t* masks = ul.masks;
    const int32_t* count = ul.count;
    const int64_t cap = ul.cap;
    dim3 grid(nsplit, units);
    const bool bf = cfg->dtype == PARISKV_BF16;
#define PKV_UNION_LAUNCH(TT, GM)                                                              \
    attend_union_kernel<TT, GM><<<grid, kAW * 32, 0, st>>>(                                   \
        static_cast<const TT*>(q), static_cast<const TT*>(K), static_cast<const TT*>(V),      \
        ld_tok, rows, masks, count, cap, scale, G, nsplit, split_base, split_total, work)
    if (bf) {
        if (G <= 2) PKV_UNION_LAUNCH(__nv_bfloat16, 2);
        else if (G <= 4) PKV_UNION_LAUNCH(__nv_bfloat16, 4);
        else PKV_UNION_LAUNCH(__nv_bfloat16, 8);
    } else {
        if (G <= 2) PKV_UNION_LAUNCH(float, 2);
        else if (G <= 4) PKV_UNION_LAUNCH(float, 4);
        else PKV_UNION_LAUNCH(float, 8);
    }
#undef PKV_UNION_LAUNCH
    return cudaGetLastError();
}

cudaError_t launch_attend_union(const pariskv_config* cfg, const void* q, const void* K,
                                const void* V, int64_t ld_tok, int64_t n, const int32_t* topk,
                                int32_t k, float scale, void* out, int32_t out_dtype,
                                float* work, int nsplit, void* scratch, cudaStream_t st) {
    cudaError_t e = launch_union_partial(cfg, q, K, V, ld_tok, n, topk, k, scale, work, nsplit, 0,
                                         nsplit, scratch, st);
    if (e != cudaSuccess) return e;
    return launch_attend_combine(cfg->batch * cfg->num_kv_heads * cfg->group, work, nsplit, out,
                                 out_dtype, st);
}

cudaError_t read_union_rows(unsigned long long* rows) {
    cudaError_t e = cudaMemcpyFromSymbol(rows, g_union_rows, sizeof(*rows));
    if (e != cudaSuccess) return e;
    const unsigned long long zero = 0;
    return cudaMemcpyToSymbol(g_union_rows, &zero, sizeof(zero));
}

cudaError_t launch_attend(const pariskv_config* cfg, const void* q, const void* K,
                          const void* V, int64_t ld_tok, int64_t n, const int32_t* topk_idx,
                          int32_t k, float scale, void* out, int32_t out_dtype, float* work,
                          int nsplit, bool mma, cudaStream_t st) {
    cudaError_t e = launch_attend_partial(cfg, q, K, V, ld_tok, n, topk_idx, k, k, scale, work,
                                          nsplit, 0, nsplit, mma, st);
    if (e != cudaSuccess) return e;
    const int heads = cfg->batch * cfg->num_kv_heads * cfg->group;
    return launch_attend_combine(heads, work, nsplit, out, out_dtype, st);
}

}  // namespace pkv
