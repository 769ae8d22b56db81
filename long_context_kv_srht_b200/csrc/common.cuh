// common.cuh -- constants, error plumbing and small PTX helpers shared by the sm_100a kernels
// of libpariskv.so. Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

// Shapes the kernels are specialised for (checked at the C ABI).
constexpr int D = 128;          // head dimension
constexpr int M = 8;            // dims per subspace
constexpr int NB = D / M;       // subspaces (16)
constexpr int NC = 1 << M;      // sign centroids per subspace (256)
constexpr int REC = 128;        // bytes per key record: 64 B of 4-bit codes + 16 fp32 factors
constexpr int NBINS = 64;       // coarse scores are < 64 (B * w_rank1 <= 48)
constexpr int SBINS_BITS = 11;  // first radix level of the top-k, counted by the rerank
constexpr int SBINS = 1 << SBINS_BITS;
constexpr int SCOPIES = 1;      // copies of that histogram (one copy per warp group spreads the reductions)
constexpr int CHUNK = 8192;     // keys per coarse-score histogram chunk (a vote work item)
constexpr int PACK = 4;         // query heads whose vote weights share one 32-bit table entry

// Device status word. ST_BADINDEX: a kernel found an index out of range and skipped the
// access. ST_TIMEOUT: a bounded device-side wait ran out (the top-k's wait for its own bulk
// copies; no kernel of the library waits on another, each stage is its own launch).
enum : int { ST_OK = 0, ST_TIMEOUT = 5, ST_BADINDEX = 6 };

// The checked build (-DPKV_CHECK=1, libpariskv_check.so) adds device-side checks of values
// that are correct by construction in a consistent run (score bytes, output positions and
// indices); a failed check records ST_BADINDEX and skips the access. Never a trap.
#ifndef PKV_CHECK
#define PKV_CHECK 0
#endif
__device__ __forceinline__ bool pkv_check(bool ok, int* status) {
    if (PKV_CHECK && !ok) {
        atomicExch(status, ST_BADINDEX);
        return false;
    }
    return true;
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
__host__ __device__ constexpr int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ constexpr int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// ---------------------------------------------------------------------------------------
// Element loads
// ---------------------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    // four consecutive elements starting at p (16-byte aligned)
    static __device__ __forceinline__ void load4(const float* p, float v[4]) {
        float4 x = *reinterpret_cast<const float4*>(p);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ void load4(const __nv_bfloat16* p, float v[4]) {
        uint2 x = *reinterpret_cast<const uint2*>(p);
        v[0] = __uint_as_float(x.x << 16); v[1] = __uint_as_float(x.x & 0xFFFF0000u);
        v[2] = __uint_as_float(x.y << 16); v[3] = __uint_as_float(x.y & 0xFFFF0000u);
    }
};

// ---------------------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
// PRMT with a compile-time selector (an immediate operand, no register to materialise).
template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt_i(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "n"(SEL));
    return r;
}

// Programmatic dependent launch. A search kernel is launched so that it may start while
// the previous kernel of the stream is finishing; pdl_wait() blocks until that kernel has
// completed and its writes are visible (every kernel calls it before reading the previous
// kernel's results and before any global write), and pdl_launch_dependents() then lets the
// next kernel begin launching. Because every kernel triggers only after its own wait, a
// kernel that has started may read anything written before its immediate predecessor.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Order-preserving 32-bit image of an fp32 value (flip all bits of negative values, set the
// sign bit of the others) and its exact inverse.
__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float value_of(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}


// 256-bit read-only global load that does not allocate in L1 (sm_100): 8 consecutive words.
struct u32x8 { uint32_t w[8]; };
__device__ __forceinline__ u32x8 ldg_stream_u256(const void* p) {
    u32x8 v;
    asm("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
          "=r"(v.w[6]), "=r"(v.w[7])
        : "l"(p));
    return v;
}

// ---- packed fp32 pairs (sm_100: one instruction, two IEEE round-to-nearest operations) ----
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t pack2u(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0,%1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return make_float2(lo, hi);
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ---- mbarrier (CTA scope) and bulk async copies (no multicast) ----
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Global -> shared bulk copy completing on an mbarrier (bytes and both addresses multiples
// of 16). The destination is this CTA's own shared memory.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace pkv
