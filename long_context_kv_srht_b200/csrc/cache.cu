// cache.cu -- four-region KV cache for unbounded decoding (pariskv_cache.h).
//
// "Technical Summary: ParisKV", System-Level Innovations 2 ("Sliding-Window Update
// Mechanism"): Sink and Local tokens stay on the GPU, older tokens are offloaded to the
// Retrieval zone and found through the index, and an Update Buffer collects new tokens;
// when it fills, the oldest Local tokens are evicted to Retrieval and the buffer becomes
// Local. System-Level Innovations 1 (UVA offloading): the attention reads the offloaded
// K/V rows of the retrieved tokens directly from pinned host memory.
//
// Region bookkeeping is host-side (the counts are the same for every (sequence, KV head)),
// and every data movement is a kernel on the caller's stream (no copy-engine calls while
// decoding):
//  - put_token_kernel writes the new token's K/V row at the end of the device pool;
//  - a promotion that evicts runs spill_kernel (evicted rows -> the host Retrieval arrays,
//    written over UVA; the rows that stay -> a scratch buffer), the index's encode kernel
//    (which reads the evicted keys from the pool) and slide_kernel (scratch -> pool rows right
//    after Sink), so Sink, Local and buffer always occupy pool rows [0, n_dense);
//  - the search runs on the index of the Retrieval zone; the attention writes split-K
//    partials for the dense rows (every head reads rows 0..n_dense-1 of its unit's pool)
//    and for the retrieved rows (pinned host memory) into one workspace, and one merge
//    (log-sum-exp) gives a single softmax over the union.
#include <cuda_runtime.h>

#include <new>

#include "common.cuh"
#include "internal.hpp"
#include "pariskv_cache.h"

using namespace pkv;

struct pariskv_cache {
    pariskv_config cfg;           // capacity = retrieval_capacity
    pariskv_cache_config cc;
    int device = 0;
    int units = 0, heads = 0;
    int64_t P = 0;                // pool rows per unit: n_sink + n_local + n_buffer
    size_t row = 0;               // bytes per K or V row
    uint8_t* poolK = nullptr;     // device [units][P][d]
    uint8_t* poolV = nullptr;
    uint8_t* tmp = nullptr;       // device [2][units][n_local + n_buffer][d] (K, then V)
    uint8_t* hostK = nullptr;     // pinned host [units][R][d]
    uint8_t* hostV = nullptr;
    int32_t* dense_idx = nullptr; // device [P]: 0, 1, ..., P - 1 (every head reads it)
    int32_t* topk = nullptr;      // device [heads][k]
    float* work = nullptr;        // device [heads][max_splits][partial]
    void* uscratch = nullptr;     // GQA-group union of the retrieved rows (NULL: per head)
    int max_splits = 0;           // per source (dense, retrieved)
    int sms = 0;
    pariskv_index* ix = nullptr;
    int64_t sink = 0, local = 0, buffer = 0, retr = 0;
};

namespace {

__global__ void iota_kernel(int32_t* p, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) p[i] = static_cast<int32_t>(i);
}

// Row copies in 16-byte words (every buffer here is allocation-aligned and a row is 256 or 512
// bytes). blockIdx.z picks the tensor (0: K, 1: V), blockIdx.y the unit.
struct Rows {
    uint4* pool[2];   // [units][P][vpr]
    uint4* host[2];   // [units][R][vpr]
    uint4* tmp[2];    // [units][L][vpr]
    int64_t P, R, L;
    int vpr;          // 16-byte words per row
};

// Rows sink + j, j in [0, move + rest): the first `move` go to host rows retr + j, the others
// to scratch rows j - move.
__global__ void __launch_bounds__(256)
spill_kernel(Rows r, int64_t sink, int64_t move, int64_t rest, int64_t retr) {
    const int t = blockIdx.z;
    const int64_t u = blockIdx.y;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= (move + rest) * r.vpr) return;
    const int64_t j = i / r.vpr, c = i - j * r.vpr;
    const uint4 v = r.pool[t][(u * r.P + sink + j) * r.vpr + c];
    if (j < move)
        r.host[t][(u * r.R + retr + j) * r.vpr + c] = v;
    else
        r.tmp[t][(u * r.L + j - move) * r.vpr + c] = v;
}

// Scratch rows [0, rest) -> pool rows sink + j.
__global__ void __launch_bounds__(256)
slide_kernel(Rows r, int64_t sink, int64_t rest) {
    const int t = blockIdx.z;
    const int64_t u = blockIdx.y;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= rest * r.vpr) return;
    const int64_t j = i / r.vpr, c = i - j * r.vpr;
    r.pool[t][(u * r.P + sink + j) * r.vpr + c] = r.tmp[t][(u * r.L + j) * r.vpr + c];
}

// The new token's rows ([units][vpr8] 8-byte words each; the caller's pointers are 8-byte
// aligned) -> pool row `at`.
__global__ void __launch_bounds__(256)
put_token_kernel(const uint2* __restrict__ kn, const uint2* __restrict__ vn, uint2* poolK,
                 uint2* poolV, int64_t P, int64_t at, int units, int vpr8) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * units * vpr8) return;
    const int t = i / (units * vpr8), r = i - t * units * vpr8;
    const int u = r / vpr8, c = r - u * vpr8;
    (t ? poolV : poolK)[(static_cast<int64_t>(u) * P + at) * vpr8 + c] = (t ? vn : kn)[r];
}

void free_cache(pariskv_cache* c) {
    if (!c) return;
    if (c->ix) pariskv_destroy(c->ix);
    cudaFree(c->poolK);
    cudaFree(c->poolV);
    cudaFree(c->tmp);
    cudaFree(c->dense_idx);
    cudaFree(c->topk);
    cudaFree(c->work);
    cudaFree(c->uscratch);
    if (c->hostK) cudaFreeHost(c->hostK);
    if (c->hostV) cudaFreeHost(c->hostV);
    delete c;
}

template <typename T>
bool dev_alloc(T** p, size_t bytes) {
    *p = nullptr;
    if (alloc_fault_injected()) return false;
    if (cudaMalloc(reinterpret_cast<void**>(p), bytes) != cudaSuccess) {
        cudaGetLastError();
        *p = nullptr;
        return false;
    }
    return true;
}

bool host_alloc(uint8_t** p, size_t bytes) {
    *p = nullptr;
    if (alloc_fault_injected()) return false;
    if (cudaHostAlloc(reinterpret_cast<void**>(p), bytes, cudaHostAllocMapped) != cudaSuccess) {
        cudaGetLastError();
        *p = nullptr;
        return false;
    }
    return true;
}

pariskv_status check_cache(const pariskv_cache* c) {
    if (!c) return fail(PARISKV_EINVAL, "cache is NULL");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != c->device)
        return fail(PARISKV_EINVAL, "cache lives on device %d but device %d is current",
                    c->device, dev);
    return PARISKV_OK;
}

// rows [r0, r0 + nr) of every unit: src (pitch src_rows rows) -> dst (pitch dst_rows rows)
cudaError_t copy_rows(void* dst, int64_t dst_rows, int64_t dst_r0, const void* src,
                      int64_t src_rows, int64_t src_r0, int64_t nr, int units, size_t row,
                      cudaStream_t st) {
    if (nr <= 0) return cudaSuccess;
    return cudaMemcpy2DAsync(static_cast<uint8_t*>(dst) + dst_r0 * row, dst_rows * row,
                             static_cast<const uint8_t*>(src) + src_r0 * row, src_rows * row,
                             nr * row, units, cudaMemcpyDefault, st);
}

Rows rows_of(const pariskv_cache* c) {
    Rows r;
    const int64_t L = c->cc.n_local + c->cc.n_buffer;
    const size_t tmp_bytes = static_cast<size_t>(c->units) * L * c->row;
    r.pool[0] = reinterpret_cast<uint4*>(c->poolK);
    r.pool[1] = reinterpret_cast<uint4*>(c->poolV);
    r.host[0] = reinterpret_cast<uint4*>(c->hostK);
    r.host[1] = reinterpret_cast<uint4*>(c->hostV);
    r.tmp[0] = reinterpret_cast<uint4*>(c->tmp);
    r.tmp[1] = reinterpret_cast<uint4*>(c->tmp + tmp_bytes);
    r.P = c->P;
    r.R = c->cc.retrieval_capacity;
    r.L = L;
    r.vpr = static_cast<int>(c->row / 16);
    return r;
}

// Evicts the oldest `move` Local rows to the Retrieval zone (host rows and index) and slides
// the rest of Local and the buffer down over them. Three launches.
pariskv_status evict(pariskv_cache* c, int64_t move, cudaStream_t st) {
    const int64_t rest = c->local + c->buffer - move;   // rows that stay after Sink
    const Rows r = rows_of(c);
    const dim3 g1(static_cast<unsigned>(ceil_div((move + rest) * r.vpr, 256)),
                  static_cast<unsigned>(c->units), 2);
    spill_kernel<<<g1, 256, 0, st>>>(r, c->sink, move, rest, c->retr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "eviction launch");
    pariskv_status s = pariskv_append(c->ix, c->poolK + c->sink * c->row, c->P, move, st);
    if (s != PARISKV_OK) return s;
    if (rest > 0) {
        const dim3 g2(static_cast<unsigned>(ceil_div(rest * r.vpr, 256)),
                      static_cast<unsigned>(c->units), 2);
        slide_kernel<<<g2, 256, 0, st>>>(r, c->sink, rest);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "compaction launch");
    }
    c->retr += move;
    return PARISKV_OK;
}

// Partials of the dense rows and of the retrieved rows, merged into `out`. The dense rows are
// pool rows [0, n_dense) of every unit: with bf16 K/V one tensor-core pass per unit serves
// all query heads of the group; fp32 caches use the row-gather kernel over an iota index list.
pariskv_status attend(pariskv_cache* c, const void* q, float scale, int32_t k_eff, void* out,
                      int32_t out_dtype, cudaStream_t st, int32_t* launches) {
    const int64_t n_dense = c->sink + c->local + c->buffer;
    const bool dense_mma = c->cfg.dtype == PARISKV_BF16 && c->cfg.group <= 8;
    const int nd = dense_mma ? min(dense_splits(c->units, n_dense, c->sms), c->max_splits)
                             : min(attend_splits(c->heads, static_cast<int32_t>(n_dense), c->sms,
                                                 false),
                                   c->max_splits);
    // the retrieved rows: over the GQA group's union (each row read once over PCIe) when the
    // cache has its scratch, else per head
    const int nr = k_eff <= 0 ? 0
                   : c->uscratch ? min(union_splits(c->units, c->cfg.group, k_eff, c->sms),
                                       c->max_splits)
                                 : min(attend_splits(c->heads, k_eff, c->sms, false),
                                       c->max_splits);
    cudaError_t e =
        dense_mma ? launch_dense_partial(&c->cfg, q, c->poolK, c->poolV, c->P, n_dense, scale,
                                         c->work, nd, 0, nd + nr, st)
                  : launch_attend_partial(&c->cfg, q, c->poolK, c->poolV, c->P, n_dense,
                                          c->dense_idx, static_cast<int32_t>(n_dense), 0, scale,
                                          c->work, nd, 0, nd + nr, false, st);
    *launches += 1;
    if (e == cudaSuccess && nr > 0) {
        if (c->uscratch) {
            e = launch_union_partial(&c->cfg, q, c->hostK, c->hostV, c->cc.retrieval_capacity,
                                     c->retr, c->topk, k_eff, scale, c->work, nr, nd, nd + nr,
                                     c->uscratch, st);
            *launches += 4;   // the union's mark, count and write kernels, then the partials
        } else {
            e = launch_attend_partial(&c->cfg, q, c->hostK, c->hostV, c->cc.retrieval_capacity,
                                      c->retr, c->topk, k_eff, k_eff, scale, c->work, nr, nd,
                                      nd + nr, false, st);
            *launches += 1;
        }
    }
    if (e == cudaSuccess) {
        e = launch_attend_combine(c->heads, c->work, nd + nr, out, out_dtype, st);
        *launches += 1;
    }
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return PARISKV_OK;
}

}  // namespace

extern "C" {

pariskv_status pariskv_cache_create(const pariskv_config* cfg, const pariskv_cache_config* cc,
                                    const int8_t* srht_signs, void* stream,
                                    pariskv_cache** out) {
    if (!out) return fail(PARISKV_EINVAL, "out is NULL");
    *out = nullptr;
    if (!cfg || !cc) return fail(PARISKV_EINVAL, "config is NULL");
    if (cc->n_sink < 0 || cc->n_buffer < 1 || cc->n_local < cc->n_buffer || cc->k < 1 ||
        cc->retrieval_capacity < 1)
        return fail(PARISKV_EINVAL, "cache config needs n_sink >= 0, n_buffer >= 1, "
                    "n_local >= n_buffer, k >= 1, retrieval_capacity >= 1");
    pariskv_config icfg = *cfg;
    icfg.capacity = cc->retrieval_capacity;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    pariskv_index* ix = nullptr;
    // an empty index validates the configuration and the signs
    pariskv_status s = pariskv_build_index(&icfg, srht_signs, nullptr, 0, 0, stream, &ix);
    if (s != PARISKV_OK) return s;
    pariskv_cache* c = new (std::nothrow) pariskv_cache();
    if (!c) {
        pariskv_destroy(ix);
        return fail(PARISKV_ENOMEM, "host allocation failed");
    }
    c->cfg = icfg;
    c->cc = *cc;
    c->ix = ix;
    cudaGetDevice(&c->device);
    cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->device);
    c->units = icfg.batch * icfg.num_kv_heads;
    c->heads = c->units * icfg.group;
    c->P = static_cast<int64_t>(cc->n_sink) + cc->n_local + cc->n_buffer;
    c->row = static_cast<size_t>(D) * (icfg.dtype == PARISKV_BF16 ? 2 : 4);
    // per source: the row-gather kernel takes up to 2*sms/heads splits, the dense pass
    // ceil(2*sms/units)
    c->max_splits = max(max(1, 2 * c->sms / c->heads) + 1,
                        static_cast<int>(ceil_div(2 * c->sms, c->units)));
    const size_t pool = static_cast<size_t>(c->units) * c->P * c->row;
    const size_t host = static_cast<size_t>(c->units) * cc->retrieval_capacity * c->row;
    const bool ok =
        dev_alloc(&c->poolK, pool) && dev_alloc(&c->poolV, pool) &&
        dev_alloc(&c->tmp, 2 * static_cast<size_t>(c->units) * (cc->n_local + cc->n_buffer) *
                               c->row) &&
        dev_alloc(&c->dense_idx, static_cast<size_t>(c->P) * 4) &&
        dev_alloc(&c->topk, static_cast<size_t>(c->heads) * cc->k * 4) &&
        dev_alloc(&c->work, attend_workspace_floats(c->heads, 2 * c->max_splits) * 4) &&
        host_alloc(&c->hostK, host) && host_alloc(&c->hostV, host);
    // the union scratch for the Retrieval zone (bitmaps over its capacity, union lists for k
    // rows per head); skipped (per-head fetching) when the union does not apply
    const size_t ub = union_workspace_bytes(&icfg, cc->retrieval_capacity, cc->k);
    if (ok && ub && !dev_alloc(&c->uscratch, ub)) c->uscratch = nullptr;
    if (!ok) {
        free_cache(c);
        return fail(PARISKV_ENOMEM, "cache allocation failed");
    }
    iota_kernel<<<static_cast<unsigned>(ceil_div(c->P, 256)), 256, 0, st>>>(c->dense_idx, c->P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        free_cache(c);
        return cuda_fail(e, "cache initialisation");
    }
    *out = c;
    return PARISKV_OK;
}

pariskv_status pariskv_cache_prefill(pariskv_cache* c, const void* K, const void* V,
                                     int64_t ld_tok, int64_t n, void* stream) {
    pariskv_status s = check_cache(c);
    if (s != PARISKV_OK) return s;
    if (c->sink + c->local + c->buffer + c->retr != 0)
        return fail(PARISKV_EINVAL, "prefill needs an empty cache");
    if (n < 0 || (n > 0 && ld_tok < n)) return fail(PARISKV_EINVAL, "n < 0 or ld_tok < n");
    if (n == 0) return PARISKV_OK;
    const size_t al = c->cfg.dtype == PARISKV_BF16 ? 8 : 16;
    if ((s = check_device_pointer(K, al, "K")) != PARISKV_OK) return s;
    if ((s = check_device_pointer(V, al, "V")) != PARISKV_OK) return s;
    const int64_t ns = min64(n, c->cc.n_sink), rest = n - ns;
    const int64_t nl = min64(rest, c->cc.n_local), nr = rest - nl;
    if (nr > c->cc.retrieval_capacity)
        return fail(PARISKV_ECAPACITY, "prefill puts %lld tokens in a Retrieval zone of %lld",
                    static_cast<long long>(nr),
                    static_cast<long long>(c->cc.retrieval_capacity));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t R = c->cc.retrieval_capacity;
    cudaError_t e = cudaSuccess;
    for (int t = 0; t < 2 && e == cudaSuccess; ++t) {
        const void* src = t ? V : K;
        uint8_t* pool = t ? c->poolV : c->poolK;
        uint8_t* hostz = t ? c->hostV : c->hostK;
        e = copy_rows(pool, c->P, 0, src, ld_tok, 0, ns, c->units, c->row, st);
        if (e == cudaSuccess)
            e = copy_rows(pool, c->P, ns, src, ld_tok, ns + nr, nl, c->units, c->row, st);
        if (e == cudaSuccess)
            e = copy_rows(hostz, R, 0, src, ld_tok, ns, nr, c->units, c->row, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "prefill copy");
    if (nr > 0) {
        s = pariskv_append(c->ix, static_cast<const uint8_t*>(K) + ns * c->row, ld_tok, nr,
                           stream);
        if (s != PARISKV_OK) return s;
    }
    c->sink = ns;
    c->local = nl;
    c->buffer = 0;
    c->retr = nr;
    set_last_launches(nr > 0 ? 1 : 0);
    return PARISKV_OK;
}

pariskv_status pariskv_cache_step(pariskv_cache* c, const void* q, const void* k_new,
                                  const void* v_new, float scale, void* out, int32_t out_dtype,
                                  int32_t* topk_idx, void* stream) {
    pariskv_status s = check_cache(c);
    if (s != PARISKV_OK) return s;
    const size_t al = c->cfg.dtype == PARISKV_BF16 ? 8 : 16;
    if ((s = check_device_pointer(q, al, "q")) != PARISKV_OK) return s;
    if ((s = check_device_pointer(k_new, al, "k_new")) != PARISKV_OK) return s;
    if ((s = check_device_pointer(v_new, al, "v_new")) != PARISKV_OK) return s;
    if ((s = check_device_pointer(out, out_dtype == PARISKV_BF16 ? 8 : 16, "out")) != PARISKV_OK)
        return s;
    if (out_dtype != PARISKV_F32 && out_dtype != PARISKV_BF16)
        return fail(PARISKV_EINVAL, "out_dtype %d unknown", out_dtype);
    if (topk_idx && (s = check_device_pointer(topk_idx, 4, "topk_idx")) != PARISKV_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // where the new token goes, and whether this step promotes the buffer
    const bool to_sink = c->sink < c->cc.n_sink;
    const int64_t nb = c->buffer + (to_sink ? 0 : 1);
    const bool promote = !to_sink && nb == c->cc.n_buffer;
    const int64_t move = promote ? max64(0, c->local + nb - c->cc.n_local) : 0;
    if (c->retr + move > c->cc.retrieval_capacity)
        return fail(PARISKV_ECAPACITY, "the Retrieval zone (%lld tokens) is full",
                    static_cast<long long>(c->cc.retrieval_capacity));

    int32_t launches = 1;
    const int64_t at = c->sink + c->local + c->buffer;   // first free pool row
    const int vpr8 = static_cast<int>(c->row / 8);
    put_token_kernel<<<static_cast<unsigned>(ceil_div(2 * c->units * vpr8, 256)), 256, 0, st>>>(
        static_cast<const uint2*>(k_new), static_cast<const uint2*>(v_new),
        reinterpret_cast<uint2*>(c->poolK), reinterpret_cast<uint2*>(c->poolV), c->P, at,
        c->units, vpr8);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "token copy");
    if (to_sink) {
        ++c->sink;
    } else {
        c->buffer = nb;
        if (promote) {
            if (move > 0) {
                if ((s = evict(c, move, st)) != PARISKV_OK) return s;
                launches += c->local + c->buffer - move > 0 ? 3 : 2;
            }
            c->local = c->local + c->buffer - move;
            c->buffer = 0;
        }
    }

    int32_t k_eff = 0;
    if (c->retr > 0) {
        k_eff = static_cast<int32_t>(min64(c->cc.k, c->retr));
        s = pariskv_search(c->ix, q, k_eff, c->topk, nullptr, stream);
        if (s != PARISKV_OK) return s;
        launches += last_launches();
    }
    if ((s = attend(c, q, scale, k_eff, out, out_dtype, st, &launches)) != PARISKV_OK) return s;
    if (topk_idx) {
        const size_t bytes = static_cast<size_t>(c->heads) * c->cc.k * 4;
        e = cudaMemsetAsync(topk_idx, 0xff, bytes, st);
        if (e == cudaSuccess && k_eff > 0)
            e = cudaMemcpy2DAsync(topk_idx, static_cast<size_t>(c->cc.k) * 4, c->topk,
                                  static_cast<size_t>(k_eff) * 4,
                                  static_cast<size_t>(k_eff) * 4, c->heads,
                                  cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "top-k copy");
    }
    set_last_launches(launches);
    return PARISKV_OK;
}

pariskv_status pariskv_cache_counts(const pariskv_cache* c, int64_t* counts) {
    if (!c || !counts) return fail(PARISKV_EINVAL, "NULL argument");
    counts[0] = c->sink;
    counts[1] = c->local;
    counts[2] = c->buffer;
    counts[3] = c->retr;
    return PARISKV_OK;
}

pariskv_index* pariskv_cache_index(pariskv_cache* c) { return c ? c->ix : nullptr; }

pariskv_status pariskv_cache_destroy(pariskv_cache* c) {
    if (!c) return PARISKV_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    cudaDeviceSynchronize();
    free_cache(c);
    cudaSetDevice(prev);
    return PARISKV_OK;
}

}  // extern "C"
