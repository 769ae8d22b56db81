// api.cu -- the C ABI of libpariskv.so: argument validation, memory ownership and the
// launch sequence of each call. Every step of the retrieval path runs in the kernels of this
// library; the host only validates, allocates and launches.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "internal.hpp"
#include "pariskv_dense.h"
#include "pariskv_learned.h"
#include "pariskv_debug.h"

using namespace pkv;

namespace {

thread_local char g_err[512] = "";
thread_local int32_t g_launches = 0;

void set_err(const char* fmt, va_list ap) { vsnprintf(g_err, sizeof(g_err), fmt, ap); }

// Test hooks (failures made on the host; no device fault is involved):
//  PARISKV_FAULT=alloc makes every device allocation of the library fail, so the ENOMEM
//  paths (and their cleanup) run without exhausting a real device;
//  PARISKV_FAULT=launch makes every call that launches kernels (search, append, the
//  attentions) fail with ECUDA before its first launch, as a launch error would, so that the
//  callers' error paths and the index's unchanged state can be checked.
bool fault_alloc() {
    const char* f = getenv("PARISKV_FAULT");
    return f && strcmp(f, "alloc") == 0;
}

bool fault_launch() {
    const char* f = getenv("PARISKV_FAULT");
    return f && strcmp(f, "launch") == 0;
}

pariskv_status injected_launch_failure() {
    return fail(PARISKV_ECUDA, "injected launch failure (PARISKV_FAULT=launch)");
}

// Guard bytes (a test aid standing in for a memory checker): with PARISKV_GUARD=1 in the
// environment when the library makes its first index allocation, every device buffer an
// index owns gets kGuard bytes of a fixed pattern before and after it. They are checked when
// the buffer is freed and by pariskv_debug_check_guards; a kernel that wrote past either end
// of a buffer is reported there by the buffer's size and the side it overran.
constexpr size_t kGuard = 256;            // keeps the buffer 256-byte aligned
constexpr unsigned char kGuardByte = 0xA5;
struct Guarded {
    char* base;
    size_t bytes;
};
std::mutex g_guard_mu;
std::vector<Guarded> g_guarded;           // live guarded buffers
char g_guard_bad[256] = "";               // first overrun seen (empty: none)

bool guards_on() {
    static const bool on = [] {
        const char* v = getenv("PARISKV_GUARD");
        return v && v[0] == '1';
    }();
    return on;
}

// Checks one buffer's guards (synchronous); records the first overrun in g_guard_bad.
bool guard_ok(const Guarded& g) {
    unsigned char h[2][kGuard];
    if (cudaMemcpy(h[0], g.base, kGuard, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(h[1], g.base + kGuard + g.bytes, kGuard, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return true;   // unreadable (device error): reported by the call that failed
    }
    for (int side = 0; side < 2; ++side)
        for (size_t i = 0; i < kGuard; ++i)
            if (h[side][i] != kGuardByte) {
                if (!g_guard_bad[0])
                    snprintf(g_guard_bad, sizeof(g_guard_bad),
                             "guard bytes %s a %zu-byte index buffer were overwritten (byte %zu)",
                             side ? "after" : "before", g.bytes, i);
                return false;
            }
    return true;
}

void* raw_alloc(size_t bytes) {
    void* p = nullptr;
    if (!guards_on()) {
        if (cudaMalloc(&p, bytes) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return p;
    }
    char* base = nullptr;
    if (cudaMalloc(reinterpret_cast<void**>(&base), bytes + 2 * kGuard) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (cudaMemset(base, kGuardByte, kGuard) != cudaSuccess ||
        cudaMemset(base + kGuard + bytes, kGuardByte, kGuard) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(base);
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_guard_mu);
    g_guarded.push_back({base, bytes});
    return base + kGuard;
}

void raw_free(void* p) {
    if (!p) return;
    if (guards_on()) {
        std::lock_guard<std::mutex> lk(g_guard_mu);
        for (size_t i = 0; i < g_guarded.size(); ++i)
            if (g_guarded[i].base + kGuard == p) {
                cudaDeviceSynchronize();
                guard_ok(g_guarded[i]);
                cudaFree(g_guarded[i].base);
                g_guarded[i] = g_guarded.back();
                g_guarded.pop_back();
                return;
            }
    }
    cudaFree(p);
}

template <typename T>
bool dalloc(T** p, size_t count) {
    *p = nullptr;
    if (count == 0) count = 1;
    if (fault_alloc()) return false;
    *p = static_cast<T*>(raw_alloc(count * sizeof(T)));
    return *p != nullptr;
}

template <typename T>
void dfree(T*& p) {
    raw_free(p);
    p = nullptr;
}

int64_t candidate_count(int64_t n, int64_t k, int32_t bp) {
    int64_t c = (n * bp + 9999) / 10000;
    if (c < k) c = k;
    if (c > n) c = n;
    return c;
}

pariskv_status check_config(const pariskv_config* c) {
    if (!c) return fail(PARISKV_EINVAL, "config is NULL");
    if (c->d != D || c->m != M || c->B != NB)
        return fail(PARISKV_EINVAL, "shape d=%d B=%d m=%d unsupported (need d=128, B=16, m=8)",
                    c->d, c->B, c->m);
    if (c->rho < 1 || c->rho > NC) return fail(PARISKV_EINVAL, "rho=%d not in [1, 256]", c->rho);
    if (c->w_rank1 < 1 || c->w_rank1 > 3 || c->w_rest < 0 || c->w_rest > c->w_rank1)
        return fail(PARISKV_EINVAL, "vote weights (%d, %d) need 1 <= w_rank1 <= 3 and "
                    "0 <= w_rest <= w_rank1", c->w_rank1, c->w_rest);
    if (c->cand_bp < 1 || c->cand_bp > 10000)
        return fail(PARISKV_EINVAL, "cand_bp=%d not in [1, 10000]", c->cand_bp);
    if (c->batch < 1 || c->num_kv_heads < 1 || c->group < 1)
        return fail(PARISKV_EINVAL, "batch, num_kv_heads and group must be >= 1");
    const int64_t heads = static_cast<int64_t>(c->batch) * c->num_kv_heads * c->group;
    if (heads > 65535) return fail(PARISKV_EINVAL, "batch * query heads = %lld > 65535",
                                   static_cast<long long>(heads));
    if (c->capacity < 0 || c->capacity > (int64_t(1) << 31) - CHUNK)
        return fail(PARISKV_EINVAL, "capacity %lld out of range",
                    static_cast<long long>(c->capacity));
    if (c->dtype != PARISKV_F32 && c->dtype != PARISKV_BF16)
        return fail(PARISKV_EINVAL, "dtype %d unknown", c->dtype);
    if (c->levels != PARISKV_LEVELS_UNIFORM && c->levels != PARISKV_LEVELS_PRIOR &&
        c->levels != PARISKV_LEVELS_TABLE)
        return fail(PARISKV_EINVAL, "levels=%d unknown", c->levels);
    if (c->levels == PARISKV_LEVELS_TABLE)
        for (int i = 0; i < 8; ++i)
            if (!std::isfinite(c->level_table[i]) ||
                (i == 0 ? c->level_table[0] < 0.0f : !(c->level_table[i] > c->level_table[i - 1])))
                return fail(PARISKV_EINVAL, "level_table must be finite with 0 <= c0 < ... < c7");
    return PARISKV_OK;
}

// A pointer the current device can dereference: device memory, managed memory, or host
// memory that is pinned/registered (UVA maps it into the device address space).
pariskv_status check_dev_ptr(const void* p, size_t align, const char* name) {
    if (!p) return fail(PARISKV_EINVAL, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % align)
        return fail(PARISKV_EINVAL, "%s is not %zu-byte aligned", name, align);
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return fail(PARISKV_EINVAL, "%s is not a CUDA-visible pointer", name);
    }
    if (a.type == cudaMemoryTypeUnregistered)
        return fail(PARISKV_EINVAL, "%s is pageable host memory (pin or register it)", name);
    if (a.type == cudaMemoryTypeHost && a.devicePointer != p)
        return fail(PARISKV_EINVAL, "%s: pinned host memory without an identical device "
                    "mapping", name);
    return PARISKV_OK;
}

// true for device (or managed) memory, false for pinned host memory
bool device_memory(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

}  // namespace

namespace pkv {
bool alloc_fault_injected() { return fault_alloc(); }
pariskv_status check_device_pointer(const void* p, size_t align, const char* name) {
    return check_dev_ptr(p, align, name);
}
pariskv_status validate_config(const pariskv_config* cfg) { return check_config(cfg); }
void set_last_launches(int32_t n) { g_launches = n; }
int32_t last_launches() { return g_launches; }
}  // namespace pkv

namespace {

pariskv_status check_index(const pariskv_index* ix) {
    if (!ix) return fail(PARISKV_EINVAL, "index is NULL");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != ix->device)
        return fail(PARISKV_EINVAL, "index lives on device %d but device %d is current",
                    ix->device, dev);
    return PARISKV_OK;
}

void free_index(pariskv_index* ix) {
    if (!ix) return;
    dfree(ix->signs); dfree(ix->ids); dfree(ix->rec); dfree(ix->lut); dfree(ix->qt);
    dfree(ix->qnorm); dfree(ix->scores); dfree(ix->hist); dfree(ix->thr); dfree(ix->cbase);
    dfree(ix->cand); dfree(ix->S); dfree(ix->shist); dfree(ix->status); dfree(ix->lvt);
    dfree(ix->cent);
    for (auto& e : ix->ev)
        if (e) cudaEventDestroy(e);
    delete ix;
}

pariskv_status ensure_candidates(pariskv_index* ix, int64_t C);

pariskv_status create_index(const pariskv_config* cfg, const int8_t* signs, cudaStream_t st,
                            pariskv_index** out) {
    *out = nullptr;
    for (int j = 0; j < D; ++j)
        if (signs[j] != 1 && signs[j] != -1)
            return fail(PARISKV_EINVAL, "srht_signs[%d] = %d is not +-1", j, signs[j]);
    pariskv_index* ix = new (std::nothrow) pariskv_index();
    if (!ix) return fail(PARISKV_ENOMEM, "host allocation failed");
    ix->cfg = *cfg;
    memcpy(ix->hsigns, signs, sizeof(ix->hsigns));
    cudaGetDevice(&ix->device);
    ix->units = cfg->batch * cfg->num_kv_heads;
    ix->hq = cfg->num_kv_heads * cfg->group;
    ix->packs = static_cast<int>(ceil_div(cfg->group, PACK));
    ix->cap_pad = round_up(cfg->capacity > 0 ? cfg->capacity : 1, CHUNK);
    const int64_t up = static_cast<int64_t>(ix->units) * ix->packs;
    const int64_t heads = static_cast<int64_t>(ix->units) * cfg->group;
    const int64_t nch = ix->cap_pad / CHUNK;
    bool ok = dalloc(&ix->signs, D) && dalloc(&ix->ids, ix->units * ix->cap_pad * 16) &&
              dalloc(&ix->rec, ix->units * ix->cap_pad * REC) &&
              dalloc(&ix->lut, up * NB * NC) && dalloc(&ix->qt, heads * D) &&
              dalloc(&ix->qnorm, heads) && dalloc(&ix->scores, up * ix->cap_pad) &&
              dalloc(&ix->hist, up * nch * PACK * NBINS) && dalloc(&ix->thr, heads * 4) &&
              dalloc(&ix->cbase, heads * nch * 2) && dalloc(&ix->shist, heads * SCOPIES * SBINS) &&
              dalloc(&ix->status, 1) && dalloc(&ix->lvt, kLevelTableFloats);
    if (!ok) {
        free_index(ix);
        return fail(PARISKV_ENOMEM, "device allocation for the index failed");
    }
    // candidate buffers for a full index up front, so a search on a growing index never
    // reallocates them (a cudaFree synchronises the device) unless k exceeds the pruned count
    pariskv_status s = ensure_candidates(ix, candidate_count(cfg->capacity, 1, cfg->cand_bp));
    if (s != PARISKV_OK) {
        free_index(ix);
        return s;
    }
    float hs[D], tab[kLevelTableFloats];
    for (int j = 0; j < D; ++j) hs[j] = static_cast<float>(signs[j]);
    if ((s = level_tables(cfg, tab)) != PARISKV_OK) {
        free_index(ix);
        return s;
    }
    if (cfg->levels == PARISKV_LEVELS_PRIOR)   // record the levels the index is coded with
        for (int i = 0; i < 8; ++i) ix->cfg.level_table[i] = tab[i];
    cudaError_t e = cudaMemcpyAsync(ix->signs, hs, sizeof(hs), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(ix->lvt, tab, sizeof(tab), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ix->lut, 0, up * NB * NC * sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ix->status, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);  // hs, tab live on this stack frame
    if (e != cudaSuccess) {
        free_index(ix);
        return cuda_fail(e, "index initialisation");
    }
    *out = ix;
    return PARISKV_OK;
}

pariskv_status ensure_candidates(pariskv_index* ix, int64_t C) {
    if (C <= ix->cmax) return PARISKV_OK;
    C = round_up(C, 32);  // every head's slice starts on a 128-byte boundary
    const int64_t heads = static_cast<int64_t>(ix->units) * ix->cfg.group;
    int32_t* c2 = nullptr;
    float* s2 = nullptr;
    if (!dalloc(&c2, heads * C) || !dalloc(&s2, heads * C)) {
        dfree(c2);
        dfree(s2);
        return fail(PARISKV_ENOMEM, "candidate buffers (%lld per head)", static_cast<long long>(C));
    }
    dfree(ix->cand);
    dfree(ix->S);
    ix->cand = c2;
    ix->S = s2;
    ix->cmax = C;
    return PARISKV_OK;
}

pariskv_status run_search(pariskv_index* ix, const void* q, const float* qt, const float* qn,
                          bool rotated, int32_t k, int32_t* topk_idx, float* topk_est,
                          cudaStream_t st) {
    if (k < 1 || k > ix->n)
        return fail(PARISKV_EINVAL, "k=%d not in [1, size=%lld]", k, static_cast<long long>(ix->n));
    const int64_t C = candidate_count(ix->n, k, ix->cfg.cand_bp);
    pariskv_status s = ensure_candidates(ix, C);
    if (s != PARISKV_OK) return s;
    // a slot past C is refused, except (with guard bytes on) one inside the guard that
    // follows the candidate buffer, which tests that an overrun is detected
    const int64_t slot = static_cast<int64_t>(ix->inject_head) * ix->cmax + ix->inject_pos;
    const int64_t cand_end = static_cast<int64_t>(ix->units) * ix->cfg.group * ix->cmax;
    const bool into_guard = guards_on() && slot >= cand_end &&
                            slot < cand_end + static_cast<int64_t>(kGuard / sizeof(int32_t));
    if (ix->inject_head >= 0 && ix->inject_pos >= C && !into_guard) {
        ix->inject_head = -1;
        return fail(PARISKV_EINVAL, "injected candidate position %lld >= C = %lld",
                    static_cast<long long>(ix->inject_pos), static_cast<long long>(C));
    }
    if (ix->inject_wait && (ix->topk_mode == 4 || C > 4 * 16384)) {
        ix->inject_wait = false;
        return fail(PARISKV_EINVAL, "the top-k of C = %lld candidates stages no copies to wait for",
                    static_cast<long long>(C));
    }
    if (ix->topk_mode != 0 && !topk_mode_fits(ix->topk_mode, C))
        return fail(PARISKV_EINVAL, "top-k launch shape %d cannot hold C = %lld candidates",
                    ix->topk_mode, static_cast<long long>(C));
    if (fault_launch()) return injected_launch_failure();
    g_launches = 0;
    int ne = 0;
    auto mark = [&]() {
        if (ix->profile) cudaEventRecord(ix->ev[ne++], st);
    };
    mark();
    cudaError_t e = launch_query_prep(ix, q, qt, qn, rotated, st);
    if (e == cudaSuccess) { ++g_launches; mark(); e = launch_vote(ix, st); }
    if (e == cudaSuccess) { ++g_launches; mark(); e = launch_threshold(ix, C, st); }
    if (e == cudaSuccess) { ++g_launches; mark(); e = launch_compact(ix, st); }
    if (e == cudaSuccess && ix->inject_head >= 0) {   // test hook: one bad candidate index
        e = launch_poke(ix->cand + ix->inject_head * ix->cmax + ix->inject_pos, ix->inject_value, st);
        ix->inject_head = -1;
    }
    if (e == cudaSuccess) { ++g_launches; mark(); e = launch_rerank(ix, C, st); }
    if (e == cudaSuccess) { ++g_launches; mark(); e = launch_topk(ix, C, k, topk_idx, topk_est, st); }
    ix->inject_wait = false;
    if (e == cudaSuccess) { ++g_launches; mark(); }
    ix->nev = ne;
    if (e != cudaSuccess) return cuda_fail(e, "search launch");
    ix->last_C = C;
    ix->last_k = k;
    ix->searched = true;
    return PARISKV_OK;
}

}  // namespace

namespace pkv {

pariskv_status fail(pariskv_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    set_err(fmt, ap);
    va_end(ap);
    return s;
}

pariskv_status cuda_fail(cudaError_t e, const char* what) {
    cudaGetLastError();
    snprintf(g_err, sizeof(g_err), "%s: %s", what, cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? PARISKV_ENOMEM : PARISKV_ECUDA;
}

}  // namespace pkv

// =========================================================================================
// Product surface
// =========================================================================================
extern "C" {

pariskv_status pariskv_config_default(pariskv_config* cfg) {
    if (!cfg) return fail(PARISKV_EINVAL, "config is NULL");
    memset(cfg, 0, sizeof(*cfg));
    cfg->d = D; cfg->B = NB; cfg->m = M; cfg->rho = 4; cfg->w_rank1 = 2; cfg->w_rest = 1;
    cfg->cand_bp = 500; cfg->batch = 1; cfg->num_kv_heads = 1; cfg->group = 1;
    cfg->capacity = 0; cfg->dtype = PARISKV_BF16;
    return PARISKV_OK;
}

static pariskv_status build_common(const pariskv_config* cfg, const int8_t* srht_signs,
                                   const void* keys, const float* knorm, bool rotated,
                                   int64_t ld_tok, int64_t n, void* stream,
                                   pariskv_index** out) {
    if (!out) return fail(PARISKV_EINVAL, "out is NULL");
    *out = nullptr;
    pariskv_status s = check_config(cfg);
    if (s != PARISKV_OK) return s;
    if (!srht_signs) return fail(PARISKV_EINVAL, "srht_signs is NULL");
    if (n < 0 || n > cfg->capacity)
        return fail(PARISKV_EINVAL, "n=%lld not in [0, capacity=%lld]", static_cast<long long>(n),
                    static_cast<long long>(cfg->capacity));
    if (n > 0) {
        if (ld_tok < n) return fail(PARISKV_EINVAL, "ld_tok < n");
        s = check_dev_ptr(keys, rotated ? 16 : (cfg->dtype == PARISKV_BF16 ? 8 : 16), "keys");
        if (s != PARISKV_OK) return s;
        if (rotated && (s = check_dev_ptr(knorm, 4, "knorm")) != PARISKV_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    pariskv_index* ix = nullptr;
    s = create_index(cfg, srht_signs, st, &ix);
    if (s != PARISKV_OK) return s;
    cudaError_t e = launch_encode(ix, keys, knorm, ld_tok, n, 0, rotated, st);
    if (e != cudaSuccess) {
        free_index(ix);
        return cuda_fail(e, "encode launch");
    }
    ix->n = n;
    *out = ix;
    return PARISKV_OK;
}

pariskv_status pariskv_build_index(const pariskv_config* cfg, const int8_t* srht_signs,
                                   const void* keys, int64_t ld_tok, int64_t n, void* stream,
                                   pariskv_index** out) {
    return build_common(cfg, srht_signs, keys, nullptr, false, ld_tok, n, stream, out);
}

static pariskv_status append_common(pariskv_index* ix, const void* keys, const float* knorm,
                                    bool rotated, int64_t ld_tok, int64_t t, void* stream) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (t < 0) return fail(PARISKV_EINVAL, "t < 0");
    if (t == 0) return PARISKV_OK;
    if (ix->n + t > ix->cfg.capacity)
        return fail(PARISKV_ECAPACITY, "append of %lld keys exceeds capacity %lld (size %lld)",
                    static_cast<long long>(t), static_cast<long long>(ix->cfg.capacity),
                    static_cast<long long>(ix->n));
    if (ld_tok < t) return fail(PARISKV_EINVAL, "ld_tok < t");
    s = check_dev_ptr(keys, rotated ? 16 : (ix->cfg.dtype == PARISKV_BF16 ? 8 : 16), "keys");
    if (s != PARISKV_OK) return s;
    if (rotated && (s = check_dev_ptr(knorm, 4, "knorm")) != PARISKV_OK) return s;
    if (fault_launch()) return injected_launch_failure();
    cudaError_t e = launch_encode(ix, keys, knorm, ld_tok, t, ix->n, rotated,
                                  static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "encode launch");
    ix->n += t;
    return PARISKV_OK;
}

pariskv_status pariskv_append(pariskv_index* index, const void* keys, int64_t ld_tok, int64_t t,
                              void* stream) {
    return append_common(index, keys, nullptr, false, ld_tok, t, stream);
}

pariskv_status pariskv_search(pariskv_index* index, const void* q, int32_t k, int32_t* topk_idx,
                              float* topk_est, void* stream) {
    pariskv_status s = check_index(index);
    if (s != PARISKV_OK) return s;
    if ((s = check_dev_ptr(q, index->cfg.dtype == PARISKV_BF16 ? 8 : 16, "q")) != PARISKV_OK)
        return s;
    if ((s = check_dev_ptr(topk_idx, 4, "topk_idx")) != PARISKV_OK) return s;
    if (topk_est && (s = check_dev_ptr(topk_est, 4, "topk_est")) != PARISKV_OK) return s;
    return run_search(index, q, nullptr, nullptr, false, k, topk_idx, topk_est,
                      static_cast<cudaStream_t>(stream));
}

// Stream-ordered workspaces of the allocating attention call come from a library-owned pool
// per device that keeps its memory mapped (release threshold: unlimited). Freed workspaces
// are reused by later calls, so a call never maps or unmaps device memory once the pool has
// grown to its working size; with the default pool, memory released at every synchronisation
// and mapped again by the next call was measured to slow the following host-memory gathers
// (first-touch and TLB costs) by up to 4x.
static cudaError_t workspace_pool(cudaMemPool_t* out) {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        e = cudaMemPoolCreate(&p, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = ~uint64_t{0};
        e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(p);
            return e;
        }
        pools[dev] = p;
    }
    *out = pools[dev];
    return cudaSuccess;
}

pariskv_status pariskv_sparse_attend(const pariskv_config* cfg, const void* q, const void* K,
                                     const void* V, int64_t ld_tok, int64_t n,
                                     const int32_t* topk_idx, int32_t k, float scale, void* out,
                                     int32_t out_dtype, void* stream) {


    pariskv_status s = check_config(cfg);
    if (s != PARISKV_OK) return s;
    const size_t al = cfg->dtype == PARISKV_BF16 ? 8 : 16;
    if (k < 1 || k > n) return fail(PARISKV_EINVAL, "k=%d not in [1, n=%lld]", k,
                                    static_cast<long long>(n));
    if (ld_tok < n) return fail(PARISKV_EINVAL, "ld_tok < n");
    if ((s = check_dev_ptr(q, al, "q")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(K, al, "K")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(V, al, "V")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(topk_idx, 4, "topk_idx")) != PARISKV_OK) return s;
    if (out_dtype != PARISKV_F32 && out_dtype != PARISKV_BF16)
        return fail(PARISKV_EINVAL, "out_dtype %d unknown", out_dtype);
    if ((s = check_dev_ptr(out, out_dtype == PARISKV_BF16 ? 8 : 16, "out")) != PARISKV_OK)
        return s;
    if (!(scale == scale)) return fail(PARISKV_EINVAL, "scale is NaN");
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int heads = cfg->batch * cfg->num_kv_heads * cfg->group;
    const bool mma = attend_uses_mma(cfg, device_memory(K) && device_memory(V));
    // the row-gather kernel fetches each row of a GQA group's union once when it can
    const size_t ubytes = mma ? 0 : union_workspace_bytes(cfg, n, k);
    const int nsplit = ubytes ? union_splits(cfg->batch * cfg->num_kv_heads, cfg->group, k, sms)
                              : attend_splits(heads, k, sms, mma);
    const size_t pbytes = round_up(attend_workspace_floats(heads, nsplit) * sizeof(float), 256);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* work = nullptr;
    if (fault_alloc()) return fail(PARISKV_ENOMEM, "attention workspace");
    if (fault_launch()) return injected_launch_failure();
    cudaMemPool_t pool = nullptr;
    cudaError_t e = workspace_pool(&pool);
    if (e == cudaSuccess)
        e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&work), pbytes + ubytes, pool, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention workspace");
    g_launches = 0;
    if (ubytes) {
        e = launch_attend_union(cfg, q, K, V, ld_tok, n, topk_idx, k, scale, out, out_dtype, work,
                                nsplit, reinterpret_cast<char*>(work) + pbytes, st);
        if (e == cudaSuccess) g_launches = 5;   // mark, count, write, attention, merge
    } else {
        e = launch_attend(cfg, q, K, V, ld_tok, n, topk_idx, k, scale, out, out_dtype, work,
                          nsplit, mma, st);
        if (e == cudaSuccess) g_launches = 2;
    }
    cudaFreeAsync(work, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return PARISKV_OK;
}

pariskv_status pariskv_dense_attend(const pariskv_config* cfg, const void* q, const void* K,
                                    const void* V, int64_t ld_tok, int64_t n, float scale,
                                    void* out, int32_t out_dtype, void* stream) {
    pariskv_status s = check_config(cfg);
    if (s != PARISKV_OK) return s;
    if (cfg->dtype != PARISKV_BF16) return fail(PARISKV_EINVAL, "dense attention reads bf16 K/V");
    if (cfg->group > 8) return fail(PARISKV_EINVAL, "group %d > 8", cfg->group);
    if (n < 1 || ld_tok < n) return fail(PARISKV_EINVAL, "need 1 <= n <= ld_tok");
    if ((s = check_dev_ptr(q, 4, "q")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(K, 16, "K")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(V, 16, "V")) != PARISKV_OK) return s;
    if (out_dtype != PARISKV_F32 && out_dtype != PARISKV_BF16)
        return fail(PARISKV_EINVAL, "out_dtype %d unknown", out_dtype);
    if ((s = check_dev_ptr(out, out_dtype == PARISKV_BF16 ? 8 : 16, "out")) != PARISKV_OK)
        return s;
    if (!(scale == scale)) return fail(PARISKV_EINVAL, "scale is NaN");
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int units = cfg->batch * cfg->num_kv_heads;
    const int heads = units * cfg->group;
    const int nsplit = dense_splits(units, n, sms);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* work = nullptr;
    if (fault_alloc()) return fail(PARISKV_ENOMEM, "attention workspace");
    if (fault_launch()) return injected_launch_failure();
    cudaMemPool_t pool = nullptr;
    cudaError_t e = workspace_pool(&pool);
    if (e == cudaSuccess)
        e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&work),
                                    attend_workspace_floats(heads, nsplit) * sizeof(float), pool,
                                    st);
    if (e != cudaSuccess) return cuda_fail(e, "attention workspace");
    g_launches = 0;
    e = launch_dense_partial(cfg, q, K, V, ld_tok, n, scale, work, nsplit, 0, nsplit, st);
    if (e == cudaSuccess) e = launch_attend_combine(heads, work, nsplit, out, out_dtype, st);
    if (e == cudaSuccess) g_launches = 2;
    cudaFreeAsync(work, st);
    if (e != cudaSuccess) return cuda_fail(e, "dense attention launch");
    return PARISKV_OK;
}

pariskv_status pariskv_sparse_attend_noalloc(const pariskv_config* cfg, const void* q,
                                             const void* K, const void* V, int64_t ld_tok,
                                             int64_t n, const int32_t* topk_idx, int32_t k,
                                             float scale, void* out, int32_t out_dtype,
                                             void* stream) {
    pariskv_status s = check_config(cfg);
    if (s != PARISKV_OK) return s;
    const size_t al = cfg->dtype == PARISKV_BF16 ? 8 : 16;
    if (k < 1 || k > n) return fail(PARISKV_EINVAL, "k=%d not in [1, n=%lld]", k,
                                    static_cast<long long>(n));
    if (ld_tok < n) return fail(PARISKV_EINVAL, "ld_tok < n");
    if ((s = check_dev_ptr(q, al, "q")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(K, al, "K")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(V, al, "V")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(topk_idx, 4, "topk_idx")) != PARISKV_OK) return s;
    if (out_dtype != PARISKV_F32 && out_dtype != PARISKV_BF16)
        return fail(PARISKV_EINVAL, "out_dtype %d unknown", out_dtype);
    if ((s = check_dev_ptr(out, out_dtype == PARISKV_BF16 ? 8 : 16, "out")) != PARISKV_OK)
        return s;
    if (!(scale == scale)) return fail(PARISKV_EINVAL, "scale is NaN");
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int heads = cfg->batch * cfg->num_kv_heads * cfg->group;
    // the split count is capped so that the partials fit the fixed workspace
    const size_t per_split = attend_workspace_floats(heads, 1);
    const int fit = static_cast<int>(kAttendScratchFloats / per_split);
    if (fit < 1)
        return fail(PARISKV_EINVAL, "%d query heads exceed the fixed attention workspace "
                    "(at most %zu heads)", heads, kAttendScratchFloats / attend_workspace_floats(1, 1));
    // the tensor-core gather kernel needs a minimum split count; with too small a fixed
    // workspace the row-gather kernel runs instead
    const bool mma = attend_uses_mma(cfg, device_memory(K) && device_memory(V)) &&
                     gather_min_splits(k) <= fit;
    const int nsplit = min(attend_splits(heads, k, sms, mma), fit);
    float* work = nullptr;
    if (fault_launch()) return injected_launch_failure();
    cudaError_t e = attend_static_scratch(&work);
    if (e != cudaSuccess) return cuda_fail(e, "fixed attention workspace lookup");
    g_launches = 0;
    e = launch_attend(cfg, q, K, V, ld_tok, n, topk_idx, k, scale, out, out_dtype, work, nsplit,
                      mma, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    g_launches = 2;
    return PARISKV_OK;
}

// ------------------------------------------------------------------------- index images
namespace {

constexpr char kMagic[8] = {'P', 'A', 'R', 'I', 'S', 'K', 'V', '\0'};
constexpr uint32_t kImageVersion = 2;

struct ImageHeader {
    char magic[8];
    uint32_t version;
    uint32_t header_bytes;
    pariskv_config cfg;
    int64_t n;
    int32_t units;
    int32_t reserved;
    int8_t signs[D];
    uint8_t pad[256 - 120 - D];
};
static_assert(sizeof(pariskv_config) == 88, "image header layout");
static_assert(sizeof(ImageHeader) == 256, "image header layout");

constexpr size_t kKeyBytes = 16 + REC;   // bucket ids + code record per key

}  // namespace

pariskv_status pariskv_export_bytes(const pariskv_index* ix, size_t* bytes) {
    if (!ix || !bytes) return fail(PARISKV_EINVAL, "NULL argument");
    *bytes = sizeof(ImageHeader) + static_cast<size_t>(ix->units) * ix->n * kKeyBytes;
    return PARISKV_OK;
}

pariskv_status pariskv_export(pariskv_index* ix, void* buf, size_t bytes, void* stream) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (ix->cent) return fail(PARISKV_EINVAL, "an index with learned centroids has no image");
    size_t need = 0;
    pariskv_export_bytes(ix, &need);
    if (!buf) return fail(PARISKV_EINVAL, "buf is NULL");
    if (bytes < need)
        return fail(PARISKV_EINVAL, "buffer of %zu bytes; the image needs %zu", bytes, need);
    ImageHeader h;
    memset(&h, 0, sizeof(h));
    memcpy(h.magic, kMagic, sizeof(kMagic));
    h.version = kImageVersion;
    h.header_bytes = sizeof(ImageHeader);
    h.cfg = ix->cfg;
    h.n = ix->n;
    h.units = ix->units;
    memcpy(h.signs, ix->hsigns, sizeof(h.signs));
    uint8_t* out = static_cast<uint8_t*>(buf);
    memcpy(out, &h, sizeof(h));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t nid = static_cast<size_t>(ix->n) * 16, nrec = static_cast<size_t>(ix->n) * REC;
    uint8_t* ids = out + sizeof(h);
    uint8_t* rec = ids + static_cast<size_t>(ix->units) * nid;
    cudaError_t e = cudaSuccess;
    for (int u = 0; u < ix->units && ix->n > 0 && e == cudaSuccess; ++u) {
        e = cudaMemcpyAsync(ids + u * nid, ix->ids + u * ix->cap_pad * 16, nid,
                            cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(rec + u * nrec, ix->rec + u * ix->cap_pad * REC, nrec,
                                cudaMemcpyDeviceToHost, st);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "export copy");
    return PARISKV_OK;
}

pariskv_status pariskv_import(const void* buf, size_t bytes, int64_t capacity, void* stream,
                              pariskv_index** out) {
    if (!out) return fail(PARISKV_EINVAL, "out is NULL");
    *out = nullptr;
    if (!buf) return fail(PARISKV_EINVAL, "buf is NULL");
    if (bytes < sizeof(ImageHeader))
        return fail(PARISKV_EINVAL, "%zu bytes cannot hold an image header", bytes);
    ImageHeader h;
    memcpy(&h, buf, sizeof(h));
    if (memcmp(h.magic, kMagic, sizeof(kMagic)) != 0)
        return fail(PARISKV_EINVAL, "not a ParisKV index image");
    if (h.version != kImageVersion || h.header_bytes != sizeof(ImageHeader))
        return fail(PARISKV_EINVAL, "image format version %u (this library reads %u)",
                    h.version, kImageVersion);
    if (h.n < 0 || h.units < 1 || h.cfg.batch < 1 || h.cfg.num_kv_heads < 1 ||
        static_cast<int64_t>(h.cfg.batch) * h.cfg.num_kv_heads != h.units)
        return fail(PARISKV_EINVAL, "inconsistent image header");
    if (capacity == 0) capacity = h.n > 0 ? h.n : 1;
    if (capacity < h.n)
        return fail(PARISKV_EINVAL, "capacity %lld below the image's size %lld",
                    static_cast<long long>(capacity), static_cast<long long>(h.n));
    pariskv_config cfg = h.cfg;
    cfg.capacity = capacity;
    // an index coded with the prior-derived levels keeps exactly the levels it was coded with
    if (cfg.levels == PARISKV_LEVELS_PRIOR) cfg.levels = PARISKV_LEVELS_TABLE;
    pariskv_status s = check_config(&cfg);
    if (s != PARISKV_OK) return s;
    const size_t nid = static_cast<size_t>(h.n) * 16, nrec = static_cast<size_t>(h.n) * REC;
    if ((bytes - sizeof(h)) / kKeyBytes / h.units < static_cast<size_t>(h.n))
        return fail(PARISKV_EINVAL, "image truncated: %zu bytes for %d units of %lld keys",
                    bytes, h.units, static_cast<long long>(h.n));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    pariskv_index* ix = nullptr;
    if ((s = create_index(&cfg, h.signs, st, &ix)) != PARISKV_OK) return s;
    const uint8_t* ids = static_cast<const uint8_t*>(buf) + sizeof(h);
    const uint8_t* rec = ids + static_cast<size_t>(h.units) * nid;
    cudaError_t e = cudaSuccess;
    for (int u = 0; u < ix->units && h.n > 0 && e == cudaSuccess; ++u) {
        e = cudaMemcpyAsync(ix->ids + u * ix->cap_pad * 16, ids + u * nid, nid,
                            cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(ix->rec + u * ix->cap_pad * REC, rec + u * nrec, nrec,
                                cudaMemcpyHostToDevice, st);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        free_index(ix);
        return cuda_fail(e, "import copy");
    }
    ix->n = h.n;
    *out = ix;
    return PARISKV_OK;
}

pariskv_status pariskv_set_centroids(pariskv_index* ix, const float* centroids, void* stream) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (ix->n != 0) return fail(PARISKV_EINVAL, "centroids can only be set on an empty index");
    if ((s = check_dev_ptr(centroids, 16, "centroids")) != PARISKV_OK) return s;
    const size_t count = static_cast<size_t>(ix->units) * NB * NC * 8;
    if (!ix->cent && !dalloc(&ix->cent, count))
        return fail(PARISKV_ENOMEM, "centroid table");
    cudaError_t e = cudaMemcpyAsync(ix->cent, centroids, count * sizeof(float),
                                    cudaMemcpyDefault, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "centroid copy");
    return PARISKV_OK;
}

pariskv_status pariskv_sync(pariskv_index* index, void* stream) {
    pariskv_status s = check_index(index);
    if (s != PARISKV_OK) return s;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronise");
    int st = 0;
    e = cudaMemcpy(&st, index->status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (st != ST_OK) {
        cudaMemset(index->status, 0, sizeof(int));
        if (st == ST_TIMEOUT) return fail(PARISKV_ETIMEOUT, "a bounded device-side wait expired");
        if (st == ST_BADINDEX)
            return fail(PARISKV_ECUDA,
                        "a kernel found an index out of range and skipped the access (device "
                        "status %d); the results of the affected heads are invalid", st);
        return fail(PARISKV_ECUDA, "internal consistency check failed on the device (%d)", st);
    }
    return PARISKV_OK;
}

pariskv_status pariskv_destroy(pariskv_index* index) {
    if (!index) return PARISKV_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(index->device);
    cudaDeviceSynchronize();
    free_index(index);
    cudaSetDevice(prev);
    return PARISKV_OK;
}

int64_t pariskv_size(const pariskv_index* index) { return index ? index->n : -1; }

int32_t pariskv_last_launch_count(void) { return g_launches; }

const char* pariskv_status_string(pariskv_status s) {
    switch (s) {
        case PARISKV_OK: return "ok";
        case PARISKV_EINVAL: return "invalid argument";
        case PARISKV_ENOMEM: return "out of device memory";
        case PARISKV_ECUDA: return "CUDA error";
        case PARISKV_ECAPACITY: return "index capacity exceeded";
        case PARISKV_ETIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

const char* pariskv_last_error(void) { return g_err; }

// =========================================================================================
// Test-only surface (pariskv_debug.h)
// =========================================================================================
pariskv_status pariskv_debug_rotate(const pariskv_config* cfg, const int8_t* srht_signs,
                                    const void* x, int64_t n, float* y, float* norm,
                                    void* stream) {
    pariskv_status s = check_config(cfg);
    if (s != PARISKV_OK) return s;
    if (!srht_signs) return fail(PARISKV_EINVAL, "srht_signs is NULL");
    if (n < 0) return fail(PARISKV_EINVAL, "n < 0");
    if (n == 0) return PARISKV_OK;
    if ((s = check_dev_ptr(x, cfg->dtype == PARISKV_BF16 ? 8 : 16, "x")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(y, 16, "y")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(norm, 4, "norm")) != PARISKV_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float hs[D];
    for (int j = 0; j < D; ++j) hs[j] = static_cast<float>(srht_signs[j]);
    float* ds = nullptr;
    if (!dalloc(&ds, D)) return fail(PARISKV_ENOMEM, "signs");
    cudaError_t e = cudaMemcpy(ds, hs, sizeof(hs), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = launch_rotate(cfg, ds, x, n, y, norm, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    dfree(ds);
    if (e != cudaSuccess) return cuda_fail(e, "rotate");
    return PARISKV_OK;
}

pariskv_status pariskv_debug_build_index_rotated(const pariskv_config* cfg,
                                                 const int8_t* srht_signs, const float* y,
                                                 const float* knorm, int64_t ld_tok, int64_t n,
                                                 void* stream, pariskv_index** out) {
    return build_common(cfg, srht_signs, y, knorm, true, ld_tok, n, stream, out);
}

pariskv_status pariskv_debug_append_rotated(pariskv_index* index, const float* y,
                                            const float* knorm, int64_t ld_tok, int64_t t,
                                            void* stream) {
    return append_common(index, y, knorm, true, ld_tok, t, stream);
}

pariskv_status pariskv_debug_search_rotated(pariskv_index* index, const float* qt,
                                            const float* qnorm, int32_t k, int32_t* topk_idx,
                                            float* topk_est, void* stream) {
    pariskv_status s = check_index(index);
    if (s != PARISKV_OK) return s;
    if ((s = check_dev_ptr(qt, 16, "qt")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(qnorm, 4, "qnorm")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(topk_idx, 4, "topk_idx")) != PARISKV_OK) return s;
    if (topk_est && (s = check_dev_ptr(topk_est, 4, "topk_est")) != PARISKV_OK) return s;
    return run_search(index, nullptr, qt, qnorm, true, k, topk_idx, topk_est,
                      static_cast<cudaStream_t>(stream));
}

pariskv_status pariskv_debug_profile(pariskv_index* ix, int32_t enable) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (enable && !ix->ev[0]) {
        for (auto& e : ix->ev) {
            cudaError_t r = cudaEventCreate(&e);
            if (r != cudaSuccess) return cuda_fail(r, "event create");
        }
    }
    ix->profile = enable != 0;
    ix->nev = 0;
    return PARISKV_OK;
}

pariskv_status pariskv_debug_inject_bad_candidate(pariskv_index* ix, int32_t head, int64_t pos,
                                                 int32_t value) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    const int heads = ix->units * ix->cfg.group;
    if (head < 0 || head >= heads) return fail(PARISKV_EINVAL, "head %d not in [0, %d)", head, heads);
    if (pos < 0) return fail(PARISKV_EINVAL, "pos < 0");
    if (value >= 0 && value < ix->n)
        return fail(PARISKV_EINVAL, "value %d is a valid key index (size %lld)", value,
                    static_cast<long long>(ix->n));
    ix->inject_head = head;
    ix->inject_pos = pos;
    ix->inject_value = value;
    return PARISKV_OK;
}

pariskv_status pariskv_debug_inject_wait_timeout(pariskv_index* ix) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    ix->inject_wait = true;
    return PARISKV_OK;
}

pariskv_status pariskv_debug_set_launch(pariskv_index* ix, int32_t vote_ctas, int32_t rerank_ctas,
                                        int32_t topk_mode) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (vote_ctas < 0 || rerank_ctas < 0 || topk_mode < 0 || topk_mode > kTopkModes)
        return fail(PARISKV_EINVAL, "launch shape (%d, %d, %d) out of range", vote_ctas,
                    rerank_ctas, topk_mode);
    ix->vote_ctas = vote_ctas;
    ix->rerank_ctas = rerank_ctas;
    ix->topk_mode = topk_mode;
    return PARISKV_OK;
}

pariskv_status pariskv_debug_union_rows(int64_t* rows) {
    if (!rows) return fail(PARISKV_EINVAL, "rows is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    unsigned long long r = 0;
    if (e == cudaSuccess) e = read_union_rows(&r);
    if (e != cudaSuccess) return cuda_fail(e, "union row counter");
    *rows = static_cast<int64_t>(r);
    return PARISKV_OK;
}

pariskv_status pariskv_debug_check_guards(void) {
    if (!guards_on()) return fail(PARISKV_EINVAL, "guard bytes are off (PARISKV_GUARD=1 not set)");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "device synchronise");
    std::lock_guard<std::mutex> lk(g_guard_mu);
    for (const Guarded& g : g_guarded) guard_ok(g);
    if (g_guard_bad[0]) {
        const pariskv_status r = fail(PARISKV_ECUDA, "%s", g_guard_bad);
        g_guard_bad[0] = 0;
        return r;
    }
    return PARISKV_OK;
}

pariskv_status pariskv_debug_gather_candidates(pariskv_index* ix, uint32_t* sink, void* stream) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (!ix->searched) return fail(PARISKV_EINVAL, "no search has run on this index");
    if ((s = check_dev_ptr(sink, 4, "sink")) != PARISKV_OK) return s;
    const int64_t heads = static_cast<int64_t>(ix->units) * ix->cfg.group;
    cudaError_t e = launch_gather_candidates(ix->rec, ix->cap_pad, ix->cand, ix->cmax,
                                             static_cast<int32_t>(ix->last_C), ix->cfg.group,
                                             heads, ix->n, sink, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gather launch");
    return PARISKV_OK;
}

pariskv_status pariskv_debug_read_stream(const void* src, int64_t bytes, uint32_t* sink,
                                        void* stream) {
    if (bytes <= 0 || bytes % 16 != 0)
        return fail(PARISKV_EINVAL, "bytes=%lld is not a positive multiple of 16",
                    static_cast<long long>(bytes));
    pariskv_status s;
    if ((s = check_dev_ptr(src, 16, "src")) != PARISKV_OK) return s;
    if ((s = check_dev_ptr(sink, 4, "sink")) != PARISKV_OK) return s;
    g_launches = 0;
    cudaError_t e = launch_read_stream(src, bytes, sink, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "read stream");
    g_launches = 1;
    return PARISKV_OK;
}

pariskv_status pariskv_debug_stage_ms(pariskv_index* ix, float* ms, int32_t* nstages) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (!ms || !nstages) return fail(PARISKV_EINVAL, "NULL output");
    *nstages = 0;
    if (ix->nev < 2) return fail(PARISKV_EINVAL, "no profiled search has run");
    cudaError_t e = cudaEventSynchronize(ix->ev[ix->nev - 1]);
    if (e != cudaSuccess) return cuda_fail(e, "event synchronise");
    for (int i = 0; i + 1 < ix->nev; ++i) {
        e = cudaEventElapsedTime(&ms[i], ix->ev[i], ix->ev[i + 1]);
        if (e != cudaSuccess) return cuda_fail(e, "event elapsed");
    }
    *nstages = ix->nev - 1;
    return PARISKV_OK;
}

pariskv_status pariskv_debug_export_index(pariskv_index* ix, uint8_t* ids, uint8_t* codes,
                                          float* factors) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "synchronise");
    const int64_t n = ix->n;
    std::vector<uint8_t> hid, hrec;
    try {
        hid.resize(static_cast<size_t>(n) * 16);
        hrec.resize(static_cast<size_t>(n) * REC);
    } catch (...) {
        return fail(PARISKV_ENOMEM, "host staging");
    }
    for (int u = 0; u < ix->units; ++u) {
        if (n == 0) break;
        e = cudaMemcpy(hid.data(), ix->ids + u * ix->cap_pad * 16, n * 16, cudaMemcpyDeviceToHost);
        if (e == cudaSuccess)
            e = cudaMemcpy(hrec.data(), ix->rec + u * ix->cap_pad * REC, n * REC,
                           cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "export copy");
        for (int64_t i = 0; i < n; ++i) {
            const int64_t o = static_cast<int64_t>(u) * n + i;
            for (int b = 0; b < NB; ++b) {
                const uint8_t id = hid[i * 16 + ((b - (i >> 1)) & 15)];
                if (ids) ids[o * NB + b] = id;
                const int64_t at = i * REC + 32 * (b >> 2) + 4 * (b & 3);
                uint32_t w;
                memcpy(&w, &hrec[at], 4);
                // stored nibble u: uniform levels store vt + 8, table levels 8 + mag (y >= 0)
                // or 7 - mag (y < 0); canonical code = sign << 3 | magnitude, the sign being
                // bit j of the bucket id
                const bool table = ix->cfg.levels != PARISKV_LEVELS_UNIFORM;
                if (codes)
                    for (int j = 0; j < M; ++j) {
                        const int u = static_cast<int>((w >> (4 * j)) & 15u);
                        const int mag = u >= 8 ? u - 8 : (table ? 7 - u : 8 - u);
                        // the nibble carries the sign except for a zero uniform level, whose
                        // sign is the id bit (not recorded when ids come from learned
                        // centroids: reported as +)
                        const uint32_t neg = (table || u != 8) ? (u < 8 ? 1u : 0u)
                                             : (ix->cent ? 0u : (id >> j) & 1u);
                        codes[o * D + b * M + j] =
                            static_cast<uint8_t>((neg << 3) | static_cast<uint32_t>(mag));
                    }
                if (factors) memcpy(&factors[o * NB + b], &hrec[at + 16], 4);
            }
        }
    }
    return PARISKV_OK;
}

pariskv_status pariskv_debug_export_search(pariskv_index* ix, uint8_t* lut, int32_t* scores,
                                           int64_t* ncand, int32_t* cand, float* S) {
    pariskv_status s = check_index(ix);
    if (s != PARISKV_OK) return s;
    if (!ix->searched) return fail(PARISKV_EINVAL, "no search has run on this index");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "synchronise");
    const int G = ix->cfg.group;
    const int64_t n = ix->n, C = ix->last_C;
    if (ncand) *ncand = C;
    std::vector<uint32_t> buf;
    for (int u = 0; u < ix->units; ++u) {
        for (int g = 0; g < G; ++g) {
            const int64_t head = static_cast<int64_t>(u) * G + g;
            const int64_t up = static_cast<int64_t>(u) * ix->packs + g / PACK;
            const int sh = 8 * (g % PACK);
            if (lut) {
                buf.resize(NB * NC);
                e = cudaMemcpy(buf.data(), ix->lut + up * NB * NC, NB * NC * 4,
                               cudaMemcpyDeviceToHost);
                if (e != cudaSuccess) return cuda_fail(e, "export lut");
                for (int i = 0; i < NB * NC; ++i) lut[head * NB * NC + i] = (buf[i] >> sh) & 0xff;
            }
            if (scores && n > 0) {
                buf.resize(n);
                e = cudaMemcpy(buf.data(), ix->scores + up * ix->cap_pad, n * 4,
                               cudaMemcpyDeviceToHost);
                if (e != cudaSuccess) return cuda_fail(e, "export scores");
                for (int64_t i = 0; i < n; ++i) scores[head * n + i] = (buf[i] >> sh) & 0xff;
            }
            if (cand && C > 0) {
                e = cudaMemcpy(cand + head * C, ix->cand + head * ix->cmax, C * 4,
                               cudaMemcpyDeviceToHost);
                if (e != cudaSuccess) return cuda_fail(e, "export candidates");
            }
            if (S && C > 0) {
                e = cudaMemcpy(S + head * C, ix->S + head * ix->cmax, C * 4,
                               cudaMemcpyDeviceToHost);
                if (e != cudaSuccess) return cuda_fail(e, "export S");
            }
        }
    }
    return PARISKV_OK;
}

}  // extern "C"
