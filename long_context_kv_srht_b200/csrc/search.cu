// search.cu -- one decode-step retrieval (query prep, collision vote, candidate selection,
// RSQ-IP rerank, top-k) as a single persistent, warp-specialised kernel.
//
// "Technical Summary: ParisKV", Methodology, Core Algorithmic Innovations 2 ("Coarse
// Candidate Generation", "Candidate Reranking (RSQ-IP)", "Estimation") and the Problem
// Statement (top-k keys per query head, found on the GPU). What each step computes:
//   query prep  q~ = R q / ||q||; per subspace the query's top-rho centroids (penalty
//               ascending, id ascending) get vote weight w_rank1 (rank 1) or w_rest;
//   vote        score_i = sum_b W_b[id_{i,b}] for every cached key, per query head;
//   select      the C = min(n, max(k, ceil(n bp / 10^4))) first keys in the order (score
//               descending, key index ascending), returned in key order;
//   rerank      S_i = sum_b f_{i,b} p_{i,b}, p_{i,b} = sum_j vt_{i,b,j} q~_{b,j}, both fp32
//               FMA chains in ascending order (p over j, then S over b);
//   top-k       the k largest S (ties to the lower key index) in key order, est = ||q|| S.
//
// Why one kernel. The step is two bandwidth passes -- 16 bytes of bucket ids per key and KV
// head (vote), then one 128-byte code record per candidate and query head (rerank) -- with
// latency-bound passes between them (threshold, compaction, top-k). Launched as a chain of
// kernels every stage waits for the previous one over all heads, and the latency-bound
// stages leave HBM idle. Here the work of all (sequence, KV head, vote pack) units is cut
// into items, and two kinds of workers on every SM take items from two global queues, so
// the latency-bound work of one unit runs while another unit's ids or records stream:
//
//  * the vote group (warps 0..7 of each CTA, working together) takes, in this order, the
//    query-prep items Q(p) of every pack-unit p, the vote items V(p, c) of every 16384-key
//    chunk c, the compaction items C(p, c) -- placed two packs behind the votes they
//    depend on -- and finally the top-k items K(h) of every query head. The vote group that
//    completes the last vote item of a pack-unit also finalises it (F: threshold T, ties E
//    and the candidate offset of every chunk, from the per-chunk histograms);
//  * the rerank warps (warps 8..15, each on its own) take rerank items R(h, r): 256
//    consecutive candidates of query head h, gathered record by record with bulk async
//    copies into a per-warp ring in shared memory and scored one record per lane.
//
// An item waits (bounded, see wait_flag) only for items that precede it in the order the
// queues hand them out: V(p, .) for Q(p); C(p, .) for the finalisation of V(p, .); R(h, .)
// for all C(p(h), .); K(h) for all R(h', .) of its pack-unit. Items are claimed in that
// order by workers that are already running, and a claimed item only ever waits for items
// claimed before it, so the earliest unfinished item never waits: no deadlock, whether or
// not every CTA is resident. A wait that runs past its limit records ST_TIMEOUT and the
// worker stops; pariskv_sync reports it.
//
// Data written for each search (layouts shared with the stage-export debug call):
//   qt, qnorm [heads][128], [heads]; lut u32 [P][16][256] (byte g = head 4 pack + g);
//   scores u32 [P][cap_pad] (byte g = that head's coarse score); hist u32 [P][nch][4][64];
//   thr [heads][4] = (T, E, C, #above T); cbase [heads][nch][2]; cand, S [heads][cmax];
//   shist u32 [heads][2048] (counts of S by the top 11 bits of its order key).
#include "common.cuh"
#include "internal.hpp"
#include "rotate.cuh"

namespace pkv {

namespace {

// ---------------------------------------------------------------------------------------
// Shape of the kernel
// ---------------------------------------------------------------------------------------
constexpr int kW = 8;                         // warps per CTA (two CTAs per SM)
constexpr int kThreads = 32 * kW;
constexpr int kVW = kW;                       // every item is worked on by the whole CTA
constexpr int kVT = kThreads;
constexpr int kBarV = 1;                      // named barrier of the CTA

constexpr int kTileKeys = 64;                 // vote warp-tile: two keys per lane
constexpr int kKeysPerThr = CHUNK / kVT;      // compaction: consecutive keys per thread
constexpr int kCWords = kKeysPerThr / 32;     // 32-bit key masks per head and kind
static_assert(kKeysPerThr % 32 == 0, "chunk shape");

constexpr int kStage = 32;                    // records per rerank stage (one per lane)
constexpr int kSlots = 2;                     // stages per rerank warp ring
constexpr int kRItem = 2048;                  // candidates per rerank item
constexpr int kBins = 2048;                   // top-k radix bins of the later levels
constexpr int kBins1 = SBINS;                 // first top-k level: counted by the rerank
constexpr int kBits1 = SBINS_BITS;
constexpr int kNR = 49;                       // byte-histogram rows per vote warp (scores 0..48)
constexpr int kSub = 512;                     // keys per streamed block of bucket ids (8 KB)
constexpr int kVSlots = 3;                    // id blocks in the vote ring

// Dynamic shared memory of a CTA (two CTAs per SM). Vote items, rerank items and top-k
// items use the same bytes in turn (a vote item rebuilds its table and clears its counters
// when another kind of item has used them since):
//  table   256 rows x 256 B: row c, bytes 4 (2b + k): vote weights of centroid c, subspace b
//          (copies k = 0, 1); bytes 128..255 of rows 49 w .. 49 w + 48: byte counters of
//          warp w < 4 (row s: one 32-bit word per lane, byte g = head g, score s)
//  h2      the same counters of warps 4..7 (128-byte rows)
//  vring   kVSlots blocks of bucket ids streamed by bulk copies; between vote items also the
//          scratch of query-prep, finalisation and compaction items
//  a rerank item's per-warp rings (kSlots stages of 32 records, 128-byte rows, 16-byte
//  piece c of row r at c ^ (r mod 8)) and query pairs start at 0; a top-k item uses it all
constexpr uint32_t kOffTab = 0;
constexpr uint32_t kTabBytes = 256 * 256;
constexpr uint32_t kOffH2 = kOffTab + kTabBytes;
constexpr uint32_t kH2Bytes = 4 * kNR * 128;
constexpr uint32_t kOffVRing = kOffH2 + kH2Bytes;
constexpr uint32_t kVRingBytes = kVSlots * kSub * 16;
constexpr uint32_t kOffScr = kOffVRing;
constexpr int kSmem = static_cast<int>(kOffVRing + kVRingBytes);
constexpr int kRingWarp = kSlots * kStage * REC;
constexpr uint32_t kOffRing = 0;
constexpr uint32_t kOffQry = kW * kRingWarp;
static_assert(kOffQry + 512 <= static_cast<uint32_t>(kSmem), "rerank rings");
static_assert(2 * kBins * 4 + 1024 <= kVRingBytes, "item scratch");

// Optional phase trace (a measurement aid, off when SearchArgs::trace is NULL): per kind of
// work, the earliest start (stored as ~t so that atomicMax keeps the minimum), the latest
// end and the summed busy time, in %globaltimer nanoseconds.
enum : int { TR_Q = 0, TR_V = 1, TR_C = 2, TR_K = 3, TR_F = 4, TR_R = 5,
             TR_VWAIT = 6, TR_RWAIT = 7, TR_KERNEL = 8, TR_POLLS = 9, TR_KSEL = 10,
             TR_KWRITE = 11, TR_SLOTS = 12 };
__device__ __forceinline__ uint64_t gtime() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void trace_add(unsigned long long* tr, int slot, uint64_t t0, uint64_t t1) {
    atomicMax(tr + 3 * slot + 0, ~static_cast<unsigned long long>(t0));
    atomicMax(tr + 3 * slot + 1, static_cast<unsigned long long>(t1));
    atomicAdd(tr + 3 * slot + 2, static_cast<unsigned long long>(t1 - t0));
}

// control block (int32 words)


struct SearchArgs {
    const uint8_t* ids;
    const uint8_t* rec;
    const float* signs;
    const float* cent;       // learned centroids or NULL
    const float* lvt;        // level table (table decode)
    const void* q;           // raw queries (bf16 / f32) or NULL
    const float* qt_in;      // rotated queries (debug path) or NULL
    const float* qn_in;
    float* qt;
    float* qnorm;
    uint32_t* lut;
    uint32_t* scores;
    uint32_t* hist;
    int32_t* thr;
    int32_t* cbase;
    int32_t* cand;
    float* S;
    uint32_t* shist;
    int32_t* topk_idx;
    float* topk_est;
    int* ctrl;
    int* status;
    unsigned long long* trace;   // phase trace [TR_SLOTS][3], or NULL
    int* progress;               // per-CTA item board in mapped host memory, or NULL
    int64_t n, cap_pad, cmax;
    long long spin_limit;
    int units, G, packs, P, nc, nch, heads;
    int rho, w1, wr, nr;     // nr = rows per head of the byte histograms (max score + 1)
    int C, k, nrh;           // nrh = rerank items per head
    int qbf16, rotated, nostall;
};

// control block: one 128-byte line per word (queue counters and flags polled by many warps
// must not share lines): queue counters, exit count, then per pack-unit p the query-prep
// count, the threshold-ready flag and the vote, compaction and rerank done-counts
enum : int { CT_Q = 0, CT_EXIT = 2, CT_HDR = 4 };
constexpr int kCtlStride = 32;
enum : int { PK_Q = 0, PK_F = 1, PK_V = 2, PK_C = 3, PK_R = 4, PK_N = 5 };
__device__ __forceinline__ int* ctl(const SearchArgs& a, int word) { return a.ctrl + word * kCtlStride; }
__device__ __forceinline__ int* pk(const SearchArgs& a, int kind, int p) {
    return a.ctrl + (CT_HDR + kind * a.P + p) * kCtlStride;
}

// ---------------------------------------------------------------------------------------
// The work queue
// ---------------------------------------------------------------------------------------
// Every CTA takes items from one queue, in this order: the query-prep item Q(h) of every
// query head; then segments s = 0, 1, ...: the compaction items C(s - 2, .) of pack-unit
// s - 2, the vote items V(s, .) of pack-unit s and the rerank items R(., .) of the heads of
// pack-unit s - 3 (evenly interleaved, so that the two CTAs of an SM usually stream ids and
// gather records at the same time), and the top-k items K(h) of the heads of pack-unit
// s - 4. Each item waits only for items handed out before it: V(p) for the Q items of p, C(p)
// for the finalisation of p (done by the CTA that completed its last vote item), R for all
// C of its pack-unit, K for all R of its pack-unit.
enum : int { IT_NONE = -1, IT_Q = 0, IT_V = 1, IT_C = 2, IT_K = 3, IT_R = 4 };
struct Item {
    int type, x, y;   // Q, K: query head x; V, C: pack-unit x, chunk y; R: head x, range y
};
constexpr int kLagC = 2, kLagR = 3, kLagK = 4;
__device__ __forceinline__ int heads_of(const SearchArgs& a, int p) {
    return min(PACK, a.G - (p % a.packs) * PACK);
}
// query heads of pack-units [0, q)
__device__ __forceinline__ int heads_before(const SearchArgs& a, int q) {
    return (q / a.packs) * a.G + min(PACK * (q % a.packs), a.G);
}
__device__ __forceinline__ int64_t seg_start(const SearchArgs& a, int s) {
    auto cl = [&](int v) { return max(0, min(v, a.P)); };
    return static_cast<int64_t>(a.heads) + static_cast<int64_t>(a.nc) * (cl(s) + cl(s - kLagC)) +
           static_cast<int64_t>(a.nrh) * heads_before(a, cl(s - kLagR)) +
           heads_before(a, cl(s - kLagK));
}
__device__ Item queue_item(const SearchArgs& a, int64_t i) {
    if (i < a.heads) return {IT_Q, static_cast<int>(i), 0};
    const int S = a.P + kLagK;   // segments 0 .. S - 1
    if (i >= seg_start(a, S)) return {IT_NONE, 0, 0};
    int lo = 0, hi = S - 1;      // the last segment starting at or before i
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (seg_start(a, mid) <= i) lo = mid;
        else hi = mid - 1;
    }
    const int s = lo;
    int64_t o = i - seg_start(a, s);
    const int pc = s - kLagC, pr = s - kLagR, pkk = s - kLagK;
    const int nC = (pc >= 0 && pc < a.P) ? a.nc : 0;
    if (o < nC) return {IT_C, pc, static_cast<int>(o)};
    o -= nC;
    const int64_t nV = s < a.P ? a.nc : 0;
    const int64_t nR = (pr >= 0 && pr < a.P) ? static_cast<int64_t>(heads_of(a, pr)) * a.nrh : 0;
    if (o < nV + nR) {
        const int64_t N = nV + nR;
        const int64_t v0 = o * nV / N, v1 = (o + 1) * nV / N;
        if (v1 > v0) return {IT_V, s, static_cast<int>(v0)};
        const int r = static_cast<int>(o - v0);   // rerank item within the pack-unit
        const int unit = pr / a.packs, pack = pr % a.packs;
        return {IT_R, unit * a.G + pack * PACK + r / a.nrh, r % a.nrh};
    }
    o -= nV + nR;
    const int unit = pkk / a.packs, pack = pkk % a.packs;
    return {IT_K, unit * a.G + pack * PACK + static_cast<int>(o), 0};
}


// The kernel's dynamic shared memory, referenced directly by the hot loops so that its
// (constant) shared-window address folds into the load instructions.
extern __shared__ __align__(128) uint8_t g_smem[];

// ---------------------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------------------
// The non-aligned form: thread 0 often reaches a barrier later than the other lanes of its
// warp (it claims items and waits on flags alone), and an aligned barrier reached by a
// diverged warp may count the warp before all of its threads have arrived.
__device__ __forceinline__ void bar_v() {
    asm volatile("barrier.sync %0, %1;" :: "n"(kBarV), "n"(kVT) : "memory");
}
// Loads that bypass L1: data written by other CTAs during this kernel.
__device__ __forceinline__ uint32_t ldcg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ int32_t ldcg_i32(const int32_t* p) {
    return static_cast<int32_t>(ldcg_u32(p));
}
__device__ __forceinline__ float ldcg_f32(const float* p) { return __uint_as_float(ldcg_u32(p)); }
__device__ __forceinline__ uint4 ldcg_u128(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// Waits until *flag == target (mode 0) or *flag >= target (mode 1). Bounded: past
// spin_limit clock cycles it records ST_TIMEOUT and returns false. One thread calls it.
__device__ __forceinline__ int ld_relaxed(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ bool wait_flag(const int* flag, int target, bool geq, long long limit, int* status,
                          unsigned long long* trace, const int* ctrl) {
    int v = ld_acquire(flag);
    if (geq ? v >= target : v == target) return true;
    // relaxed polling with exponential backoff (many warps may wait on one flag: keep its
    // L2 line cool), and one fence once the value is seen
    const long long t0 = clock64();
    unsigned ns = 512;
    for (;;) {
        __nanosleep(ns);
        if (ns < 4096) ns <<= 1;
        if (trace) atomicAdd(trace + 3 * TR_POLLS + 2, 1ull);
        v = ld_relaxed(flag);
        if (geq ? v >= target : v == target) {
            __threadfence();
            return true;
        }
        if (clock64() - t0 > limit) {
            if (atomicExch(status, ST_TIMEOUT) != ST_TIMEOUT) {   // the first expiry: where and what
                status[1] = static_cast<int>(flag - ctrl) / kCtlStride;
                status[2] = target;
                status[3] = v;
            }
            return false;
        }
    }
}

// Bounded mbarrier wait (rerank rings). False (and ST_TIMEOUT recorded) past the limit.
__device__ __forceinline__ bool mbar_wait_limit(uint32_t bar, uint32_t parity, long long limit,
                                                int* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) {
            if (atomicExch(status, ST_TIMEOUT) != ST_TIMEOUT) status[1] = -1;   // an mbarrier
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ uint32_t tab_ld(uint32_t off) {
    return *reinterpret_cast<const uint32_t*>(g_smem + kOffTab + off);
}

// ---------------------------------------------------------------------------------------
// Q: rotated query and vote weights of one query head
// ---------------------------------------------------------------------------------------
// Warp 0 rotates the query; then warp w ranks the 256 centroids of subspaces w and w + 8,
// eight per lane, as 64-bit keys (pen bits << 32 | id), by rho rounds of a warp-wide
// minimum (rho <= 32) or an all-pairs rank count, and writes the head's byte of every
// packed table entry. The last Q item of a pack-unit makes its table ready.
__device__ void q_item(const SearchArgs& a, int head, uint8_t* scr) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = head / a.G, g = head - unit * a.G;
    const int p = unit * a.packs + g / PACK, slot = g % PACK;
    float* sq = reinterpret_cast<float*>(scr);             // [128]
    if (warp == 0) {
        float v[4];
        float nr;
        if (a.rotated) {
            Elem<float>::load4(a.qt_in + static_cast<int64_t>(head) * D + 4 * lane, v);
            nr = a.qn_in[head];
        } else {
            float sg[4];
            load_signs(a.signs, sg);
            if (a.qbf16)
                Elem<__nv_bfloat16>::load4(
                    static_cast<const __nv_bfloat16*>(a.q) + static_cast<int64_t>(head) * D + 4 * lane, v);
            else
                Elem<float>::load4(static_cast<const float*>(a.q) + static_cast<int64_t>(head) * D + 4 * lane, v);
            nr = normalize_rotate_warp(v, sg);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) sq[4 * lane + i] = v[i];
        *reinterpret_cast<float4*>(a.qt + static_cast<int64_t>(head) * D + 4 * lane) =
            make_float4(v[0], v[1], v[2], v[3]);
        if (lane == 0) a.qnorm[head] = nr;
    }
    bar_v();
    for (int b = warp; b < NB; b += kVW) {
        const float* qb = sq + 8 * b;
        unsigned long long key[8];
        if (a.cent) {
            // learned centroids: rank by <mu_c, q~_b> (fp32 FMA chain over j ascending)
            // descending, ties to the lower id
            const float* cb = a.cent + (static_cast<int64_t>(unit) * NB + b) * NC * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t c = static_cast<uint32_t>(lane + 32 * i);
                float sim = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) sim = __fmaf_rn(cb[c * 8 + j], qb[j], sim);
                key[i] = (static_cast<unsigned long long>(~order_key(sim)) << 32) | c;
            }
        } else {
            float av[8];
            uint32_t c1 = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float x = qb[j];
                av[j] = fabsf(x);
                c1 |= (x < 0.0f ? 1u : 0u) << j;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t c = static_cast<uint32_t>(lane + 32 * i);
                const uint32_t diff = c ^ c1;
                float pen = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if ((diff >> j) & 1u) pen = __fadd_rn(pen, av[j]);
                key[i] = (static_cast<unsigned long long>(__float_as_uint(pen)) << 32) | c;
            }
        }
        uint32_t wgt[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) wgt[i] = 0;
        if (a.rho <= 32) {
            uint32_t taken = 0;
            for (int r = 0; r < a.rho; ++r) {
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
                        wgt[i] = r == 0 ? a.w1 : a.wr;
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
                wgt[i] = rank[i] == 0 ? a.w1
                                      : (rank[i] < static_cast<uint32_t>(a.rho) ? a.wr : 0u);
        }
        uint8_t* out = reinterpret_cast<uint8_t*>(a.lut + (static_cast<int64_t>(p) * NB + b) * NC);
#pragma unroll
        for (int i = 0; i < 8; ++i) out[4 * (lane + 32 * i) + slot] = static_cast<uint8_t>(wgt[i]);
    }
    __threadfence();
    bar_v();
    if (threadIdx.x == 0) atomicAdd(pk(a, PK_Q, p), 1);
}

// ---------------------------------------------------------------------------------------
// V: collision vote over one chunk of one pack-unit
// ---------------------------------------------------------------------------------------
// The ids of keys L and L + 32 of a 64-key tile (lane L): two 128-bit non-allocating loads,
// each a fully coalesced 512-byte warp access.
__device__ __forceinline__ u32x8 ldg_ids(const uint8_t* p) {
    u32x8 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]) : "l"(p));
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7]) : "l"(p + 512));
    return v;
}

// Table entry of step t: byte0 <- column (byte t % 3 of colp[t / 3]), byte1 <- id byte t % 4,
// bytes 2, 3 <- the zero top byte of colp[t / 3]: row id, 256-byte rows.
template <int T>
__device__ __forceinline__ uint32_t look(const uint32_t* wd, const uint32_t* colp) {
    constexpr uint32_t sel = 0x7700u | ((T & 3u) << 4) | (4u + (T % 3));
    return tab_ld(prmt_i<sel>(wd[T >> 2], colp[T / 3]));
}

// Packed coarse score of one key: the sum of its 16 table entries (byte g = query head g).
__device__ __forceinline__ uint32_t score_key(const uint32_t* wd, const uint32_t* colp) {
    const uint32_t v0 = look<0>(wd, colp), v1 = look<1>(wd, colp);
    const uint32_t v2 = look<2>(wd, colp), v3 = look<3>(wd, colp);
    const uint32_t v4 = look<4>(wd, colp), v5 = look<5>(wd, colp);
    const uint32_t v6 = look<6>(wd, colp), v7 = look<7>(wd, colp);
    const uint32_t v8 = look<8>(wd, colp), v9 = look<9>(wd, colp);
    const uint32_t v10 = look<10>(wd, colp), v11 = look<11>(wd, colp);
    const uint32_t v12 = look<12>(wd, colp), v13 = look<13>(wd, colp);
    const uint32_t v14 = look<14>(wd, colp), v15 = look<15>(wd, colp);
    const uint32_t x = v0 + v1 + v2, y = v3 + v4 + v5, z = v6 + v7 + v8, w = v9 + v10 + v11;
    const uint32_t e = v12 + v13 + v14;
    return (x + y + z) + (w + e + v15);
}

// Loads pack-unit p's vote table into rows c, columns 2b + k (copies k = 0, 1) of the
// table area (the lower 128 bytes of each 256-byte row).
__device__ void load_table(const SearchArgs& a, int p, uint8_t* tab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t* src = a.lut + static_cast<int64_t>(p) * NB * NC + (lane >> 1) * NC;
    constexpr int kRows = NC / kVW;
    uint32_t v[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) v[i] = ldcg_u32(src + warp + kVW * i);
#pragma unroll
    for (int i = 0; i < kRows; ++i)
        *reinterpret_cast<uint32_t*>(tab + (warp + kVW * i) * 256 + 4 * lane) = v[i];
}

// Lane-private byte counters of the vote group: vote warp w, score s, lane L owns one 32-bit
// word whose byte g counts head g's keys with that score (one bank per lane, so the
// increments of a warp never conflict). Warps 0..3 keep theirs in the upper halves of the
// table rows 49 w + s, warps 4..7 in h2 rows 49 (w - 4) + s.
__device__ __forceinline__ uint32_t counter_base(uint8_t* smem, int warp, int lane) {
    return warp < 4 ? smem_addr(smem + kOffTab + 49 * warp * 256 + 128 + 4 * lane)
                    : smem_addr(smem + kOffH2 + 49 * (warp - 4) * 128 + 4 * lane);
}

// Counts one key's HP packed scores (byte g of acc = head g's score) in this lane's byte
// counters: the HP bytes live in one word per score (byte g of word s), so the HP
// read-modify-writes of a key touch distinct bytes and go out as one group of loads, then
// one group of stores.
template <int HP>
__device__ __forceinline__ void count_scores(uint32_t acc, uint32_t cb, uint32_t pitch) {
    uint32_t ad[HP], v[HP];
#pragma unroll
    for (int g = 0; g < HP; ++g) ad[g] = cb + prmt(acc, 0u, 0x4440u + g) * pitch + g;
    if constexpr (HP == 4) {
        asm volatile(
            "{\n ld.shared.u8 %0, [%4];\n ld.shared.u8 %1, [%5];\n ld.shared.u8 %2, [%6];\n"
            " ld.shared.u8 %3, [%7];\n}"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
            : "r"(ad[0]), "r"(ad[1]), "r"(ad[2]), "r"(ad[3]));
        asm volatile(
            "{\n st.shared.u8 [%0], %4;\n st.shared.u8 [%1], %5;\n st.shared.u8 [%2], %6;\n"
            " st.shared.u8 [%3], %7;\n}"
            :: "r"(ad[0]), "r"(ad[1]), "r"(ad[2]), "r"(ad[3]),
               "r"(v[0] + 1u), "r"(v[1] + 1u), "r"(v[2] + 1u), "r"(v[3] + 1u));
    } else {
#pragma unroll
        for (int g = 0; g < HP; ++g) {
            asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v[g]) : "r"(ad[g]));
            asm volatile("st.shared.u8 [%0], %1;" :: "r"(ad[g]), "r"(v[g] + 1u));
        }
    }
}

struct VRing {
    uint32_t bar0;   // kVSlots mbarriers
    int seq;         // blocks consumed so far by this vote group (slot = seq % kVSlots)
};

__device__ __forceinline__ void v_item(const SearchArgs& a, int p, int c, uint8_t* smem,
                                      const uint32_t colp[6], VRing& vr) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = p / a.packs, pack = p % a.packs;
    const int hp = min(PACK, a.G - pack * PACK);
    const uint32_t pitch = warp < 4 ? 256u : 128u;
    const uint32_t cb = counter_base(smem, warp, lane);

    const int64_t k0 = static_cast<int64_t>(c) * CHUNK;
    const int nkeys = static_cast<int>(min64(a.n - k0, CHUNK));
    const int nsub = (nkeys + kSub - 1) / kSub;
    const uint8_t* src = a.ids + (static_cast<int64_t>(unit) * a.cap_pad + k0) * 16;
    uint32_t* sc_out = a.scores + static_cast<int64_t>(p) * a.cap_pad + k0;
    // blocks of 1024 keys (16 KB) stream through the ring; whole blocks are copied (a chunk
    // lies inside the padded capacity), keys past n are masked
    auto issue = [&](int b) {
        const int slot = (vr.seq + b) % kVSlots;
        const uint32_t bar = vr.bar0 + 8 * slot;
        mbar_arrive_expect_tx(bar, kSub * 16);
        bulk_g2s(smem_addr(smem + kOffVRing + slot * kSub * 16), src + static_cast<int64_t>(b) * kSub * 16,
                 kSub * 16, bar);
    };
    if (threadIdx.x == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        for (int b = 0; b < min(kVSlots, nsub); ++b) issue(b);
    }
    for (int b = 0; b < nsub; ++b) {
        const int slot = (vr.seq + b) % kVSlots;
        const uint32_t par = static_cast<uint32_t>((vr.seq + b) / kVSlots) & 1u;
        mbar_wait_limit(vr.bar0 + 8 * slot, par, a.spin_limit, a.status);
        const uint8_t* blk = smem + kOffVRing + slot * kSub * 16;
        // warp w scores tile w of the block: keys lane and lane + 32
        const int kb = b * kSub + warp * kTileKeys;      // first key of the warp's tile
        if (kb < nkeys) {
            uint32_t acc[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint4 x = *reinterpret_cast<const uint4*>(blk + (warp * kTileKeys + 32 * i + lane) * 16);
                const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
                acc[i] = score_key(wd, colp);
            }
            if (kb + kTileKeys <= nkeys && hp == PACK) {
#pragma unroll
                for (int i = 0; i < 2; ++i) sc_out[kb + 32 * i + lane] = acc[i];
#pragma unroll
                for (int i = 0; i < 2; ++i) count_scores<PACK>(acc[i], cb, pitch);
            } else {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (kb + 32 * i + lane < nkeys) {
                        sc_out[kb + 32 * i + lane] = acc[i];
                        if (hp == 4) count_scores<4>(acc[i], cb, pitch);
                        else if (hp == 3) count_scores<3>(acc[i], cb, pitch);
                        else if (hp == 2) count_scores<2>(acc[i], cb, pitch);
                        else count_scores<1>(acc[i], cb, pitch);
                    }
                }
            }
        }
        bar_v();   // every warp is done with the block: its slot may be refilled
        if (threadIdx.x == 0 && b + kVSlots < nsub) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(b + kVSlots);
        }
    }
    vr.seq += nsub;
    // flush: per score s, every warp's word of every lane; bytes summed as 16-bit fields
    // (a counter reaches at most 64 per item, 512 over the eight warps)
    uint32_t* hout = a.hist + (static_cast<int64_t>(p) * a.nch + c) * (PACK * 64);
    for (int sv = warp; sv < a.nr; sv += kVW) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int w = 0; w < kVW; ++w) {
            uint32_t* q = reinterpret_cast<uint32_t*>(
                w < 4 ? smem + kOffTab + (49 * w + sv) * 256 + 128 + 4 * lane
                      : smem + kOffH2 + (49 * (w - 4) + sv) * 128 + 4 * lane);
            const uint32_t x = *q;
            *q = 0u;
            lo += x & 0x00ff00ffu;
            hi += (x >> 8) & 0x00ff00ffu;
        }
        lo = __reduce_add_sync(0xffffffffu, lo);
        hi = __reduce_add_sync(0xffffffffu, hi);
        if (lane < PACK) {
            const uint32_t v = lane == 0 ? (lo & 0xffffu) : lane == 1 ? (hi & 0xffffu)
                             : lane == 2 ? (lo >> 16) : (hi >> 16);
            hout[lane * 64 + sv] = v;
        }
    }
}

// ---------------------------------------------------------------------------------------
// F: finalise a pack-unit once all its votes are in
// ---------------------------------------------------------------------------------------
// Block-wide (vote group) exclusive scan of a 64-bit value; *total receives the sum.
__device__ __forceinline__ uint64_t vgroup_excl_scan(uint64_t v, uint64_t* total,
                                                     uint64_t* sh /* [kVW + 1] */) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    bar_v();
    uint64_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kVW; ++w) {
        const uint64_t t = sh[w];
        before += w < warp ? t : 0u;
        tot += t;
    }
    *total = tot;
    bar_v();
    return before + x - v;
}

__device__ void f_item(const SearchArgs& a, int p, uint8_t* scr) {
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int unit = p / a.packs, pack = p % a.packs;
    const int hp = min(PACK, a.G - pack * PACK);
    const int head0 = unit * a.G + pack * PACK;
    uint32_t* tot = reinterpret_cast<uint32_t*>(scr);                  // [4][64]
    int32_t* sT = reinterpret_cast<int32_t*>(scr + 1024);              // [4]
    int32_t* sE = sT + 4;                                              // [4]
    uint64_t* scan = reinterpret_cast<uint64_t*>(scr + 1024 + 64);     // [kVW]
    const uint32_t* hp_base = a.hist + static_cast<int64_t>(p) * a.nch * (PACK * 64);
    constexpr int kQ = 13;   // 16-byte words per (chunk, head) histogram (bins 0..51)
    // thread (g = t / 64, chunk cb + t % 64) reads that chunk's histogram of head g, four
    // 16-byte words at a time (bins past the largest score were never written: skipped)
    const int g = t >> 6, cl = t & 63;
    auto words = [&](int cb, int i0, uint32_t v[16]) {
        const int c = cb + cl;
        const bool ok = g < hp && c < a.nc;
        const uint4* src = reinterpret_cast<const uint4*>(hp_base + (static_cast<int64_t>(c) * PACK + g) * 64);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 x = ok && i0 + i < kQ ? ldcg_u128(src + i0 + i) : make_uint4(0, 0, 0, 0);
            v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (4 * i0 + i >= a.nr) v[i] = 0u;
    };
    tot[t] = 0u;
    bar_v();
    for (int cb = 0; cb < a.nc; cb += 64) {
#pragma unroll 1
        for (int i0 = 0; i0 < kQ; i0 += 4) {
            uint32_t v[16];
            words(cb, i0, v);
            // per bin: the warp's sum, then the head's two warps add into the totals
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t sum = __reduce_add_sync(0xffffffffu, v[i]);
                if (lane == 0 && sum) atomicAdd(&tot[g * 64 + 4 * i0 + i], sum);
            }
        }
    }
    bar_v();
    if (warp < hp) {
        // T = the largest t with #{score >= t} >= C (suffix sums over the 64 bins)
        const uint32_t lo = tot[warp * 64 + lane], hi = tot[warp * 64 + 32 + lane];
        uint32_t shi = hi;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, shi, o);
            if (lane + o < 32) shi += y;
        }
        const uint32_t tot_hi = __shfl_sync(0xffffffffu, shi, 0);
        uint32_t slo = lo;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, slo, o);
            if (lane + o < 32) slo += y;
        }
        slo += tot_hi;
        const uint32_t Cu = static_cast<uint32_t>(a.C);
        const uint32_t mhi = __ballot_sync(0xffffffffu, shi >= Cu);
        const uint32_t mlo = __ballot_sync(0xffffffffu, slo >= Cu);
        int T;
        uint32_t ge_T, cnt_T;
        if (mhi) {
            T = 31 - __clz(mhi) + 32;
            ge_T = __shfl_sync(0xffffffffu, shi, T - 32);
            cnt_T = __shfl_sync(0xffffffffu, hi, T - 32);
        } else {
            T = 31 - __clz(mlo);
            ge_T = __shfl_sync(0xffffffffu, slo, T);
            cnt_T = __shfl_sync(0xffffffffu, lo, T);
        }
        if (lane == 0) {
            const int32_t above = static_cast<int32_t>(ge_T - cnt_T);   // #{score > T}
            const int32_t E = a.C - above;
            sT[warp] = T;
            sE[warp] = E;
            int32_t* th = a.thr + (head0 + warp) * 4;
            th[0] = T;
            th[1] = E;
            th[2] = a.C;
            th[3] = above;
        }
    }
    bar_v();
    // per chunk: keys above T and ties at T, exclusive scans over the chunks of each head
    // (the 64 threads of head g are warps 2g, 2g + 1)
    uint64_t run = 0;   // (eq << 32) | gt before this block of chunks, for head g
    const int T = g < hp ? sT[g] : 0;
    for (int cb = 0; cb < a.nc; cb += 64) {
        const int c = cb + cl;
        uint32_t gt = 0, eq = 0;
#pragma unroll 1
        for (int i0 = 0; i0 < kQ; i0 += 4) {
            uint32_t v[16];
            words(cb, i0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                gt += 4 * i0 + i > T ? v[i] : 0u;
                eq += 4 * i0 + i == T ? v[i] : 0u;
            }
        }
        const uint64_t mine = (static_cast<uint64_t>(eq) << 32) | gt;
        uint64_t x = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) scan[warp] = x;
        bar_v();
        const uint64_t wtot0 = scan[warp & ~1], wtot1 = scan[warp | 1];
        const uint64_t pre = run + ((warp & 1) ? wtot0 : 0u) + x - mine;
        if (g < hp && c < a.nc) {
            const int64_t E = sE[g];
            const int64_t gt_before = static_cast<int64_t>(pre & 0xffffffffu);
            const int64_t eq_before = static_cast<int64_t>(pre >> 32);
            int32_t* cb2 = a.cbase + ((static_cast<int64_t>(head0 + g)) * a.nch + c) * 2;
            cb2[0] = static_cast<int32_t>(gt_before + min64(eq_before, E));
            cb2[1] = static_cast<int32_t>(eq_before);
        }
        run += wtot0 + wtot1;
        bar_v();
    }
    // the top-k's first radix level is counted by the rerank: start it at zero
    for (int i = t; i < hp * kBins1; i += kVT) a.shist[static_cast<int64_t>(head0) * kBins1 + i] = 0u;
    __threadfence();
    bar_v();
    if (t == 0) st_release(pk(a, PK_F, p), 1);
}

// ---------------------------------------------------------------------------------------
// C: compaction of one chunk (the candidates of every head of the pack-unit, in key order)
// ---------------------------------------------------------------------------------------
__device__ void c_item(const SearchArgs& a, int p, int c, uint8_t* scr) {
    const int t = threadIdx.x;
    const int unit = p / a.packs, pack = p % a.packs;
    const int hp = min(PACK, a.G - pack * PACK);
    const int head0 = unit * a.G + pack * PACK;
    uint64_t* scan = reinterpret_cast<uint64_t*>(scr);   // [kVW + 1] (two scans)
    const int64_t k0 = static_cast<int64_t>(c) * CHUNK + static_cast<int64_t>(t) * kKeysPerThr;
    const int nv = static_cast<int>(max64(0, min64(kKeysPerThr, a.n - k0)));

    // Per-head thresholds packed one per byte; a head outside the pack gets T = 127, which
    // no score (< 64) reaches. Byte g of (s + gt_add) has bit 7 set iff score_g > T_g, and of
    // (s + ge_add) iff score_g >= T_g; bytes never carry (score + 128 <= 191).
    uint32_t gt_add = 0, ge_add = 0;
#pragma unroll
    for (int g = 0; g < PACK; ++g) {
        const int T = g < hp ? ldcg_i32(a.thr + (head0 + g) * 4) : 127;
        gt_add |= static_cast<uint32_t>(127 - T) << (8 * g);
        ge_add |= static_cast<uint32_t>(128 - T) << (8 * g);
    }
    uint32_t gm[PACK][kCWords], em[PACK][kCWords];
    const uint32_t* src = a.scores + static_cast<int64_t>(p) * a.cap_pad + k0;
    // all of the thread's packed scores are loaded first (one round trip)
    uint32_t sv[kKeysPerThr];
#pragma unroll
    for (int i = 0; i < kKeysPerThr / 4; ++i) {
        const uint4 x = 4 * i < nv ? ldcg_u128(src + 4 * i) : make_uint4(0, 0, 0, 0);
        sv[4 * i] = x.x; sv[4 * i + 1] = x.y; sv[4 * i + 2] = x.z; sv[4 * i + 3] = x.w;
    }
#pragma unroll
    for (int w = 0; w < kCWords; ++w) {
        uint32_t G4[4], GE4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t g1 = 0, g2 = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t x = sv[32 * w + 8 * q + i];
                g1 |= (((x + gt_add) >> 7) & 0x01010101u) << i;
                g2 |= (((x + ge_add) >> 7) & 0x01010101u) << i;
            }
            G4[q] = g1;
            GE4[q] = g2;
        }
        const int vw = nv - 32 * w;
        const uint32_t vbits = vw >= 32 ? 0xffffffffu : (vw <= 0 ? 0u : ((1u << vw) - 1u));
#define PKV_HEAD_MASK(W, H)                                                              \
    (prmt_i<0x5410u>(prmt_i<((4u + (H)) << 4) | (H)>(W[0], W[1]),                      \
                     prmt_i<((4u + (H)) << 4) | (H)>(W[2], W[3])))
        gm[0][w] = PKV_HEAD_MASK(G4, 0) & vbits;  em[0][w] = PKV_HEAD_MASK(GE4, 0) & vbits & ~gm[0][w];
        gm[1][w] = PKV_HEAD_MASK(G4, 1) & vbits;  em[1][w] = PKV_HEAD_MASK(GE4, 1) & vbits & ~gm[1][w];
        gm[2][w] = PKV_HEAD_MASK(G4, 2) & vbits;  em[2][w] = PKV_HEAD_MASK(GE4, 2) & vbits & ~gm[2][w];
        gm[3][w] = PKV_HEAD_MASK(G4, 3) & vbits;  em[3][w] = PKV_HEAD_MASK(GE4, 3) & vbits & ~gm[3][w];
#undef PKV_HEAD_MASK
    }
    uint64_t gb = 0, eb = 0;
#pragma unroll
    for (int g = 0; g < PACK; ++g) {
        uint32_t ng = 0, ne = 0;
#pragma unroll
        for (int w = 0; w < kCWords; ++w) { ng += __popc(gm[g][w]); ne += __popc(em[g][w]); }
        gb |= static_cast<uint64_t>(ng) << (16 * g);
        eb |= static_cast<uint64_t>(ne) << (16 * g);
    }
    uint64_t tg, te;
    gb = vgroup_excl_scan(gb, &tg, scan);
    eb = vgroup_excl_scan(eb, &te, scan);

    const int32_t kbase = static_cast<int32_t>(k0);
#pragma unroll
    for (int g = 0; g < PACK; ++g) {
        if (g >= hp) break;
        const int head = head0 + g;
        const int32_t* cb2 = a.cbase + (static_cast<int64_t>(head) * a.nch + c) * 2;
        const int32_t E = ldcg_i32(a.thr + head * 4 + 1);
        const int32_t B = max(0, E - ldcg_i32(cb2 + 1));
        const int32_t gbefore = static_cast<int32_t>((gb >> (16 * g)) & 0xffffu);
        const int32_t ebefore = static_cast<int32_t>((eb >> (16 * g)) & 0xffffu);
        uint32_t sel[kCWords];
        int mine_e = 0, nsel = 0;
#pragma unroll
        for (int w = 0; w < kCWords; ++w) mine_e += __popc(em[g][w]);
        const int take = min(max(B - ebefore, 0), mine_e);
#pragma unroll
        for (int w = 0; w < kCWords; ++w) sel[w] = gm[g][w] | (take == mine_e ? em[g][w] : 0u);
        if (take != mine_e) {                 // the one thread where the E-th tie falls
            int left = take;
#pragma unroll
            for (int w = 0; w < kCWords; ++w) {
                uint32_t m = em[g][w];
                for (; left > 0 && m; --left) {
                    const uint32_t low = m & (0u - m);
                    sel[w] |= low;
                    m ^= low;
                }
            }
        }
#pragma unroll
        for (int w = 0; w < kCWords; ++w) nsel += __popc(sel[w]);
        const int32_t start = ldcg_i32(cb2) + gbefore + min(B, ebefore);
        if (start + nsel > a.C) {            // never taken when the histograms are consistent
            atomicExch(a.status, ST_BADINDEX);
            continue;
        }
        int32_t* out = a.cand + static_cast<int64_t>(head) * a.cmax + start;
#pragma unroll
        for (int w = 0; w < kCWords; ++w) {
            uint32_t m = sel[w];
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1u;
                *out++ = kbase + 32 * w + j;
            }
        }
    }
    __threadfence();
    bar_v();
    if (t == 0) atomicAdd(pk(a, PK_C, p), 1);
}

// ---------------------------------------------------------------------------------------
// K: top-k of one query head (vote group, 256 threads)
// ---------------------------------------------------------------------------------------
// Exact selection on the order-preserving image u of S (ties to the lower key index,
// output in key order, est = ||q|| S). The head's S values (and, for the last pass, its
// candidate indices) are streamed into shared memory in 16 KB chunks by bulk async copies,
// two chunks in flight.
//  1. The rerank counted u's top 11 bits: that histogram names the bin holding the k-th
//     largest value and how many of the k lie above it.
//  2. Radix levels narrow [lo, hi] to the k-th largest value T: a level streams S,
//     histograms the values inside [lo, hi] by their next bits and keeps them in a list in
//     shared memory when they fit; once they do, further levels run on the list alone.
//  3. A final pass streams S and the indices, counts per warp-tile the values above T and
//     the ties at T, scans them in key order chunk by chunk, and writes every value above T
//     and the first E ties at T.
// The vote group's whole shared-memory area is scratch: top-k items are the last items the
// vote group takes, so no vote table or histogram is needed after them.
constexpr int kKChunk = 4096;               // values per streamed chunk
constexpr int kKBuf = 9216;                 // offset of the four chunk buffers (S0, S1, I0, I1)
constexpr int kKList = kKBuf + 4 * kKChunk * 4;
static_assert(kKList + 4 * 8192 <= kVRingBytes + kTabBytes + kH2Bytes, "top-k list");

__device__ void k_item(const SearchArgs& a, int head, uint8_t* kscr, uint32_t kscr_bytes) {
    const int kKListCap = static_cast<int>((kscr_bytes - kKList) / 4);
    constexpr int BPT = kBins / kVT;    // 8 bins per thread
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int C = a.C, k = a.k;
    uint32_t* hist = reinterpret_cast<uint32_t*>(kscr);                // [kBins]
    uint32_t* wa = reinterpret_cast<uint32_t*>(kscr + 8192);           // [kVW]
    uint32_t* wb = wa + kVW;                                            // [kVW]
    uint32_t* pick = wb + kVW;                                          // [2]
    uint32_t* listn = pick + 2;                                         // [1]
    uint32_t* list = reinterpret_cast<uint32_t*>(kscr + kKList);
    const uint32_t bar0 = smem_addr(kscr + 8448);                       // 2 mbarriers
    const float* Sh = a.S + static_cast<int64_t>(head) * a.cmax;
    const int32_t* ch = a.cand + static_cast<int64_t>(head) * a.cmax;
    const int nchk = (C + kKChunk - 1) / kKChunk;

    if (t == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        mbar_fence_init();
        // S and the indices were written by the rerank warps (generic stores, acquired by the
        // wait before this item) and are read here by the async proxy
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    bar_v();
    uint32_t par = 0;   // bit s: parity of mbarrier s's next phase
    // streams chunks 0..nchk-1 through the two buffer pairs; body(chunk, S, idx) runs on
    // every thread with the chunk resident
    auto stream = [&](bool with_idx, auto&& body) {
        auto issue = [&](int c) {
            const int len = min(kKChunk, C - c * kKChunk);
            const uint32_t bytes = static_cast<uint32_t>((len * 4 + 15) & ~15);
            const uint32_t bar = bar0 + 8 * (c & 1);
            mbar_arrive_expect_tx(bar, with_idx ? 2 * bytes : bytes);
            bulk_g2s(smem_addr(kscr + kKBuf + (c & 1) * kKChunk * 4), Sh + c * kKChunk, bytes, bar);
            if (with_idx)
                bulk_g2s(smem_addr(kscr + kKBuf + (2 + (c & 1)) * kKChunk * 4), ch + c * kKChunk,
                         bytes, bar);
        };
        if (t == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            for (int c = 0; c < min(2, nchk); ++c) issue(c);
        }
        for (int c = 0; c < nchk; ++c) {
            const int sl = c & 1;
            mbar_wait_limit(bar0 + 8 * sl, (par >> sl) & 1u, a.spin_limit, a.status);
            par ^= 1u << sl;
            body(c, reinterpret_cast<const uint32_t*>(kscr + kKBuf + sl * kKChunk * 4),
                 reinterpret_cast<const int32_t*>(kscr + kKBuf + (2 + sl) * kKChunk * 4));
            bar_v();   // the buffers of chunk c are free again
            if (t == 0 && c + 2 < nchk) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue(c + 2);
            }
        }
    };

    const uint64_t tk0 = a.trace ? gtime() : 0;
    uint32_t krem = static_cast<uint32_t>(k);
    uint32_t lo = 0u, hi = 0xffffffffu;
    // finds, from each thread's BPT bins, the bin holding the krem-th largest value and
    // narrows [lo, hi] to it (every thread makes the same choice)
    auto choose = [&](const auto& h, int sh) {
        constexpr int NB = sizeof(h) / sizeof(h[0]);   // bins per thread
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < NB; ++j) mine += h[j];
        uint32_t x = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += y;
        }
        if (lane == 0) wa[warp] = x;
        bar_v();
        if (warp == 0) {
            const uint32_t tv = lane < kVW ? wa[lane] : 0u;
            uint32_t y = tv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t z = __shfl_down_sync(0xffffffffu, y, o);
                if (lane + o < 32) y += z;
            }
            if (lane < kVW) wb[lane] = y - tv;
        }
        if (t == 0) pick[0] = 0xffffffffu;
        bar_v();
        uint32_t above = wb[warp] + x - mine;
#pragma unroll
        for (int j = NB - 1; j >= 0; --j) {
            if (above < krem && krem <= above + h[j]) {
                pick[0] = NB * t + j;
                pick[1] = above;
            }
            above += h[j];
        }
        bar_v();
        if (pick[0] == 0xffffffffu) {   // the counts do not hold the k-th value: give up
            if (t == 0) atomicExch(a.status, ST_BADINDEX);
            lo = hi;
            bar_v();
            return;
        }
        const uint32_t b = pick[0];
        krem -= pick[1];
        const uint32_t nlo = lo + (b << sh);
        const uint64_t bin_hi = static_cast<uint64_t>(nlo) + ((uint64_t{1} << sh) - 1u);
        lo = nlo;
        hi = static_cast<uint32_t>(min(static_cast<uint64_t>(hi), bin_hi));
        bar_v();
    };
    // 1. first level, counted by the rerank (kBins1 bins of the top kBits1 bits)
    {
        constexpr int NB1 = kBins1 / kVT;
        uint32_t h[NB1];
        const uint32_t* hs = a.shist + static_cast<int64_t>(head) * kBins1 + NB1 * t;
#pragma unroll
        for (int i = 0; i < NB1 / 4; ++i) {
            const uint4 v = ldcg_u128(hs + 4 * i);
            h[4 * i] = v.x; h[4 * i + 1] = v.y; h[4 * i + 2] = v.z; h[4 * i + 3] = v.w;
        }
        choose(h, 32 - kBits1);
    }
    // 2. radix levels until the k-th largest value is isolated
    bool listed = false;   // the list holds every value inside [lo, hi]
    for (int level = 0; lo != hi && level < 4; ++level) {
        const uint32_t span = hi - lo;
        const int bitlen = 32 - __clz(span);
        const int sh = bitlen > 11 ? bitlen - 11 : 0;
#pragma unroll
        for (int j = 0; j < BPT; ++j) hist[t + kVT * j] = 0u;
        if (t == 0) *listn = 0u;
        bar_v();
        if (listed) {
            const int n1 = static_cast<int>(*reinterpret_cast<volatile uint32_t*>(pick + 3));
            for (int i = t; i < n1; i += kVT) {
                const uint32_t u = list[i];
                if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
            }
        } else {
            const uint32_t l0 = lo, h0 = hi;
            if (a.trace && t == 0) atomicAdd(a.trace + 3 * TR_KSEL + 0, 1ull);   // stream passes
            stream(false, [&](int c, const uint32_t* sb, const int32_t*) {
                const int len = min(kKChunk, C - c * kKChunk);
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int p0 = (warp + kVW * r) * 256 + 8 * lane;   // within the chunk
                    const uint4 x = *reinterpret_cast<const uint4*>(sb + p0);
                    const uint4 y = *reinterpret_cast<const uint4*>(sb + p0 + 4);
                    const uint32_t w[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t u = order_key(__uint_as_float(w[j]));
                        const bool in = p0 + j < len && u >= l0 && u <= h0;
                        if (in) atomicAdd(&hist[(u - l0) >> sh], 1u);
                        const uint32_t m = __ballot_sync(0xffffffffu, in);
                        if (m) {
                            uint32_t base = 0;
                            if (lane == 0) base = atomicAdd(listn, static_cast<uint32_t>(__popc(m)));
                            base = __shfl_sync(0xffffffffu, base, 0);
                            const uint32_t slot = base + __popc(m & ((1u << lane) - 1u));
                            if (in && slot < static_cast<uint32_t>(kKListCap)) list[slot] = u;
                        }
                    }
                }
            });
            // stream() ends with a barrier: the list count is final
            listed = *listn <= static_cast<uint32_t>(kKListCap);
            if (t == 0) pick[3] = *listn;
            bar_v();
        }
        bar_v();
        uint32_t h[BPT];
#pragma unroll
        for (int j = 0; j < BPT; ++j) h[j] = hist[BPT * t + j];
        choose(h, sh);
    }
    const uint32_t T = lo, E = krem;
    const uint64_t tk1 = a.trace ? gtime() : 0;
    if (a.trace && t == 0) {
        atomicAdd(a.trace + 3 * TR_KSEL + 2, static_cast<unsigned long long>(tk1 - tk0));
        if (!listed) atomicAdd(a.trace + 3 * TR_KSEL + 1, 1ull);   // selections without a list
    }
    // 3. winners in key order: warp w scans tiles 2w, 2w + 1 of every chunk
    const float qn = ldcg_f32(a.qnorm + head);
    int32_t* oi = a.topk_idx + static_cast<int64_t>(head) * k;
    float* oe = a.topk_est ? a.topk_est + static_cast<int64_t>(head) * k : nullptr;
    uint32_t gt_run = 0, eq_run = 0;   // values above T / ties at T before the chunk
    stream(true, [&](int c, const uint32_t* sb, const int32_t* ib) {
        const int len = min(kKChunk, C - c * kKChunk);
        uint32_t u[2][8];
        uint32_t ng[2], ne[2], gp[2], ep[2], tg[2], te[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int p0 = (2 * warp + r) * 256 + 8 * lane;
            const uint4 x = *reinterpret_cast<const uint4*>(sb + p0);
            const uint4 y = *reinterpret_cast<const uint4*>(sb + p0 + 4);
            const uint32_t w[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
            ng[r] = 0;
            ne[r] = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                u[r][j] = p0 + j < len ? order_key(__uint_as_float(w[j])) : 0u;
                const bool v = p0 + j < len;
                ng[r] += v && u[r][j] > T;
                ne[r] += v && u[r][j] == T;
            }
            gp[r] = ng[r];
            ep[r] = ne[r];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t xg = __shfl_up_sync(0xffffffffu, gp[r], o);
                const uint32_t xe = __shfl_up_sync(0xffffffffu, ep[r], o);
                if (lane >= o) { gp[r] += xg; ep[r] += xe; }
            }
            tg[r] = __shfl_sync(0xffffffffu, gp[r], 31);
            te[r] = __shfl_sync(0xffffffffu, ep[r], 31);
            gp[r] -= ng[r];
            ep[r] -= ne[r];
        }
        if (lane == 0) { wa[warp] = tg[0] + tg[1]; wb[warp] = te[0] + te[1]; }
        bar_v();
        uint32_t gw = gt_run, ew = eq_run, gc = 0, ec = 0;
#pragma unroll
        for (int w = 0; w < kVW; ++w) {
            const uint32_t x = wa[w], y = wb[w];
            gw += w < warp ? x : 0u;
            ew += w < warp ? y : 0u;
            gc += x;
            ec += y;
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            // ties before this lane's first value, and where its first winner goes
            uint32_t eb = ew + ep[r] + (r ? te[0] : 0u);
            uint32_t pos = gw + gp[r] + (r ? tg[0] : 0u) + min(eb, E);
            if (ng[r] + ne[r]) {
                const int p0 = (2 * warp + r) * 256 + 8 * lane;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const bool v = p0 + j < len;
                    bool take = v && u[r][j] > T;
                    if (v && u[r][j] == T) take = eb++ < E;
                    if (take) {
                        if (pos < static_cast<uint32_t>(k)) {
                            oi[pos] = ib[p0 + j];
                            if (oe) oe[pos] = __fmul_rn(qn, value_of(u[r][j]));
                        } else {
                            atomicExch(a.status, ST_BADINDEX);   // never taken when counts agree
                        }
                        ++pos;
                    }
                }
            }
        }
        gt_run += gc;
        eq_run += ec;
    });
    if (t == 0) {
        asm volatile("mbarrier.inval.shared::cta.b64 [%0];" :: "r"(bar0) : "memory");
        asm volatile("mbarrier.inval.shared::cta.b64 [%0];" :: "r"(bar0 + 8) : "memory");
        if (a.trace) atomicAdd(a.trace + 3 * TR_KWRITE + 2, static_cast<unsigned long long>(gtime() - tk1));
    }
}

// ---------------------------------------------------------------------------------------
// R: rerank warps
// ---------------------------------------------------------------------------------------
// Decode constants, held in registers for a whole stage: the bytes 0x4B000000 (the
// exponent of 2^23) and the fp32 pair (-(2^23 + 8), -(2^23 + 8)). Produced by opaque moves so
// that they are not re-created at every use.
struct DecodeConsts {
    uint32_t k4b;
    uint64_t koff;
};
__device__ __forceinline__ DecodeConsts decode_consts() {
    DecodeConsts d;
    asm volatile("mov.b32 %0, 0x4B000000;" : "=r"(d.k4b));
    asm volatile("mov.b64 %0, 0xCB000008CB000008;" : "=l"(d.koff));
    return d;
}

template <int K>
__device__ __forceinline__ uint64_t level_pair(uint32_t xa, uint32_t xb, const DecodeConsts& dc) {
    // byte K of each word into the mantissa of 2^23: 2^23 + u exactly; minus (2^23 + 8) = vt
    return add2(pack2u(prmt_i<0x7650u + K>(xa, dc.k4b), prmt_i<0x7650u + K>(xb, dc.k4b)), dc.koff);
}
template <int K>
__device__ __forceinline__ uint64_t table_pair(uint32_t xa, uint32_t xb, const float* dec) {
    return pack2(dec[(xa >> (8 * K)) & 15u], dec[(xb >> (8 * K)) & 15u]);
}

// p chains of the subspace pair (a, b) from their code words, with the query pairs
// q[j] = (q~_{a,j}, q~_{b,j}) for j = 0..7.
template <bool TABLE>
__device__ __forceinline__ float2 pair_dots(uint32_t wa, uint32_t wb, const uint64_t q[8],
                                            const float* dec, const DecodeConsts& dc) {
    const uint32_t ea = wa & 0x0F0F0F0Fu, oa = (wa >> 4) & 0x0F0F0F0Fu;
    const uint32_t eb = wb & 0x0F0F0F0Fu, ob = (wb >> 4) & 0x0F0F0F0Fu;
    uint64_t p = pack2(0.0f, 0.0f);
    if constexpr (TABLE) {
        p = fma2(table_pair<0>(ea, eb, dec), q[0], p);
        p = fma2(table_pair<0>(oa, ob, dec), q[1], p);
        p = fma2(table_pair<1>(ea, eb, dec), q[2], p);
        p = fma2(table_pair<1>(oa, ob, dec), q[3], p);
        p = fma2(table_pair<2>(ea, eb, dec), q[4], p);
        p = fma2(table_pair<2>(oa, ob, dec), q[5], p);
        p = fma2(table_pair<3>(ea, eb, dec), q[6], p);
        p = fma2(table_pair<3>(oa, ob, dec), q[7], p);
    } else {
        p = fma2(level_pair<0>(ea, eb, dc), q[0], p);
        p = fma2(level_pair<0>(oa, ob, dc), q[1], p);
        p = fma2(level_pair<1>(ea, eb, dc), q[2], p);
        p = fma2(level_pair<1>(oa, ob, dc), q[3], p);
        p = fma2(level_pair<2>(ea, eb, dc), q[4], p);
        p = fma2(level_pair<2>(oa, ob, dc), q[5], p);
        p = fma2(level_pair<3>(ea, eb, dc), q[6], p);
        p = fma2(level_pair<3>(oa, ob, dc), q[7], p);
    }
    return unpack2(p);
}

__device__ __forceinline__ void load_qpairs(const uint64_t* qp, uint64_t q[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const ulonglong2 v = reinterpret_cast<const ulonglong2*>(qp)[i];
        q[2 * i] = v.x;
        q[2 * i + 1] = v.y;
    }
}

// S of the record in `row` (piece q at 16 ((q ^ sw) mod 8) bytes) for the query pairs qp
// (pair t at qp + 8 t).
template <bool TABLE>
__device__ __forceinline__ float score_record(const uint8_t* row, int sw, const uint64_t* qp,
                                              const float* dec, const DecodeConsts& dc) {
    float S = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {   // chunk c: subspaces 4c..4c+3
        const uint4 cw = *reinterpret_cast<const uint4*>(row + (((2 * c) ^ sw) << 4));
        const uint4 fw = *reinterpret_cast<const uint4*>(row + (((2 * c + 1) ^ sw) << 4));
        uint64_t q[8];
        load_qpairs(qp + 16 * c, q);
        const float2 pa = pair_dots<TABLE>(cw.x, cw.y, q, dec, dc);
        S = __fmaf_rn(__uint_as_float(fw.x), pa.x, S);
        S = __fmaf_rn(__uint_as_float(fw.y), pa.y, S);
        load_qpairs(qp + 16 * c + 8, q);
        const float2 pb = pair_dots<TABLE>(cw.z, cw.w, q, dec, dc);
        S = __fmaf_rn(__uint_as_float(fw.z), pb.x, S);
        S = __fmaf_rn(__uint_as_float(fw.w), pb.y, S);
    }
    return S;
}

// ---------------------------------------------------------------------------------------
// R: rerank of one range of up to kRItem candidates of one query head (whole CTA)
// ---------------------------------------------------------------------------------------
// Warp w takes the stages w, w + 8, ... of 32 candidates; each warp gathers its stages' records
// with 16-byte cp.async copies (eight lanes per record, so one warp instruction moves four
// records) into a ring of kSlots stages and scores one record per lane. Every value is also
// counted, by the top 13 bits of its order-preserving image, into the head's first top-k
// level (lanes with the same bin are grouped by a warp match; one global add per group).
template <bool TABLE>
__device__ void r_item(const SearchArgs& a, int head, int r, uint8_t* smem, const float* dec) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c0 = r * kRItem, c1 = min(a.C, c0 + kRItem);
    const int nst = (c1 - c0 + kStage - 1) / kStage;
    uint8_t* ring = smem + kOffRing + warp * kRingWarp;
    float2* qs = reinterpret_cast<float2*>(smem + kOffQry);
    const uint64_t* qp = reinterpret_cast<const uint64_t*>(qs);
    if (threadIdx.x < 64) {   // the head's rotated query as (subspace 2t, 2t + 1) pairs
        const float* qh = a.qt + static_cast<int64_t>(head) * D;
        const int tt = threadIdx.x >> 3, j = threadIdx.x & 7;
        qs[threadIdx.x] = make_float2(ldcg_f32(qh + 16 * tt + j), ldcg_f32(qh + 16 * tt + 8 + j));
    }
    bar_v();
    const uint8_t* ubase = a.rec + static_cast<int64_t>(head / a.G) * a.cap_pad * REC;
    const int32_t* cbase = a.cand + static_cast<int64_t>(head) * a.cmax;
    const int nmine = nst > warp ? (nst - warp + kW - 1) / kW : 0;   // this warp's stages
    // commits one ring step: the copies of this warp's k-th stage, or an empty group
    auto issue = [&](int k) {
        if (k < nmine) {
            const int pos = c0 + (warp + kW * k) * kStage;
            const int cnt = min(kStage, c1 - pos);
            uint32_t idx = 0xffffffffu;
            if (lane < cnt) {
                idx = static_cast<uint32_t>(ldcg_i32(cbase + pos + lane));
                if (idx >= static_cast<uint64_t>(a.n)) {
                    atomicExch(a.status, ST_BADINDEX);   // never taken when selection is consistent
                    idx = 0xffffffffu;
                }
            }
            uint8_t* dst0 = ring + (k % kSlots) * (kStage * REC);
            const int piece = lane & 7, sub = lane >> 3;
#pragma unroll
            for (int j = 0; j < kStage / 4; ++j) {
                const int rr = 4 * j + sub;
                const uint32_t ri = __shfl_sync(0xffffffffu, idx, rr);
                if (ri != 0xffffffffu) {
                    const uint32_t dst = smem_addr(dst0 + rr * REC + ((piece ^ (rr & 7)) << 4));
                    const uint8_t* srcp = ubase + static_cast<uint64_t>(ri) * REC + piece * 16;
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(srcp) : "memory");
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    for (int k = 0; k < kSlots; ++k) issue(k);
    for (int k = 0; k < nmine; ++k) {
        asm volatile("cp.async.wait_group %0;" :: "n"(kSlots - 1) : "memory");
        __syncwarp();
        const int pos = c0 + (warp + kW * k) * kStage;
        const int cnt = min(kStage, c1 - pos);
        if (lane < cnt) {
            const DecodeConsts dc = decode_consts();
            const float sv = score_record<TABLE>(ring + (k % kSlots) * (kStage * REC) + lane * REC,
                                                 lane & 7, qp, dec, dc);
            a.S[static_cast<int64_t>(head) * a.cmax + pos + lane] = sv;
            const uint32_t bin = order_key(sv) >> (32 - kBits1);
            const uint32_t peers = __match_any_sync(__activemask(), bin);
            if (lane == __ffs(peers) - 1)
                atomicAdd(&a.shist[static_cast<int64_t>(head) * kBins1 + bin],
                          static_cast<uint32_t>(__popc(peers)));
        }
        __syncwarp();   // every lane has read the slot
        issue(k + kSlots);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // no copy in flight past the item
    __threadfence();
    bar_v();
    if (threadIdx.x == 0) {
        const int unit = head / a.G, g = head - unit * a.G;
        atomicAdd(pk(a, PK_R, unit * a.packs + g / PACK), 1);
    }
}

}  // namespace

// ---------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------
namespace {

// Progress board checkpoints (debugging aid): threads 1, 32, 224 and 0 report 100 * (loop
// iteration) + checkpoint into words 4..7 of their CTA's board entry.
__device__ __forceinline__ void mark(const SearchArgs& a, int iter, int v) {
    if (!a.progress) return;
    const int t = threadIdx.x;
    const int slot = t == 0 ? 7 : t == 1 ? 4 : t == 32 ? 5 : t == 224 ? 6 : -1;
    if (slot >= 0) reinterpret_cast<volatile int*>(a.progress)[8 * blockIdx.x + slot] = 100 * iter + v;
}

template <bool TABLE>
__global__ void __launch_bounds__(kThreads, 2) search_kernel(const SearchArgs a) {
    uint8_t* smem = g_smem;
    __shared__ float dec[16];
    __shared__ int vbuf[4];      // claimed item (type, x, y), abort flag
    __shared__ __align__(8) uint64_t vbar[kVSlots];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x < 16) dec[threadIdx.x] = TABLE ? a.lvt[16 + threadIdx.x] : 0.0f;
    if (threadIdx.x == 0) {
        vbuf[3] = 0;
        for (int s = 0; s < kVSlots; ++s) mbar_init(smem_addr(&vbar[s]), 1);
        mbar_fence_init();
    }
    const uint64_t tk0 = a.trace ? gtime() : 0;
    __syncthreads();

    // per-lane address parts of the vote lookups: at step t lane L reads subspace
    // (t + L / 2) mod 16 of both its keys (the encoder rotates key i's bytes by (i / 2) mod
    // 16), in copy L mod 2, which owns bank column 2 * subspace + copy; three columns per
    // register with a zero top byte, so one PRMT builds an address
    uint32_t colp[6];
#pragma unroll
    for (int r = 0; r < 6; ++r) {
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int tt = 3 * r + j;
            if (tt < 16) w |= (4u * (2u * ((tt + (lane >> 1)) & 15) + (lane & 1))) << (8 * j);
        }
        colp[r] = w;
    }
    int cur_table = -1;          // pack-unit whose vote table is in shared memory
    bool counters_clean = false; // the vote counters are zero (cleared lazily)
    VRing vr{smem_addr(&vbar[0]), 0};
    uint8_t* scr = smem + kOffScr;
    for (int iter = 0;; ++iter) {
        mark(a, iter, 1);
        if (threadIdx.x == 0) {
            const int64_t it = atomicAdd(ctl(a, CT_Q), 1);
            const Item vi = queue_item(a, it);
            vbuf[0] = vi.type;
            vbuf[1] = vi.x;
            vbuf[2] = vi.y;
            const uint64_t tw = a.trace ? gtime() : 0;
            bool ok = true;
            if (vi.type == IT_V && vi.x != cur_table) {
                ok = wait_flag(pk(a, PK_Q, vi.x), heads_of(a, vi.x), true, a.spin_limit, a.status, a.trace, a.ctrl);
            } else if (vi.type == IT_C) {
                ok = wait_flag(pk(a, PK_F, vi.x), 1, false, a.spin_limit, a.status, a.trace, a.ctrl);
            } else if (vi.type == IT_R || vi.type == IT_K) {
                const int unit = vi.x / a.G, g = vi.x - unit * a.G;
                const int p = unit * a.packs + g / PACK;
                ok = vi.type == IT_R
                         ? wait_flag(pk(a, PK_C, p), a.nc, true, a.spin_limit, a.status, a.trace, a.ctrl)
                         : wait_flag(pk(a, PK_R, p), heads_of(a, p) * a.nrh, true, a.spin_limit,
                                     a.status, a.trace, a.ctrl);
            }
            if (!ok) vbuf[3] = 1;
            if (a.progress) {
                volatile int* pb = a.progress + 8 * blockIdx.x;
                pb[0] = static_cast<int>(it); pb[1] = vi.type; pb[2] = vi.x; pb[3] = ok ? 1 : -1;
            }
            if (a.trace && vi.type != IT_NONE)
                trace_add(a.trace, vi.type == IT_R ? TR_RWAIT : TR_VWAIT, tw, gtime());
        }
        __syncwarp();
        bar_v();
        mark(a, iter, 2);
        const int type = vbuf[0], x = vbuf[1], y = vbuf[2];
        if (type == IT_NONE || vbuf[3]) break;
        const uint64_t t0 = a.trace ? gtime() : 0;
        if (type == IT_Q) {
            q_item(a, x, scr);
        } else if (type == IT_V) {
            if (!counters_clean) {
                for (int i = threadIdx.x; i < 256 * 8; i += kThreads)   // upper halves of the table rows
                    *reinterpret_cast<uint4*>(smem + kOffTab + (i >> 3) * 256 + 128 + 16 * (i & 7)) =
                        make_uint4(0, 0, 0, 0);
                for (int i = threadIdx.x; i < static_cast<int>(kH2Bytes / 16); i += kThreads)
                    reinterpret_cast<uint4*>(smem + kOffH2)[i] = make_uint4(0, 0, 0, 0);
                counters_clean = true;
            }
            if (x != cur_table) {
                bar_v();
                load_table(a, x, smem + kOffTab);
                cur_table = x;
            }
            bar_v();
            mark(a, iter, 5);
            v_item(a, x, y, smem, colp, vr);
            mark(a, iter, 6);
            __threadfence();
            bar_v();
            if (threadIdx.x == 0) {
                vbuf[2] = atomicAdd(pk(a, PK_V, x), 1);
                __threadfence();   // the other vote items' histograms are visible after this
            }
            bar_v();
            mark(a, iter, 7);
            if (vbuf[2] == a.nc - 1) {
                if (a.trace && threadIdx.x == 0) trace_add(a.trace, TR_V, t0, gtime());
                const uint64_t t1 = a.trace ? gtime() : 0;
                f_item(a, x, scr);
                mark(a, iter, 8);
                if (a.trace && threadIdx.x == 0) trace_add(a.trace, TR_F, t1, gtime());
                bar_v();
                continue;
            }
        } else if (type == IT_C) {
            c_item(a, x, y, scr);
        } else if (type == IT_R) {
            r_item<TABLE>(a, x, y, smem, dec);
            counters_clean = false;
            cur_table = -1;
        } else {
            k_item(a, x, smem, kSmem);
            counters_clean = false;
            cur_table = -1;
        }
        if (a.trace && threadIdx.x == 0)
            trace_add(a.trace, type == IT_R ? TR_R : type, t0, gtime());
        if (a.progress && threadIdx.x == 0) reinterpret_cast<volatile int*>(a.progress)[8 * blockIdx.x + 3] = 2;
        mark(a, iter, 9);
        bar_v();
    }
    mark(a, 99, 3);
    __syncthreads();
    mark(a, 99, 4);
    if (threadIdx.x == 0) {
        if (a.progress) reinterpret_cast<volatile int*>(a.progress)[8 * blockIdx.x + 3] = 3;
        if (a.trace) trace_add(a.trace, TR_KERNEL, tk0, gtime());
        __threadfence();
        const int done = atomicAdd(ctl(a, CT_EXIT), 1);
        if (done == static_cast<int>(gridDim.x) - 1) {
            // the last CTA out resets the queue and the per-pack counters for the next search
            *ctl(a, CT_Q) = 0;
            for (int i = 0; i < PK_N * a.P; ++i) *ctl(a, CT_HDR + i) = 0;
            __threadfence();
            *ctl(a, CT_EXIT) = 0;
        }
    }
}

}  // namespace

// ---------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------
int search_ctrl_words(int P) { return (CT_HDR + PK_N * P) * kCtlStride; }
static_assert(kTraceWords == 3 * TR_SLOTS, "trace layout");


cudaError_t launch_search(pariskv_index* ix, const void* q, const float* qt_in,
                          const float* qn_in, bool rotated, int64_t C, int32_t k,
                          int32_t* topk_idx, float* topk_est, cudaStream_t st) {
    const auto& c = ix->cfg;
    const bool table = c.levels != PARISKV_LEVELS_UNIFORM;
    static std::atomic<uint64_t> raised{0}, raised_t{0};
    cudaError_t e = table ? raise_smem_limit(search_kernel<true>, kSmem, raised_t)
                          : raise_smem_limit(search_kernel<false>, kSmem, raised);
    if (e != cudaSuccess) return e;
    const int nc = static_cast<int>(ceil_div(ix->n, CHUNK));
    const int P = ix->units * ix->packs;
    const int heads = ix->units * c.group;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    SearchArgs a{};
    a.ids = ix->ids; a.rec = ix->rec; a.signs = ix->signs; a.cent = ix->cent; a.lvt = ix->lvt;
    a.q = q; a.qt_in = qt_in; a.qn_in = qn_in;
    a.qt = ix->qt; a.qnorm = ix->qnorm; a.lut = ix->lut; a.scores = ix->scores;
    a.hist = ix->hist; a.thr = ix->thr; a.cbase = ix->cbase; a.cand = ix->cand; a.S = ix->S;
    a.shist = ix->shist; a.topk_idx = topk_idx; a.topk_est = topk_est;
    a.ctrl = ix->ctrl; a.status = ix->status; a.trace = ix->profile ? ix->trace : nullptr;
    a.progress = ix->progress;
    a.n = ix->n; a.cap_pad = ix->cap_pad; a.cmax = ix->cmax;
    a.spin_limit = ix->spin_limit;
    a.units = ix->units; a.G = c.group; a.packs = ix->packs; a.P = P; a.nc = nc;
    a.nch = static_cast<int>(ix->cap_pad / CHUNK); a.heads = heads;
    a.rho = c.rho; a.w1 = c.w_rank1; a.wr = c.w_rest; a.nr = NB * c.w_rank1 + 1;
    a.C = static_cast<int>(C); a.k = k; a.nrh = static_cast<int>(ceil_div(C, kRItem));
    a.qbf16 = c.dtype == PARISKV_BF16; a.rotated = rotated ? 1 : 0;
    if (a.trace) {
        e = cudaMemsetAsync(ix->trace, 0, kTraceWords * sizeof(unsigned long long), st);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * sms));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    return table ? cudaLaunchKernelEx(&cfg, search_kernel<true>, a)
                 : cudaLaunchKernelEx(&cfg, search_kernel<false>, a);
}

}  // namespace pkv
