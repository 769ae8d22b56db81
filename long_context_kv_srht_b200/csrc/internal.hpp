// internal.hpp -- the index object and the kernel launchers behind the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "pariskv.h"

struct pariskv_index {
    pariskv_config cfg;
    int device = 0;
    int64_t n = 0;        // tokens indexed per unit
    int64_t cap_pad = 0;  // capacity rounded up to a whole histogram chunk
    int units = 0;        // batch * num_kv_heads
    int hq = 0;           // query heads per sequence
    int packs = 0;        // ceil(group / 4): vote-table packs per KV head

    int8_t hsigns[128] = {};    // the SRHT signs as given (host copy, for index images)
    float* lvt = nullptr;       // [32] code levels: [0..7] magnitudes, [9..15] thresholds,
                                //      [16..31] signed level of each code nibble
    float* cent = nullptr;      // learned centroids [units][16][256][8], or NULL (analytic)
    float* signs = nullptr;     // [128] +-1.0f
    uint8_t* ids = nullptr;     // [units][cap_pad][16] bucket ids, byte-rotated per key
    uint8_t* rec = nullptr;     // [units][cap_pad][128] codes (64 B) + factors (16 x f32)

    // per-search scratch (library-owned)
    uint32_t* lut = nullptr;    // [units*packs][16][256] packed vote weights
    float* qt = nullptr;        // [units*group][128] rotated queries
    float* qnorm = nullptr;     // [units*group]
    uint32_t* scores = nullptr; // [units*packs][cap_pad] packed coarse scores
    uint32_t* hist = nullptr;   // [units*packs][chunks][4][64] per-chunk score histograms
    int32_t* thr = nullptr;     // [units*group][4] threshold T, ties E, candidate count C
    int32_t* cbase = nullptr;   // [units*group][chunks][2] selected/ties before each chunk
    int32_t* cand = nullptr;    // [units*group][cmax] candidate indices (ascending)
    float* S = nullptr;         // [units*group][cmax] rerank values
    uint32_t* shist = nullptr;  // [units*group][SCOPIES][SBINS] counts of S by its top order-key bits
    int64_t cmax = 0;
    int* status = nullptr;      // device status word (ST_OK / ST_TIMEOUT)

    // test hooks: one out-of-range candidate index written before the next rerank (head < 0:
    // none), and launch shapes forced for the determinism tests (0: automatic)
    int32_t inject_head = -1;
    int64_t inject_pos = 0;
    int32_t inject_value = 0;
    bool inject_wait = false;   // test hook: the next top-k's copy wait runs out
    int32_t vote_ctas = 0, rerank_ctas = 0, topk_mode = 0;

    // optional per-stage timing of searches (test and benchmark use)
    bool profile = false;
    cudaEvent_t ev[8] = {};
    int nev = 0;

    int64_t last_C = 0;
    int32_t last_k = 0;
    bool searched = false;
};

namespace pkv {

// Raises a kernel's dynamic shared-memory limit on the current device, once per device
// (devices 0..63 are remembered in `done`; others set the attribute on every call).
template <typename Kern>
cudaError_t raise_smem_limit(Kern kernel, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Launches a search kernel with programmatic stream serialization (see pdl_wait), in
// thread-block clusters of `cluster` CTAs along x when cluster > 1.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, unsigned cluster, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    unsigned na = 1;
    if (cluster > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
    return launch_pdl_cluster(kernel, grid, block, smem, st, 1u, std::forward<Args>(args)...);
}

// levels.cu: the code level table of a config ([0..7] magnitude levels, [8 + i] the fp32
// threshold between levels i-1 and i, [16 + u] the signed level of code nibble u)
constexpr int kLevelTableFloats = 32;
pariskv_status level_tables(const pariskv_config* cfg, float tab[kLevelTableFloats]);
void prior_levels(float out[8]);

// status helpers (defined in api.cu)
pariskv_status fail(pariskv_status s, const char* fmt, ...);
pariskv_status cuda_fail(cudaError_t e, const char* what);
bool alloc_fault_injected();   // PARISKV_FAULT=alloc: every device allocation fails
pariskv_status check_device_pointer(const void* p, size_t align, const char* name);
pariskv_status validate_config(const pariskv_config* cfg);   // the checks every call makes
void set_last_launches(int32_t n);   // what pariskv_last_launch_count reports
int32_t last_launches();

// encode.cu
cudaError_t launch_encode(const pariskv_index* ix, const void* keys, const float* knorm,
                          int64_t ld_tok, int64_t t, int64_t pos0, bool rotated,
                          cudaStream_t st);
cudaError_t launch_rotate(const pariskv_config* cfg, const float* signs, const void* x,
                          int64_t n, float* y, float* norm, cudaStream_t st);

// query.cu
cudaError_t launch_query_prep(const pariskv_index* ix, const void* q, const float* qt_in,
                              const float* qn_in, bool rotated, cudaStream_t st);

// vote.cu
cudaError_t launch_vote(const pariskv_index* ix, cudaStream_t st);

// select.cu
cudaError_t launch_threshold(const pariskv_index* ix, int64_t C, cudaStream_t st);
cudaError_t launch_compact(const pariskv_index* ix, cudaStream_t st);
// writes `value` to *dst on the stream (the bad-candidate test hook)
cudaError_t launch_poke(int32_t* dst, int32_t value, cudaStream_t st);
// top-k launch shapes that pariskv_debug_set_launch may force: 1 one 1024-thread CTA per head
// (C <= 8192), 2 one 256-thread CTA (C <= 8192), 3 a cluster of four 1024-thread CTAs with the
// values in shared memory (C <= 65536), 4 the same cluster reading global memory (any C)
constexpr int kTopkModes = 4;
bool topk_mode_fits(int mode, int64_t C);

// rerank.cu
cudaError_t launch_rerank(const pariskv_index* ix, int64_t C, cudaStream_t st);

// topk.cu
cudaError_t launch_topk(const pariskv_index* ix, int64_t C, int32_t k, int32_t* topk_idx,
                        float* topk_est, cudaStream_t st);

// attend.cu
cudaError_t launch_read_stream(const void* src, int64_t bytes, uint32_t* sink,
                               cudaStream_t st);
// the rerank's record gathers alone (no arithmetic): the candidates' records of every head
cudaError_t launch_gather_candidates(const uint8_t* rec, int64_t cap_pad, const int32_t* cand,
                                     int64_t cmax, int32_t C, int group, int64_t heads,
                                     int64_t n, uint32_t* sink, cudaStream_t st);
// Sparse attention has two kernels: with bf16 K/V in device memory, the tensor-core gather
// kernel of dense.cu (`mma` = true); otherwise (K/V in pinned host memory, or fp32) the
// latency-tolerant row-gather kernel of attend.cu. attend_splits gives the split count for
// the chosen kernel; the launchers take the same choice.
bool attend_uses_mma(const pariskv_config* cfg, bool kv_device);
int attend_splits(int heads, int32_t k, int num_sms, bool mma);
cudaError_t launch_attend(const pariskv_config* cfg, const void* q, const void* K,
                          const void* V, int64_t ld_tok, int64_t n, const int32_t* topk_idx,
                          int32_t k, float scale, void* out, int32_t out_dtype, float* work,
                          int nsplit, bool mma, cudaStream_t st);
// the two halves of launch_attend: split-K partials of `k` indices per head (row `head` of
// idx starts at head * k_stride) written to splits [split_base, split_base + nsplit) of
// split_total per head, and the log-sum-exp merge of split_total splits per head
cudaError_t launch_attend_partial(const pariskv_config* cfg, const void* q, const void* K,
                                  const void* V, int64_t ld_tok, int64_t n,
                                  const int32_t* idx, int32_t k, int32_t k_stride, float scale,
                                  float* work, int nsplit, int split_base, int split_total,
                                  bool mma, cudaStream_t st);
cudaError_t launch_attend_combine(int heads, const float* work, int split_total, void* out,
                                  int32_t out_dtype, cudaStream_t st);
// GQA-group union (attend.cu): for the row-gather kernel with 1 < group <= 8, the group's
// top-k lists are merged into one ascending union of rows per unit with a membership mask per
// row; each union row is fetched once and scored for every query head that selected it.
// union_workspace_bytes is the scratch launch_attend_union needs (0: the union is not used for
// this shape); the partials then take union_splits splits per head.
size_t union_workspace_bytes(const pariskv_config* cfg, int64_t n, int32_t k);
int union_splits(int units, int group, int32_t k, int num_sms);
cudaError_t launch_attend_union(const pariskv_config* cfg, const void* q, const void* K,
                                const void* V, int64_t ld_tok, int64_t n, const int32_t* topk,
                                int32_t k, float scale, void* out, int32_t out_dtype,
                                float* work, int nsplit, void* scratch, cudaStream_t st);
// the union lists of a call (inside its scratch): rows [units][cap], masks [units][cap],
// count [units]; launch_union_build fills them from the heads' top-k lists
struct UnionLists {
    int32_t* rows;
    uint8_t* masks;
    int32_t* count;
    int64_t cap;
};
cudaError_t launch_union_build(const pariskv_config* cfg, int64_t n, const int32_t* topk,
                               int32_t k, void* scratch, cudaStream_t st, UnionLists* out);
// the union's split-K partials only, into splits [split_base, split_base + nsplit) of
// split_total per head (the four-region cache merges them with its dense rows' partials)
cudaError_t launch_union_partial(const pariskv_config* cfg, const void* q, const void* K,
                                 const void* V, int64_t ld_tok, int64_t n, const int32_t* topk,
                                 int32_t k, float scale, float* work, int nsplit,
                                 int split_base, int split_total, void* scratch,
                                 cudaStream_t st);
cudaError_t read_union_rows(unsigned long long* rows);   // rows fetched since the last read
// floats per split partial in the attention workspace: 128 accumulators, the running max
// (natural-log units) and the denominator, padded so every partial starts 16-byte aligned
constexpr int kAttendPart = 128 + 4;

// dense.cu (tensor-core attention, bf16 K/V in device memory): split-K partials of dense
// attention over rows [0, n) of every unit (group <= 8), and of the rows named by each head's
// indices (gather mode), written like launch_attend_partial's
int dense_splits(int units, int64_t n, int num_sms);
int gather_splits(int heads, int32_t k, int num_sms);
int gather_min_splits(int32_t k);   // the gather kernel needs at least this many splits
cudaError_t launch_dense_partial(const pariskv_config* cfg, const void* q, const void* K,
                                 const void* V, int64_t ld_tok, int64_t n, float scale,
                                 float* work, int nsplit, int split_base, int split_total,
                                 cudaStream_t st);
cudaError_t launch_gather_partial(const pariskv_config* cfg, const void* q, const void* K,
                                  const void* V, int64_t ld_tok, int64_t n, const int32_t* idx,
                                  int32_t k, int32_t k_stride, float scale, float* work,
                                  int nsplit, int split_base, int split_total, cudaStream_t st);
// Allocation-free attention: floats in the fixed per-device workspace and its address on the
// current device (looked up on first use per device).
constexpr size_t kAttendScratchFloats = size_t(1) << 20;
cudaError_t attend_static_scratch(float** ptr);
size_t attend_workspace_floats(int heads, int nsplit);

}  // namespace pkv
