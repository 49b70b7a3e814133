// C ABI of the DSA hot path (declared in include/dsa.h): argument checks,
// workspace layout and kernel dispatch. All kernels live in the headers
// included below and are compiled here as one translation unit for sm_100a.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "dsa.h"
#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "mha_tc.cuh"
#include "attn_simple.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "debug_checks.cuh"
#include "indexer_chunked.cuh"
#include "indexer_kl.cuh"
#include "indexer_scores.cuh"
#include "indexer_tc.cuh"
#include "mha_attn.cuh"
#include "topk_select.cuh"

namespace dsa {

// One warp waits on a barrier that nothing ever signals: the bounded wait
// gives up after limit_ns, records DSA_ERR_TIMEOUT (barrier tag 999) in the
// device status word and the kernel returns. Exercises the failure-detection
// path without faulting or hanging the GPU.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t b = sm100::smem_u32(&bar);
    if (threadIdx.x == 0) {
        sm100::mbar_init(b, 1);
        abort_flag = 0;
    }
    __syncthreads();
    const bool got = sm100::mbar_wait(b, 0, &abort_flag, 999, 0, limit_ns);
    __syncwarp();
    (void)got;
}

}  // namespace dsa

namespace {

thread_local char g_err[512] = {0};
std::atomic<unsigned long long> g_launches{0};

int fail(int code, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_fail(cudaError_t e, const char* where)
{
    return fail(DSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// cuTensorMapEncodeTiled, looked up through the runtime so the library does
// not link the driver library directly (it loads on machines without a GPU).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

#define DSA_LAUNCH_CHECK(where)                                      \
    do {                                                             \
        g_launches.fetch_add(1, std::memory_order_relaxed);          \
        cudaError_t e_ = cudaGetLastError();                         \
        if (e_ != cudaSuccess) return cuda_fail(e_, where);          \
    } while (0)

// Debug build (-DDSA_DEBUG): validate an index set on the device (counts
// violations, never traps; debug_checks.cuh). `selector`: the set is a
// selector result. The release build launches nothing here.
int debug_check(const int32_t* idx, const int32_t* pos, const int32_t* k_base, int T, int S, int k,
                const dsa::PagedRows& pg, bool selector, cudaStream_t st)
{
#ifdef DSA_DEBUG
    dsa::debug_check_idx_kernel<<<T, dsa::kCheckThreads, 0, st>>>(idx, pos, k_base, T, S, k, pg, selector ? 1 : 0);
    DSA_LAUNCH_CHECK("debug_check_idx_kernel");
#else
    (void)idx; (void)pos; (void)k_base; (void)T; (void)S; (void)k; (void)pg; (void)selector; (void)st;
#endif
    return DSA_OK;
}

// ------------------------------------------------------------ phase timing
//
// Diagnostic: with timing on, the indexer brackets each of its phases with a
// pair of CUDA events on the caller's stream; dsa_phase_times() sums them.
enum Phase : int { kPhaseScores = 0, kPhaseThreshold = 1, kPhaseSelect = 2, kNumPhases = 3 };

struct PhaseRec {
    int phase;
    cudaEvent_t a, b;
};
std::mutex g_phase_mu;
std::atomic<bool> g_phase_on{false};
std::vector<PhaseRec> g_phase_recs;

// Records the start of a phase; the returned handle closes it.
struct PhaseMark {
    int phase = -1;
    cudaEvent_t a = nullptr;
    cudaStream_t st = nullptr;
};

PhaseMark phase_begin(int phase, cudaStream_t st)
{
    PhaseMark m;
    if (!g_phase_on.load(std::memory_order_relaxed)) return m;
    if (cudaEventCreate(&m.a) != cudaSuccess) return PhaseMark{};
    cudaEventRecord(m.a, st);
    m.phase = phase;
    m.st = st;
    return m;
}

void phase_end(const PhaseMark& m)
{
    if (m.phase < 0) return;
    cudaEvent_t b;
    if (cudaEventCreate(&b) != cudaSuccess) {
        cudaEventDestroy(m.a);
        return;
    }
    cudaEventRecord(b, m.st);
    std::lock_guard<std::mutex> lock(g_phase_mu);
    g_phase_recs.push_back({m.phase, m.a, b});
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream drains (it calls griddep_wait() before
// reading global memory), which hides the launch gap between the short
// kernels of a decode step.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------ workspace plan

constexpr size_t kAlign = 256;
constexpr size_t kScoreBlockBytes = size_t(1) << 30;  // score rows kept per block of queries

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Query rows whose full score rows fit in one block of the score buffer.
// Chunked indexer (per-row key ranges): rows per launch block, the per-row
// strides (most chunks of a row times k pairs, times the sampled positions)
// and the buffers it needs.
struct ChunkPlan {
    int RB, max_chunks;
    long long cand_ld, samp_ld;
    size_t off_work, off_tau, off_ccnt, off_samp, off_cand, bytes;
};

constexpr int kMaxChunksPerRow = 16384;   // S <= 2^27 keys on this path

ChunkPlan chunk_plan(int T, int S, int k)
{
    using namespace dsa::idx_chunk;
    ChunkPlan p;
    p.max_chunks = dsa::ceil_div(S, kChunkKeys);
    const bool multi = p.max_chunks > 1;
    p.cand_ld = multi ? (long long)p.max_chunks * k : 0;
    p.samp_ld = multi ? (long long)p.max_chunks * kSamplesPerChunk : 0;
    const size_t per_row = (size_t)p.cand_ld * sizeof(uint2) + (size_t)p.samp_ld * sizeof(float) +
                           (size_t)p.max_chunks * sizeof(int) + 2 * sizeof(int);
    p.RB = (int)std::min<size_t>((size_t)T, std::max<size_t>(1, kScoreBlockBytes / per_row));
    p.off_work = 0;
    p.off_tau = align_up((size_t)(p.RB + 1) * sizeof(int));
    p.off_ccnt = p.off_tau + align_up((size_t)p.RB * sizeof(uint32_t));
    p.off_samp = p.off_ccnt + align_up((size_t)p.RB * p.max_chunks * sizeof(int));
    p.off_cand = p.off_samp + align_up((size_t)p.RB * p.samp_ld * sizeof(float));
    p.bytes = p.off_cand + align_up((size_t)p.RB * p.cand_ld * sizeof(uint2));
    return p;
}

// Few rows over long key ranges (decode) with d_I = 128: every key scored into
// a dense score row, then a cluster per row thresholds, filters and selects
// (indexer_chunked.cuh, rs). Rows per launch block and the buffers they need:
// the score rows (ld floats each, at most rs::kMaxKeys keys) and the rows'
// 16-key and 4-key group maxima.
struct RowScorePlan {
    int RB;
    long long ld, g16_ld, g4_ld;
    size_t off_g16, off_g4, bytes;
};

bool use_row_scores(int T, int S, int d_I)
{
    using namespace dsa::idx_chunk;
    return d_I == 128 && S > kChunkKeys && T <= rs::kMaxRows;
}

RowScorePlan row_score_plan(int T, int S)
{
    using namespace dsa::idx_chunk;
    RowScorePlan p;
    p.ld = (long long)dsa::ceil_div(std::min(S, rs::kMaxKeys), rs::kTileKeys) * rs::kTileKeys;
    p.g16_ld = p.ld / rs::kTileKeys * rs::kGroupsPerTile;
    p.g4_ld = p.ld / 4;
    const size_t per_row = (size_t)p.ld * sizeof(float) + (size_t)(p.g16_ld + p.g4_ld) * sizeof(uint32_t);
    p.RB = (int)std::min<size_t>({(size_t)T, (size_t)rs::kMaxRows,
                                  std::max<size_t>(1, kScoreBlockBytes / per_row)});
    p.off_g16 = align_up((size_t)p.RB * p.ld * sizeof(float));
    p.off_g4 = p.off_g16 + align_up((size_t)p.RB * p.g16_ld * sizeof(uint32_t));
    p.bytes = p.off_g4 + align_up((size_t)p.RB * p.g4_ld * sizeof(uint32_t));
    return p;
}

// Streaming (tensor-core) indexer: query rows per launch block and the
// per-row buffers it needs.
constexpr int kFusedRowsPerBlock = 32768;

struct FusedPlan {
    int RB, samp_ld, cap;
    size_t off_samp, off_tau, off_cand, off_cnt, bytes;
};

FusedPlan fused_plan(int T, int S, int k)
{
    using namespace dsa::idx_tc;
    FusedPlan p;
    p.RB = std::min(T, kFusedRowsPerBlock);
    p.samp_ld = ((num_tiles(S) + kSampleStride - 1) / kSampleStride) * kKeys;
    p.cap = 2 * kAlpha * k;
    p.off_samp = 0;
    p.off_tau = align_up(p.off_samp + (size_t)p.RB * p.samp_ld * sizeof(float));
    p.off_cand = align_up(p.off_tau + (size_t)p.RB * sizeof(float));
    p.off_cnt = align_up(p.off_cand + (size_t)p.RB * p.cap * sizeof(uint2));
    p.bytes = align_up(p.off_cnt + (size_t)p.RB * sizeof(int));
    return p;
}

// Workspace of the indexer paths these head shapes can take (the streaming
// tensor-core path exists for H_I = 8, d_I = 128 only).
size_t indexer_workspace(int T, int S, int k, int H_I, int d_I)
{
    size_t chunked = chunk_plan(T, S, k).bytes;
    if (use_row_scores(T, S, d_I)) chunked = std::max(chunked, row_score_plan(T, S).bytes);
    if (H_I != dsa::idx_tc::kHI || d_I != dsa::idx_tc::kDI) return chunked;
    return std::max(chunked, fused_plan(T, S, k).bytes);
}

int num_sms()
{
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

// Tensor-core attention: one 2-CTA cluster per query row (Hq=128, d_qk=576,
// d_v=512, k a multiple of 4).
bool attn_tc_supported(int Hq, int d_qk, int d_v, int k)
{
    return Hq == dsa::attn_tc::kHeads && d_qk == dsa::attn_tc::kDqk && d_v == dsa::attn_tc::kDv &&
           k % 4 == 0;
}

// Parts each row's selected set is split into when the caller leaves it to
// the library: only as many as add no wave of work. CUDA-core kernel: CTAs
// of 8 heads, two per SM; tensor-core kernel: one cluster per SM pair.
int attn_auto_splits(int T, int Hq, int d_qk, int d_v, int k)
{
    const int max_split = std::max(1, std::min(16, k / 64));
    if (attn_tc_supported(Hq, d_qk, d_v, k)) {
        const int slots = num_sms() / 2;
        if (T >= slots) return 1;
        return std::max(1, std::min(max_split, slots / T));
    }
    const long long ctas = (long long)T * dsa::ceil_div(Hq, dsa::kAttnHeads);
    const long long want = 2LL * num_sms();
    if (ctas >= want) return 1;
    const int s = (int)((want + ctas - 1) / ctas);
    return std::max(1, std::min(s, max_split));
}

// Workspace of a split attention: the parts' fp32 outputs and log-sum-exps.
size_t attn_split_workspace(int T, int Hq, int d_v, int splits)
{
    if (splits <= 1) return 0;
    return align_up((size_t)T * splits * Hq * d_v * sizeof(float)) +
           align_up((size_t)T * splits * Hq * sizeof(float));
}

size_t attn_workspace(int T, int Hq, int d_qk, int d_v, int k)
{
    return attn_split_workspace(T, Hq, d_v, attn_auto_splits(T, Hq, d_qk, d_v, k));
}

// ---------------------------------------------------------- argument checks

int check_rows(const int32_t* pos, const int32_t* k_base, int T, int S)
{
    if (T <= 0 || S <= 0) return fail(DSA_ERR_ARG, "T=%d and S=%d must be positive", T, S);
    if (!pos && T > S) return fail(DSA_ERR_ARG, "pos == NULL needs T <= S (T=%d, S=%d)", T, S);
    if ((pos && !al16(pos)) || (k_base && !al16(k_base)))
        return fail(DSA_ERR_ARG, "pos / k_base must be 16-byte aligned");
    return DSA_OK;
}

int check_indexer(const void* q_idx, const float* w, const void* k_idx, const int32_t* pos,
                  const int32_t* k_base, int T, int S, int H_I, int d_I, int k, const int32_t* idx)
{
    if (!q_idx || !w || !k_idx || !idx) return fail(DSA_ERR_ARG, "NULL q_idx, w, k_idx or idx");
    if (!al16(q_idx) || !al16(w) || !al16(k_idx) || !al16(idx))
        return fail(DSA_ERR_ARG, "q_idx, w, k_idx and idx must be 16-byte aligned");
    if (int rc = check_rows(pos, k_base, T, S)) return rc;
    if (H_I <= 0 || H_I > 16) return fail(DSA_ERR_UNSUPPORTED, "H_I=%d (supported: 1..16)", H_I);
    if (d_I != 32 && d_I != 64 && d_I != 128 && d_I != 256)
        return fail(DSA_ERR_UNSUPPORTED, "d_I=%d (supported: 32, 64, 128, 256)", d_I);
    if (k <= 0 || k > 4096) return fail(DSA_ERR_UNSUPPORTED, "k=%d (supported: 1..4096)", k);
    return DSA_OK;
}

int check_attn(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
               const int32_t* k_base, int T, int S, int Hq, int d_qk, int d_v, int k,
               const void* out, const float* lse)
{
    if (!q || !kv || !idx || !out || !lse) return fail(DSA_ERR_ARG, "NULL q, kv, idx, out or lse");
    if (!al16(q) || !al16(kv) || !al16(idx) || !al16(out) || !al16(lse))
        return fail(DSA_ERR_ARG, "q, kv, idx, out and lse must be 16-byte aligned");
    if (int rc = check_rows(pos, k_base, T, S)) return rc;
    if (Hq <= 0 || Hq > 1024) return fail(DSA_ERR_UNSUPPORTED, "Hq=%d (supported: 1..1024)", Hq);
    if (d_qk <= 0 || d_qk > 1024 || d_qk % 8)
        return fail(DSA_ERR_UNSUPPORTED, "d_qk=%d (supported: multiples of 8 up to 1024)", d_qk);
    if (d_v <= 0 || d_v > d_qk || d_v % 2)
        return fail(DSA_ERR_UNSUPPORTED, "d_v=%d (supported: even, <= d_qk)", d_v);
    if (k <= 0 || k > 4096) return fail(DSA_ERR_UNSUPPORTED, "k=%d (supported: 1..4096)", k);
    return DSA_OK;
}

// ----------------------------------------------------------------- indexer

template <int NT, int DI>
void launch_scores(dim3 grid, cudaStream_t st, const uint8_t* q_idx, const float* w,
                   const uint8_t* k_idx, const int* pos, const int* k_base, int T, int S, int H_I,
                   int row0, float* scores, long long ld, int keys_per_cta)
{
    dsa::indexer_scores_kernel<NT, DI><<<grid, dsa::kScoreThreads, 0, st>>>(
        q_idx, w, k_idx, pos, k_base, T, S, H_I, row0, scores, ld, keys_per_cta);
}

using ScoresFn = void (*)(dim3, cudaStream_t, const uint8_t*, const float*, const uint8_t*,
                          const int*, const int*, int, int, int, int, float*, long long, int);

ScoresFn pick_scores(int H_I, int d_I)
{
    const bool two = H_I > 8;
    switch (d_I) {
        case 32: return two ? launch_scores<2, 32> : launch_scores<1, 32>;
        case 64: return two ? launch_scores<2, 64> : launch_scores<1, 64>;
        case 128: return two ? launch_scores<2, 128> : launch_scores<1, 128>;
        default: return two ? launch_scores<2, 256> : launch_scores<1, 256>;
    }
}

int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows);

struct ChunkArgs {
    const uint8_t* q_idx;
    const float* w;
    const uint8_t* k_idx;
    const int* pos;
    const int* k_base;
    int T, S, H_I, k, row0, rows;
    const int* work_off;
    dsa::PagedRows pg;
};

template <int NT, int DI>
struct ChunkKernels {
    // plan + sampled scores + threshold in one launch
    static void sample_tau(cudaStream_t st, const ChunkArgs& a, int* work_off, float* samp, long long samp_ld,
                           uint32_t* tau)
    {
        using namespace dsa::idx_chunk;
        launch_pdl(chunk_sample_tau_kernel<NT, DI>, dim3(a.rows), dim3(kFusedTauThreads), 0, st, a.q_idx, a.w,
                   a.k_idx, a.pos, a.k_base, a.T, a.S, a.H_I, a.row0, a.rows, a.k, work_off, samp, samp_ld, tau,
                   a.pg);
    }
    static void topk(int grid, cudaStream_t st, const ChunkArgs& a, const uint32_t* tau, uint2* cand,
                     long long cand_ld, int* ccnt, int max_chunks, int32_t* idx)
    {
        using namespace dsa::idx_chunk;
        cudaFuncSetAttribute(chunk_topk_kernel<NT, DI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
        launch_pdl(chunk_topk_kernel<NT, DI>, dim3(grid), dim3(kThreads), kSmemBytes, st, a.q_idx, a.w, a.k_idx,
                   a.pos, a.k_base, a.T, a.S, a.H_I, a.row0, a.rows, a.k, a.work_off, tau, cand, cand_ld, ccnt,
                   max_chunks, idx);
    }
};

// d_I = 128: key rows streamed by TMA (tm_k over k_idx, 128-key boxes)
template <int NT>
void chunk_topk_tma(int grid, cudaStream_t st, const CUtensorMap& tm_k, const ChunkArgs& a,
                    const uint32_t* tau, uint2* cand, long long cand_ld, int* ccnt, int max_chunks,
                    int32_t* idx)
{
    using namespace dsa::idx_chunk;
    cudaFuncSetAttribute(chunk_topk_tma_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tma::kSmemBytes);
    launch_pdl(chunk_topk_tma_kernel<NT>, dim3(grid), dim3(tma::kThreads), tma::kSmemBytes, st, tm_k, a.q_idx,
               a.w, a.pos, a.k_base, a.T, a.S, a.H_I, a.row0, a.rows, a.k, a.work_off, tau, cand, cand_ld, ccnt,
               max_chunks, idx, a.pg);
}

// d_I = 128, few rows: the dense score rows (tm_k as for chunk_topk_tma)
template <int NT>
void row_scores_tma(int grid, cudaStream_t st, const CUtensorMap& tm_k, const ChunkArgs& a, float* scores,
                    long long ld, uint32_t* g16, long long g16_ld, uint32_t* g4, long long g4_ld)
{
    using namespace dsa::idx_chunk;
    cudaFuncSetAttribute(row_scores_tma_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         rs::kSmemBytes);
    launch_pdl(row_scores_tma_kernel<NT>, dim3(grid), dim3(rs::kThreads), rs::kSmemBytes, st, tm_k, a.q_idx,
               a.w, a.pos, a.k_base, a.T, a.S, a.H_I, a.row0, a.rows, a.k, scores, ld, g16, g16_ld, g4, g4_ld,
               a.pg);
}

struct ChunkFns {
    void (*row_scores)(int, cudaStream_t, const CUtensorMap&, const ChunkArgs&, float*, long long, uint32_t*,
                       long long, uint32_t*, long long);
    void (*sample_tau)(cudaStream_t, const ChunkArgs&, int*, float*, long long, uint32_t*);
    void (*topk)(int, cudaStream_t, const ChunkArgs&, const uint32_t*, uint2*, long long, int*, int,
                 int32_t*);
    void (*topk_tma)(int, cudaStream_t, const CUtensorMap&, const ChunkArgs&, const uint32_t*, uint2*,
                     long long, int*, int, int32_t*);
};

template <int NT, int DI>
ChunkFns chunk_fns()
{
    return {DI == 128 ? row_scores_tma<NT> : nullptr, ChunkKernels<NT, DI>::sample_tau,
            ChunkKernels<NT, DI>::topk, DI == 128 ? chunk_topk_tma<NT> : nullptr};
}

ChunkFns pick_chunk(int H_I, int d_I)
{
    const bool two = H_I > 8;
    switch (d_I) {
        case 32: return two ? chunk_fns<2, 32>() : chunk_fns<1, 32>();
        case 64: return two ? chunk_fns<2, 64>() : chunk_fns<1, 64>();
        case 128: return two ? chunk_fns<2, 128>() : chunk_fns<1, 128>();
        default: return two ? chunk_fns<2, 256>() : chunk_fns<1, 256>();
    }
}

// Rows with their own key ranges (indexer_chunked.cuh): chunk scores and
// sampled thresholds, chunk filters, and the merge of the chunks' pairs (with
// the exact fallback for a row the threshold left short).
// S: the most keys a row can have; a paged cache (pg.block_table) holds
// pg.num_pages * pg.page_size key rows.
int indexer_chunked(const uint8_t* q_idx, const float* w, const uint8_t* k_idx, const int32_t* pos,
                    const int32_t* k_base, int T, int S, int H_I, int d_I, int k, int32_t* idx,
                    void* workspace, cudaStream_t st, const dsa::PagedRows& pg = {})
{
    using namespace dsa::idx_chunk;
    const ChunkPlan p = chunk_plan(T, S, k);
    if (p.max_chunks > kMaxChunksPerRow)
        return fail(DSA_ERR_UNSUPPORTED, "S=%d: at most %d keys per row on this path", S,
                    kMaxChunksPerRow * kChunkKeys);
    char* ws = reinterpret_cast<char*>(workspace);
    int* work_off = reinterpret_cast<int*>(ws + p.off_work);
    uint32_t* tau = reinterpret_cast<uint32_t*>(ws + p.off_tau);
    int* ccnt = reinterpret_cast<int*>(ws + p.off_ccnt);
    float* samp = reinterpret_cast<float*>(ws + p.off_samp);
    uint2* cand = reinterpret_cast<uint2*>(ws + p.off_cand);
    const ChunkFns fn = pick_chunk(H_I, d_I);
    const bool paged = pg.block_table != nullptr;
    if (paged && !fn.topk_tma)
        return fail(DSA_ERR_UNSUPPORTED, "a paged key cache needs d_I = 128 (got %d)", d_I);
    CUtensorMap tm_k;
    if (fn.topk_tma) {
        const uint64_t key_rows = paged ? (uint64_t)pg.num_pages * pg.page_size : (uint64_t)S;
        if (int rc = make_tmap_u8(&tm_k, k_idx, 128, key_rows, paged ? tma::kTileKeys / 2 : tma::kTileKeys))
            return rc;
    }
    if (fn.row_scores && use_row_scores(T, S, d_I)) {
        // every key into a dense score row, then a cluster per row
        // thresholds, filters and selects
        const RowScorePlan q = row_score_plan(T, S);
        float* scores = reinterpret_cast<float*>(ws);
        uint32_t* g16 = reinterpret_cast<uint32_t*>(ws + q.off_g16);
        uint32_t* g4 = reinterpret_cast<uint32_t*>(ws + q.off_g4);
        cudaError_t e = cudaFuncSetAttribute(row_select_cluster_kernel<rs::kCsThreads>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, rs::kCsSmem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(row select kernels)");
        for (int row0 = 0; row0 < T; row0 += q.RB) {
            const int rows = std::min(q.RB, T - row0);
            const ChunkArgs a{q_idx, w, k_idx, pos, k_base, T, S, H_I, k, row0, rows, nullptr, pg};
            PhaseMark ph = phase_begin(kPhaseScores, st);
            fn.row_scores(rs::kCtasPerSm * num_sms(), st, tm_k, a, scores, q.ld, g16, q.g16_ld, g4, q.g4_ld);
            DSA_LAUNCH_CHECK("row_scores_tma_kernel");
            phase_end(ph);
            ph = phase_begin(kPhaseSelect, st);
            launch_pdl(row_select_cluster_kernel<rs::kCsThreads>, dim3(rs::kClusterCtas * rows),
                       dim3(rs::kCsThreads), rs::kCsSmem, st, scores, q.ld, g16, q.g16_ld, g4, q.g4_ld, q_idx, w,
                       k_idx, H_I, d_I, pos, k_base, T, S, row0, k, idx, pg);
            DSA_LAUNCH_CHECK("row_select_cluster_kernel");
            phase_end(ph);
        }
        return DSA_OK;
    }
    const int resident = (fn.topk_tma ? tma::kCtasPerSm : kCtasPerSm) * num_sms();
    auto topk = [&](const ChunkArgs& a, int grid, const uint32_t* tk) {
        if (fn.topk_tma)
            fn.topk_tma(grid, st, tm_k, a, tk, cand, p.cand_ld, ccnt, p.max_chunks, idx);
        else
            fn.topk(grid, st, a, tk, cand, p.cand_ld, ccnt, p.max_chunks, idx);
    };
    const size_t merge_smem = (size_t)((p.max_chunks + 2) & ~1) * sizeof(int) +
                              (size_t)kMergeSmemPairs * sizeof(uint2);
    {
        cudaError_t e = cudaFuncSetAttribute(merge_topk_kernel<kMergeThreads>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)merge_smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(merge_topk_kernel)");
    }
    for (int row0 = 0; row0 < T; row0 += p.RB) {
        const int rows = std::min(p.RB, T - row0);
        const int n_max = pos ? S : std::min(S, row0 + rows + S - T);
        const bool multi = n_max > kChunkKeys;
        const int grid = (int)std::min<long long>(
            (long long)rows * std::max(1, dsa::ceil_div(n_max, kChunkKeys)), resident);
        const ChunkArgs a{q_idx, w, k_idx, pos, k_base, T, S, H_I, k, row0, rows, work_off, pg};
        PhaseMark ph = phase_begin(kPhaseThreshold, st);
        if (multi) {
            // plan, sampled scores and threshold in one launch
            fn.sample_tau(st, a, work_off, samp, p.samp_ld, tau);
            DSA_LAUNCH_CHECK("chunk_sample_tau_kernel");
        } else {
            launch_pdl(chunk_plan_kernel, dim3(1), dim3(kPlanThreads), 0, st, pos, k_base, T, S, row0, rows,
                       work_off, pg);
            DSA_LAUNCH_CHECK("chunk_plan_kernel");
        }
        phase_end(ph);
        ph = phase_begin(kPhaseScores, st);
        topk(a, grid, multi ? tau : nullptr);
        DSA_LAUNCH_CHECK("chunk_topk_kernel");
        phase_end(ph);
        if (!multi) continue;
        ph = phase_begin(kPhaseSelect, st);
        launch_pdl(merge_topk_kernel<kMergeThreads>, dim3(rows), dim3(kMergeThreads), merge_smem, st, cand,
                   p.cand_ld, ccnt, p.max_chunks, q_idx, w, k_idx, H_I, d_I, pos, k_base, T, S, row0, k, idx, pg);
        DSA_LAUNCH_CHECK("merge_topk_kernel");
        phase_end(ph);
    }
    return DSA_OK;
}

// Shared memory the streaming indexer's threshold and select kernels stage a
// row in (its samples, its candidates).
constexpr size_t kFusedStageMax = 200 * 1024;

// One causal sequence (pos and k_base NULL), H_I = 8, d_I = 128, and a row's
// samples and candidates fit the select kernels' shared memory: streamed FP8
// tensor-core scan with sampled thresholds (indexer_tc.cuh).
bool indexer_fused_supported(const int32_t* pos, const int32_t* k_base, int H_I, int d_I, int S, int k)
{
    using namespace dsa::idx_tc;
    if (pos || k_base || H_I != kHI || d_I != kDI) return false;
    const size_t samp_bytes = (size_t)((num_tiles(S) + kSampleStride - 1) / kSampleStride) * kKeys * sizeof(float);
    const size_t bitmap_bytes = (size_t)std::max((S + 31) / 32, dsa::pow2_ceil(k)) * sizeof(uint32_t);
    return samp_bytes <= kFusedStageMax && bitmap_bytes <= kFusedStageMax;
}

int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                 uint32_t box_rows)
{
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)row_bytes, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const CUresult r = enc(
        m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return DSA_OK;
}

int indexer_fused(const uint8_t* q_idx, const float* w, const uint8_t* k_idx, int T, int S, int k,
                  int32_t* idx, void* workspace, cudaStream_t st)
{
    using namespace dsa::idx_tc;
    const FusedPlan p = fused_plan(T, S, k);
    char* ws = reinterpret_cast<char*>(workspace);
    float* samp = reinterpret_cast<float*>(ws + p.off_samp);
    float* tau = reinterpret_cast<float*>(ws + p.off_tau);
    uint2* cand = reinterpret_cast<uint2*>(ws + p.off_cand);
    int* cnt = reinterpret_cast<int*>(ws + p.off_cnt);
    CUtensorMap tq, tk;
    if (int rc = make_tmap_u8(&tq, q_idx, kDI, (uint64_t)T * kHI, kN)) return rc;
    if (int rc = make_tmap_u8(&tk, k_idx, kDI, (uint64_t)S, kKeys)) return rc;
    for (auto* f : {indexer_scan_kernel<true>, indexer_scan_kernel<false>}) {
        cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(indexer_scan_kernel)");
    }
    // staged samples (tau) and candidates (select) of one row
    const size_t tau_smem = (size_t)p.samp_ld * sizeof(float);
    // select: a bitmap over the row's keys (S bits), at least pow2_ceil(k)
    // ints for the sort a longer row falls back to
    const int bitmap_words = std::max((S + 31) / 32, dsa::pow2_ceil(k));
    const size_t sel_smem = (size_t)bitmap_words * sizeof(uint32_t);
    {
        cudaError_t e = cudaFuncSetAttribute(indexer_tau_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)tau_smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(indexer_select_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sel_smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(indexer_tau/select_kernel)");
    }
    for (int row0 = 0; row0 < T; row0 += p.RB) {
        const int rows = std::min(p.RB, T - row0);
        ScanArgs a{w, T, S, k, row0, rows, samp, p.samp_ld, tau, cand, cnt, p.cap};
        const int ctas = (rows + kRows - 1) / kRows;
        PhaseMark ph = phase_begin(kPhaseScores, st);
        indexer_scan_kernel<true><<<ctas, kThreads, kSmemBytes, st>>>(tq, tk, a);
        DSA_LAUNCH_CHECK("indexer_scan_kernel<sample>");
        phase_end(ph);
        ph = phase_begin(kPhaseThreshold, st);
        indexer_tau_kernel<256><<<rows, 256, tau_smem, st>>>(samp, p.samp_ld, T, S, k, row0, tau);
        DSA_LAUNCH_CHECK("indexer_tau_kernel");
        phase_end(ph);
        ph = phase_begin(kPhaseScores, st);
        indexer_scan_kernel<false><<<ctas, kThreads, kSmemBytes, st>>>(tq, tk, a);
        DSA_LAUNCH_CHECK("indexer_scan_kernel<filter>");
        phase_end(ph);
        // ~2k candidates per row: 256 threads keep the radix passes busy
        ph = phase_begin(kPhaseSelect, st);
        indexer_select_kernel<256><<<rows, 256, sel_smem, st>>>(cand, cnt, p.cap, q_idx, w, k_idx, T, S, k,
                                                                row0, idx, bitmap_words);
        DSA_LAUNCH_CHECK("indexer_select_kernel");
        phase_end(ph);
    }
    return DSA_OK;
}

// --------------------------------------------------------------- attention

int attn_simple(const __nv_bfloat16* q, const __nv_bfloat16* kv, const int32_t* idx,
                const int32_t* pos, const int32_t* k_base, int T, int S, int Hq, int d_qk,
                int d_v, int k, float scale, int splits, __nv_bfloat16* out, float* lse, void* workspace,
                cudaStream_t st)
{
    const int kcap = dsa::ceil_div(k, splits);
    const size_t smem = dsa::attn_simple_smem(d_qk, kcap);
    cudaError_t e = cudaFuncSetAttribute(dsa::sparse_attn_simple_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(sparse_attn_simple_kernel)");
    float* part_o = nullptr;
    float* part_lse = nullptr;
    if (splits > 1) {
        part_o = reinterpret_cast<float*>(workspace);
        part_lse = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                            align_up((size_t)T * splits * Hq * d_v * sizeof(float)));
    }
    dim3 grid(T, dsa::ceil_div(Hq, dsa::kAttnHeads), splits);
    dsa::sparse_attn_simple_kernel<<<grid, dsa::kAttnThreads, smem, st>>>(
        q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, kcap, scale, out, lse, part_o, part_lse);
    DSA_LAUNCH_CHECK("sparse_attn_simple_kernel");
    if (splits > 1) {
        dsa::lse_combine_kernel<<<dim3(T, Hq), 128, 0, st>>>(part_o, part_lse, T, Hq, d_v, splits,
                                                             out, lse);
        DSA_LAUNCH_CHECK("lse_combine_kernel");
    }
    return DSA_OK;
}

// 2D bf16 tensor map over a row-major [rows, cols] matrix, box [box_rows, box_cols].
int make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                   uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const CUresult r = enc(
        m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return DSA_OK;
}

int attn_tc(const __nv_bfloat16* q, const __nv_bfloat16* kv, const int32_t* idx,
            const int32_t* pos, const int32_t* k_base, int T, int S, int k, float scale,
            __nv_bfloat16* out, float* lse, cudaStream_t st, const dsa::PagedRows& pg = {},
            int splits = 1, void* workspace = nullptr)
{
    using namespace dsa::attn_tc;
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_attn_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(sparse_mla_attn_tc_kernel)");
    // Q as [T*128, 576]: TMA boxes of 128 heads; 64 latent columns with 128B
    // swizzle, the 32 rope columns with 64B swizzle. Half of the latent slice
    // is written to TMEM by the kernel itself.
    CUtensorMap tq128, tq64;
    if (int rc = make_tmap_bf16(&tq128, q, kDqk, (uint64_t)T * kHeads, 64, kHeads,
                                CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
    if (int rc = make_tmap_bf16(&tq64, q, kDqk, (uint64_t)T * kHeads, 32, kHeads,
                                CU_TENSOR_MAP_SWIZZLE_64B)) return rc;
    const float scale_log2 = scale * 1.4426950408889634f;
    float* part_o = nullptr;
    float* part_lse = nullptr;
    if (splits > 1) {
        part_o = reinterpret_cast<float*>(workspace);
        part_lse = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                            align_up((size_t)T * splits * kHeads * kDv * sizeof(float)));
    }
    // persistent: one cluster per SM pair, each walking units cid, cid + clusters, ...
    const int clusters = (int)std::min<long long>((long long)T * splits, std::max(1, num_sms() / 2));
    launch_pdl(sparse_mla_attn_tc_kernel, dim3(2 * clusters), dim3(kThreads), kSmemBytes, st, tq128, tq64, q,
               kv, idx, pos, k_base, T, S, k, scale_log2, out, lse, pg, splits, part_o, part_lse);
    DSA_LAUNCH_CHECK("sparse_mla_attn_tc_kernel");
    if (splits > 1) {
        launch_pdl(lse_merge_kernel, dim3(T, kHeads / kMergeHeads), dim3(128), 0, st, part_o, part_lse, T, splits,
                   out, lse);
        DSA_LAUNCH_CHECK("lse_merge_kernel");
    }
    return DSA_OK;
}

// Sparse attention with `splits` parts per row (0: the library's choice).
int attn_dispatch(const void* q, const void* kv, const int32_t* idx, const int32_t* pos, const int32_t* k_base,
                  int T, int S, int Hq, int d_qk, int d_v, int k, float scale, int splits, void* out, float* lse,
                  void* workspace, size_t ws_bytes, void* stream)
{
    using bf = __nv_bfloat16;
    if (splits < 0 || splits > dsa::attn_tc::kMaxSplits)
        return fail(DSA_ERR_ARG, "splits=%d (supported: 0..%d)", splits, dsa::attn_tc::kMaxSplits);
    if (splits == 0) splits = attn_auto_splits(T, Hq, d_qk, d_v, k);
    const size_t need = attn_split_workspace(T, Hq, d_v, splits);
    if (need && (!workspace || ws_bytes < need || !al16(workspace)))
        return fail(DSA_ERR_WORKSPACE, "attention with %d parts per row needs %zu workspace bytes (got %zu)",
                    splits, need, ws_bytes);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (int rc = debug_check(idx, pos, k_base, T, S, k, {}, false, st)) return rc;
    if (attn_tc_supported(Hq, d_qk, d_v, k)) {
        if ((long long)T * splits > 0x3FFFFFFF)
            return fail(DSA_ERR_UNSUPPORTED, "T * splits = %lld clusters", (long long)T * splits);
        return attn_tc(reinterpret_cast<const bf*>(q), reinterpret_cast<const bf*>(kv), idx, pos, k_base, T, S,
                       k, scale, reinterpret_cast<bf*>(out), lse, st, {}, splits, workspace);
    }
    return attn_simple(reinterpret_cast<const bf*>(q), reinterpret_cast<const bf*>(kv), idx, pos, k_base, T, S,
                       Hq, d_qk, d_v, k, scale, splits, reinterpret_cast<bf*>(out), lse, workspace, st);
}

// ---------------------------------------------------------- attention backward

constexpr int kBwdRowsMax = 8192;   // query rows per pass of the backward (workspace size)

// Per row of a pass: g (bf16 [heads_pad][slots_pad]) and D (fp32 [heads_pad]).
size_t attn_bwd_row_bytes(int Hq, int k)
{
    return (size_t)dsa::bwd::heads_pad(Hq) * (dsa::bwd::slots_pad(k) * sizeof(__nv_bfloat16) + sizeof(float));
}

int check_attn_bwd(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
                   const int32_t* k_base, const void* out, const float* lse, const void* dout, int T,
                   int S, int Hq, int d_qk, int d_v, int k, const float* dq, const float* dkv)
{
    if (int rc = check_attn(q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, out, lse)) return rc;
    if (!dout || !dq || !dkv) return fail(DSA_ERR_ARG, "NULL dout, dq or dkv");
    if (!al16(dout) || !al16(dq) || !al16(dkv))
        return fail(DSA_ERR_ARG, "dout, dq and dkv must be 16-byte aligned");
    if (Hq > dsa::bwd::kMaxHeads)
        return fail(DSA_ERR_UNSUPPORTED, "Hq=%d (backward supports 1..%d)", Hq, dsa::bwd::kMaxHeads);
    if (d_qk % 16 || d_qk > dsa::bwd::kMaxDqk || d_v % 16)
        return fail(DSA_ERR_UNSUPPORTED, "d_qk=%d, d_v=%d (backward: multiples of 16, d_qk <= %d)", d_qk,
                    d_v, dsa::bwd::kMaxDqk);
    return DSA_OK;
}

int attn_bwd(const __nv_bfloat16* q, const __nv_bfloat16* kv, const int32_t* idx, const int32_t* pos,
             const int32_t* k_base, const __nv_bfloat16* out, const float* lse,
             const __nv_bfloat16* dout, int T, int S, int Hq, int d_qk, int d_v, int k, float scale,
             float* dq, float* dkv, void* workspace, size_t ws_bytes, cudaStream_t st)
{
    using namespace dsa::bwd;
    const size_t row_bytes = attn_bwd_row_bytes(Hq, k);
    const size_t fit = workspace && al16(workspace) ? ws_bytes / row_bytes : 0;
    if (fit < 1)
        return fail(DSA_ERR_WORKSPACE, "attention backward needs %zu workspace bytes per row (got %zu)",
                    row_bytes, ws_bytes);
    const int rows = (int)std::min<size_t>(std::min<size_t>(fit, (size_t)T), 65535);
    const size_t s_dkv = dkv_smem(Hq, d_qk), s_dq = dq_smem(Hq);
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)s_dkv);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_bwd_dkv_kernel)");
    e = cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_dq);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_bwd_dq_kernel)");
    __nv_bfloat16* g_ws = reinterpret_cast<__nv_bfloat16*>(workspace);
    // D per row after the pass's g rows (16-byte aligned: heads_pad * slots_pad * 2 is)
    float* d_ws = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                           (size_t)rows * heads_pad(Hq) * slots_pad(k) * sizeof(__nv_bfloat16));
    // the MLA head shape runs the dkv part on the tensor-core kernel
    const bool tc = Hq == dsa::bwd_tc::kHeads && d_qk == dsa::bwd_tc::kDqk && d_v == dsa::bwd_tc::kDv;
    CUtensorMap tq, tdo, tg;
    if (tc) {
        e = cudaFuncSetAttribute(dsa::bwd_tc::attn_bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::bwd_tc::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_bwd_dkv_tc_kernel)");
        if (int rc = make_tmap_bf16(&tq, q, d_qk, (uint64_t)T * Hq, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
        if (int rc = make_tmap_bf16(&tdo, dout, d_v, (uint64_t)T * Hq, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
            return rc;
        // g_ws as [rows * 128, kp]: boxes of 64 slots x 128 heads
        if (int rc = make_tmap_bf16(&tg, g_ws, slots_pad(k), (uint64_t)rows * Hq, 64, 128,
                                    CU_TENSOR_MAP_SWIZZLE_128B))
            return rc;
        e = cudaFuncSetAttribute(dsa::bwd_tc::attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::bwd_tc::kDqSmem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_bwd_dq_tc_kernel)");
    }
    for (int r0 = 0; r0 < T; r0 += rows) {
        const int n = std::min(rows, T - r0);
        if (tc) {
            dsa::bwd_tc::attn_bwd_delta_kernel<<<n, 256, 0, st>>>(out, dout, r0, d_ws);
            DSA_LAUNCH_CHECK("attn_bwd_delta_kernel");
            dsa::bwd_tc::attn_bwd_dkv_tc_kernel<<<dim3(slots_pad(k) / kSlots, n), dsa::bwd_tc::kThreads,
                                                  dsa::bwd_tc::kSmemBytes, st>>>(
                tq, tdo, kv, idx, pos, k_base, out, lse, dout, r0, T, S, k, slots_pad(k), scale, dkv, g_ws, d_ws);
            DSA_LAUNCH_CHECK("attn_bwd_dkv_tc_kernel");
        } else {
            attn_bwd_dkv_kernel<<<dim3(slots_pad(k) / kSlots, n), kThreads, s_dkv, st>>>(
                q, kv, idx, pos, k_base, out, lse, dout, r0, T, S, Hq, d_qk, d_v, k, scale, dkv, g_ws);
            DSA_LAUNCH_CHECK("attn_bwd_dkv_kernel");
        }
        if (tc) {
            dsa::bwd_tc::attn_bwd_dq_tc_kernel<<<dim3(d_qk / dsa::bwd_tc::kDqCols, n), dsa::bwd_tc::kDqThreads,
                                                 dsa::bwd_tc::kDqSmem, st>>>(tg, kv, idx, pos, k_base, r0, T, S, k,
                                                                             dq);
            DSA_LAUNCH_CHECK("attn_bwd_dq_tc_kernel");
        } else {
            attn_bwd_dq_kernel<<<dim3(dsa::ceil_div(d_qk, kCols), n), kThreads, s_dq, st>>>(
                kv, idx, pos, k_base, g_ws, r0, T, S, Hq, d_qk, k, dq);
            DSA_LAUNCH_CHECK("attn_bwd_dq_kernel");
        }
    }
    return DSA_OK;
}

// ------------------------------------------------------------ indexer KL loss

constexpr int kKlRowsMax = 8192;   // query rows per pass (workspace size)

size_t kl_row_bytes(int k) { return (size_t)dsa::bwd::slots_pad(k) * sizeof(float); }

int check_kl(const void* q, const void* kv, const int32_t* idx, const int32_t* pos, const int32_t* k_base,
             const float* lse, const void* q_idx, const float* w, const void* k_idx, int T, int S, int Hq,
             int d_qk, int H_I, int d_I, int k, const float* loss, const float* dw, const float* dqi,
             const float* dki)
{
    if (!q || !kv || !idx || !lse || !q_idx || !w || !k_idx || !loss || !dw || !dqi || !dki)
        return fail(DSA_ERR_ARG, "NULL argument");
    if (!al16(q) || !al16(kv) || !al16(idx) || !al16(lse) || !al16(q_idx) || !al16(w) || !al16(k_idx) ||
        !al16(loss) || !al16(dw) || !al16(dqi) || !al16(dki))
        return fail(DSA_ERR_ARG, "every array must be 16-byte aligned");
    if (int rc = check_rows(pos, k_base, T, S)) return rc;
    if (Hq <= 0 || Hq > dsa::bwd::kMaxHeads || d_qk <= 0 || d_qk % 16 || d_qk > dsa::bwd::kMaxDqk)
        return fail(DSA_ERR_UNSUPPORTED, "Hq=%d, d_qk=%d (supported: Hq <= 128, d_qk a multiple of 16 <= 576)",
                    Hq, d_qk);
    if (H_I <= 0 || H_I > dsa::kl::kMaxHI || d_I <= 0 || d_I % 16 || d_I > dsa::kl::kMaxDI ||
        H_I * d_I > dsa::kl::kMaxQElems)
        return fail(DSA_ERR_UNSUPPORTED, "H_I=%d, d_I=%d (supported: H_I <= 16, d_I a multiple of 16 <= 256, "
                    "H_I * d_I <= 4096)", H_I, d_I);
    if (k <= 0 || k > 4096) return fail(DSA_ERR_UNSUPPORTED, "k=%d (supported: 1..4096)", k);
    return DSA_OK;
}

int indexer_kl(const __nv_bfloat16* q, const __nv_bfloat16* kv, const int32_t* idx, const int32_t* pos,
               const int32_t* k_base, const float* lse, const uint8_t* q_idx, const float* w,
               const uint8_t* k_idx, int T, int S, int Hq, int d_qk, int H_I, int d_I, int k, float scale,
               float* loss, float* dw, float* dqi, float* dki, void* workspace, size_t ws_bytes, cudaStream_t st)
{
    using namespace dsa::kl;
    const size_t row_bytes = kl_row_bytes(k);
    const size_t fit = workspace && al16(workspace) ? ws_bytes / row_bytes : 0;
    if (fit < 1)
        return fail(DSA_ERR_WORKSPACE, "indexer KL loss needs %zu workspace bytes per row (got %zu)", row_bytes,
                    ws_bytes);
    const int rows = (int)std::min<size_t>(std::min<size_t>(fit, (size_t)T), 65535);
    const size_t s_prob = prob_smem(Hq, d_qk), s_row = row_smem(H_I, d_I, k);
    cudaError_t e = cudaFuncSetAttribute(head_prob_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)s_prob);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(head_prob_sum_kernel)");
    e = cudaFuncSetAttribute(indexer_kl_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_row);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(indexer_kl_row_kernel)");
    float* psum = reinterpret_cast<float*>(workspace);
    // the MLA head shape forms the head-summed probabilities on the tensor cores
    const bool tc = Hq == dsa::bwd_tc::kHeads && d_qk == dsa::bwd_tc::kDqk;
    CUtensorMap tq;
    if (tc) {
        e = cudaFuncSetAttribute(dsa::bwd_tc::head_prob_sum_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::bwd_tc::kPsSmem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(head_prob_sum_tc_kernel)");
        if (int rc = make_tmap_bf16(&tq, q, d_qk, (uint64_t)T * Hq, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
    }
    for (int r0 = 0; r0 < T; r0 += rows) {
        const int n = std::min(rows, T - r0);
        if (tc) {
            dsa::bwd_tc::head_prob_sum_tc_kernel<<<dim3(dsa::bwd::slots_pad(k) / dsa::bwd::kSlots, n),
                                                   dsa::bwd_tc::kThreads, dsa::bwd_tc::kPsSmem, st>>>(
                tq, kv, idx, pos, k_base, lse, r0, T, S, k, dsa::bwd::slots_pad(k), scale, psum);
            DSA_LAUNCH_CHECK("head_prob_sum_tc_kernel");
        } else {
            head_prob_sum_kernel<<<dim3(dsa::bwd::slots_pad(k) / dsa::bwd::kSlots, n), dsa::bwd::kThreads, s_prob,
                                   st>>>(q, kv, idx, pos, k_base, lse, r0, T, S, Hq, d_qk, k, scale, psum);
            DSA_LAUNCH_CHECK("head_prob_sum_kernel");
        }
        indexer_kl_row_kernel<<<n, kRowThreads, s_row, st>>>(q_idx, w, k_idx, idx, pos, k_base, psum, r0, T, S,
                                                             H_I, d_I, k, loss, dw, dqi, dki);
        DSA_LAUNCH_CHECK("indexer_kl_row_kernel");
    }
    return DSA_OK;
}

// ------------------------------------------------------------- MLA MHA mode

template <int DH, int DV>
int mha_launch(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int T, int S, int Hq,
               float scale, __nv_bfloat16* out, float* lse, cudaStream_t st)
{
    using namespace dsa::mha;
    auto kern = mha_causal_kernel<DH, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Shape<DH, DV>::kSmem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(mha_causal_kernel)");
    kern<<<dim3(dsa::ceil_div(T, kRows), Hq), kThreads, Shape<DH, DV>::kSmem, st>>>(q, k, v, T, S, Hq, scale,
                                                                                   out, lse);
    DSA_LAUNCH_CHECK("mha_causal_kernel");
    return DSA_OK;
}

}  // namespace

// ===================================================================== C ABI

extern "C" {

int dsa_abi_version(void) { return 1; }

int dsa_selftest_bounded_wait(int limit_ms, void* stream)
{
    g_err[0] = 0;
    if (limit_ms < 1 || limit_ms > 2000) return fail(DSA_ERR_ARG, "limit_ms=%d (1..2000)", limit_ms);
    dsa::bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (uint64_t)limit_ms * 1000000ull);
    DSA_LAUNCH_CHECK("bounded_wait_selftest_kernel");
    return DSA_OK;
}

uint64_t dsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* dsa_last_error(void) { return g_err; }

size_t dsa_workspace_size(int T, int S, int H_I, int d_I, int k, int Hq, int d_qk, int d_v)
{
    if (T <= 0 || S <= 0 || k <= 0 || Hq <= 0 || d_v <= 0) return 0;
    return std::max(indexer_workspace(T, S, k, H_I, d_I), attn_workspace(T, Hq, d_qk, d_v, k));
}

int dsa_indexer_topk(const void* q_idx, const float* w, const void* k_idx, const int32_t* pos,
                     const int32_t* k_base, int T, int S, int H_I, int d_I, int k, int32_t* idx,
                     void* workspace, size_t ws_bytes, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_indexer(q_idx, w, k_idx, pos, k_base, T, S, H_I, d_I, k, idx)) return rc;
    const size_t need = indexer_workspace(T, S, k, H_I, d_I);
    if (need && (!workspace || ws_bytes < need || !al16(workspace)))
        return fail(DSA_ERR_WORKSPACE, "indexer needs %zu workspace bytes (got %zu)", need, ws_bytes);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int rc = indexer_fused_supported(pos, k_base, H_I, d_I, S, k)
                       ? indexer_fused(reinterpret_cast<const uint8_t*>(q_idx), w,
                                       reinterpret_cast<const uint8_t*>(k_idx), T, S, k, idx, workspace, st)
                       : indexer_chunked(reinterpret_cast<const uint8_t*>(q_idx), w,
                                         reinterpret_cast<const uint8_t*>(k_idx), pos, k_base, T, S, H_I, d_I, k,
                                         idx, workspace, st);
    if (rc) return rc;
    return debug_check(idx, pos, k_base, T, S, k, {}, true, st);
}

int dsa_indexer_topk_varlen(const void* q_idx, const float* w, const void* k_idx, const int32_t* cu_q,
                            const int32_t* cu_k, int n_seqs, int H_I, int d_I, int k, int32_t* idx,
                            void* workspace, size_t ws_bytes, void* stream)
{
    g_err[0] = 0;
    if (!cu_q || !cu_k || n_seqs <= 0) return fail(DSA_ERR_ARG, "cu_q, cu_k NULL or n_seqs=%d", n_seqs);
    if (cu_q[0] != 0 || cu_k[0] != 0) return fail(DSA_ERR_ARG, "cu_q[0] and cu_k[0] must be 0");
    size_t need = 0;
    for (int b = 0; b < n_seqs; ++b) {
        const int Tb = cu_q[b + 1] - cu_q[b], Sb = cu_k[b + 1] - cu_k[b];
        if (Tb < 0 || Sb < 0 || Tb > Sb)
            return fail(DSA_ERR_ARG, "sequence %d: %d query rows over %d keys (need 0 <= T <= S)", b, Tb, Sb);
        if (Tb > 0) need = std::max(need, indexer_workspace(Tb, Sb, k, H_I, d_I));
    }
    const int T = cu_q[n_seqs], S = cu_k[n_seqs];
    if (int rc = check_indexer(q_idx, w, k_idx, nullptr, nullptr, T, S, H_I, d_I, k, idx)) return rc;
    if (need && (!workspace || ws_bytes < need || !al16(workspace)))
        return fail(DSA_ERR_WORKSPACE, "indexer needs %zu workspace bytes (got %zu)", need, ws_bytes);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint8_t* q8 = reinterpret_cast<const uint8_t*>(q_idx);
    const uint8_t* k8 = reinterpret_cast<const uint8_t*>(k_idx);
    for (int b = 0; b < n_seqs; ++b) {
        const int Tb = cu_q[b + 1] - cu_q[b], Sb = cu_k[b + 1] - cu_k[b];
        if (Tb == 0) continue;
        const uint8_t* qb = q8 + (size_t)cu_q[b] * H_I * d_I;
        const float* wb = w + (size_t)cu_q[b] * H_I;
        const uint8_t* kb = k8 + (size_t)cu_k[b] * d_I;
        int32_t* ib = idx + (size_t)cu_q[b] * k;
        if (!al16(qb) || !al16(wb) || !al16(kb) || !al16(ib))
            return fail(DSA_ERR_ARG, "sequence %d: its rows of q_idx, w, k_idx or idx are not 16-byte "
                                     "aligned (cu_q[b] * H_I * 4 and cu_q[b] * k * 4 must be multiples "
                                     "of 16)", b);
        const int rc = indexer_fused_supported(nullptr, nullptr, H_I, d_I, Sb, k)
                           ? indexer_fused(qb, wb, kb, Tb, Sb, k, ib, workspace, st)
                           : indexer_chunked(qb, wb, kb, nullptr, nullptr, Tb, Sb, H_I, d_I, k, ib,
                                             workspace, st);
        if (rc) return rc;
        if (int rc2 = debug_check(ib, nullptr, nullptr, Tb, Sb, k, {}, true, st)) return rc2;
    }
    return DSA_OK;
}

namespace {
int check_paged(const void* cache, int num_pages, int page_size, const int32_t* block_table, int n_seqs,
                int max_pages, const int32_t* seq, const int32_t* pos, int T)
{
    if (!cache || !block_table || !seq || !pos) return fail(DSA_ERR_ARG, "NULL cache, block_table, seq or pos");
    if (!al16(cache) || !al16(block_table) || !al16(seq) || !al16(pos))
        return fail(DSA_ERR_ARG, "cache, block_table, seq and pos must be 16-byte aligned");
    if (T <= 0 || num_pages <= 0 || n_seqs <= 0 || max_pages <= 0)
        return fail(DSA_ERR_ARG, "T=%d, num_pages=%d, n_seqs=%d, max_pages=%d must be positive", T,
                    num_pages, n_seqs, max_pages);
    if (page_size <= 0 || page_size % 64 != 0)
        return fail(DSA_ERR_UNSUPPORTED, "page_size=%d (supported: multiples of 64)", page_size);
    if ((long long)num_pages * page_size > INT32_MAX || (long long)max_pages * page_size > INT32_MAX)
        return fail(DSA_ERR_UNSUPPORTED, "cache of more than 2^31 rows");
    return DSA_OK;
}
}  // namespace

int dsa_indexer_topk_paged(const void* q_idx, const float* w, const void* k_pages, int num_pages,
                           int page_size, const int32_t* block_table, int n_seqs, int max_pages,
                           const int32_t* seq, const int32_t* pos, int T, int H_I, int d_I, int k,
                           int32_t* idx, void* workspace, size_t ws_bytes, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_paged(k_pages, num_pages, page_size, block_table, n_seqs, max_pages, seq, pos, T))
        return rc;
    const int S = max_pages * page_size;   // the most keys a row can have
    if (int rc = check_indexer(q_idx, w, k_pages, pos, nullptr, T, S, H_I, d_I, k, idx)) return rc;
    if (d_I != 128) return fail(DSA_ERR_UNSUPPORTED, "a paged key cache needs d_I = 128 (got %d)", d_I);
    const size_t need = indexer_workspace(T, S, k, H_I, d_I);
    if (need && (!workspace || ws_bytes < need || !al16(workspace)))
        return fail(DSA_ERR_WORKSPACE, "indexer needs %zu workspace bytes (got %zu)", need, ws_bytes);
    dsa::PagedRows pg;
    pg.block_table = block_table;
    pg.seq = seq;
    pg.n_seqs = n_seqs;
    pg.max_pages = max_pages;
    pg.page_size = page_size;
    pg.num_pages = num_pages;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (int rc = indexer_chunked(reinterpret_cast<const uint8_t*>(q_idx), w,
                                 reinterpret_cast<const uint8_t*>(k_pages), pos, nullptr, T, S, H_I, d_I, k, idx,
                                 workspace, st, pg))
        return rc;
    return debug_check(idx, pos, nullptr, T, S, k, pg, true, st);
}

int dsa_sparse_mla_attn_paged(const void* q, const void* kv_pages, int num_pages, int page_size,
                              const int32_t* block_table, int n_seqs, int max_pages, const int32_t* seq,
                              const int32_t* pos, const int32_t* idx, int T, int Hq, int d_qk, int d_v,
                              int k, float scale, void* out, float* lse, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_paged(kv_pages, num_pages, page_size, block_table, n_seqs, max_pages, seq, pos, T))
        return rc;
    const int S = num_pages * page_size;
    if (int rc = check_attn(q, kv_pages, idx, pos, nullptr, T, S, Hq, d_qk, d_v, k, out, lse)) return rc;
    if (!attn_tc_supported(Hq, d_qk, d_v, k))
        return fail(DSA_ERR_UNSUPPORTED, "a paged latent cache needs Hq = 128, d_qk = 576, d_v = 512");
    dsa::PagedRows pg;
    pg.block_table = block_table;
    pg.seq = seq;
    pg.n_seqs = n_seqs;
    pg.max_pages = max_pages;
    pg.page_size = page_size;
    pg.num_pages = num_pages;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (int rc = debug_check(idx, pos, nullptr, T, S, k, pg, false, st)) return rc;
    return attn_tc(reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(kv_pages),
                   idx, pos, nullptr, T, S, k, scale, reinterpret_cast<__nv_bfloat16*>(out), lse, st, pg);
}

int dsa_sparse_mla_attn(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
                        const int32_t* k_base, int T, int S, int Hq, int d_qk, int d_v, int k,
                        float scale, void* out, float* lse, void* workspace, size_t ws_bytes,
                        void* stream)
{
    g_err[0] = 0;
    if (int rc = check_attn(q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, out, lse)) return rc;
    return attn_dispatch(q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, scale, 0, out, lse, workspace, ws_bytes,
                         stream);
}

size_t dsa_sparse_mla_attn_split_workspace_size(int T, int Hq, int d_v, int splits)
{
    if (T <= 0 || Hq <= 0 || d_v <= 0 || splits < 0) return 0;
    return attn_split_workspace(T, Hq, d_v, splits);
}

int dsa_sparse_mla_attn_split(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
                              const int32_t* k_base, int T, int S, int Hq, int d_qk, int d_v, int k, float scale,
                              int splits, void* out, float* lse, void* workspace, size_t ws_bytes, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_attn(q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, out, lse)) return rc;
    return attn_dispatch(q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, scale, splits, out, lse, workspace,
                         ws_bytes, stream);
}

size_t dsa_sparse_mla_attn_bwd_workspace_size(int T, int Hq, int k)
{
    if (T <= 0 || Hq <= 0 || k <= 0) return 0;
    return (size_t)std::min(T, kBwdRowsMax) * attn_bwd_row_bytes(Hq, k);
}

int dsa_sparse_mla_attn_bwd(const void* q, const void* kv, const int32_t* idx, const int32_t* pos,
                            const int32_t* k_base, const void* out, const float* lse, const void* dout,
                            int T, int S, int Hq, int d_qk, int d_v, int k, float scale, float* dq,
                            float* dkv, void* workspace, size_t ws_bytes, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_attn_bwd(q, kv, idx, pos, k_base, out, lse, dout, T, S, Hq, d_qk, d_v, k, dq, dkv))
        return rc;
    using bf = __nv_bfloat16;
    return attn_bwd(reinterpret_cast<const bf*>(q), reinterpret_cast<const bf*>(kv), idx, pos, k_base,
                    reinterpret_cast<const bf*>(out), lse, reinterpret_cast<const bf*>(dout), T, S, Hq,
                    d_qk, d_v, k, scale, dq, dkv, workspace, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_indexer_kl_workspace_size(int T, int k)
{
    if (T <= 0 || k <= 0) return 0;
    return (size_t)std::min(T, kKlRowsMax) * kl_row_bytes(k);
}

int dsa_indexer_kl(const void* q, const void* kv, const int32_t* idx, const int32_t* pos, const int32_t* k_base,
                   const float* lse, const void* q_idx, const float* w, const void* k_idx, int T, int S, int Hq,
                   int d_qk, int H_I, int d_I, int k, float scale, float* loss, float* dw, float* dq_idx,
                   float* dk_idx, void* workspace, size_t ws_bytes, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_kl(q, kv, idx, pos, k_base, lse, q_idx, w, k_idx, T, S, Hq, d_qk, H_I, d_I, k, loss, dw,
                          dq_idx, dk_idx))
        return rc;
    using bf = __nv_bfloat16;
    return indexer_kl(reinterpret_cast<const bf*>(q), reinterpret_cast<const bf*>(kv), idx, pos, k_base, lse,
                      reinterpret_cast<const uint8_t*>(q_idx), w, reinterpret_cast<const uint8_t*>(k_idx), T, S,
                      Hq, d_qk, H_I, d_I, k, scale, loss, dw, dq_idx, dk_idx, workspace, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

// MHA mode, (d_h, d_hv) = (192, 128), on the tensor cores: TMA maps over the
// head-interleaved rows of q, k and v.
int mha_tc_launch(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int T, int S, int Hq,
                  float scale, __nv_bfloat16* out, float* lse, cudaStream_t st)
{
    using namespace dsa::mha_tc;
    cudaError_t e = cudaFuncSetAttribute(mha_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(mha_tc_kernel)");
    CUtensorMap tq, tk, tv;
    if (int rc = make_tmap_bf16(&tq, q, (uint64_t)Hq * kDh, (uint64_t)T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return rc;
    if (int rc = make_tmap_bf16(&tk, k, (uint64_t)Hq * kDh, (uint64_t)S, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return rc;
    if (int rc = make_tmap_bf16(&tv, v, (uint64_t)Hq * kDv, (uint64_t)S, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return rc;
    // persistent: one CTA per SM walking the (query tile, head) units
    const int units = dsa::ceil_div(T, kRows) * Hq;
    mha_tc_kernel<<<std::min(units, num_sms()), kThreads, kSmemBytes, st>>>(
        tq, tk, tv, T, S, Hq, scale * 1.4426950408889634f, out, lse);
    DSA_LAUNCH_CHECK("mha_tc_kernel");
    return DSA_OK;
}

int dsa_mla_mha_attn(const void* q, const void* k, const void* v, int T, int S, int Hq, int d_h, int d_hv,
                     float scale, void* out, float* lse, void* stream)
{
    g_err[0] = 0;
    if (!q || !k || !v || !out || !lse) return fail(DSA_ERR_ARG, "NULL q, k, v, out or lse");
    if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || !al16(lse))
        return fail(DSA_ERR_ARG, "q, k, v, out and lse must be 16-byte aligned");
    if (T <= 0 || S <= 0 || T > S) return fail(DSA_ERR_ARG, "T=%d, S=%d (need 0 < T <= S)", T, S);
    if (Hq <= 0 || Hq > 65535) return fail(DSA_ERR_UNSUPPORTED, "Hq=%d (supported: 1..65535)", Hq);
    using bf = __nv_bfloat16;
    auto st = reinterpret_cast<cudaStream_t>(stream);
    const bf *qq = reinterpret_cast<const bf*>(q), *kk = reinterpret_cast<const bf*>(k),
             *vv = reinterpret_cast<const bf*>(v);
    bf* oo = reinterpret_cast<bf*>(out);
    if (d_h == 192 && d_hv == 128) return mha_tc_launch(qq, kk, vv, T, S, Hq, scale, oo, lse, st);
    if (d_h == 64 && d_hv == 64) return mha_launch<64, 64>(qq, kk, vv, T, S, Hq, scale, oo, lse, st);
    return fail(DSA_ERR_UNSUPPORTED, "d_h=%d, d_hv=%d (supported: (192, 128), (64, 64))", d_h, d_hv);
}

int dsa_forward(const void* q_idx, const float* w, const void* k_idx, const void* q,
                const void* kv, const int32_t* pos, const int32_t* k_base, int T, int S, int H_I,
                int d_I, int Hq, int d_qk, int d_v, int k, float scale, int32_t* idx, void* out,
                float* lse, void* workspace, size_t ws_bytes, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_indexer(q_idx, w, k_idx, pos, k_base, T, S, H_I, d_I, k, idx)) return rc;
    if (int rc = check_attn(q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, out, lse)) return rc;
    if (int rc = dsa_indexer_topk(q_idx, w, k_idx, pos, k_base, T, S, H_I, d_I, k, idx, workspace,
                                  ws_bytes, stream))
        return rc;
    return dsa_sparse_mla_attn(q, kv, idx, pos, k_base, T, S, Hq, d_qk, d_v, k, scale, out, lse,
                               workspace, ws_bytes, stream);
}

// ------------------------------------------------------- multi-GPU partition
//
// The path shards by query rows and by sequences with no exchange between
// ranks; these host-only functions pick the contiguous ranges.

namespace {

// Split items with costs c[0..n) into `parts` contiguous ranges of about
// equal total cost: range r ends at the first item where the running cost
// reaches (r+1)/parts of the total. bounds[0] = 0, bounds[parts] = n.
void balanced_bounds(const double* prefix, int n, int parts, int32_t* bounds)
{
    const double total = prefix[n];
    bounds[0] = 0;
    int i = 0;
    for (int r = 1; r < parts; ++r) {
        const double goal = total * r / parts;
        while (i < n && prefix[i + 1] < goal) ++i;
        // item i straddles the goal: end the range before or after it,
        // whichever lands closer
        int b = i;
        if (i < n && prefix[i + 1] - goal < goal - prefix[i]) b = i + 1;
        bounds[r] = std::max(b, (int)bounds[r - 1]);
    }
    bounds[parts] = n;
}

}  // namespace

int dsa_partition_prefill_rows(int T, int S, int k, int H_I, int d_I, int Hq, int d_qk, int d_v, int parts,
                               int32_t* bounds)
{
    g_err[0] = 0;
    if (!bounds) return fail(DSA_ERR_ARG, "NULL bounds");
    if (T <= 0 || S < T || k <= 0 || H_I <= 0 || d_I <= 0 || Hq <= 0 || d_qk <= 0 || d_v <= 0 || parts <= 0)
        return fail(DSA_ERR_ARG, "T=%d, S=%d, k=%d, H_I=%d, d_I=%d, Hq=%d, d_qk=%d, d_v=%d, parts=%d",
                    T, S, k, H_I, d_I, Hq, d_qk, d_v, parts);
    // modelled time of row t (position p = t + S - T, n = p + 1 candidates):
    // indexer FP8 MMA work over its n keys when n > k (FP8 at twice the BF16
    // rate), then the BF16 attention work over min(n, k) selected rows
    std::vector<double> prefix((size_t)T + 1, 0.0);
    const double w_idx = 2.0 * H_I * d_I / 2.0, w_attn = 2.0 * Hq * (double)(d_qk + d_v);
    for (int t = 0; t < T; ++t) {
        const double n = (double)t + (S - T) + 1;
        prefix[t + 1] = prefix[t] + (n > k ? n * w_idx : 0.0) + std::min(n, (double)k) * w_attn;
    }
    balanced_bounds(prefix.data(), T, parts, bounds);
    return DSA_OK;
}

int dsa_partition_decode_seqs(const int32_t* ctx, int n_seqs, int k, int d_I, int d_qk, int parts,
                              int32_t* bounds)
{
    g_err[0] = 0;
    if (!ctx || !bounds) return fail(DSA_ERR_ARG, "NULL ctx or bounds");
    if (n_seqs <= 0 || k <= 0 || d_I <= 0 || d_qk <= 0 || parts <= 0)
        return fail(DSA_ERR_ARG, "n_seqs=%d, k=%d, d_I=%d, d_qk=%d, parts=%d", n_seqs, k, d_I, d_qk, parts);
    // modelled time of a sequence: the bytes its step reads (every cached
    // indexer key once, the selected latent rows once)
    std::vector<double> prefix((size_t)n_seqs + 1, 0.0);
    for (int b = 0; b < n_seqs; ++b) {
        if (ctx[b] < 0) return fail(DSA_ERR_ARG, "ctx[%d] = %d", b, ctx[b]);
        prefix[b + 1] = prefix[b] + (double)ctx[b] * d_I + std::min(ctx[b], k) * 2.0 * d_qk;
    }
    balanced_bounds(prefix.data(), n_seqs, parts, bounds);
    return DSA_OK;
}

int dsa_device_status(void* stream)
{
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, dsa::g_status, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "read device status");
    if (v != 0) {
        const int zero = 0;
        if (v == dsa::kStatusCheck) {
            cudaMemcpyToSymbol(dsa::g_status, &zero, sizeof zero);
            return fail(v, "a debug-build check counted invalid index-set entries (dsa_debug_counters)");
        }
        int info[4] = {0, 0, 0, 0};
        cudaMemcpyFromSymbol(info, dsa::g_timeout_info, sizeof info);
        cudaMemcpyToSymbol(dsa::g_status, &zero, sizeof zero);
        return fail(v, "a kernel reported status %d: bounded wait gave up (barrier tag %d, chunk %d, "
                       "block %d, parity %d)", v, info[0], info[1], info[2], info[3]);
    }
    return DSA_OK;
}

int dsa_phase_timing(int enable)
{
    g_phase_on.store(enable != 0, std::memory_order_relaxed);
    return DSA_OK;
}

int dsa_phase_times(double* ms, int n)
{
    g_err[0] = 0;
    if (!ms || n < 0 || n > kNumPhases) return fail(DSA_ERR_ARG, "ms NULL or n=%d outside 0..%d", n, (int)kNumPhases);
    std::vector<PhaseRec> recs;
    {
        std::lock_guard<std::mutex> lock(g_phase_mu);
        recs.swap(g_phase_recs);
    }
    double sum[kNumPhases] = {0.0, 0.0, 0.0};
    int rc = DSA_OK;
    for (const PhaseRec& r : recs) {
        float t = 0.f;
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
        if (e != cudaSuccess && rc == DSA_OK) rc = cuda_fail(e, "phase timing events");
        sum[r.phase] += t;
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    for (int i = 0; i < n; ++i) ms[i] = sum[i];
    return rc;
}

int dsa_debug_build(void)
{
#ifdef DSA_DEBUG
    return 1;
#else
    return 0;
#endif
}

int dsa_debug_counters(uint64_t* out, int n, int reset)
{
    g_err[0] = 0;
    if (!out || n < 0 || n > dsa::kNumDebugCounts)
        return fail(DSA_ERR_ARG, "out NULL or n=%d outside 0..%d", n, (int)dsa::kNumDebugCounts);
    unsigned long long v[dsa::kNumDebugCounts] = {0};
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    e = cudaMemcpyFromSymbol(v, dsa::g_debug_counts, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "read debug counters");
    for (int i = 0; i < n; ++i) out[i] = v[i];
    if (reset) {
        const unsigned long long z[dsa::kNumDebugCounts] = {0};
        e = cudaMemcpyToSymbol(dsa::g_debug_counts, z, sizeof z);
        if (e != cudaSuccess) return cuda_fail(e, "clear debug counters");
    }
    return DSA_OK;
}

}  // extern "C"

// ============================================== indexer with library-held scratch
//
// dsa_indexer_topk_noalloc runs the same two kernels as dsa_indexer_topk, but
// its score scratch is a fixed array that the library itself holds in device
// memory, so the caller passes no workspace and nothing is allocated per call.

namespace {

// 4,194,304 fp32 scores = 16 MiB. Every GPU on which the library is loaded
// holds this array until the process exits.
constexpr size_t kStaticScoreFloats = size_t(4) << 20;
static __device__ __align__(256) float g_static_scores[kStaticScoreFloats];

// In host code `g_static_scores` only names a host-side stand-in for the
// array, not a device address; kernels get the address that
// cudaGetSymbolAddress returns, looked up once per device with that device
// current.
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
float* g_static_ptr[kMaxDevices] = {nullptr};

int static_scores_on_current_device(float** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scores);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_static_scores)");
        g_static_ptr[dev] = reinterpret_cast<float*>(p);
    }
    *out = g_static_ptr[dev];
    return DSA_OK;
}

}  // namespace

extern "C" int dsa_indexer_topk_noalloc(const void* q_idx, const float* w, const void* k_idx,
                                        const int32_t* pos, const int32_t* k_base, int T, int S,
                                        int H_I, int d_I, int k, int32_t* idx, void* stream)
{
    g_err[0] = 0;
    if (int rc = check_indexer(q_idx, w, k_idx, pos, k_base, T, S, H_I, d_I, k, idx)) return rc;
    if ((size_t)S > kStaticScoreFloats)
        return fail(DSA_ERR_UNSUPPORTED,
                    "S=%d: the library-held scratch takes at most %zu candidate keys", S,
                    kStaticScoreFloats);
    float* scores = nullptr;
    if (int rc = static_scores_on_current_device(&scores)) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // rows per block: as many score rows as the array holds, at most 65535
    // (the launches below put the block's rows on gridDim.y)
    const int RB = (int)std::min<size_t>({(size_t)T, kStaticScoreFloats / (size_t)S, (size_t)65535});
    const long long ld = S;
    constexpr int kKeysPerCta = 2048;
    ScoresFn scores_fn = pick_scores(H_I, d_I);
    const uint8_t* q8 = reinterpret_cast<const uint8_t*>(q_idx);
    const uint8_t* k8 = reinterpret_cast<const uint8_t*>(k_idx);
    for (int row0 = 0; row0 < T; row0 += RB) {
        const int rb = std::min(RB, T - row0);
        const int n_max = pos ? S : std::min(S, row0 + rb + S - T);
        dim3 grid(dsa::ceil_div(n_max, kKeysPerCta), rb);
        scores_fn(grid, st, q8, w, k8, pos, k_base, T, S, H_I, row0, scores, ld, kKeysPerCta);
        DSA_LAUNCH_CHECK("indexer_scores_kernel");
        dsa::topk_dense_rows_kernel<dsa::kSelectThreads>
            <<<rb, dsa::kSelectThreads, 0, st>>>(scores, ld, pos, k_base, T, S, row0, k, idx);
        DSA_LAUNCH_CHECK("topk_dense_rows_kernel");
    }
    return debug_check(idx, pos, k_base, T, S, k, {}, true, st);
}
