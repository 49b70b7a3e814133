// Lightning indexer + Top-k for rows with their own key ranges (decode, packed
// sequences, head shapes the tensor-core scan does not cover).
//
//   I_{t,s} = sum_{j<H_I} w_{t,j} * ReLU(q^I_{t,j} . k^I_s), then the k
//   largest I_{t,s} of each row ("Paper Breakdown: DeepSeek-V3.2", section 2,
//   "Index score" and "Top-k selector")
//
// A row's candidate range is cut into chunks of kChunkKeys keys; one CTA
// scores a chunk into shared memory (mma.sync e4m3, HBM-bound on the key rows)
// and keeps part of it as (score, s) pairs; a second kernel selects the row's
// Top-k from the union of its chunks' pairs. A row of a single chunk is
// finished exactly by the first kernel.
//
// What a chunk keeps: a sampled threshold tau (every 32nd tile of 128 keys is
// scored first; tau is the sample whose rank predicts about 2k entries of the
// row above it) filters the chunk, which then keeps its entries >= tau in s
// order; if more than k pass, it keeps its own Top-k instead. Under the total
// order (score descending, s ascending) both keep every member of the row's
// Top-k whenever at least k entries of the row pass tau; the merge checks that
// count, and a row short of it is run again without tau, where each chunk
// keeps its own Top-k. The result is the row's exact Top-k either way.
//
// Work items (row, chunk) are numbered through a per-row prefix of chunk
// counts computed on the device, so a fixed grid of persistent CTAs covers
// rows of any length mix without empty blocks.
#pragma once
#include "common.cuh"
#include "indexer_scores.cuh"
#include "topk_select.cuh"

namespace dsa {
namespace idx_chunk {

constexpr int kChunkKeys = 8192;
constexpr int kThreads = 512;
constexpr int kCtasPerSm = 2;
constexpr int kMergeThreads = 1024;
constexpr int kPlanThreads = 1024;
constexpr int kTauThreads = 256;
constexpr size_t kSmemBytes = kChunkKeys * sizeof(float) + sizeof(SelectSmem<kThreads>);
// sampling: tiles of 128 keys, every 32nd tile of a row (two per chunk)
constexpr int kSampleTile = 128;
constexpr int kSampleStride = 32 * kSampleTile;
constexpr int kSamplesPerChunk = kChunkKeys / kSampleStride * kSampleTile;
constexpr int kAlpha = 2;   // tau aims at about kAlpha * k entries of the row

__device__ __forceinline__ int row_chunks(int n) { return n <= kChunkKeys ? 1 : ceil_div(n, kChunkKeys); }

// work_off[r] = number of work items of rows row0 .. row0+r-1, r = 0..rows.
// mode 0: every row has row_chunks(n) items and flags[r] is cleared;
// mode 1: only rows with flags[r] set have items.
__global__ void __launch_bounds__(kPlanThreads)
chunk_plan_kernel(const int* __restrict__ pos, const int* __restrict__ k_base, int T, int S, int row0,
                  int rows, int mode, int* __restrict__ flags, int* __restrict__ work_off)
{
    __shared__ int part[kPlanThreads];
    const int per = ceil_div(rows, kPlanThreads);
    const int r0 = threadIdx.x * per, r1 = min(rows, r0 + per);
    auto items = [&](int r) -> int {
        long long base;
        const int c = row_chunks(row_candidates(pos, k_base, row0 + r, T, S, &base));
        return mode == 0 ? c : (flags[r] ? c : 0);
    };
    int sum = 0;
    for (int r = r0; r < r1; ++r) sum += items(r);
    part[threadIdx.x] = sum;
    __syncthreads();
    // inclusive scan of the per-thread sums (Hillis-Steele in shared memory)
    for (int off = 1; off < kPlanThreads; off <<= 1) {
        const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int acc = part[threadIdx.x] - sum;
    for (int r = r0; r < r1; ++r) {
        work_off[r] = acc;
        acc += items(r);
        if (mode == 0) flags[r] = 0;
    }
    if (threadIdx.x == kPlanThreads - 1) work_off[rows] = part[kPlanThreads - 1];
}

// Local row of work item `item`: the last r with work_off[r] <= item (rows
// without items share their offset with the next row and are skipped).
__device__ __forceinline__ int item_row(const int* __restrict__ work_off, int rows, int item)
{
    int lo = 0, hi = rows - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (work_off[mid] <= item) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Scores of keys [0, m) of a chunk into sc[0..m); kq points at key 0 of the
// chunk (this lane's quarter). kB 16-key blocks per warp and step (two when
// the key fragments fit the register budget), all loads before the MMAs.
template <int NT, int DI, int THREADS>
__device__ __forceinline__ void score_chunk(const QueryFrag<NT, DI>& qf, const uint8_t* kq, int m,
                                            float* sc)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tid4 = lane & 3;
    constexpr int kWarps = THREADS / 32;
    constexpr int kB = NT * DI <= 128 ? 2 : 1;
    for (int j0 = warp * 16 * kB; j0 < m; j0 += kWarps * 16 * kB) {
        KeyQuarter<DI> A[kB], B[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int a = j0 + 16 * u + gid, b = a + 8;
            if (a < m) A[u].load(kq + (size_t)a * DI); else A[u].zero();
            if (b < m) B[u].load(kq + (size_t)b * DI); else B[u].zero();
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int a = j0 + 16 * u + gid, b = a + 8;
            float ia, ib;
            qf.score(A[u], B[u], ia, ib);
            if (tid4 == 0) {
                if (a < m) sc[a] = ia;
                if (b < m) sc[b] = ib;
            }
        }
    }
}

// Sample tiles of every chunk of multi-chunk rows: samp[r * samp_ld +
// chunk * kSamplesPerChunk + j]; positions beyond the row hold -inf.
template <int NT, int DI>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
chunk_sample_kernel(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                    const uint8_t* __restrict__ k_idx, const int* __restrict__ pos,
                    const int* __restrict__ k_base, int T, int S, int H_I, int row0, int rows,
                    const int* __restrict__ work_off, float* __restrict__ samp, long long samp_ld)
{
    __shared__ float sc[kSamplesPerChunk];
    const int lane = threadIdx.x & 31;
    const int total = work_off[rows];
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int r = item_row(work_off, rows, item), t = row0 + r;
        const int chunk = item - work_off[r];
        long long base;
        const int n = row_candidates(pos, k_base, t, T, S, &base);
        if (row_chunks(n) < 2) continue;   // uniform over the CTA
        QueryFrag<NT, DI> qf;
        qf.load(q_idx, w, t, H_I, lane);
        const int tid4 = lane & 3;
#pragma unroll 1
        for (int u = 0; u < kSamplesPerChunk / kSampleTile; ++u) {
            const int s0 = chunk * kChunkKeys + u * kSampleStride;
            const int m = max(0, min(kSampleTile, n - s0));
            score_chunk<NT, DI, kThreads>(qf, k_idx + (size_t)(base + s0) * DI + tid4 * (DI / 4), m,
                                          sc + u * kSampleTile);
            for (int j = m + (int)threadIdx.x; j < kSampleTile; j += kThreads) sc[u * kSampleTile + j] = -INFINITY;
        }
        __syncthreads();
        float* out = samp + (size_t)r * samp_ld + (size_t)chunk * kSamplesPerChunk;
        for (int j = threadIdx.x; j < kSamplesPerChunk; j += kThreads) out[j] = sc[j];
        __syncthreads();
    }
}

// Number of sampled positions inside a row of n keys.
__device__ __forceinline__ int row_samples(int n)
{
    const int full = n / kSampleStride;
    return full * kSampleTile + min(kSampleTile, n - full * kSampleStride);
}

// tau[r] = order key of the sample of rank ceil(kAlpha * k * m / n) (m valid
// samples), or 0 (no filtering) where that rank is out of reach.
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
chunk_tau_kernel(const float* __restrict__ samp, long long samp_ld, const int* __restrict__ pos,
                 const int* __restrict__ k_base, int T, int S, int row0, int k,
                 uint32_t* __restrict__ tau)
{
    __shared__ SelectSmem<THREADS> sm;
    const int r = blockIdx.x, t = row0 + r;
    long long base;
    const int n = row_candidates(pos, k_base, t, T, S, &base);
    const int nchunks = row_chunks(n);
    const int m = row_samples(n);
    const long long want = ((long long)kAlpha * k * m + n - 1) / n;
    const int n_s = nchunks * kSamplesPerChunk;
    if (nchunks < 2 || want >= m || want >= n_s) {
        if (threadIdx.x == 0) tau[r] = 0u;
        return;
    }
    int take_eq, count_eq;
    const uint32_t key = radix_kth_key<THREADS>(DenseScores{samp + (size_t)r * samp_ld}, n_s, (int)want,
                                                sm, &take_eq, &count_eq);
    if (threadIdx.x == 0) tau[r] = key;
}

// Persistent CTAs over the work items of rows row0 .. row0+rows-1. Chunk c of
// local row r keeps its pairs at cand[r * cand_ld + c * k ...] and their count
// at ccnt[r * max_chunks + c]; tau == NULL: no filtering. A single-chunk row
// writes its final indices to idx.
template <int NT, int DI>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
chunk_topk_kernel(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                  const uint8_t* __restrict__ k_idx, const int* __restrict__ pos,
                  const int* __restrict__ k_base, int T, int S, int H_I, int row0, int rows, int k,
                  const int* __restrict__ work_off, const uint32_t* __restrict__ tau,
                  uint2* __restrict__ cand, long long cand_ld, int* __restrict__ ccnt, int max_chunks,
                  int32_t* __restrict__ idx)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float* sc = reinterpret_cast<float*>(smem);
    SelectSmem<kThreads>& sm = *reinterpret_cast<SelectSmem<kThreads>*>(smem + kChunkKeys * sizeof(float));
    const int lane = threadIdx.x & 31, tid4 = lane & 3;
    const int total = work_off[rows];

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int r = item_row(work_off, rows, item), t = row0 + r;
        const int chunk = item - work_off[r];
        long long base;
        const int n = row_candidates(pos, k_base, t, T, S, &base);
        const int nchunks = row_chunks(n);
        const int c0 = chunk * kChunkKeys;
        const int m = min(n - c0, kChunkKeys);   // 0 for an empty row

        QueryFrag<NT, DI> qf;
        qf.load(q_idx, w, t, H_I, lane);
        score_chunk<NT, DI, kThreads>(qf, k_idx + (size_t)(base + c0) * DI + tid4 * (DI / 4), m, sc);
        __syncthreads();
        if (nchunks == 1) {
            block_topk<kThreads>(SmemScores{sc, 0}, m, k, idx + (size_t)t * k, sm);
        } else {
            uint2* out = cand + (size_t)r * cand_ld + (size_t)chunk * k;
            auto emit = [&](int slot, int i) {
                out[slot] = make_uint2(__float_as_uint(sc[i]), (uint32_t)(c0 + i));
            };
            const uint32_t tk = tau ? tau[r] : 0u;
            // entries >= tau in s order (all entries when tau is 0)
            int kept = block_emit_if<kThreads>(m, [&](int i) { return score_key(sc[i]) >= tk; }, emit, k, sm);
            if (kept > k) {
                // more than k pass: the chunk's own Top-k
                block_select<kThreads>(SmemScores{sc, c0}, m, k, emit, sm);
                kept = k;
            }
            if (threadIdx.x == 0) ccnt[(size_t)r * max_chunks + chunk] = kept;
        }
        __syncthreads();   // sc and sm are reused by the next item
    }
}

// The pairs of a row: chunk c's ccnt[c] pairs at c * k; entry i of the
// concatenation is found through the prefix pre[] (shared memory).
struct ChunkPairs {
    const uint2* p;
    const int* pre;
    int nchunks, k;
    __device__ __forceinline__ uint2 at(int i) const
    {
        int lo = 0, hi = nchunks - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pre[mid] <= i) lo = mid; else hi = mid - 1;
        }
        return p[(size_t)lo * k + (i - pre[lo])];
    }
    __device__ __forceinline__ uint32_t key(int i) const { return score_key(__uint_as_float(at(i).x)); }
    __device__ __forceinline__ int s(int i) const { return (int)at(i).y; }
};

// Row Top-k from the chunks' pairs (rows of two or more chunks). mode 0: a row
// whose chunks kept fewer than k pairs in all is flagged for the rerun; mode 1:
// only flagged rows. Pairs are in ascending s, and so is the emitted row.
// Dynamic shared memory: (max_chunks + 1) ints.
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
merge_topk_kernel(const uint2* __restrict__ cand, long long cand_ld, const int* __restrict__ ccnt,
                  int max_chunks, const int* __restrict__ pos, const int* __restrict__ k_base, int T,
                  int S, int row0, int k, int mode, int* __restrict__ flags, int32_t* __restrict__ idx)
{
    __shared__ SelectSmem<THREADS> sm;
    extern __shared__ int pre[];
    const int r = blockIdx.x, t = row0 + r;
    long long base;
    const int n = row_candidates(pos, k_base, t, T, S, &base);
    const int nchunks = row_chunks(n);
    if (nchunks < 2 || (mode == 1 && !flags[r])) return;
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int c = 0; c < nchunks; ++c) {
            pre[c] = acc;
            acc += ccnt[(size_t)r * max_chunks + c];
        }
        pre[nchunks] = acc;
    }
    __syncthreads();
    const int n_pairs = pre[nchunks];
    if (n_pairs < k) {
        // fewer than k entries passed tau: rerun this row without it
        if (threadIdx.x == 0) flags[r] = 1;
        return;
    }
    block_topk<THREADS>(ChunkPairs{cand + (size_t)r * cand_ld, pre, nchunks, k}, n_pairs, k,
                        idx + (size_t)t * k, sm);
}

}  // namespace idx_chunk
}  // namespace dsa
