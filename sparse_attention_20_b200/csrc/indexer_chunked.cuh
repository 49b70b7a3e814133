// Lightning indexer + Top-k for rows with their own key ranges (decode, packed
// sequences, head shapes the tensor-core scan does not cover).
//
//   I_{t,s} = sum_{j<H_I} w_{t,j} * ReLU(q^I_{t,j} . k^I_s), then the k
//   largest I_{t,s} of each row ("Paper Breakdown: DeepSeek-V3.2", section 2,
//   "Index score" and "Top-k selector")
//
// A row's candidate range is cut into chunks of kChunkKeys keys. One CTA
// scores a chunk into shared memory (mma.sync e4m3, HBM-bound on the key
// rows) and keeps the chunk's own Top-k as (score, s) pairs; a second kernel
// selects the row's Top-k from the union of its chunks' pairs. Under the total
// order (score descending, s ascending) every member of the row's Top-k is
// also in the Top-k of its chunk, so the two steps give exactly the row's
// Top-k. A row of a single chunk is finished by the first kernel.
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
constexpr size_t kSmemBytes = kChunkKeys * sizeof(float) + sizeof(SelectSmem<kThreads>);

__device__ __forceinline__ int row_chunks(int n) { return n <= kChunkKeys ? 1 : ceil_div(n, kChunkKeys); }

// work_off[r] = sum of row_chunks over rows row0 .. row0+r-1, r = 0..rows.
__global__ void __launch_bounds__(kPlanThreads)
chunk_plan_kernel(const int* __restrict__ pos, const int* __restrict__ k_base, int T, int S, int row0,
                  int rows, int* __restrict__ work_off)
{
    __shared__ int part[kPlanThreads];
    const int per = ceil_div(rows, kPlanThreads);
    const int r0 = threadIdx.x * per, r1 = min(rows, r0 + per);
    int sum = 0;
    for (int r = r0; r < r1; ++r) {
        long long base;
        sum += row_chunks(row_candidates(pos, k_base, row0 + r, T, S, &base));
    }
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
        long long base;
        acc += row_chunks(row_candidates(pos, k_base, row0 + r, T, S, &base));
    }
    if (threadIdx.x == kPlanThreads - 1) work_off[rows] = part[kPlanThreads - 1];
}

// Persistent CTAs over the work items of rows row0 .. row0+rows-1. Pairs of
// chunk c of local row r go to cand[r * cand_ld + c * k ...]; a single-chunk
// row writes its final indices to idx.
template <int NT, int DI>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
chunk_topk_kernel(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                  const uint8_t* __restrict__ k_idx, const int* __restrict__ pos,
                  const int* __restrict__ k_base, int T, int S, int H_I, int row0, int rows, int k,
                  const int* __restrict__ work_off, uint2* __restrict__ cand, long long cand_ld,
                  int32_t* __restrict__ idx)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float* sc = reinterpret_cast<float*>(smem);
    SelectSmem<kThreads>& sm = *reinterpret_cast<SelectSmem<kThreads>*>(smem + kChunkKeys * sizeof(float));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tid4 = lane & 3;
    constexpr int kWarps = kThreads / 32;
    const int total = work_off[rows];

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        // row of this item: the last r with work_off[r] <= item
        int lo = 0, hi = rows - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (work_off[mid] <= item) lo = mid; else hi = mid - 1;
        }
        const int r = lo, t = row0 + r;
        const int chunk = item - work_off[r];
        long long base;
        const int n = row_candidates(pos, k_base, t, T, S, &base);
        const int nchunks = row_chunks(n);
        const int c0 = chunk * kChunkKeys;
        const int m = min(n - c0, kChunkKeys);   // 0 for an empty row

        QueryFrag<NT, DI> qf;
        qf.load(q_idx, w, t, H_I, lane);
        const uint8_t* kq = k_idx + (size_t)(base + c0) * DI + tid4 * (DI / 4);
        // kB 16-key blocks per warp and step (two when the key fragments fit
        // the register budget), all loads issued before the MMAs
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
        __syncthreads();
        if (nchunks == 1) {
            block_topk<kThreads>(SmemScores{sc, 0}, m, k, idx + (size_t)t * k, sm);
        } else {
            uint2* out = cand + (size_t)r * cand_ld + (size_t)chunk * k;
            if (m <= k) {
                for (int i = threadIdx.x; i < m; i += kThreads)
                    out[i] = make_uint2(__float_as_uint(sc[i]), (uint32_t)(c0 + i));
            } else {
                block_select<kThreads>(
                    SmemScores{sc, c0}, m, k,
                    [&](int slot, int i) { out[slot] = make_uint2(__float_as_uint(sc[i]), (uint32_t)(c0 + i)); },
                    sm);
            }
        }
        __syncthreads();   // sc and sm are reused by the next item
    }
}

// Row Top-k from the chunks' pairs (rows of two or more chunks). Chunks hold
// k pairs each except the last (min(its keys, k)), so a row's pairs are
// contiguous; they are in ascending s, and so is the emitted row.
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
merge_topk_kernel(const uint2* __restrict__ cand, long long cand_ld, const int* __restrict__ pos,
                  const int* __restrict__ k_base, int T, int S, int row0, int k,
                  int32_t* __restrict__ idx)
{
    __shared__ SelectSmem<THREADS> sm;
    const int r = blockIdx.x, t = row0 + r;
    long long base;
    const int n = row_candidates(pos, k_base, t, T, S, &base);
    const int nchunks = row_chunks(n);
    if (nchunks < 2) return;
    const int last = n - (nchunks - 1) * kChunkKeys;
    const int n_pairs = (nchunks - 1) * k + min(last, k);
    block_topk<THREADS>(PairScores{cand + (size_t)r * cand_ld}, n_pairs, k, idx + (size_t)t * k, sm);
}

}  // namespace idx_chunk
}  // namespace dsa
