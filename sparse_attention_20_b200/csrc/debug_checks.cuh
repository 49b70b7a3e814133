// Checks of the debug build (libdsa_debug.so, compiled with -DDSA_DEBUG):
// device-side validation of the index sets that flow between the selector
// and the attention, standing in for an external memory checker. They never
// trap: each violation is counted in g_debug_counts and the first call that
// finds one sets the device status word to kStatusCheck, which
// dsa_device_status reports. The release build compiles none of this.
//
// What a row t of an index set may hold (include/dsa.h, dsa_indexer_topk and
// dsa_sparse_mla_attn): the attention reads the first m = min(k, n) entries
// (n = pos[t] + 1 candidates), ignores those < 0 or > pos[t], and reads
// nothing past m. Counted, per entry:
//   kCntBeyondPos   an entry in [0, m) greater than pos[t] (ignored)
//   kCntPadInside   an entry in [0, m) below 0 (ignored)
//   kCntDropped     a valid entry at or past m (never read)
//   kCntDuplicate   a valid entry in [0, m) equal to an earlier one
//   kCntBadPage     a valid entry whose block-table page is outside the pool
//                   (read from page 0 instead)
//   kCntSelection   a selector result that is not min(k, n) distinct valid
//                   entries followed by -1 padding
#pragma once
#include "common.cuh"

namespace dsa {

enum : int { kCntBeyondPos = 0, kCntPadInside, kCntDropped, kCntDuplicate, kCntBadPage, kCntSelection,
             kNumDebugCounts };
enum : int { kStatusCheck = -6 };

__device__ unsigned long long g_debug_counts[kNumDebugCounts];

constexpr int kCheckThreads = 256;
constexpr int kCheckMaxK = 4096;

#ifdef DSA_DEBUG

// Bitonic sort of the first `n` values of a shared array of `cap` (a power
// of two >= n); the tail is filled with INT_MAX.
__device__ void block_sort_ints(int* v, int n, int cap)
{
    for (int i = n + (int)threadIdx.x; i < cap; i += blockDim.x) v[i] = 0x7FFFFFFF;
    __syncthreads();
    for (int size = 2; size <= cap; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < cap; i += blockDim.x) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool up = (i & size) == 0;
                    const int a = v[i], b = v[j];
                    if ((a > b) == up) {
                        v[i] = b;
                        v[j] = a;
                    }
                }
            }
            __syncthreads();
        }
}

// One CTA per row: counts the violations of one index set. `selector`: the
// set came from the selector, so it must also be exactly min(k, n) distinct
// valid entries then -1 padding.
__global__ void __launch_bounds__(kCheckThreads)
debug_check_idx_kernel(const int* __restrict__ idx, const int* __restrict__ pos, const int* __restrict__ k_base,
                       int T, int S, int k, const PagedRows pg, int selector)
{
    __shared__ int vals[kCheckMaxK];
    __shared__ unsigned long long cnt[kNumDebugCounts];
    __shared__ int n_valid;
    const int t = blockIdx.x;
    long long base;
    const int* bt;
    const int n = row_keys(pg, pos, k_base, t, T, S, &base, &bt);
    const int m = min(k, n);
    if (threadIdx.x < kNumDebugCounts) cnt[threadIdx.x] = 0;
    if (threadIdx.x == 0) n_valid = 0;
    __syncthreads();
    const int* row = idx + (size_t)t * k;
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const int v = row[i];
        const bool valid = v >= 0 && v < n;
        if (i < m) {
            if (v >= n) atomicAdd(&cnt[kCntBeyondPos], 1ull);
            if (v < 0) atomicAdd(&cnt[kCntPadInside], 1ull);
        } else if (valid) {
            atomicAdd(&cnt[kCntDropped], 1ull);
        }
        if (valid && bt && (unsigned)bt[v / pg.page_size] >= (unsigned)pg.num_pages)
            atomicAdd(&cnt[kCntBadPage], 1ull);
        if (selector && (i < m ? !valid : v != -1)) atomicAdd(&cnt[kCntSelection], 1ull);
        vals[i] = (i < m && valid) ? v : 0x7FFFFFFF;
        if (i < m && valid) atomicAdd(&n_valid, 1);
    }
    __syncthreads();
    int cap = 1;
    while (cap < k) cap <<= 1;
    block_sort_ints(vals, k, cap);
    for (int i = threadIdx.x + 1; i < n_valid; i += blockDim.x)
        if (vals[i] == vals[i - 1]) atomicAdd(&cnt[kCntDuplicate], 1ull);
    __syncthreads();
    if (threadIdx.x < kNumDebugCounts && cnt[threadIdx.x]) {
        atomicAdd(&g_debug_counts[threadIdx.x], cnt[threadIdx.x]);
        report_status(kStatusCheck);
    }
}

#endif  // DSA_DEBUG

}  // namespace dsa
