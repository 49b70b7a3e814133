// Exact per-row Top-k selection ("Top-k selector on I_{t,s}", section 2 of
// "Paper Breakdown: DeepSeek-V3.2") over scores that are already in memory.
//
// One CTA per row. The k-th largest score is found by an MSD radix select on
// the order-preserving 32-bit key of the fp32 score (four 8-bit digits, one
// pass over the row each, per-warp shared-memory histograms). Equal scores are
// broken towards the lower index: if more entries tie at the k-th score than
// slots are left, a second radix select over the candidates' indices finds the
// cut. The emitted set is therefore the unique Top-k under (score desc, s asc).
#pragma once
#include "common.cuh"

namespace dsa {

template <int THREADS>
struct SelectSmem {
    uint32_t hist[THREADS / 32][256];
    uint32_t total[256];
    int misc[4];
    int counter[2];
};

// Threads that run a block-level selection together: the whole CTA (the
// default) or a warp-aligned subset meeting at a named barrier.
struct CtaGroup {
    __device__ static __forceinline__ int tid() { return (int)threadIdx.x; }
    __device__ static __forceinline__ void sync() { __syncthreads(); }
};
template <int ID, int NTHREADS, int FIRST>
struct NamedGroup {
    static_assert(NTHREADS % 32 == 0 && FIRST % 32 == 0, "warp-aligned group");
    __device__ static __forceinline__ int tid() { return (int)threadIdx.x - FIRST; }
    __device__ static __forceinline__ void sync()
    {
        asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(NTHREADS) : "memory");
    }
};

// Scores stored densely: entry i is candidate s = i.
struct DenseScores {
    const float* p;
    __device__ __forceinline__ uint32_t key(int i) const { return score_key(p[i]); }
    __device__ __forceinline__ int s(int i) const { return i; }
};

// Scores of keys s0, s0+1, ... held in shared memory.
struct SmemScores {
    const float* p;
    int s0;
    __device__ __forceinline__ uint32_t key(int i) const { return score_key(p[i]); }
    __device__ __forceinline__ int s(int i) const { return s0 + i; }
};

// Candidates stored as (fp32 score bits, s) pairs.
struct PairScores {
    const uint2* p;
    __device__ __forceinline__ uint32_t key(int i) const { return score_key(__uint_as_float(p[i].x)); }
    __device__ __forceinline__ int s(int i) const { return (int)p[i].y; }
};

// Merge the per-warp histograms into total[], then find the digit whose bin
// holds the need-th entry counted from the top (descending) or from the
// bottom (ascending). Results: misc[0] = digit, misc[1] = rank inside the bin
// (1-based), misc[2] = entries in the bin.
template <int THREADS, class G = CtaGroup>
__device__ __forceinline__ void select_digit(SelectSmem<THREADS>& sm, int need, bool descending)
{
    constexpr int W = THREADS / 32;
    for (int b = G::tid(); b < 256; b += THREADS) {
        uint32_t s = 0;
#pragma unroll 8
        for (int w = 0; w < W; ++w) s += sm.hist[w][b];
        sm.total[b] = s;
    }
    G::sync();
    if (G::tid() < 32) {
        const int lane = G::tid();
        // lane owns 8 bins; in the descending case lane 0 owns the top bins
        uint32_t c[8];
        uint32_t local = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int b = descending ? 255 - (lane * 8 + j) : lane * 8 + j;
            c[j] = sm.total[b];
            local += c[j];
        }
        uint32_t incl = local;  // inclusive prefix over lanes 0..lane
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const uint32_t before = incl - local;
        if (before < (uint32_t)need && incl >= (uint32_t)need) {
            uint32_t cum = before;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (cum + c[j] >= (uint32_t)need) {
                    sm.misc[0] = descending ? 255 - (lane * 8 + j) : lane * 8 + j;
                    sm.misc[1] = need - (int)cum;
                    sm.misc[2] = (int)c[j];
                    break;
                }
                cum += c[j];
            }
        }
    }
    G::sync();
}

template <int THREADS, class G = CtaGroup>
__device__ __forceinline__ void clear_hist(SelectSmem<THREADS>& sm)
{
    uint32_t* h = &sm.hist[0][0];
    for (int i = G::tid(); i < (THREADS / 32) * 256; i += THREADS) h[i] = 0u;
    G::sync();
}

// Returns the key of the k-th largest entry; *take_eq = entries equal to it
// that belong to the Top-k, *count_eq = entries equal to it. Requires n > k.
// With digits < 4 only the top 8 * digits bits are resolved: the result is
// the k-th largest key with its lower bits cleared, a lower bound of it (and
// *take_eq, *count_eq refer to that bucket).
template <int THREADS, class G = CtaGroup, class Row>
__device__ uint32_t radix_kth_key(const Row& row, int n, int k, SelectSmem<THREADS>& sm,
                                  int* take_eq, int* count_eq, int digits = 4)
{
    const int warp = G::tid() >> 5;
    uint32_t prefix = 0u, mask = 0u;
    int need = k, cnt = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 32 - 8 * digits; shift -= 8) {
        clear_hist<THREADS, G>(sm);
        for (int i = G::tid(); i < n; i += THREADS) {
            const uint32_t key = row.key(i);
            if ((key & mask) == prefix) atomicAdd(&sm.hist[warp][(key >> shift) & 255u], 1u);
        }
        G::sync();
        select_digit<THREADS, G>(sm, need, true);
        prefix |= (uint32_t)sm.misc[0] << shift;
        mask |= 255u << shift;
        need = sm.misc[1];
        cnt = sm.misc[2];
        G::sync();
    }
    *take_eq = need;
    *count_eq = cnt;
    return prefix;
}

// Ordered compaction: emit(slot, i) for the entries i < n with pred(i), in
// storage order, for slots below cap. Returns the number of such entries
// (which may exceed cap). Every thread of the CTA takes part; thread j looks
// at kEmitPer consecutive entries of each batch of THREADS * kEmitPer.
constexpr int kEmitPer = 4;

template <int THREADS, class G = CtaGroup, class Pred, class Emit>
__device__ int block_emit_if(int n, const Pred& pred, const Emit& emit, int cap, SelectSmem<THREADS>& sm)
{
    constexpr int W = THREADS / 32;
    const int warp = G::tid() >> 5, lane = G::tid() & 31;
    int running = 0;
    for (int b0 = 0; b0 < n; b0 += THREADS * kEmitPer) {
        const int i0 = b0 + G::tid() * kEmitPer;
        uint32_t bits = 0u;
#pragma unroll
        for (int e = 0; e < kEmitPer; ++e)
            if (i0 + e < n && pred(i0 + e)) bits |= 1u << e;
        const int cnt = __popc(bits);
        int incl = cnt;   // inclusive prefix over the lanes of the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) sm.hist[0][warp] = (uint32_t)incl;
        G::sync();
        int slot = running + incl - cnt, total = 0;
#pragma unroll 4
        for (int w = 0; w < W; ++w) {
            const int v = (int)sm.hist[0][w];
            if (w < warp) slot += v;
            total += v;
        }
#pragma unroll
        for (int e = 0; e < kEmitPer; ++e)
            if (bits >> e & 1u) {
                if (slot < cap) emit(slot, i0 + e);
                ++slot;
            }
        running += total;
        G::sync();   // hist[0] is rewritten by the next batch
    }
    return running;
}

// Emits the Top-k of `row` (n > k entries) as emit(slot, i) for slots
// 0..k-1 in storage order (for dense rows: ascending s), so the result is
// deterministic.
template <int THREADS, class G = CtaGroup, class Row, class Emit>
__device__ void block_select(const Row& row, int n, int k, const Emit& emit, SelectSmem<THREADS>& sm)
{
    int take_eq, count_eq;
    const uint32_t kth = radix_kth_key<THREADS, G>(row, n, k, sm, &take_eq, &count_eq);
    const int warp = G::tid() >> 5;
    // Index cut among the ties: the take_eq-th smallest s with key == kth.
    uint32_t s_cut = 0xFFFFFFFFu;
    if (count_eq > take_eq) {
        uint32_t prefix = 0u, mask = 0u;
        int need = take_eq;
#pragma unroll 1
        for (int shift = 24; shift >= 0; shift -= 8) {
            clear_hist<THREADS, G>(sm);
            for (int i = G::tid(); i < n; i += THREADS) {
                if (row.key(i) != kth) continue;
                const uint32_t s = (uint32_t)row.s(i);
                if ((s & mask) == prefix) atomicAdd(&sm.hist[warp][(s >> shift) & 255u], 1u);
            }
            G::sync();
            select_digit<THREADS, G>(sm, need, false);
            prefix |= (uint32_t)sm.misc[0] << shift;
            mask |= 255u << shift;
            need = sm.misc[1];
            G::sync();
        }
        s_cut = prefix;
    }
    // Emit in storage order (ascending s for dense rows): ordered compaction.
    block_emit_if<THREADS, G>(
        n,
        [&](int i) {
            const uint32_t key = row.key(i);
            return key > kth || (key == kth && (uint32_t)row.s(i) <= s_cut);
        },
        emit, k, sm);
}

// Exact Top-k of `row` (n >= k entries; order: key descending, then s
// ascending) marked in a bitmap over s, in three reads of the row: the key
// range, a histogram of kRangeBins equal-width bins over that range, and a
// pass that marks every entry of a bin above the one holding the k-th entry
// and collects that bin's entries, which are then ranked in shared memory.
// Returns false, with the bitmap untouched, when every key is equal or the
// boundary bin holds more than kRangeListCap entries (the caller then takes
// the radix path). The caller synchronises before reading the bitmap.
constexpr int kRangeBins = 2048;
constexpr int kRangeListCap = 128;   // uint2 entries in SelectSmem::total

// With the kRangeBins-bin histogram in sm.hist complete and visible: the bin
// holding the k-th entry from the top goes to sm.misc[0], k minus the entries
// of the bins above it to misc[1], the bin's count to misc[2] (visible to
// every thread on return). If the histogram holds fewer than k entries,
// misc[2] is INT_MAX.
template <int THREADS>
__device__ void range_kth_bin(int k, SelectSmem<THREADS>& sm)
{
    constexpr int W = THREADS / 32;
    constexpr int PER = kRangeBins / THREADS;
    __shared__ uint32_t wsum[W];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t* h = &sm.hist[0][0];
    // thread j owns the PER bins just below the top j * PER
    uint32_t c[PER], local = 0u;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        c[j] = h[kRangeBins - 1 - (tid * PER + j)];
        local += c[j];
    }
    uint32_t incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    if (tid == 0) {
        sm.counter[0] = 0;
        // what a histogram of fewer than k entries leaves: no bin, and a
        // boundary "count" above any list capacity (range_select_core declines)
        sm.misc[0] = 0;
        sm.misc[1] = k;
        sm.misc[2] = 0x7FFFFFFF;
    }
    __syncthreads();
    uint32_t before = incl - local;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (before < (uint32_t)k && before + local >= (uint32_t)k) {
        uint32_t cum = before;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            if (cum + c[j] >= (uint32_t)k) {
                sm.misc[0] = kRangeBins - 1 - (tid * PER + j);
                sm.misc[1] = k - (int)cum;
                sm.misc[2] = (int)c[j];
                break;
            }
            cum += c[j];
        }
    }
    __syncthreads();
}

// Steps 2-5 with the block's key range [lo, hi] known and the histogram
// (sm.hist) zeroed and visible to every thread.
// each(f) calls f(key, s) for every entry of the row (every thread of the
// CTA calls it, each thread for its own share of the entries).
template <int THREADS, class Each>
__device__ bool range_select_core(const Each& each, int k, uint32_t lo, uint32_t hi, uint32_t* bm,
                                  SelectSmem<THREADS>& sm)
{
    constexpr int W = THREADS / 32;
    static_assert(W * 256 >= kRangeBins && kRangeBins % THREADS == 0, "histogram space");
    static_assert(2 * kRangeListCap <= 256 && 2 * W <= 256, "list space");
    const int tid = threadIdx.x;
    uint32_t* h = &sm.hist[0][0];
    if (lo == hi) return false;
    const int shift = max(0, 32 - __clz(hi - lo) - 11);   // (hi - lo) >> shift < 2048
    // 2. histogram
    each([&](uint32_t key, uint32_t) { atomicAdd(&h[(key - lo) >> shift], 1u); });
    __syncthreads();
    // 3. the bin of the k-th entry from the top
    range_kth_bin<THREADS>(k, sm);
    const uint32_t kb = (uint32_t)sm.misc[0];
    const int need = sm.misc[1], inb = sm.misc[2];
    if (inb > kRangeListCap) return false;
    // 4. mark the entries above bin kb, collect bin kb
    uint2* list = reinterpret_cast<uint2*>(sm.total);
    each([&](uint32_t key, uint32_t s) {
        const uint32_t b = (key - lo) >> shift;
        if (b > kb)
            atomicOr(&bm[s >> 5], 1u << (s & 31));
        else if (b == kb)
            list[atomicAdd(&sm.counter[0], 1)] = make_uint2(key, s);
    });
    __syncthreads();
    // 5. the first `need` entries of the bin by (key descending, s ascending)
    for (int j = tid; j < inb; j += THREADS) {
        const uint2 e = list[j];
        int rank = 0;
        for (int q = 0; q < inb; ++q) {
            const uint2 f = list[q];
            rank += (f.x > e.x) || (f.x == e.x && f.y < e.y);
        }
        if (rank < need) atomicOr(&bm[e.y >> 5], 1u << (e.y & 31));
    }
    return true;
}

template <int THREADS, class Row>
__device__ bool range_select_bitmap(const Row& row, int n, int k, uint32_t* bm, SelectSmem<THREADS>& sm)
{
    constexpr int W = THREADS / 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t* h = &sm.hist[0][0];
    // 1. key range
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int i = tid; i < n; i += THREADS) {
        const uint32_t key = row.key(i);
        lo = min(lo, key);
        hi = max(hi, key);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
        sm.total[warp] = lo;
        sm.total[W + warp] = hi;
    }
    for (int b = tid; b < kRangeBins; b += THREADS) h[b] = 0u;
    __syncthreads();
    lo = sm.total[0];
    hi = sm.total[W];
#pragma unroll
    for (int w = 1; w < W; ++w) {
        lo = min(lo, sm.total[w]);
        hi = max(hi, sm.total[W + w]);
    }
    const auto each = [&](const auto& f) {
        for (int i = tid; i < n; i += THREADS) f(row.key(i), (uint32_t)row.s(i));
    };
    return range_select_core<THREADS>(each, k, lo, hi, bm, sm);
}

// The same with the row's key range [lo, hi] given by the caller (every
// thread passes the same values) and its entries visited by each(f), which
// calls f(key, s) for this thread's share of them.
template <int THREADS, class Each>
__device__ bool range_select_bitmap_in(const Each& each, int k, uint32_t lo, uint32_t hi, uint32_t* bm,
                                       SelectSmem<THREADS>& sm)
{
    uint32_t* h = &sm.hist[0][0];
    for (int b = threadIdx.x; b < kRangeBins; b += THREADS) h[b] = 0u;
    __syncthreads();
    return range_select_core<THREADS>(each, k, lo, hi, bm, sm);
}

// A lower bound of the k-th largest of the non-zero order keys among
// v[0..m) (shared or global memory; key 0 marks an empty entry), or 0 when
// fewer than k are non-zero. The k-th largest is located in a kRangeBins-bin
// histogram over the keys' range, then in a kRangeBins-bin histogram over
// that bin; the result is the lower edge of the sub-bin holding it, so at
// least k of the keys are >= it. Every thread of the CTA takes part and
// returns it.
template <int THREADS>
__device__ uint32_t range_floor(const uint32_t* v, int m, int k, SelectSmem<THREADS>& sm)
{
    constexpr int W = THREADS / 32;
    static_assert(W * 256 >= kRangeBins && kRangeBins % THREADS == 0, "histogram space");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t* h = &sm.hist[0][0];
    uint32_t lo = 0xFFFFFFFFu, hi = 0u, cnt = 0u;
    for (int i = tid; i < m; i += THREADS) {
        const uint32_t x = v[i];
        if (x) {
            lo = min(lo, x);
            hi = max(hi, x);
            ++cnt;
        }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    }
    if (lane == 0) {
        sm.total[warp] = lo;
        sm.total[W + warp] = hi;
        sm.total[2 * W + warp] = cnt;
    }
    for (int b = tid; b < kRangeBins; b += THREADS) h[b] = 0u;
    __syncthreads();
    lo = sm.total[0];
    hi = sm.total[W];
    cnt = sm.total[2 * W];
#pragma unroll
    for (int w = 1; w < W; ++w) {
        lo = min(lo, sm.total[w]);
        hi = max(hi, sm.total[W + w]);
        cnt += sm.total[2 * W + w];
    }
    __syncthreads();   // sm.total is free again
    if (cnt < (uint32_t)k) return 0u;
    if (lo == hi) return lo;
    // level 1: bins of 2^shift keys over [lo, hi]
    const int shift = max(0, 32 - __clz(hi - lo) - 11);   // (hi - lo) >> shift < 2048
    for (int i = tid; i < m; i += THREADS) {
        const uint32_t x = v[i];
        if (x) atomicAdd(&h[(x - lo) >> shift], 1u);
    }
    __syncthreads();
    range_kth_bin<THREADS>(k, sm);
    const uint32_t kb = (uint32_t)sm.misc[0];
    const int need = sm.misc[1];
    __syncthreads();   // sm.misc is read; the histogram is cleared next
    const uint32_t b0 = lo + (kb << shift);
    if (shift == 0) return b0;
    // level 2: sub-bins of 2^shift2 keys over bin kb
    const int shift2 = max(0, shift - 11);
    for (int b = tid; b < kRangeBins; b += THREADS) h[b] = 0u;
    __syncthreads();
    for (int i = tid; i < m; i += THREADS) {
        const uint32_t x = v[i];
        if (x && ((x - lo) >> shift) == kb) atomicAdd(&h[(x - b0) >> shift2], 1u);
    }
    __syncthreads();
    range_kth_bin<THREADS>(need, sm);
    const uint32_t kb2 = (uint32_t)sm.misc[0];
    __syncthreads();   // sm.misc is free again
    return b0 + (kb2 << shift2);
}

// Writes the Top-k of `row` (n entries) to out[0..k) in storage order; slots
// beyond n (n < k) get -1.
template <int THREADS, class G = CtaGroup, class Row>
__device__ void block_topk(const Row& row, int n, int k, int32_t* __restrict__ out,
                           SelectSmem<THREADS>& sm)
{
    if (n <= k) {
        for (int i = G::tid(); i < k; i += THREADS) out[i] = i < n ? row.s(i) : -1;
        return;
    }
    block_select<THREADS, G>(row, n, k, [&](int slot, int i) { out[slot] = row.s(i); }, sm);
}

// Sorts v[0..n) ascending in shared memory (bitonic network over cap, a power
// of two >= n; the tail is padded with INT_MAX). Every thread of the CTA takes
// part.
__device__ __forceinline__ void block_sort_ascending(int* v, int n, int cap)
{
    for (int i = n + (int)threadIdx.x; i < cap; i += blockDim.x) v[i] = 0x7FFFFFFF;
    __syncthreads();
    for (int size = 2; size <= cap; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < cap / 2; i += blockDim.x) {
                // i-th compare-exchange pair of this stage: (lo, lo + stride)
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const int a = v[lo], b = v[hi];
                if ((a > b) == up) {
                    v[lo] = b;
                    v[hi] = a;
                }
            }
            __syncthreads();
        }
}

// Writes map(position) of the set bits of bm (words covering [0, n)) to
// out[0..) in ascending order of position: every thread emits the set bits of its run of
// words at an offset from a block-wide prefix of their counts. warp_sums
// holds THREADS / 32 ints of shared memory. Every thread of the CTA takes
// part.
struct SamePosition {
    __device__ __forceinline__ int operator()(int i) const { return i; }
};

template <int THREADS, class Map = SamePosition>
__device__ void block_emit_bitmap(const uint32_t* bm, int n, int* out, int* warp_sums, const Map& map = {})
{
    const int words = (n + 31) >> 5;
    const int per = (words + THREADS - 1) / THREADS;
    const int w0 = min(words, (int)threadIdx.x * per), w1 = min(words, w0 + per);
    int cnt = 0;
    for (int i = w0; i < w1; ++i) cnt += __popc(bm[i]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int pos = incl - cnt;
    for (int q = 0; q < warp; ++q) pos += warp_sums[q];
    for (int i = w0; i < w1; ++i)
        for (uint32_t b = bm[i]; b; b &= b - 1u) out[pos++] = map((i << 5) + __ffs(b) - 1);
}

__host__ __device__ __forceinline__ int pow2_ceil(int x)
{
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

constexpr int kSelectThreads = 1024;

// One CTA per query row t = row0 + blockIdx.x; its scores are row blockIdx.x
// of `scores` (dense, s = 0..pos[t]).
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
topk_dense_rows_kernel(const float* __restrict__ scores, long long ld, const int* __restrict__ pos,
                       const int* __restrict__ k_base, int T, int S, int row0, int k,
                       int32_t* __restrict__ idx)
{
    __shared__ SelectSmem<THREADS> sm;
    const int t = row0 + blockIdx.x;
    long long base;
    const int n = row_candidates(pos, k_base, t, T, S, &base);
    DenseScores row{scores + (size_t)blockIdx.x * ld};
    block_topk<THREADS>(row, n, k, idx + (size_t)t * k, sm);
}

}  // namespace dsa
