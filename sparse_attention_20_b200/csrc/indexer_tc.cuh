// Lightning indexer + Top-k selector for one causal sequence, streamed on the
// 5th-generation tensor cores (FP8). The L x L score matrix is never stored.
//
//   I_{t,s} = sum_{j<8} w_{t,j} * ReLU(q^I_{t,j} . k^I_s),  s <= pos[t]
//   ("Paper Breakdown: DeepSeek-V3.2", section 2, "Index score"; few FP8
//   heads: the research summary's "Key points"), then Top-k of I_{t,:}.
//
// Scan kernel (one CTA per 32 query rows): keys are the M dimension of the
// MMA and (row, head) pairs the N dimension: D[128 keys, 256] = K[128, 128] .
// Q^T where Q is the 32 rows x 8 heads of q^I (a contiguous 32 KB block, loaded
// once by TMA). Each key tile is one 16 KB TMA box; four tcgen05 kind::f8f6f4
// instructions (K = 32 each) score 4096 (row, key) pairs into TMEM. The
// epilogue thread that owns a key (TMEM lane) forms the weighted ReLU head-sum
// of the 32 rows, masks s > pos[t], and either
//   - sample mode: writes every score of the sampled tiles (every G-th tile),
//     from which a per-row threshold tau_t is drawn, or
//   - filter mode: appends the (score, s) with score >= tau_t to the row's
//     bounded candidate buffer.
// A final per-row select takes the exact Top-k from the candidates (ties to
// the lower s). Rows whose buffer ended up with fewer than k entries (tau too
// high) or overflowed are recomputed exactly in the same select kernel, so
// the result never depends on the sampling.
//
// Warp roles (640 threads): warp 0 TMA, warp 1 MMA (one thread), warps 4-19
// four epilogue groups of four warps: groups 0/1 share TMEM buffer 0 (even
// key tiles), groups 2/3 buffer 1 (odd tiles); within a pair each group takes
// 16 of the 32 query rows.
#pragma once
#include <cuda.h>

#include "sm100.cuh"
#include "topk_select.cuh"

#include <type_traits>

namespace dsa {
namespace idx_tc {

using namespace sm100;

constexpr int kHI = 8;            // indexer heads
constexpr int kDI = 128;          // indexer width (bytes per row, e4m3)
constexpr int kRows = 32;         // query rows per CTA (N = 32 * 8 = 256)
constexpr int kN = kRows * kHI;
constexpr int kKeys = 128;        // keys per tile (M)
constexpr int kStages = 6;
constexpr int kThreads = 640;            // 20 warps: TMA, MMA, 2 idle, 16 epilogue
constexpr int kQBytes = kN * kDI;             // 32 KB
constexpr int kTileBytes = kKeys * kDI;       // 16 KB
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffW = kOffK + kStages * kTileBytes;    // [32][8] fp32 head weights
constexpr int kOffTau = kOffW + kRows * kHI * 4;      // [32] thresholds
constexpr int kOffCnt = kOffTau + kRows * 4;          // [32] candidate counters
constexpr int kOffBar = kOffCnt + kRows * 4;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;              // two buffers of 256 columns

enum : int { B_Q = 0, B_KFULL = 1, B_KEMPTY = 1 + kStages, B_DFULL = 1 + 2 * kStages,
             B_DEMPTY = 3 + 2 * kStages, B_DRAIN = 5 + 2 * kStages, B_COUNT = 6 + 2 * kStages };

static_assert(kOffK % 1024 == 0 && kTileBytes % 1024 == 0, "alignment");
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kThreads == 32 * (4 + 16), "four role warps + four epilogue groups of four warps");

// Sampling: every kSampleStride-th key tile is scored in the sample pass; a
// row keeps about kAlpha * k candidates in the filter pass.
constexpr int kSampleStride = 32;
constexpr int kAlpha = 2;

struct ScanArgs {
    const float* w;       // [T, 8]
    int T, S, k;
    int row0;             // first query row of this launch
    int rows;             // rows in this launch
    // sample mode
    float* samp;          // [rows, samp_ld]
    int samp_ld;
    // filter mode
    const float* tau;     // [rows]
    uint2* cand;          // [rows, cap]
    int* cnt;             // [rows]
    int cap;
};

__host__ __device__ inline int num_tiles(int n) { return (n + kKeys - 1) / kKeys; }

template <bool kSample>
__global__ void __launch_bounds__(kThreads, 1)
indexer_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    ScanArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + kOffBar;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sgen + kOffBar + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kOffBar + 8 * B_COUNT + 8);
    float* w_s = reinterpret_cast<float*>(sgen + kOffW);
    float* tau_s = reinterpret_cast<float*>(sgen + kOffTau);
    int* cnt_s = reinterpret_cast<int*>(sgen + kOffCnt);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = (a.rows + kRows - 1) / kRows;
    const int tile_id = tiles - 1 - (int)blockIdx.x;          // long rows first
    const int r0 = tile_id * kRows;                            // first row (launch-relative)
    const int t0 = a.row0 + r0;
    const int shift = a.S - a.T;                               // pos[t] = t + shift
    const int t_last = min(a.T - 1, t0 + kRows - 1);
    const int n_max = min(a.S, t_last + shift + 1);
    // rows with n <= k need no scores (every candidate is selected)
    const bool needed = n_max > a.k;
    const int NK = needed ? num_tiles(n_max) : 0;
    const int NIT = kSample ? (NK + kSampleStride - 1) / kSampleStride : NK;

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B_KFULL + s), 1);
            mbar_init(bar(B_KEMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_DFULL + b), 1);
            mbar_init(bar(B_DEMPTY + b), 8);   // two groups of four warps per buffer
        }
        mbar_init(bar(B_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init_cluster();
    }
    for (int e = threadIdx.x; e < kRows * kHI; e += kThreads) {
        const int t = t0 + e / kHI;
        w_s[e] = t < a.T ? a.w[(size_t)t * kHI + (e % kHI)] : 0.f;
    }
    if (threadIdx.x < kRows) {
        const int r = r0 + threadIdx.x;
        tau_s[threadIdx.x] = (!kSample && r < a.rows) ? a.tau[r] : 0.f;
        cnt_s[threadIdx.x] = 0;
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(taddr_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_slot;
    const uint32_t qs = sbase + kOffQ;
    const int tile_step = kSample ? kSampleStride : 1;

    if (warp == 0) {
        // ------------------------------------------------------------- TMA
        if (lane == 0 && NIT > 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            mbar_arrive_expect_tx(bar(B_Q), kQBytes);
            tma_load_2d(qs, &tm_q, 0, t0 * kHI, bar(B_Q));
            for (int it = 0; it < NIT; ++it) {
                const int st = it % kStages;
                if (it >= kStages &&
                    !mbar_wait(bar(B_KEMPTY + st), ((it - kStages) / kStages) & 1, abort_flag, 100 + B_KEMPTY, it))
                    break;
                mbar_arrive_expect_tx(bar(B_KFULL + st), kTileBytes);
                tma_load_2d(sbase + kOffK + st * kTileBytes, &tm_k, 0, it * tile_step * kKeys,
                            bar(B_KFULL + st));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0 && NIT > 0) {
            const uint32_t id = idesc_e4m3(kKeys, kN);
            bool ok = mbar_wait(bar(B_Q), 0, abort_flag, B_Q, 0);
            for (int it = 0; ok && it < NIT; ++it) {
                const int st = it % kStages, g = it & 1;
                ok = mbar_wait(bar(B_KFULL + st), (it / kStages) & 1, abort_flag, B_KFULL, it);
                if (ok && it >= 2) ok = mbar_wait(bar(B_DEMPTY + g), ((it - 2) >> 1) & 1, abort_flag, B_DEMPTY, it);
                if (!ok) break;
                tc_fence_after();
                const uint32_t ks = sbase + kOffK + st * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kDI / 32; ++kk) {
                    const uint64_t ad = smem_desc(ks + kk * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = smem_desc(qs + kk * 32, 16, 1024, kSwizzle128B);
                    mma_f8_ss(tmem + g * 256, ad, bd, id, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(B_DFULL + g));
                mma_commit(bar(B_KEMPTY + st));
            }
            mma_commit(bar(B_DRAIN));
            const uint64_t t0n = globaltimer_ns();
            while (!mbar_try_wait(bar(B_DRAIN), 0) && globaltimer_ns() - t0n < kWaitLimitNs) {
            }
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------- epilogue
        const int grp = (warp - 4) >> 2;                   // epilogue group 0..3
        const int g = grp >> 1;                            // TMEM buffer / tile parity
        const int rh = grp & 1;                            // row half: rows [16rh, 16rh+16)
        const int key_lane = (warp & 3) * 32 + lane;       // key within the tile
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        for (int it = g; it < NIT; it += 2) {
            const bool got = mbar_wait(bar(B_DFULL + g), (it >> 1) & 1, abort_flag, 200 + B_DFULL, it);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const int s = it * tile_step * kKeys + key_lane;     // this thread's key
            // every row of the CTA exists and sees every key of this warp: no
            // per-row validity test (the common case on long rows)
            const bool full = r0 + kRows <= a.rows &&
                              it * tile_step * kKeys + (warp & 3) * 32 + 31 <= t0 + shift;
            // eight rows at a time: two TMEM loads (4 rows x 8 heads each), the
            // weighted ReLU head-sums, then the rows' mask / sample / filter step
#pragma unroll 1
            for (int q8 = 4 * rh; q8 < 4 * rh + 4; q8 += 2) {
                uint32_t v0[32], v1[32];
                tmem_ld32(tmem + lane_addr + g * 256 + q8 * 32, v0);
                tmem_ld32(tmem + lane_addr + g * 256 + q8 * 32 + 32, v1);
                tmem_wait_ld();
                if (q8 == 4 * rh + 2) {
                    // every column of this buffer has been read: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_DEMPTY + g));
                }
                auto rows8 = [&](auto full_tag) {
                    constexpr bool kFull = decltype(full_tag)::value;
                    float accs[8];
                    uint32_t pass = 0u;                        // bit rr: row q8 * 4 + rr passes
#pragma unroll
                    for (int rr = 0; rr < 8; ++rr) {
                        const uint32_t* v = rr < 4 ? v0 : v1;
                        const int rb = (rr & 3) * 8;
                        const int r = q8 * 4 + rr;
                        const float4 wa = *reinterpret_cast<const float4*>(w_s + r * kHI);
                        const float4 wb = *reinterpret_cast<const float4*>(w_s + r * kHI + 4);
                        float acc = wa.x * fmaxf(__uint_as_float(v[rb + 0]), 0.f);
                        acc = fmaf(wa.y, fmaxf(__uint_as_float(v[rb + 1]), 0.f), acc);
                        acc = fmaf(wa.z, fmaxf(__uint_as_float(v[rb + 2]), 0.f), acc);
                        acc = fmaf(wa.w, fmaxf(__uint_as_float(v[rb + 3]), 0.f), acc);
                        acc = fmaf(wb.x, fmaxf(__uint_as_float(v[rb + 4]), 0.f), acc);
                        acc = fmaf(wb.y, fmaxf(__uint_as_float(v[rb + 5]), 0.f), acc);
                        acc = fmaf(wb.z, fmaxf(__uint_as_float(v[rb + 6]), 0.f), acc);
                        acc = fmaf(wb.w, fmaxf(__uint_as_float(v[rb + 7]), 0.f), acc);
                        const int rl = r0 + r;                   // launch-relative row
                        const int t = t0 + r;
                        const bool valid = kFull || (rl < a.rows && t < a.T && s <= t + shift && s < a.S);
                        if (kSample) {
                            if (kFull || rl < a.rows)
                                a.samp[(size_t)rl * a.samp_ld + it * kKeys + key_lane] = valid ? acc : -INFINITY;
                        } else {
                            accs[rr] = acc;
                            if (valid && acc >= tau_s[r]) pass |= 1u << rr;
                        }
                    }
                    // the rows' appends, once per eight rows (about 3% of the
                    // pairs pass on long rows)
                    if (!kSample) {
                        while (pass) {
                            const int rr = __ffs(pass) - 1;
                            pass &= pass - 1u;
                            const int r = q8 * 4 + rr;
                            const int slot = atomicAdd(&cnt_s[r], 1);
                            if (slot < a.cap)
                                a.cand[(size_t)(r0 + r) * a.cap + slot] =
                                    make_uint2(__float_as_uint(accs[rr]), (uint32_t)s);
                        }
                    }
                };
                if (full) rows8(std::true_type{}); else rows8(std::false_type{});
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (!kSample && threadIdx.x < kRows && r0 + (int)threadIdx.x < a.rows)
        a.cnt[r0 + threadIdx.x] = needed ? cnt_s[threadIdx.x] : -1;
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Number of sampled keys (s <= pos) of a row with n candidates.
__device__ __forceinline__ int sampled_valid(int n)
{
    int m = 0;
    for (int j = 0; j * kSampleStride * kKeys < n; ++j) m += min(kKeys, n - j * kSampleStride * kKeys);
    return m;
}

// tau_t: the r-th largest sampled score with r = ceil(alpha * k * m / n),
// rounded down to its order key's top 16 bits (two radix passes; the
// threshold only steers how many candidates the filter keeps, which it
// raises by about a hundredth); rows that can keep every candidate get -inf.
// The row's samples are staged in shared memory (dynamic, samp_ld floats).
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
indexer_tau_kernel(const float* __restrict__ samp, int samp_ld, int T, int S, int k, int row0,
                   float* __restrict__ tau)
{
    __shared__ SelectSmem<THREADS> sm;
    extern __shared__ float samp_s[];
    const int rl = blockIdx.x;
    const int t = row0 + rl;
    const int n = min(S, t + (S - T) + 1);
    float out = -INFINITY;
    if (n > kAlpha * k) {
        const int m = sampled_valid(n);
        const long long r = ((long long)kAlpha * k * m + n - 1) / n;
        const int stored = ((num_tiles(n) + kSampleStride - 1) / kSampleStride) * kKeys;
        if (r < m) {
            const float4* src = reinterpret_cast<const float4*>(samp + (size_t)rl * samp_ld);
            for (int i = threadIdx.x; i < stored / 4; i += THREADS) reinterpret_cast<float4*>(samp_s)[i] = src[i];
            __syncthreads();
            int take_eq, count_eq;
            const uint32_t kth = radix_kth_key<THREADS>(SmemScores{samp_s, 0}, stored, (int)r, sm, &take_eq,
                                                        &count_eq, 2);
            out = key_score(kth);
        }
    }
    if (threadIdx.x == 0) tau[rl] = out;
}

// Exact score recomputation for rows whose candidate buffer cannot be used.
struct RecomputedScores {
    const float* qf;      // [8][128] fp32 (shared memory)
    const float* wf;      // [8]
    const uint8_t* keys;  // row 0 of this sequence
    __device__ uint32_t key(int i) const
    {
        const uint4* kr = reinterpret_cast<const uint4*>(keys + (size_t)i * kDI);
        float dot[kHI];
#pragma unroll
        for (int j = 0; j < kHI; ++j) dot[j] = 0.f;
#pragma unroll 2
        for (int c = 0; c < kDI / 16; ++c) {
            const uint4 x = __ldg(kr + c);
            const uint32_t wds[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 lo = e4m3x2_to_float2((uint16_t)(wds[h] & 0xFFFFu));
                const float2 hi = e4m3x2_to_float2((uint16_t)(wds[h] >> 16));
                const int d = c * 16 + h * 4;
#pragma unroll
                for (int j = 0; j < kHI; ++j) {
                    const float* qj = qf + j * kDI + d;
                    dot[j] = fmaf(qj[0], lo.x, fmaf(qj[1], lo.y, fmaf(qj[2], hi.x, fmaf(qj[3], hi.y, dot[j]))));
                }
            }
        }
        float sc = 0.f;
#pragma unroll
        for (int j = 0; j < kHI; ++j) sc = fmaf(wf[j], fmaxf(dot[j], 0.f), sc);
        return score_key(sc);
    }
    __device__ __forceinline__ int s(int i) const { return i; }
};

// Candidate buffer of a row viewed as one array.
struct CandScores {
    const uint2* p;    // the row's candidate pairs
    __device__ __forceinline__ uint32_t key(int i) const { return score_key(__uint_as_float(p[i].x)); }
    __device__ __forceinline__ int s(int i) const { return (int)p[i].y; }
};

// The candidates arrive in no fixed order (appended by the scan's atomics), so
// the selected set is not written in the order it is found: each selected s
// sets its bit in a shared-memory bitmap over the row's keys (dynamic shared
// memory, bitmap_words words), and the row is written from the bitmap in
// ascending s, deterministically (attention over it then sums in a fixed
// order). A row longer than the bitmap sorts its k values instead
// (bitmap_words >= k required for that buffer).
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
indexer_select_kernel(const uint2* __restrict__ cand, const int* __restrict__ cnt, int cap,
                      const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                      const uint8_t* __restrict__ k_idx, int T, int S, int k, int row0,
                      int32_t* __restrict__ idx, int bitmap_words)
{
    __shared__ SelectSmem<THREADS> sm;
    extern __shared__ uint32_t bitmap[];
    __shared__ float qf[kHI * kDI];
    __shared__ float wf[kHI];
    const int rl = blockIdx.x;
    const int t = row0 + rl;
    const int n = min(S, t + (S - T) + 1);
    int32_t* out = idx + (size_t)t * k;
    if (n <= k) {
        for (int i = threadIdx.x; i < k; i += THREADS) out[i] = i < n ? i : -1;
        return;
    }
    const int c = cnt[rl];
    if (c >= k && c <= cap) {
        const CandScores row{cand + (size_t)rl * cap};
        if (n <= bitmap_words * 32) {
            for (int i = threadIdx.x; i < (n + 31) / 32; i += THREADS) bitmap[i] = 0u;
            __syncthreads();
            if (!range_select_bitmap<THREADS>(row, c, k, bitmap, sm))
                block_select<THREADS>(row, c, k,
                                      [&](int, int i) {
                                          const int s = row.s(i);
                                          atomicOr(&bitmap[s >> 5], 1u << (s & 31));
                                      },
                                      sm);
            __syncthreads();
            block_emit_bitmap<THREADS>(bitmap, n, out, reinterpret_cast<int*>(sm.hist[0]));
        } else {
            int* sel = reinterpret_cast<int*>(bitmap);
            block_select<THREADS>(row, c, k, [&](int slot, int i) { sel[slot] = row.s(i); }, sm);
            __syncthreads();
            block_sort_ascending(sel, k, pow2_ceil(k));
            for (int i = threadIdx.x; i < k; i += THREADS) out[i] = sel[i];
        }
        return;
    }
    // threshold too high (fewer than k candidates) or buffer overflow: exact
    for (int e = threadIdx.x; e < kHI * kDI; e += THREADS) {
        const uint8_t b = q_idx[(size_t)t * kHI * kDI + e];
        qf[e] = e4m3x2_to_float2((uint16_t)b).x;
    }
    if (threadIdx.x < kHI) wf[threadIdx.x] = w[(size_t)t * kHI + threadIdx.x];
    __syncthreads();
    block_topk<THREADS>(RecomputedScores{qf, wf, k_idx}, n, k, out, sm);
}

}  // namespace idx_tc
}  // namespace dsa
