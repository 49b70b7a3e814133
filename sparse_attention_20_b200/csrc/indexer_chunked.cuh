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
// count, and for a row short of it selects the exact Top-k of the whole row
// from scores it recomputes itself. The result is the row's exact Top-k
// either way.
//
// Work items (row, chunk) are numbered through a per-row prefix of chunk
// counts computed on the device, so a fixed grid of persistent CTAs covers
// rows of any length mix without empty blocks.
#pragma once
#include "common.cuh"
#include "indexer_scores.cuh"
#include "sm100.cuh"
#include "topk_select.cuh"

namespace dsa {
namespace idx_chunk {

constexpr int kChunkKeys = 8192;
constexpr int kThreads = 512;
constexpr int kCtasPerSm = 2;
constexpr int kMergeThreads = 1024;
constexpr int kMergeSmemPairs = 8192;   // 64 KB of staged (score, s) pairs
constexpr int kPlanThreads = 1024;
constexpr int kTauSmemSamples = 6144;   // rows up to 24 chunks stage their samples
constexpr size_t kSmemBytes = kChunkKeys * sizeof(float) + sizeof(SelectSmem<kThreads>);
// sampling: tiles of 128 keys, every 32nd tile of a row (two per chunk)
constexpr int kSampleTile = 128;
constexpr int kSampleStride = 32 * kSampleTile;
constexpr int kSamplesPerChunk = kChunkKeys / kSampleStride * kSampleTile;
constexpr int kAlpha = 2;   // tau aims at about kAlpha * k entries of the row

__device__ __forceinline__ int row_chunks(int n) { return n <= kChunkKeys ? 1 : ceil_div(n, kChunkKeys); }

// work_off[r] = number of work items of rows row0 .. row0+r-1, r = 0..rows.
__global__ void __launch_bounds__(kPlanThreads)
chunk_plan_kernel(const int* __restrict__ pos, const int* __restrict__ k_base, int T, int S, int row0,
                  int rows, int* __restrict__ work_off, const PagedRows pg)
{
    __shared__ int part[kPlanThreads];
    griddep_wait();
    const int per = ceil_div(rows, kPlanThreads);
    const int r0 = threadIdx.x * per, r1 = min(rows, r0 + per);
    auto items = [&](int r) -> int {
        long long base;
        const int* bt;
        return row_chunks(row_keys(pg, pos, k_base, row0 + r, T, S, &base, &bt));
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

// Number of sampled positions inside a row of n keys.
__device__ __forceinline__ int row_samples(int n)
{
    const int full = n / kSampleStride;
    return full * kSampleTile + min(kSampleTile, n - full * kSampleStride);
}

// One CTA per row: the work plan of the chunk kernel (block 0, as
// chunk_plan_kernel), then the row's sampled scores (every 32nd 128-key tile)
// and its threshold tau[r] = the order key of the sample of rank
// ceil(kAlpha * k * m / n) (m valid samples), or 0 (no filtering) where that
// rank is out of reach. The samples of a row of up to 24 chunks (196608 keys,
// every decode row of the 128K workload) stay in shared memory; a longer
// row's go to samp[r * samp_ld ...] in global memory.
constexpr int kFusedTauThreads = 512;

template <int NT, int DI>
__global__ void __launch_bounds__(kFusedTauThreads)
chunk_sample_tau_kernel(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                        const uint8_t* __restrict__ k_idx, const int* __restrict__ pos,
                        const int* __restrict__ k_base, int T, int S, int H_I, int row0, int rows, int k,
                        int* __restrict__ work_off, float* __restrict__ samp, long long samp_ld,
                        uint32_t* __restrict__ tau, const PagedRows pg)
{
    __shared__ SelectSmem<kFusedTauThreads> sm;
    __shared__ float ss[kTauSmemSamples];
    __shared__ int part[kFusedTauThreads];
    griddep_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tid4 = lane & 3;
    if (blockIdx.x == 0) {
        // work_off[r] = work items of rows row0 .. row0+r-1 (chunk_plan_kernel)
        const int per = ceil_div(rows, kFusedTauThreads);
        const int a0 = threadIdx.x * per, a1 = min(rows, a0 + per);
        auto items = [&](int r) -> int {
            long long base;
            const int* bt;
            return row_chunks(row_keys(pg, pos, k_base, row0 + r, T, S, &base, &bt));
        };
        int sum = 0;
        for (int r = a0; r < a1; ++r) sum += items(r);
        part[threadIdx.x] = sum;
        __syncthreads();
        for (int off = 1; off < kFusedTauThreads; off <<= 1) {
            const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
            __syncthreads();
            part[threadIdx.x] += v;
            __syncthreads();
        }
        int acc = part[threadIdx.x] - sum;
        for (int r = a0; r < a1; ++r) {
            work_off[r] = acc;
            acc += items(r);
        }
        if (threadIdx.x == kFusedTauThreads - 1) work_off[rows] = part[kFusedTauThreads - 1];
    }
    const int r = blockIdx.x, t = row0 + r;
    long long base;
    const int* bt;
    const int n = row_keys(pg, pos, k_base, t, T, S, &base, &bt);
    const int nchunks = row_chunks(n);
    const int m = row_samples(n);
    const long long want = ((long long)kAlpha * k * m + n - 1) / n;
    const int n_s = nchunks * kSamplesPerChunk;
    if (nchunks < 2 || want >= m || want >= n_s) {
        if (threadIdx.x == 0) tau[r] = 0u;
        return;
    }
    float* dst = n_s <= kTauSmemSamples ? ss : samp + (size_t)r * samp_ld;
    // sample position j: chunk j / 256, tile (j % 256) / 128 of the chunk's
    // every-32nd tiles, key j % 128; each warp scores 16 consecutive positions
    // per step, with the loads of two steps issued before their MMAs
    QueryFrag<NT, DI> qf;
    qf.load(q_idx, w, t, H_I, lane);
    constexpr int kStep = 16 * (kFusedTauThreads / 32);
    auto key_of = [&](int j) -> int {
        const int c = j / kSamplesPerChunk, jj = j % kSamplesPerChunk;
        return c * kChunkKeys + (jj / kSampleTile) * kSampleStride + jj % kSampleTile;
    };
    for (int j0 = warp * 16; j0 < n_s; j0 += 2 * kStep) {
        KeyQuarter<DI> A[2], B[2];
        int sa[2], sb[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int ja = j0 + u * kStep + gid;
            sa[u] = ja < n_s ? key_of(ja) : n;
            sb[u] = ja + 8 < n_s ? key_of(ja + 8) : n;
            if (sa[u] < n) A[u].load(k_idx + (size_t)key_row(pg, bt, base, sa[u]) * DI + tid4 * (DI / 4)); else A[u].zero();
            if (sb[u] < n) B[u].load(k_idx + (size_t)key_row(pg, bt, base, sb[u]) * DI + tid4 * (DI / 4)); else B[u].zero();
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float ia, ib;
            qf.score(A[u], B[u], ia, ib);
            const int ja = j0 + u * kStep + gid;
            if (tid4 == 0) {
                if (ja < n_s) dst[ja] = sa[u] < n ? ia : -INFINITY;
                if (ja + 8 < n_s) dst[ja + 8] = sb[u] < n ? ib : -INFINITY;
            }
        }
    }
    __syncthreads();
    int take_eq, count_eq;
    const uint32_t key = radix_kth_key<kFusedTauThreads>(DenseScores{dst}, n_s, (int)want, sm, &take_eq, &count_eq);
    if (threadIdx.x == 0) tau[r] = key;
}

// Keeps the pairs of chunk c0.. of local row r (scores sc[0..m)) and writes
// their count; a single-chunk row instead writes its final indices.
template <int THREADS>
__device__ __forceinline__ void chunk_keep(const float* sc, int m, int c0, int chunk, int nchunks, int r,
                                           int t, int k, uint32_t tk, uint2* __restrict__ cand,
                                           long long cand_ld, int* __restrict__ ccnt, int max_chunks,
                                           int32_t* __restrict__ idx, SelectSmem<THREADS>& sm)
{
    if (nchunks == 1) {
        block_topk<THREADS>(SmemScores{sc, 0}, m, k, idx + (size_t)t * k, sm);
        return;
    }
    uint2* out = cand + (size_t)r * cand_ld + (size_t)chunk * k;
    auto emit = [&](int slot, int i) { out[slot] = make_uint2(__float_as_uint(sc[i]), (uint32_t)(c0 + i)); };
    // entries >= tau in s order (all entries when tau is 0)
    int kept = block_emit_if<THREADS>(m, [&](int i) { return score_key(sc[i]) >= tk; }, emit, k, sm);
    if (kept > k) {
        // more than k pass: the chunk's own Top-k
        block_select<THREADS>(SmemScores{sc, c0}, m, k, emit, sm);
        kept = k;
    }
    if (threadIdx.x == 0) ccnt[(size_t)r * max_chunks + chunk] = kept;
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
    // contiguous key ranges only (a paged cache takes the TMA kernel below)
    extern __shared__ __align__(16) uint8_t smem[];
    float* sc = reinterpret_cast<float*>(smem);
    SelectSmem<kThreads>& sm = *reinterpret_cast<SelectSmem<kThreads>*>(smem + kChunkKeys * sizeof(float));
    const int lane = threadIdx.x & 31, tid4 = lane & 3;
    griddep_wait();
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
        chunk_keep<kThreads>(sc, m, c0, chunk, nchunks, r, t, k, tau ? tau[r] : 0u, cand, cand_ld, ccnt,
                             max_chunks, idx, sm);
        __syncthreads();   // sc and sm are reused by the next item
    }
}

// d_I = 128: the same work with the key rows streamed by TMA (128-key tiles,
// 128B-swizzled, a 4-stage ring per CTA) so that many tiles are in flight
// without holding registers. Warps 0-7 score (16 keys each per tile), warp 8
// issues the copies; all nine take part in the selection.
namespace tma {
constexpr int kTileKeys = 128;
constexpr int kTileBytes = kTileKeys * 128;
constexpr int kStages = 4;
constexpr int kScoreWarps = 8;
constexpr int kThreads = (kScoreWarps + 1) * 32;
constexpr int kCtasPerSm = 2;
constexpr int kOffScores = kStages * kTileBytes;
constexpr int kOffSel = kOffScores + kChunkKeys * 4;
constexpr int kOffBar = kOffSel + (int)((sizeof(SelectSmem<kThreads>) + 15) / 16 * 16);
constexpr int kSmemBytes = kOffBar + 128 + 1024;   // + alignment slack
enum : int { B_FULL = 0, B_EMPTY = kStages, B_COUNT = 2 * kStages };
static_assert(kTileKeys == kScoreWarps * 16, "one 16-key MMA block per scoring warp and tile");
}  // namespace tma

template <int NT>
__global__ void __launch_bounds__(tma::kThreads, tma::kCtasPerSm)
chunk_topk_tma_kernel(const __grid_constant__ CUtensorMap tm_k, const uint8_t* __restrict__ q_idx,
                      const float* __restrict__ w, const int* __restrict__ pos,
                      const int* __restrict__ k_base, int T, int S, int H_I, int row0, int rows, int k,
                      const int* __restrict__ work_off, const uint32_t* __restrict__ tau,
                      uint2* __restrict__ cand, long long cand_ld, int* __restrict__ ccnt, int max_chunks,
                      int32_t* __restrict__ idx, const PagedRows pg)
{
    // tm_k boxes: 128 key rows (contiguous ranges) or 64 (paged cache: a tile
    // is two half-tiles, each inside one page of a multiple of 64 keys)
    using namespace sm100;
    constexpr int DI = 128;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    float* sc = reinterpret_cast<float*>(sgen + tma::kOffScores);
    SelectSmem<tma::kThreads>& sm = *reinterpret_cast<SelectSmem<tma::kThreads>*>(sgen + tma::kOffSel);
    const uint32_t bar0 = sbase + tma::kOffBar;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + tma::kOffBar + 8 * tma::B_COUNT);
    int* stop_s = reinterpret_cast<int*>(sgen + tma::kOffBar + 8 * tma::B_COUNT + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tid4 = lane & 3;

    if (threadIdx.x == 0) {
        for (int s = 0; s < tma::kStages; ++s) {
            mbar_init(bar(tma::B_FULL + s), 1);
            mbar_init(bar(tma::B_EMPTY + s), tma::kScoreWarps);
        }
        *abort_flag = 0;
        fence_mbar_init_cluster();
        prefetch_tmap(&tm_k);
    }
    __syncthreads();
    griddep_wait();
    const int total = work_off[rows];
    struct Item {
        int r, t, chunk, n, nchunks, c0, m, ntiles;
        long long base;
        const int* bt;
    };
    auto item_info = [&](int item) {
        Item it;
        it.r = item_row(work_off, rows, item);
        it.t = row0 + it.r;
        it.chunk = item - work_off[it.r];
        it.n = row_keys(pg, pos, k_base, it.t, T, S, &it.base, &it.bt);
        it.nchunks = row_chunks(it.n);
        it.c0 = it.chunk * kChunkKeys;
        it.m = min(it.n - it.c0, kChunkKeys);   // 0 for an empty row
        it.ntiles = ceil_div(max(it.m, 0), tma::kTileKeys);
        return it;
    };
    // Copy warp: tiles [j0, j1) of item `it`, whose first tile is ring
    // position g0 of this CTA.
    auto issue = [&](const Item& it, int g0, int j0, int j1) -> bool {
        for (int j = j0; j < j1; ++j) {
            const int g = g0 + j, st = g % tma::kStages;
            if (g >= tma::kStages &&
                !mbar_wait(bar(tma::B_EMPTY + st), ((g - tma::kStages) / tma::kStages) & 1, abort_flag,
                           600 + tma::B_EMPTY, j))
                return false;
            mbar_arrive_expect_tx(bar(tma::B_FULL + st), tma::kTileBytes);
            const int s0 = it.c0 + j * tma::kTileKeys;
            if (it.bt) {
                tma_load_2d(sbase + st * tma::kTileBytes, &tm_k, 0, (int)key_row(pg, it.bt, 0, s0),
                            bar(tma::B_FULL + st));
                // a second half that starts past the row's keys reloads the
                // first half (never scored) instead of naming a page the row
                // does not have
                const int s1 = s0 + tma::kTileKeys / 2 < it.n ? s0 + tma::kTileKeys / 2 : s0;
                tma_load_2d(sbase + st * tma::kTileBytes + tma::kTileBytes / 2, &tm_k, 0,
                            (int)key_row(pg, it.bt, 0, s1), bar(tma::B_FULL + st));
            } else {
                tma_load_2d(sbase + st * tma::kTileBytes, &tm_k, 0, (int)(it.base + s0), bar(tma::B_FULL + st));
            }
        }
        return true;
    };
    const bool producer = warp == tma::kScoreWarps && lane == 0;
    int gt = 0;   // tiles of this CTA so far (ring position and phase)
    // the first tiles of each item are issued ahead, while the previous item
    // is still being selected
    if (producer && (int)blockIdx.x < total) {
        const Item it = item_info(blockIdx.x);
        issue(it, 0, 0, min(it.ntiles, tma::kStages));
    }
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Item it = item_info(item);
        if (warp == tma::kScoreWarps) {
            if (lane == 0) issue(it, gt, min(it.ntiles, tma::kStages), it.ntiles);
        } else {
            QueryFrag<NT, DI> qf;
            qf.load(q_idx, w, it.t, H_I, lane);
            const int ra = warp * 16 + gid, rb = ra + 8;   // tile rows; both are gid mod 8
            for (int j = 0; j < it.ntiles; ++j) {
                const int g = gt + j, st = g % tma::kStages;
                const bool got = mbar_wait(bar(tma::B_FULL + st), (g / tma::kStages) & 1, abort_flag,
                                           600 + tma::B_FULL, j);
                if (!__all_sync(0xffffffffu, got)) break;
                const uint32_t ts = sbase + st * tma::kTileBytes;
                KeyQuarter<DI> A, B;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // 16-byte chunk 2*tid4+h of the row, 128B swizzle: chunk ^ (row & 7)
                    const uint32_t col = (uint32_t)(((2 * tid4 + h) ^ gid) << 4);
                    const uint4 va = ld_shared_v4(ts + ra * 128 + col);
                    const uint4 vb = ld_shared_v4(ts + rb * 128 + col);
                    A.v[4 * h] = va.x; A.v[4 * h + 1] = va.y; A.v[4 * h + 2] = va.z; A.v[4 * h + 3] = va.w;
                    B.v[4 * h] = vb.x; B.v[4 * h + 1] = vb.y; B.v[4 * h + 2] = vb.z; B.v[4 * h + 3] = vb.w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(tma::B_EMPTY + st));
                float ia, ib;
                qf.score(A, B, ia, ib);
                const int a = j * tma::kTileKeys + ra, b = a + 8;
                if (tid4 == 0) {
                    if (a < it.m) sc[a] = ia;
                    if (b < it.m) sc[b] = ib;
                }
            }
        }
        gt += it.ntiles;
        __syncthreads();
        if (threadIdx.x == 0) *stop_s = *abort_flag;
        __syncthreads();
        if (*stop_s) break;
        if (producer && item + (int)gridDim.x < total) {
            // every stage is free now: start the next item's copies
            const Item nx = item_info(item + gridDim.x);
            issue(nx, gt, 0, min(nx.ntiles, tma::kStages));
        }
        chunk_keep<tma::kThreads>(sc, it.m, it.c0, it.chunk, it.nchunks, it.r, it.t, k, tau ? tau[it.r] : 0u,
                                  cand, cand_ld, ccnt, max_chunks, idx, sm);
        __syncthreads();   // sc and sm are reused by the next item
    }
}

// Few rows with long key ranges (decode): the rows' key tiles are concatenated
// and cut into equal contiguous ranges, one per CTA, so the key stream has no
// item boundaries, no per-item selection and at most a handful of row changes
// per CTA. Every key of a row is scored into a dense score row
// (scores[r * ld + s]) together with the largest order key of each group of
// 16 scores (gmax16[r * g16_ld + 8 * tile + warp]: one group per scoring warp
// and tile) and of each group of 4 (gmax4[r * g4_ld + 32 * tile + 4 * warp +
// q]: keys gid, gid + 1, gid + 8, gid + 9 of the warp's 16, q = gid / 2).
// The row's Top-k is selected afterwards from these
// (row_select_cluster_kernel). Rows with at most k keys, or more than
// kMaxKeys, get no tiles here (the select writes the former directly and
// recomputes the latter's scores).
namespace rs {
constexpr int kTileKeys = 128;
constexpr int kTileBytes = kTileKeys * 128;
constexpr int kStages = 6;
constexpr int kScoreWarps = 8;
constexpr int kThreads = (kScoreWarps + 1) * 32;
constexpr int kCtasPerSm = 2;
constexpr int kMaxRows = 2048;        // rows per launch: the tile table lives in shared memory
constexpr int kMaxKeys = 1 << 20;     // longest row scored into the workspace
constexpr int kGroupsPerTile = kScoreWarps;   // 16-key groups per tile
constexpr int kOffTable = kStages * kTileBytes;
constexpr int kOffBar = kOffTable + (kMaxRows + 1 + 3) / 4 * 16;
constexpr int kSmemBytes = kOffBar + 128 + 1024;   // + alignment slack
enum : int { B_FULL = 0, B_EMPTY = kStages, B_COUNT = 2 * kStages };
static_assert(kTileKeys == kScoreWarps * 16, "one 16-key MMA block per scoring warp and tile");
static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");

// Tiles of a row of n keys on this path.
__device__ __forceinline__ int row_tiles(int n, int k)
{
    return n > k && n <= kMaxKeys ? ceil_div(n, kTileKeys) : 0;
}
}  // namespace rs

template <int NT>
__global__ void __launch_bounds__(rs::kThreads, rs::kCtasPerSm)
row_scores_tma_kernel(const __grid_constant__ CUtensorMap tm_k, const uint8_t* __restrict__ q_idx,
                      const float* __restrict__ w, const int* __restrict__ pos,
                      const int* __restrict__ k_base, int T, int S, int H_I, int row0, int rows, int k,
                      float* __restrict__ scores, long long ld, uint32_t* __restrict__ gmax16,
                      long long g16_ld, uint32_t* __restrict__ gmax4, long long g4_ld, const PagedRows pg)
{
    // tm_k boxes: 128 key rows (contiguous ranges) or 64 (paged cache: a tile
    // is two half-tiles, each inside one page of a multiple of 64 keys)
    using namespace sm100;
    constexpr int DI = 128;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int wsum[rs::kThreads / 32];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    int* tbl = reinterpret_cast<int*>(sgen + rs::kOffTable);
    const uint32_t bar0 = sbase + rs::kOffBar;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + rs::kOffBar + 8 * rs::B_COUNT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tid4 = lane & 3;

    if (threadIdx.x == 0) {
        for (int s = 0; s < rs::kStages; ++s) {
            mbar_init(bar(rs::B_FULL + s), 1);
            mbar_init(bar(rs::B_EMPTY + s), rs::kScoreWarps);
        }
        *abort_flag = 0;
        fence_mbar_init_cluster();
        prefetch_tmap(&tm_k);
    }
    griddep_wait();
    // tbl[r] = tiles of rows 0 .. r-1 (exclusive prefix over the rows)
    auto tiles_of = [&](int r) -> int {
        long long b;
        const int* bt;
        return rs::row_tiles(row_keys(pg, pos, k_base, row0 + r, T, S, &b, &bt), k);
    };
    {
        const int per = ceil_div(rows, rs::kThreads);
        const int a0 = min(rows, (int)threadIdx.x * per), a1 = min(rows, a0 + per);
        int sum = 0;
        for (int r = a0; r < a1; ++r) sum += tiles_of(r);
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int acc = incl - sum, total = 0;
#pragma unroll
        for (int q = 0; q < rs::kThreads / 32; ++q) {
            if (q < warp) acc += wsum[q];
            total += wsum[q];
        }
        for (int r = a0; r < a1; ++r) {
            tbl[r] = acc;
            acc += tiles_of(r);
        }
        if (threadIdx.x == 0) tbl[rows] = total;
        __syncthreads();
    }
    const long long G = tbl[rows];
    const int g0 = (int)(G * blockIdx.x / gridDim.x), g1 = (int)(G * (blockIdx.x + 1) / gridDim.x);
    if (g0 >= g1) return;
    // the row holding tile g: the last r with tbl[r] <= g (rows without tiles
    // share their offset with the next row and are skipped)
    auto row_of = [&](int g) -> int {
        int lo = 0, hi = rows - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tbl[mid] <= g) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    int r = row_of(g0);
    long long base;
    const int* bt;
    int n = row_keys(pg, pos, k_base, row0 + r, T, S, &base, &bt);

    if (warp == rs::kScoreWarps) {
        if (lane != 0) return;
        for (int g = g0; g < g1; ++g) {
            if (g >= tbl[r + 1]) {
                do ++r; while (g >= tbl[r + 1]);
                n = row_keys(pg, pos, k_base, row0 + r, T, S, &base, &bt);
            }
            const int i = g - g0, st = i % rs::kStages;
            if (i >= rs::kStages &&
                !mbar_wait(bar(rs::B_EMPTY + st), ((i - rs::kStages) / rs::kStages) & 1, abort_flag,
                           640 + rs::B_EMPTY, i))
                return;
            mbar_arrive_expect_tx(bar(rs::B_FULL + st), rs::kTileBytes);
            const int s0 = (g - tbl[r]) * rs::kTileKeys;
            const uint32_t dst = sbase + st * rs::kTileBytes;
            if (bt) {
                tma_load_2d(dst, &tm_k, 0, (int)key_row(pg, bt, 0, s0), bar(rs::B_FULL + st));
                // a second half that starts past the row's keys reloads the
                // first half (never scored) instead of naming a page the row
                // does not have
                const int s1 = s0 + rs::kTileKeys / 2 < n ? s0 + rs::kTileKeys / 2 : s0;
                tma_load_2d(dst + rs::kTileBytes / 2, &tm_k, 0, (int)key_row(pg, bt, 0, s1),
                            bar(rs::B_FULL + st));
            } else {
                tma_load_2d(dst, &tm_k, 0, (int)(base + s0), bar(rs::B_FULL + st));
            }
        }
        return;
    }
    QueryFrag<NT, DI> qf;
    qf.load(q_idx, w, row0 + r, H_I, lane);
    const int ra = warp * 16 + gid, rb = ra + 8;   // tile rows; both are gid mod 8
    for (int g = g0; g < g1; ++g) {
        if (g >= tbl[r + 1]) {
            do ++r; while (g >= tbl[r + 1]);
            n = row_keys(pg, pos, k_base, row0 + r, T, S, &base, &bt);
            qf.load(q_idx, w, row0 + r, H_I, lane);
        }
        const int i = g - g0, st = i % rs::kStages;
        const bool got = mbar_wait(bar(rs::B_FULL + st), (i / rs::kStages) & 1, abort_flag, 640 + rs::B_FULL, i);
        if (!__all_sync(0xffffffffu, got)) break;
        const uint32_t ts = sbase + st * rs::kTileBytes;
        KeyQuarter<DI> A, B;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // 16-byte chunk 2*tid4+h of the row, 128B swizzle: chunk ^ (row & 7)
            const uint32_t col = (uint32_t)(((2 * tid4 + h) ^ gid) << 4);
            const uint4 va = ld_shared_v4(ts + ra * 128 + col);
            const uint4 vb = ld_shared_v4(ts + rb * 128 + col);
            A.v[4 * h] = va.x; A.v[4 * h + 1] = va.y; A.v[4 * h + 2] = va.z; A.v[4 * h + 3] = va.w;
            B.v[4 * h] = vb.x; B.v[4 * h + 1] = vb.y; B.v[4 * h + 2] = vb.z; B.v[4 * h + 3] = vb.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(rs::B_EMPTY + st));
        float ia, ib;
        qf.score(A, B, ia, ib);
        const int j = g - tbl[r];
        const int a = j * rs::kTileKeys + ra, b = a + 8;
        uint32_t hi = 0u;   // an empty group's maximum is the smallest key
        if (tid4 == 0) {
            float* out = scores + (size_t)r * ld;
            if (a < n) {
                out[a] = ia;
                hi = max(hi, score_key(ia));
            }
            if (b < n) {
                out[b] = ib;
                hi = max(hi, score_key(ib));
            }
        }
        // lanes 0, 4, ..., 28 hold the values; one step leaves the maxima of
        // four keys (gid, gid + 1 and their rb rows) in lanes 0, 8, 16, 24
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, 4));
        if ((lane & 7) == 0) gmax4[(size_t)r * g4_ld + (size_t)j * 32 + warp * 4 + (lane >> 3)] = hi;
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, 8));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, 16));
        if (lane == 0) gmax16[(size_t)r * g16_ld + (size_t)j * rs::kGroupsPerTile + warp] = hi;
    }
}

// Scores recomputed from the key rows (the merge's exact fallback): q^I of the
// row as fp32 in shared memory, up to 16 heads.
struct RecomputedRow {
    const float* qf;      // [H_I][d_I]
    const float* wf;      // [H_I]
    const uint8_t* k_idx; // the key cache
    PagedRows pg;
    const int* bt;        // the row's block-table line (paged), else NULL
    long long base;       // first key of the row's range (contiguous)
    int H_I, d_I;
    __device__ uint32_t key(int i) const
    {
        const uint8_t* kr = k_idx + (size_t)key_row(pg, bt, base, i) * d_I;
        float dot[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) dot[j] = 0.f;
        for (int c = 0; c < d_I; c += 16) {
            const uint4 x = __ldg(reinterpret_cast<const uint4*>(kr + c));
            const uint32_t wds[4] = {x.x, x.y, x.z, x.w};
            float kf[16];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 lo = e4m3x2_to_float2((uint16_t)(wds[h] & 0xFFFFu));
                const float2 hi = e4m3x2_to_float2((uint16_t)(wds[h] >> 16));
                kf[4 * h] = lo.x; kf[4 * h + 1] = lo.y; kf[4 * h + 2] = hi.x; kf[4 * h + 3] = hi.y;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (j >= H_I) break;
                const float* qj = qf + j * d_I + c;
#pragma unroll
                for (int e = 0; e < 16; ++e) dot[j] = fmaf(qj[e], kf[e], dot[j]);
            }
        }
        float sc = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < H_I) sc = fmaf(wf[j], fmaxf(dot[j], 0.f), sc);
        return score_key(sc);
    }
    __device__ int s(int i) const { return i; }
};

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

// Row Top-k from the chunks' pairs (rows of two or more chunks). Pairs are in
// ascending s, and so is the emitted row. A row whose chunks kept fewer than
// k pairs in all (tau overshot) gets the exact Top-k of all its keys from
// recomputed scores instead. Dynamic shared memory: (max_chunks + 2) ints
// (rounded to even) for the prefix, then kMergeSmemPairs pairs (or the row's
// q^I and w as fp32 for the fallback).
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
merge_topk_kernel(const uint2* __restrict__ cand, long long cand_ld, const int* __restrict__ ccnt,
                  int max_chunks, const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                  const uint8_t* __restrict__ k_idx, int H_I, int d_I, const int* __restrict__ pos,
                  const int* __restrict__ k_base, int T, int S, int row0, int k, int32_t* __restrict__ idx,
                  const PagedRows pg)
{
    __shared__ SelectSmem<THREADS> sm;
    extern __shared__ int pre[];
    griddep_wait();
    const int r = blockIdx.x, t = row0 + r;
    long long base;
    const int* bt;
    const int n = row_keys(pg, pos, k_base, t, T, S, &base, &bt);
    const int nchunks = row_chunks(n);
    if (nchunks < 2) return;
    // chunk counts loaded in parallel, then their prefix
    for (int c = threadIdx.x; c < nchunks; c += THREADS) pre[c + 1] = ccnt[(size_t)r * max_chunks + c];
    __syncthreads();
    if (threadIdx.x == 0) {
        pre[0] = 0;
        for (int c = 0; c < nchunks; ++c) pre[c + 1] += pre[c];
    }
    __syncthreads();
    const int n_pairs = pre[nchunks];
    uint2* ps = reinterpret_cast<uint2*>(pre + ((max_chunks + 2) & ~1));
    if (n_pairs < k) {
        // fewer than k entries passed tau: exact Top-k of the whole row
        float* qf = reinterpret_cast<float*>(ps);
        float* wf = qf + H_I * d_I;
        const uint8_t* qrow = q_idx + (size_t)t * H_I * d_I;
        for (int e = threadIdx.x; e < H_I * d_I; e += THREADS) qf[e] = e4m3x2_to_float2((uint16_t)qrow[e]).x;
        for (int j = threadIdx.x; j < H_I; j += THREADS) wf[j] = w[(size_t)t * H_I + j];
        __syncthreads();
        block_topk<THREADS>(RecomputedRow{qf, wf, k_idx, pg, bt, base, H_I, d_I}, n, k,
                            idx + (size_t)t * k, sm);
        return;
    }
    const ChunkPairs pairs{cand + (size_t)r * cand_ld, pre, nchunks, k};
    if (n_pairs <= kMergeSmemPairs) {
        // gather the kept pairs in chunk order into shared memory first (one
        // flat loop: every load is independent)
#pragma unroll 4
        for (int i = threadIdx.x; i < n_pairs; i += THREADS) ps[i] = pairs.at(i);
        __syncthreads();
        block_topk<THREADS>(PairScores{ps}, n_pairs, k, idx + (size_t)t * k, sm);
    } else {
        block_topk<THREADS>(pairs, n_pairs, k, idx + (size_t)t * k, sm);
    }
}

// Row Top-k from the dense score rows of row_scores_tma_kernel, for rows of
// k < n <= rs::kMaxKeys keys: row_select_cluster_kernel, a cluster of
// kClusterCtas CTAs per row.
//
// Every CTA first takes the row's threshold tau, a lower bound of its k-th
// largest score, from group maxima. With at least k groups, the k-th largest
// group maximum is reached by at least k groups, so by at least k scores: the
// 16-key groups where the row has k of them, else the 4-key groups, else
// tau = 0 (rows of fewer than 4k keys keep everything); range_floor rounds it
// down to a histogram sub-bin edge. Then CTA q streams the q-th contiguous
// part of the score row through a ring of kCsStages shared-memory buffers
// (1-D bulk copies; four of them in the lower half of the pair space, which is
// free until the pairs are gathered) and keeps its scores >= tau as
// (order key, s) pairs in ascending s (a scan over the CTA per two stages).
// The parts' counts are exchanged over distributed shared memory, each part's
// pairs are stored into CTA 0 after the pairs of the parts before it, so
// CTA 0 holds every score
// >= tau in ascending s, and CTA 0 takes their exact Top-k (range-histogram
// select, or the radix select where the keys' spread defeats it), marked in a
// bitmap over the pairs and written in ascending s. Parts that keep more than
// kCsLocal pairs, or more than kCsList in all (scores far from independent),
// send the row to CTA 0's exact select over the score row in global memory.
// A row of at most k keys lists them and pads with -1; a row longer than
// kMaxKeys gets the exact Top-k of scores it recomputes. Every CTA of a
// cluster takes the same path through the cluster barriers.
namespace rs {
constexpr int kMaxStaged = 16384;                          // group maxima staged in the pair space
constexpr int kClusterCtas = 4;
constexpr int kCsThreads = 512;
constexpr int kCsChunk = kCsThreads * 4;                   // scores per copy: one float4 per thread
constexpr int kCsLocal = 4096;                             // pairs one part keeps
constexpr int kCsList = 8192;                              // pairs of the row in CTA 0
constexpr int kOffCsLocal = (kCsList - kCsLocal) * 8;      // a part's pairs: the top of the list space
constexpr int kCsStages = 6;
constexpr int kOffCsBuf = kCsList * 8;                     // chunk buffers 0, 1 (2..5: the pair space)
constexpr int kOffCsBits = kOffCsBuf + 2 * kCsChunk * 4;   // bitmap over CTA 0's list
constexpr int kOffCsBars = kOffCsBits + kCsList / 8;
constexpr int kCsSmem = kOffCsBars + 8 * (kCsStages + 1);
static_assert(kCsLocal * 8 <= kOffCsLocal, "CTA 0 moves its own pairs down without overlap");
static_assert(kMaxStaged * 4 <= kOffCsBuf, "the group maxima fit the pair space");
static_assert((kCsStages - 2) * kCsChunk * 4 <= kOffCsLocal, "buffers 2.. stay below the part's pairs");
// shared-memory offset of ring buffer st
__host__ __device__ constexpr int cs_buf(int st) { return st < 2 ? kOffCsBuf + st * kCsChunk * 4 : (st - 2) * kCsChunk * 4; }
}  // namespace rs

// Pairs staged in shared memory; entry i is marked as bit i.
struct PairList {
    const uint2* p;
    __device__ __forceinline__ uint32_t key(int i) const { return p[i].x; }
    __device__ __forceinline__ int s(int i) const { return i; }
};

// The cluster kernel's rare paths, kept out of line so that its hot loop and
// the common select stay small in the instruction cache.
template <int THREADS>
__device__ __noinline__ void recomputed_row_topk(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                                                 int H_I, int d_I, const PagedRows& pg, const int* bt,
                                                 long long base, int t, int n, int k, int32_t* out, float* buf,
                                                 SelectSmem<THREADS>& sm)
{
    float* wf = buf + H_I * d_I;
    const uint8_t* qrow = q_idx + (size_t)t * H_I * d_I;
    for (int e = threadIdx.x; e < H_I * d_I; e += THREADS) buf[e] = e4m3x2_to_float2((uint16_t)qrow[e]).x;
    for (int j = threadIdx.x; j < H_I; j += THREADS) wf[j] = w[(size_t)t * H_I + j];
    __syncthreads();
    block_topk<THREADS>(RecomputedRow{buf, wf, k_idx, pg, bt, base, H_I, d_I}, n, k, out, sm);
}

template <int THREADS, class Row>
__device__ __noinline__ void radix_topk_out_of_line(const Row& row, int n, int k, int32_t* out,
                                                    SelectSmem<THREADS>& sm)
{
    block_topk<THREADS>(row, n, k, out, sm);
}

template <int THREADS>
__device__ __noinline__ void radix_mark_out_of_line(const PairList& row, int n, int k, uint32_t* bm,
                                                    SelectSmem<THREADS>& sm)
{
    block_select<THREADS>(row, n, k, [&](int, int i) { atomicOr(&bm[i >> 5], 1u << (i & 31)); }, sm);
}

template <int THREADS>
__global__ void __cluster_dims__(rs::kClusterCtas, 1, 1) __launch_bounds__(THREADS, 2)
row_select_cluster_kernel(const float* __restrict__ scores, long long ld, const uint32_t* __restrict__ gmax16,
                          long long g16_ld, const uint32_t* __restrict__ gmax4, long long g4_ld,
                          const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                          const uint8_t* __restrict__ k_idx, int H_I, int d_I, const int* __restrict__ pos,
                          const int* __restrict__ k_base, int T, int S, int row0, int k, int32_t* __restrict__ idx,
                          const PagedRows pg)
{
    using namespace sm100;
    constexpr int W = THREADS / 32;
    static_assert(THREADS == rs::kCsThreads && W <= 32, "launch shape");
    __shared__ SelectSmem<THREADS> sm;
    __shared__ int wsum[2][2][W];
    __shared__ int count_s, abort_s;
    extern __shared__ __align__(16) uint8_t dyn[];
    const uint32_t dyn_s = smem_u32(dyn);
    auto full = [&](int b) -> uint32_t { return dyn_s + rs::kOffCsBars + 8u * (uint32_t)b; };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = (int)cluster_ctarank(), r = blockIdx.x / rs::kClusterCtas, t = row0 + r;
    if (tid == 0) {
        for (int st = 0; st <= rs::kCsStages; ++st) mbar_init(full(st), 1);   // the last: the group maxima
        abort_s = 0;
        fence_mbar_init_cluster();
    }
    __syncthreads();
    griddep_wait();
    long long base;
    const int* bt;
    const int n = row_keys(pg, pos, k_base, t, T, S, &base, &bt);
    int32_t* out = idx + (size_t)t * k;
    if (n <= k) {
        if (q == 0)
            for (int i = tid; i < k; i += THREADS) out[i] = i < n ? i : -1;
        return;
    }
    if (n > rs::kMaxKeys) {
        if (q == 0)
            recomputed_row_topk<THREADS>(q_idx, w, k_idx, H_I, d_I, pg, bt, base, t, n, k, out,
                                         reinterpret_cast<float*>(dyn), sm);
        return;
    }
    const float* sc = scores + (size_t)r * ld;
    // this CTA's part [a, b) of the row, in chunks of kCsChunk scores
    const int span = ceil_div(ceil_div(n, rs::kClusterCtas), rs::kCsChunk) * rs::kCsChunk;
    const int a = min(n, q * span), b = min(n, a + span);
    const int nch = ceil_div(b - a, rs::kCsChunk);
    auto issue = [&](int j) {
        const int s0 = a + j * rs::kCsChunk, st = j % rs::kCsStages;
        // the last copy of a row is rounded up to 16 bytes: it stays inside ld
        const uint32_t bytes = (uint32_t)(min(rs::kCsChunk, b - s0) * 4 + 15) & ~15u;
        mbar_arrive_expect_tx(full(st), bytes);
        bulk_g2s(dyn_s + (uint32_t)rs::cs_buf(st), sc + s0, bytes, full(st));
    };
    // the row's group maxima (16-key groups where there are k of them)
    const int tiles = rs::row_tiles(n, k);
    const int m16 = tiles * rs::kGroupsPerTile, m4 = tiles * 32;
    const uint32_t* gm = m16 >= k ? gmax16 + (size_t)r * g16_ld : m4 >= k ? gmax4 + (size_t)r * g4_ld : nullptr;
    const int m = m16 >= k ? m16 : m4 >= k ? m4 : 0;
    const bool stage = gm && m <= rs::kMaxStaged;
    // chunks 0 and 1 go to the buffers above the pair space at once; the
    // maxima are staged in the pair space, and chunks 2.. follow once tau is
    // taken from them
    if (tid == 0) {
        if (stage) {
            mbar_arrive_expect_tx(full(rs::kCsStages), (uint32_t)m * 4u);
            bulk_g2s(dyn_s, gm, (uint32_t)m * 4u, full(rs::kCsStages));
        }
        for (int j = 0; j < min(nch, 2); ++j) issue(j);
    }
    bool bad = false;
    uint32_t tk = 0u;
    if (gm) {
        if (stage) bad = __syncthreads_or(!mbar_wait(full(rs::kCsStages), 0, (volatile int*)&abort_s, 674, 0));
        if (!bad) tk = range_floor<THREADS>(stage ? reinterpret_cast<const uint32_t*>(dyn) : gm, m, k, sm);
    }
    // (range_floor ends with a barrier: the staged maxima are no longer read)
    if (tid == 0 && !bad)
        for (int j = 2; j < min(nch, rs::kCsStages); ++j) issue(j);
    // the float whose order key is tau: x >= tf keeps every score whose key
    // is >= tau (and at most a zero of the other sign besides, which ranks
    // below k kept scores and is never selected); tau = 0 keeps all
    const float tf = tk ? key_score(tk) : -INFINITY;
    uint2* local = reinterpret_cast<uint2*>(dyn + rs::kOffCsLocal);
    int running = 0;
    // two chunks per pass of the CTA (one barrier for both): chunk j's pairs,
    // then chunk j + 1's
    for (int j = 0; j < nch && !bad; j += 2) {
        const bool two = j + 1 < nch;
        bool got = mbar_wait(full(j % rs::kCsStages), (uint32_t)((j / rs::kCsStages) & 1),
                             (volatile int*)&abort_s, 673, j);
        if (two)
            got = mbar_wait(full((j + 1) % rs::kCsStages), (uint32_t)(((j + 1) / rs::kCsStages) & 1),
                            (volatile int*)&abort_s, 673, j + 1) && got;
        float e[2][4];
        uint32_t bits[2];
        int cnt[2], incl[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int s = a + (j + h) * rs::kCsChunk + 4 * tid;
            const float4 v = *reinterpret_cast<const float4*>(dyn + rs::cs_buf((j + h) % rs::kCsStages) + 16 * tid);
            e[h][0] = v.x;
            e[h][1] = v.y;
            e[h][2] = v.z;
            e[h][3] = v.w;
            bits[h] = 0u;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if ((h == 0 || two) && s + u < b && e[h][u] >= tf) bits[h] |= 1u << u;
            cnt[h] = __popc(bits[h]);
            incl[h] = cnt[h];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, incl[h], off);
                if (lane >= off) incl[h] += x;
            }
        }
        const int par = (j >> 1) & 1;
        if (lane == 31) {
            wsum[par][0][warp] = incl[0];
            wsum[par][1][warp] = incl[1];
        }
        if (__syncthreads_or(!got)) {
            bad = true;   // a copy timed out: the row takes the global-memory select
            break;
        }
        // every thread has read both buffers: refill them
        if (tid == 0) {
            if (j + rs::kCsStages < nch) issue(j + rs::kCsStages);
            if (j + 1 + rs::kCsStages < nch) issue(j + 1 + rs::kCsStages);
        }
        int base_h = running;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int x = lane < W ? wsum[par][h][lane] : 0;
            int xi = x;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, xi, off);
                if (lane >= off) xi += y;
            }
            int at = base_h + __shfl_sync(0xffffffffu, xi - x, warp) + incl[h] - cnt[h];
            const int s = a + (j + h) * rs::kCsChunk + 4 * tid;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (bits[h] >> u & 1u) {
                    if (at < rs::kCsLocal) local[at] = make_uint2(score_key(e[h][u]), (uint32_t)(s + u));
                    ++at;
                }
            base_h += __shfl_sync(0xffffffffu, xi, W - 1);
        }
        running = base_h;
    }
    if (tid == 0) count_s = bad ? rs::kCsLocal + 1 : running;
    __syncthreads();   // every thread's pairs of the last chunk are written
    uint2* list = reinterpret_cast<uint2*>(dyn);
    if (q == 0) {
        // CTA 0's pairs go first: move them down (the two ranges do not
        // overlap), before any other part stores into the list
        for (int i = tid; i < min(running, rs::kCsLocal); i += THREADS) list[i] = local[i];
    }
    cluster_sync();   // 1: every part's count is final (and every CTA of the cluster runs)
    int before = 0, total = 0;
    bool over = false;
#pragma unroll
    for (int p = 0; p < rs::kClusterCtas; ++p) {
        const int c = (int)ld_cluster_u32(mapa(smem_u32(&count_s), (uint32_t)p));
        over |= c > rs::kCsLocal;
        if (p < q) before += c;
        total += c;
    }
    // (total >= k always holds: tau is at most the k-th largest score; a row
    // short of k pairs would still take the exact global select, so the
    // selects below never see fewer than k entries)
    over |= total > rs::kCsList || total < k;
    cluster_sync();   // 2: every CTA has read the counts (none exits before that)
    int* warp_sums = reinterpret_cast<int*>(sm.hist[0]);
    if (over) {
        // (the same decision in every CTA: no further cluster barrier)
        if (q == 0) radix_topk_out_of_line<THREADS>(DenseScores{sc}, n, k, out, sm);
        return;
    }
    if (q != 0) {
        const uint32_t dst = mapa(dyn_s, 0u) + (uint32_t)before * 8u;
        for (int i = tid; i < running; i += THREADS) st_cluster_v2(dst + 8u * (uint32_t)i, local[i]);
    }
    cluster_sync();   // 3: every part's pairs are in CTA 0 (release / acquire)
    if (q != 0) return;
    uint32_t* lbm = reinterpret_cast<uint32_t*>(dyn + rs::kOffCsBits);
    for (int i = tid; i < (total + 31) / 32; i += THREADS) lbm[i] = 0u;
    __syncthreads();
    const PairList row{list};
    if (!range_select_bitmap<THREADS>(row, total, k, lbm, sm)) radix_mark_out_of_line<THREADS>(row, total, k, lbm, sm);
    __syncthreads();
    block_emit_bitmap<THREADS>(lbm, total, out, warp_sums, [&](int i) { return (int)list[i].y; });
}

}  // namespace idx_chunk
}  // namespace dsa
