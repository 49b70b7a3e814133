// Backward of the sparse MQA attention, dkv part, on the 5th-generation
// tensor cores, for the MLA head shape (Hq = 128, d_qk = 576, d_v = 512).
// Same results as attn_bwd_dkv_kernel (attn_bwd.cuh states the chain rule):
// per query row t and chunk of 64 selected slots,
//   z = Q_t C^T, dp = dO_t V^T                      (128 heads x 64 slots)
//   p = exp(scale z - lse), g = scale p (dp - D)    (bf16, g also to g_ws)
//   dC^T = Q_t^T g + dO_t^T p                        (576 columns x 64 slots)
// and dC is scatter-added into dkv (fp32 atomics, one per element).
//
// One CTA of 256 threads per (row, 64 slots), two CTAs per SM (their phases
// overlap):
//  - warp 0 (one thread) streams Q_t and dO_t in 64-column tiles by TMA
//    (128 rows x 128 B, 128B swizzle): 17 tiles for z and dp (a 2-stage
//    ring), then 9 two-tile pairs for dC (two 32 KB buffers in the space of
//    the gathered rows, free once z and dp are done);
//  - warps 1-3 gather the 64 selected latent rows (cp.async, 128B-swizzled
//    64-column slabs, K-major B operand of z and dp); warp 1's first thread
//    then issues every MMA;
//  - warps 4-7 (one head per thread, the TMEM lane) read D (formed once per
//    row by attn_bwd_delta_kernel) and lse, then read z and dp from TMEM, write p and g as MN-major tiles
//    [head][slot] in the ring's space (the B operands of dC^T, whose A
//    operands are the Q / dO tiles read MN-major), and finally add each dC^T
//    tile (M = 128 columns, N = 64 slots) into dkv.
// TMEM (256 columns): z [0,64) and dp [64,128), then dC^T tiles 0..3 at
// [64m, 64m+64); tile 4 reuses tile 0's columns once they are drained.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace bwd_tc {

using namespace sm100;

constexpr int kHeads = 128, kDqk = 576, kDv = 512, kSlots = 64;
constexpr int kThreads = 256;
constexpr int kTile = 128 * 128;          // one [128 rows x 64 columns] bf16 tile, 128B swizzle
constexpr int kCSlab = kSlots * 128;      // 64 gathered rows x 64 columns
constexpr int kQTiles = kDqk / 64;        // 9
constexpr int kVTiles = kDv / 64;         // 8
constexpr int kRing = 2;
constexpr int kGatherThreads = 96;
constexpr int kOffC = 0;                                   // 9 slabs (72 KB); then 2 pair buffers
constexpr int kOffRing = kOffC + kQTiles * kCSlab;         // 3 x 16 KB
constexpr int kPGTile = kHeads * kSlots * 2;               // p or g: [128 heads][64 slots] bf16, 16 KB
constexpr int kOffP = kOffRing;                            // p and g take the ring's space after z, dp
constexpr int kOffG = kOffP + kPGTile;
constexpr int kOffRows = kOffRing + kRing * kTile;         // 64 x long long
constexpr int kOffBar = kOffRows + kSlots * 8;
constexpr int kSmemBytes = kOffBar + 256 + 1024;           // + alignment slack
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColZ = 0, kColDp = 64, kColDc = 0;

enum : int {
    B_CFULL = 0, B_AFULL = 1, B_AEMPTY = B_AFULL + kRing, B_ZDONE = B_AEMPTY + kRing, B_PG = B_ZDONE + 1,
    B_PFULL = B_PG + 1, B_PEMPTY = B_PFULL + 2, B_TILE = B_PEMPTY + 2, B_T0FREE = B_TILE + 5,
    B_DRAIN = B_T0FREE + 1, B_COUNT = B_DRAIN + 1
};

static_assert(2 * 2 * kTile <= kQTiles * kCSlab, "pair buffers fit in the gathered rows' space");
static_assert(kOffRing % 1024 == 0 && kOffP % 1024 == 0 && kOffG % 1024 == 0, "alignment");
static_assert(8 * B_COUNT + 16 <= 256, "barrier area");
static_assert(kPGTile == kHeads * 128 && kOffG + kPGTile <= kOffRows && kOffBar - kOffRows == kSlots * 8,
              "p / g tiles of 128-byte rows inside the ring, then the slot rows, then the barriers");
static_assert(2 * (kSmemBytes + 1024) <= 233472, "two CTAs per SM");
static_assert(kSmemBytes <= 232448, "shared memory");

// kind::f16 instruction descriptor with both operand majors given.
__host__ __device__ constexpr uint32_t idesc_bf16_ab(int M, int N, bool a_mn_major, bool b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Bounded wait whose outcome is the same for the whole warp.
__device__ __forceinline__ bool wait_all(uint32_t b_addr, uint32_t par, volatile int* abort_flag, int tag, int c)
{
    return __all_sync(0xffffffffu, mbar_wait(b_addr, par, abort_flag, tag, c));
}

__device__ __forceinline__ void red_add_f32(float* p, float v)
{
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// D_h = dout_h . o_h of every head of the pass's rows: d_ws[row][128] (fp32).
// One CTA of 256 threads per row; warp w takes heads 16w .. 16w+15, its lanes
// eight columns at a time.
__global__ void __launch_bounds__(256)
attn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout, int r0,
                      float* __restrict__ d_ws)
{
    const int tl = blockIdx.x, t = r0 + tl;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int hh = 0; hh < 16; ++hh) {
        const int h = warp * 16 + hh;
        const uint4* gr = reinterpret_cast<const uint4*>(dout + ((size_t)t * kHeads + h) * kDv);
        const uint4* orow = reinterpret_cast<const uint4*>(out + ((size_t)t * kHeads + h) * kDv);
        float acc = 0.f;
#pragma unroll
        for (int it = 0; it < kDv / 256; ++it) {
            const uint4 a = __ldg(gr + it * 32 + lane), b = __ldg(orow + it * 32 + lane);
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc = fmaf(bf16_lo(aw[e]), bf16_lo(bw[e]), fmaf(bf16_hi(aw[e]), bf16_hi(bw[e]), acc));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) d_ws[(size_t)tl * kHeads + h] = acc;
    }
}

// grid: x = slot chunk (64 slots), y = query row within the pass [r0, r0 + gridDim.y).
// g_ws: bf16 [rows][128][slots_pad(k)], as attn_bwd_dkv_kernel writes it;
// d_ws: fp32 [rows][128], from attn_bwd_delta_kernel.
__global__ void __launch_bounds__(kThreads, 2)
attn_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                       const __nv_bfloat16* __restrict__ kv, const int* __restrict__ idx,
                       const int* __restrict__ pos, const int* __restrict__ k_base,
                       const __nv_bfloat16* __restrict__ out, const float* __restrict__ lse,
                       const __nv_bfloat16* __restrict__ dout, int r0, int T, int S, int k, int kp,
                       float scale, float* __restrict__ dkv, __nv_bfloat16* __restrict__ g_ws,
                       const float* __restrict__ d_ws)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + kOffBar;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sgen + kOffBar + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kOffBar + 8 * B_COUNT + 8);
    long long* rows = reinterpret_cast<long long*>(sgen + kOffRows);

    const int tl = blockIdx.y, t = r0 + tl, i0 = blockIdx.x * kSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    if (i0 >= min(k, n_cand)) return;   // whole chunk past the row's entries (uniform per CTA)

    if (threadIdx.x < kSlots) {
        const int i = i0 + threadIdx.x;
        const int s = i < k ? idx[(size_t)t * k + i] : -1;
        rows[threadIdx.x] = (i < k && s >= 0 && s < n_cand) ? base + s : -1ll;
    }
    if (threadIdx.x == 0) {
        mbar_init(bar(B_CFULL), kGatherThreads);
        for (int s = 0; s < kRing; ++s) {
            mbar_init(bar(B_AFULL + s), 1);
            mbar_init(bar(B_AEMPTY + s), 1);
        }
        mbar_init(bar(B_ZDONE), 1);
        mbar_init(bar(B_PG), 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_PFULL + b), 1);
            mbar_init(bar(B_PEMPTY + b), 1);
        }
        for (int m = 0; m < 5; ++m) mbar_init(bar(B_TILE + m), 1);
        mbar_init(bar(B_T0FREE), 4);    // tile 0's columns read by the four epilogue warps
        mbar_init(bar(B_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init_cluster();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(taddr_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_slot;
    const uint32_t cs = sbase + kOffC, ring = sbase + kOffRing, ps = sbase + kOffP, gs = sbase + kOffG;

    if (warp == 0) {
        // ------------------------------------------------------------- TMA
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_do);
            bool ok = true;
            // z and dp: Q tiles 0..8, then dO tiles 0..7
            for (int s = 0; ok && s < kQTiles + kVTiles; ++s) {
                const int st = s % kRing;
                if (s >= kRing && !mbar_wait(bar(B_AEMPTY + st), ((s - kRing) / kRing) & 1, abort_flag, 100, s)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(bar(B_AFULL + st), kTile);
                if (s < kQTiles)
                    tma_load_2d(ring + st * kTile, &tm_q, 64 * s, t * kHeads, bar(B_AFULL + st));
                else
                    tma_load_2d(ring + st * kTile, &tm_do, 64 * (s - kQTiles), t * kHeads, bar(B_AFULL + st));
            }
            // dC^T: for column tile m, the pair of Q tiles (2m, 2m+1), then the
            // pair of dO tiles (m < 4); tile 4 has one Q tile (columns 512..575).
            // The pair buffers overwrite the gathered rows: z and dp first.
            if (ok) ok = mbar_wait(bar(B_ZDONE), 0, abort_flag, 101, 0);
            int p = 0;
            for (int m = 0; ok && m < 5; ++m) {
                for (int kind = 0; kind < (m < 4 ? 2 : 1); ++kind, ++p) {
                    const int pb = p & 1;
                    if (p >= 2 && !mbar_wait(bar(B_PEMPTY + pb), ((p - 2) >> 1) & 1, abort_flag, 102, p)) {
                        ok = false;
                        break;
                    }
                    const int n_tiles = m < 4 ? 2 : 1;
                    mbar_arrive_expect_tx(bar(B_PFULL + pb), n_tiles * kTile);
                    for (int h = 0; h < n_tiles; ++h)
                        tma_load_2d(cs + pb * 2 * kTile + h * kTile, kind == 0 ? (const void*)&tm_q : (const void*)&tm_do,
                                    128 * m + 64 * h, t * kHeads, bar(B_PFULL + pb));
                }
            }
        }
    } else if (warp <= 3) {
        // ---------------------------------------------------------- gather
        // 64 rows x 72 sixteen-byte pieces; piece j of row r goes to slab j/8
        // (64 columns), 16-byte unit (j%8) ^ (r%8) of the row's 128 bytes
        const int g = threadIdx.x - 32;
        const char* kvb = reinterpret_cast<const char*>(kv);
        for (int e = g; e < kSlots * 72; e += kGatherThreads) {
            const int r = e / 72, j = e - r * 72;
            const long long row = rows[r];
            const uint32_t dst = cs + (j >> 3) * kCSlab + r * 128 + (((j & 7) ^ (r & 7)) << 4);
            cp_async16(dst, row >= 0 ? kvb + row * (kDqk * 2) + j * 16 : kvb, row >= 0 ? 16u : 0u);
        }
        cp_async_arrive_noinc(bar(B_CFULL));
        if (warp == 1 && lane == 0) {
            // ----------------------------------------------------- MMAs
            const uint32_t id_a = idesc_bf16_ab(128, kSlots, false, false);   // z, dp
            const uint32_t id_c = idesc_bf16_ab(128, kSlots, true, true);     // dC^T
            bool ok = mbar_wait(bar(B_CFULL), 0, abort_flag, 200, 0);
            // the rows were written by cp.async (generic proxy); the MMA reads
            // them through the async proxy
            fence_proxy_async_smem();
            for (int s = 0; ok && s < kQTiles + kVTiles; ++s) {
                const int st = s % kRing;
                ok = mbar_wait(bar(B_AFULL + st), (s / kRing) & 1, abort_flag, 201, s);
                if (!ok) break;
                tc_fence_after();
                const bool is_z = s < kQTiles;
                const int slab = is_z ? s : s - kQTiles;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc(ring + st * kTile + kk * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = smem_desc(cs + slab * kCSlab + kk * 32, 16, 1024, kSwizzle128B);
                    mma_f16_ss(tmem + (is_z ? kColZ : kColDp), ad, bd, id_a, (slab > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(B_AEMPTY + st));
            }
            if (ok) mma_commit(bar(B_ZDONE));
            // dC^T tile m (columns 128m .. 128m+127) = Q^T g + dO^T p over the
            // 128 heads (8 K-steps): A = a pair buffer read MN-major (two
            // 64-column tiles, LBO = one tile), B = g or p [head][slot]
            if (ok) ok = mbar_wait(bar(B_PG), 0, abort_flag, 202, 0);
            if (ok) tc_fence_after();
            int p = 0;
            for (int m = 0; ok && m < 5; ++m) {
                // tile 4 reuses tile 0's columns once the epilogue has read them
                if (m == 4) {
                    ok = mbar_wait(bar(B_T0FREE), 0, abort_flag, 204, 0);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t dcol = kColDc + 64 * (m & 3);
                for (int kind = 0; kind < (m < 4 ? 2 : 1); ++kind, ++p) {
                    const int pb = p & 1;
                    ok = mbar_wait(bar(B_PFULL + pb), (p >> 1) & 1, abort_flag, 203, p);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a0 = cs + pb * 2 * kTile;
                    const uint32_t b0 = kind == 0 ? gs : ps;
#pragma unroll
                    for (int ks = 0; ks < kHeads / 16; ++ks) {
                        const uint64_t ad = smem_desc(a0 + ks * 2048, kTile, 1024, kSwizzle128B);
                        const uint64_t bd = smem_desc(b0 + ks * 2048, kTile, 1024, kSwizzle128B);
                        mma_f16_ss(tmem + dcol, ad, bd, id_c, (kind > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(bar(B_PEMPTY + pb));
                }
                if (ok) mma_commit(bar(B_TILE + m));
            }
            // every MMA issued completes before TMEM is released
            mma_commit(bar(B_DRAIN));
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bar(B_DRAIN), 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
            }
        }
        cp_async_wait_all();
    } else {
        // -------------------------------------------------------- epilogue
        const int h = threadIdx.x - 128;                       // head = TMEM lane
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        constexpr float kLog2e = 1.4426950408889634f;
        // D_h = dout_h . o_h (formed per row) and lse in base 2
        const float D = d_ws[(size_t)tl * kHeads + h];
        const float l2 = lse[(size_t)t * kHeads + h] * kLog2e;
        bool ok = wait_all(bar(B_ZDONE), 0, abort_flag, 300, 0);
        if (ok) {
            tc_fence_after();
            // p and g for the 64 slots, 32 at a time, as [head][slot] rows of
            // 128 B (128B swizzle: unit u of row h at (u ^ (h % 8)) * 16), and
            // g to g_ws
            const float zs = scale * kLog2e;
            uint4* gw = reinterpret_cast<uint4*>(g_ws + ((size_t)tl * kHeads + h) * kp + i0);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t z[32], dp[32];
                tmem_ld32(tmem + lane_addr + kColZ + 32 * half, z);
                tmem_ld32(tmem + lane_addr + kColDp + 32 * half, dp);
                tmem_wait_ld();
#pragma unroll
                for (int uu = 0; uu < 4; ++uu) {
                    const int u = 4 * half + uu;
                    uint32_t pp[4], gg[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float pv[2], gv[2];
#pragma unroll
                        for (int f = 0; f < 2; ++f) {
                            const int jl = 8 * uu + 2 * e + f;
                            const bool valid = rows[32 * half + jl] >= 0;
                            const float p = valid ? exp2f(fmaf(__uint_as_float(z[jl]), zs, -l2)) : 0.f;
                            pv[f] = p;
                            gv[f] = valid ? scale * p * (__uint_as_float(dp[jl]) - D) : 0.f;
                        }
                        pp[e] = pack_bf16x2(pv[0], pv[1]);
                        gg[e] = pack_bf16x2(gv[0], gv[1]);
                    }
                    const uint32_t off = (uint32_t)h * 128 + (((uint32_t)u ^ (h & 7)) << 4);
                    st_shared_v4(ps + off, make_uint4(pp[0], pp[1], pp[2], pp[3]));
                    st_shared_v4(gs + off, make_uint4(gg[0], gg[1], gg[2], gg[3]));
                    gw[u] = make_uint4(gg[0], gg[1], gg[2], gg[3]);
                }
            }
            // z and dp are read (the dC^T tiles overwrite them), and the MMA
            // reads p and g through the async proxy
            tc_fence_before();
            // the MMA reads p and g through the async proxy
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_PG));
        }
        // dC^T tiles: this thread's column of tile m, 64 slots (32 at a time)
        for (int m = 0; ok && m < 5; ++m) {
            ok = wait_all(bar(B_TILE + m), 0, abort_flag, 301, m);
            if (!ok) break;
            tc_fence_after();
            const int col = 128 * m + h;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_addr + kColDc + 64 * (m & 3) + 32 * half, v);
                tmem_wait_ld();
                if (m == 0 && half == 1) {
                    // tile 0's columns are read: tile 4 may overwrite them
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_T0FREE));
                }
                if (col < kDqk) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const long long r = rows[32 * half + j];
                        if (r >= 0) red_add_f32(dkv + (size_t)r * kDqk + col, __uint_as_float(v[j]));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------- dq kernel

// dq_t = g_t C: per query row, (128 heads x slots) times (slots x 576), fp32
// out. Three CTAs per row, each 192 output columns (a 128 x 192 fp32 TMEM
// accumulator); per chunk of 64 slots, g by TMA ([128 heads x 64 slots],
// 128B swizzle: the K-major A operand) and the slots' 192 columns of the
// latent rows by cp.async (three 128B-swizzled 64-column slabs: the B
// operand read MN-major, as the forward's PV reads them). Two stages, two
// CTAs per SM.
constexpr int kDqCols = 192;
constexpr int kDqStages = 2;
constexpr int kDqGTile = kHeads * kSlots * 2;                 // 16 KB
constexpr int kDqCSlab = kSlots * 128;                        // 64 rows x 64 columns
constexpr int kDqStage = kDqGTile + 3 * kDqCSlab;              // 40 KB
constexpr int kDqOffBar = kDqStages * kDqStage;
constexpr int kDqSmem = kDqOffBar + 256 + 1024;
constexpr int kDqThreads = 256;
constexpr int kDqGatherThreads = 64;

enum : int { D_FULL = 0, D_EMPTY = D_FULL + kDqStages, D_DONE = D_EMPTY + kDqStages, D_COUNT = D_DONE + 1 };

static_assert(kDqGTile % 1024 == 0 && kDqStage % 1024 == 0, "alignment");
static_assert(2 * (kDqSmem + 1024) <= 233472, "two CTAs per SM");

// grid: x = 192-column block (0..2), y = query row within the pass.
// tm_g: g_ws as [rows * 128, kp] bf16, box 64 slots x 128 heads, 128B swizzle.
__global__ void __launch_bounds__(kDqThreads, 2)
attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16* __restrict__ kv,
                      const int* __restrict__ idx, const int* __restrict__ pos, const int* __restrict__ k_base,
                      int r0, int T, int S, int k, float* __restrict__ dq)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + kDqOffBar;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sgen + kDqOffBar + 8 * D_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kDqOffBar + 8 * D_COUNT + 8);

    const int tl = blockIdx.y, t = r0 + tl, cb = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    const int n_ent = min(k, n_cand);
    const int n_chunks = (n_ent + kSlots - 1) / kSlots;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDqStages; ++s) {
            mbar_init(bar(D_FULL + s), kDqGatherThreads + 1);   // gather threads + the TMA arrival
            mbar_init(bar(D_EMPTY + s), 1);
        }
        mbar_init(bar(D_DONE), 1);
        *abort_flag = 0;
        fence_mbar_init_cluster();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(taddr_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_slot;

    if (warp == 0) {
        // ------------------------------------------------------------- MMA
        if (lane == 0 && n_chunks > 0) {
            const uint32_t id = idesc_bf16_ab(128, kDqCols, false, true);
            bool ok = true;
            for (int c = 0; ok && c < n_chunks; ++c) {
                const int st = c % kDqStages;
                ok = mbar_wait(bar(D_FULL + st), (c / kDqStages) & 1, abort_flag, 400, c);
                if (!ok) break;
                // the rows were written by cp.async (generic proxy)
                fence_proxy_async_smem();
                tc_fence_after();
                const uint32_t gt = sbase + st * kDqStage, ct = gt + kDqGTile;
#pragma unroll
                for (int kk = 0; kk < kSlots / 16; ++kk) {
                    const uint64_t ad = smem_desc(gt + kk * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = smem_desc(ct + kk * 2048, kDqCSlab, 1024, kSwizzle128B);
                    mma_f16_ss(tmem, ad, bd, id, (c > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(D_EMPTY + st));
            }
            mma_commit(bar(D_DONE));
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- TMA of g
        if (lane == 0) {
            prefetch_tmap(&tm_g);
            for (int c = 0; c < n_chunks; ++c) {
                const int st = c % kDqStages;
                if (c >= kDqStages &&
                    !mbar_wait(bar(D_EMPTY + st), ((c - kDqStages) / kDqStages) & 1, abort_flag, 401, c))
                    break;
                mbar_arrive_expect_tx(bar(D_FULL + st), kDqGTile);
                tma_load_2d(sbase + st * kDqStage, &tm_g, kSlots * c, tl * kHeads, bar(D_FULL + st));
            }
        }
    } else if (warp <= 3) {
        // ---------------------------------------------------------- gather
        // Thread r copies slot r's 24 sixteen-byte pieces (192 columns) of
        // every chunk: piece p goes to slab p/8, unit (p%8) ^ (r%8) of the
        // row's 128 bytes. The next chunk's index is loaded one chunk ahead.
        const int r = threadIdx.x - 64;
        const char* kvb = reinterpret_cast<const char*>(kv);
        auto slot_of = [&](int c) -> int {
            const int i = c * kSlots + r;
            const int s = i < n_ent ? idx[(size_t)t * k + i] : -1;
            return (s >= 0 && s < n_cand) ? s : -1;
        };
        int s_next = n_chunks > 0 ? slot_of(0) : -1;
        for (int c = 0; c < n_chunks; ++c) {
            const int st = c % kDqStages;
            const int s = s_next;
            if (c + 1 < n_chunks) s_next = slot_of(c + 1);
            if (c >= kDqStages) {
                const bool got = mbar_wait(bar(D_EMPTY + st), ((c - kDqStages) / kDqStages) & 1, abort_flag, 402, c);
                if (!__all_sync(0xffffffffu, got)) break;
            }
            const uint32_t ct = sbase + st * kDqStage + kDqGTile + r * 128;
            const char* src = s >= 0 ? kvb + (base + s) * (kDqk * 2) + kDqCols * cb * 2 : kvb;
#pragma unroll
            for (int pc = 0; pc < 24; ++pc)
                cp_async16(ct + (pc >> 3) * kDqCSlab + (((pc & 7) ^ (r & 7)) << 4), s >= 0 ? src + pc * 16 : kvb,
                           s >= 0 ? 16u : 0u);
            cp_async_arrive_noinc(bar(D_FULL + st));
        }
        cp_async_wait_all();
    } else {
        // -------------------------------------------------------- epilogue
        const int h = threadIdx.x - 128;                       // head = TMEM lane
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        float* dst = dq + ((size_t)t * kHeads + h) * kDqk + kDqCols * cb;
        bool ok = true;
        if (n_chunks > 0) {
            ok = wait_all(bar(D_DONE), 0, abort_flag, 403, 0);
            if (ok) tc_fence_after();
        }
        if (ok) {
#pragma unroll 1
            for (int q = 0; q < kDqCols / 32; ++q) {
                uint32_t v[32];
                if (n_chunks > 0) {
                    tmem_ld32(tmem + lane_addr + 32 * q, v);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                float4* d4 = reinterpret_cast<float4*>(dst + 32 * q);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                        __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------ head-summed probabilities

// The indexer KL loss's target for the MLA head shape: per query row and
// chunk of 64 selected slots, psum_s = sum_h exp(scale q_h.c_s - lse_h) (0
// for non-candidates), into psum [rows][kp] fp32. z = Q_t C^T as in
// attn_bwd_dkv_tc_kernel (Q_t by TMA in nine 64-column tiles, 2-stage ring;
// the gathered rows the K-major B operand; z in TMEM), then each epilogue
// thread (one head) forms its 64 probabilities and every warp sums them over
// its 32 heads with a halving exchange (lane L ends with slots 2L and
// 2L + 1), the four warps' sums meeting in shared memory.
constexpr int kPsOffRing = kQTiles * kCSlab;                 // after the gathered rows
constexpr int kPsOffRows = kPsOffRing + 2 * kTile;
constexpr int kPsOffRed = kPsOffRows + kSlots * 8;           // [4 warps][64] fp32
constexpr int kPsOffBar = kPsOffRed + 4 * kSlots * 4;
constexpr int kPsSmem = kPsOffBar + 256 + 1024;

enum : int { H_CFULL = 0, H_AFULL = 1, H_AEMPTY = 3, H_ZDONE = 5, H_COUNT = 6 };

static_assert(kPsOffRing % 1024 == 0, "alignment");
static_assert(2 * (kPsSmem + 1024) <= 233472, "two CTAs per SM");

__global__ void __launch_bounds__(kThreads, 2)
head_prob_sum_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __nv_bfloat16* __restrict__ kv,
                        const int* __restrict__ idx, const int* __restrict__ pos, const int* __restrict__ k_base,
                        const float* __restrict__ lse, int r0, int T, int S, int k, int kp, float scale,
                        float* __restrict__ psum)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + kPsOffBar;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sgen + kPsOffBar + 8 * H_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kPsOffBar + 8 * H_COUNT + 8);
    long long* rows = reinterpret_cast<long long*>(sgen + kPsOffRows);
    float* red = reinterpret_cast<float*>(sgen + kPsOffRed);

    const int tl = blockIdx.y, t = r0 + tl, i0 = blockIdx.x * kSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    if (i0 >= min(k, n_cand)) return;   // whole chunk past the row's entries (uniform per CTA)

    if (threadIdx.x < kSlots) {
        const int i = i0 + threadIdx.x;
        const int s = i < k ? idx[(size_t)t * k + i] : -1;
        rows[threadIdx.x] = (i < k && s >= 0 && s < n_cand) ? base + s : -1ll;
    }
    if (threadIdx.x == 0) {
        mbar_init(bar(H_CFULL), kGatherThreads);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(H_AFULL + s), 1);
            mbar_init(bar(H_AEMPTY + s), 1);
        }
        mbar_init(bar(H_ZDONE), 1);
        *abort_flag = 0;
        fence_mbar_init_cluster();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(taddr_slot), 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_slot;
    const uint32_t cs = sbase, ring = sbase + kPsOffRing;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            for (int s = 0; s < kQTiles; ++s) {
                const int st = s & 1;
                if (s >= 2 && !mbar_wait(bar(H_AEMPTY + st), ((s - 2) >> 1) & 1, abort_flag, 500, s)) break;
                mbar_arrive_expect_tx(bar(H_AFULL + st), kTile);
                tma_load_2d(ring + st * kTile, &tm_q, 64 * s, t * kHeads, bar(H_AFULL + st));
            }
        }
    } else if (warp <= 3) {
        const int g = threadIdx.x - 32;
        const char* kvb = reinterpret_cast<const char*>(kv);
        for (int e = g; e < kSlots * 72; e += kGatherThreads) {
            const int r = e / 72, j = e - r * 72;
            const long long row = rows[r];
            const uint32_t dst = cs + (j >> 3) * kCSlab + r * 128 + (((j & 7) ^ (r & 7)) << 4);
            cp_async16(dst, row >= 0 ? kvb + row * (kDqk * 2) + j * 16 : kvb, row >= 0 ? 16u : 0u);
        }
        cp_async_arrive_noinc(bar(H_CFULL));
        if (warp == 1 && lane == 0) {
            const uint32_t id = idesc_bf16_ab(128, kSlots, false, false);
            bool ok = mbar_wait(bar(H_CFULL), 0, abort_flag, 501, 0);
            fence_proxy_async_smem();
            for (int s = 0; ok && s < kQTiles; ++s) {
                const int st = s & 1;
                ok = mbar_wait(bar(H_AFULL + st), (s >> 1) & 1, abort_flag, 502, s);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc(ring + st * kTile + kk * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = smem_desc(cs + s * kCSlab + kk * 32, 16, 1024, kSwizzle128B);
                    mma_f16_ss(tmem, ad, bd, id, (s > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(H_AEMPTY + st));
            }
            mma_commit(bar(H_ZDONE));
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bar(H_ZDONE), 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
            }
        }
        cp_async_wait_all();
    } else {
        const int h = threadIdx.x - 128;
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        constexpr float kLog2e = 1.4426950408889634f;
        const float l2 = lse[(size_t)t * kHeads + h] * kLog2e, zs = scale * kLog2e;
        const bool ok = wait_all(bar(H_ZDONE), 0, abort_flag, 503, 0);
        float v[64];
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t z[32];
                tmem_ld32(tmem + lane_addr + 32 * half, z);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    v[32 * half + j] = rows[32 * half + j] >= 0 ? exp2f(fmaf(__uint_as_float(z[j]), zs, -l2)) : 0.f;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = 0.f;
        }
        // halving exchange: keep the lower or upper half of the current slot
        // range (by lane bit o), add the partner's copy of it
#pragma unroll
        for (int o = 16, n = 64; o >= 1; o >>= 1, n >>= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
                const float send = up ? v[i] : v[i + n / 2];
                const float keep = up ? v[i + n / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        red[(warp & 3) * kSlots + 2 * lane] = v[0];
        red[(warp & 3) * kSlots + 2 * lane + 1] = v[1];
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (ok && h < kSlots)
            psum[(size_t)tl * kp + i0 + h] = red[h] + red[kSlots + h] + red[2 * kSlots + h] + red[3 * kSlots + h];
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

}  // namespace bwd_tc
}  // namespace dsa
