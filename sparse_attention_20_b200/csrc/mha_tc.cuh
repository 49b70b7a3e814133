// MLA in MHA mode (dense causal attention, every head with its own key and
// value rows; mha_attn.cuh states the operation) on the 5th-generation tensor
// cores, for the (d_h, d_hv) = (192, 128) head shape.
//
// Persistent: one CTA of 384 threads per SM walks the work units (128 query
// rows, head) in order of decreasing causal length; every per-tile barrier
// counts tiles across units, so the K/V ring and the QK MMAs run on into the
// next unit while the softmax warps finish the current one:
//  - warp 1 (one thread) loads the Q tile and streams 128-key tiles of K and
//    V by TMA from the head's column window of the row-major tensors
//    ([rows, Hq * d] bf16; 64-column boxes of 128 rows, 128B swizzle; a
//    2-stage ring of K + V);
//  - warp 0 (one thread) issues S = Q K^T (M = 128 query rows, N = 128 keys,
//    K = 192) into a TMEM double buffer, and O += P V (A = P from TMEM, B = the
//    V tile read MN-major, N = 128) into TMEM;
//  - warps 4-11, two per TMEM lane quarter (each 64 of a tile's 128 keys),
//    run the online softmax in the log2 domain: causal mask, row maximum
//    agreed between the two halves through shared memory, lazy rescaling of
//    O (only when the maximum rises by more than 8), bf16 P into TMEM; then
//    the epilogue (O / l -> bf16, lse).
// TMEM: O [0,128), S double buffer [128,384), P double buffer [384,512).
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace mha_tc {

using namespace sm100;

constexpr int kRows = 128, kKeys = 128, kDh = 192, kDv = 128;
constexpr int kThreads = 384;
constexpr int kSlab = 128 * 128;                 // [128 rows x 64 columns] bf16
constexpr int kQBytes = 3 * kSlab;
constexpr int kStageBytes = 5 * kSlab;           // K (three slabs) + V (two slabs)
constexpr int kStages = 2;
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffRed = kOffKV + kStages * kStageBytes;   // [2 parities][2 halves][128] row maxima
constexpr int kOffLsum = kOffRed + 2 * 2 * kRows * 4;     // [2 unit parities][2 halves][128] row sums
constexpr int kOffBar = kOffLsum + 2 * 2 * kRows * 4;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 128, kColP = 384;

enum : int {
    M_Q = 0, M_KFULL = 1, M_KEMPTY = 3, M_SFULL = 5, M_SFREE = 7, M_PFULL = 9, M_PVDONE = 11, M_RED = 13,
    M_LSUM = 15, M_DRAIN = 16, M_COUNT = 17
};

static_assert(kOffKV % 1024 == 0 && kStageBytes % 1024 == 0, "alignment");
static_assert(8 * M_COUNT + 16 <= 256, "barrier area");
static_assert(kSmemBytes <= 232448, "shared memory");

__host__ __device__ constexpr uint32_t idesc(int M, int N, bool b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ bool wait_w(uint32_t b_addr, uint32_t par, volatile int* abort_flag, int tag, int c)
{
    return __all_sync(0xffffffffu, mbar_wait(b_addr, par, abort_flag, tag, c));
}

// A work unit: query tile qt (rows 128 qt ..) of head h; unit u takes the
// tiles in order of decreasing causal length, all heads of a tile together.
struct Unit {
    int t0, h, NT;
};

__device__ __forceinline__ Unit unit_of(int u, int n_qt, int Hq, int T, int S)
{
    Unit w;
    w.t0 = (n_qt - 1 - u / Hq) * kRows;
    w.h = u % Hq;
    const int kmax = min(S, w.t0 + kRows + (S - T));   // keys this tile needs
    w.NT = (kmax + kKeys - 1) / kKeys;
    return w;
}

// grid: one CTA per SM (at most one per unit).
// tm_q: q as [T, Hq * 192]; tm_k: k as [S, Hq * 192]; tm_v: v as [S, Hq * 128].
__global__ void __launch_bounds__(kThreads, 1)
mha_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, int T, int S, int Hq, float scale_log2,
              __nv_bfloat16* __restrict__ out, float* __restrict__ lse)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + kOffBar;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sgen + kOffBar + 8 * M_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kOffBar + 8 * M_COUNT + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int shift = S - T;                       // pos[t] = t + shift
    const int n_qt = (T + kRows - 1) / kRows;
    const int n_all = n_qt * Hq;
    const int cta = blockIdx.x, ncta = gridDim.x;
    const int n_units = cta < n_all ? (n_all - cta + ncta - 1) / ncta : 0;
    auto unit = [&](int j) -> Unit { return unit_of(cta + j * ncta, n_qt, Hq, T, S); };

    if (threadIdx.x == 0) {
        mbar_init(bar(M_Q), 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(M_KFULL + b), 1);
            mbar_init(bar(M_KEMPTY + b), 1);
            mbar_init(bar(M_SFULL + b), 1);
            mbar_init(bar(M_SFREE + b), 8);
            mbar_init(bar(M_PFULL + b), 8);
            mbar_init(bar(M_PVDONE + b), 1);
            mbar_init(bar(M_RED + b), 8);
        }
        mbar_init(bar(M_LSUM), 8);
        mbar_init(bar(M_DRAIN), 1);
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
    const uint32_t qs = sbase + kOffQ;

    if (warp == 1) {
        // ------------------------------------------------------------- TMA
        // Q of a unit once every QK of the previous unit has completed (they
        // read the Q tile), then its K / V tiles through the ring
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int g = 0, g_prev_last = -1;
            bool ok = true;
            for (int j = 0; ok && j < n_units; ++j) {
                const Unit w = unit(j);
                if (g_prev_last >= 0 &&
                    !mbar_wait(bar(M_SFULL + (g_prev_last & 1)), (g_prev_last >> 1) & 1, abort_flag, 102, j)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(bar(M_Q), kQBytes);
                for (int i = 0; i < 3; ++i) tma_load_2d(qs + i * kSlab, &tm_q, w.h * kDh + 64 * i, w.t0, bar(M_Q));
                for (int jt = 0; jt < w.NT; ++jt, ++g) {
                    const int st = g % kStages;
                    if (g >= kStages &&
                        !mbar_wait(bar(M_KEMPTY + st), ((g - kStages) / kStages) & 1, abort_flag, 100, g)) {
                        ok = false;
                        break;
                    }
                    const uint32_t kvs = sbase + kOffKV + st * kStageBytes;
                    mbar_arrive_expect_tx(bar(M_KFULL + st), kStageBytes);
                    for (int i = 0; i < 3; ++i)
                        tma_load_2d(kvs + i * kSlab, &tm_k, w.h * kDh + 64 * i, kKeys * jt, bar(M_KFULL + st));
                    for (int i = 0; i < 2; ++i)
                        tma_load_2d(kvs + (3 + i) * kSlab, &tm_v, w.h * kDv + 64 * i, kKeys * jt, bar(M_KFULL + st));
                }
                g_prev_last = g - 1;
            }
        }
    } else if (warp == 0) {
        // ------------------------------------------------------------- MMA
        if (lane == 0 && n_units > 0) {
            const uint32_t id_qk = idesc(128, kKeys, false);
            const uint32_t id_pv = idesc(128, kDv, true);
            bool ok = true;
            int qj = 0, qc = 0, qg = 0;   // QK cursor: unit, tile of the unit, global tile
            int pj = 0, pc = 0, pg = 0;   // PV cursor
            Unit qu = unit(0), pu = qu;
            uint64_t t_idle = globaltimer_ns();
            while (ok && pj < n_units) {
                bool progressed = false;
                if (qj < n_units && mbar_test_wait(bar(M_KFULL + qg % kStages), (qg / kStages) & 1) &&
                    (qg < 2 || mbar_test_wait(bar(M_SFREE + (qg & 1)), ((qg - 2) >> 1) & 1)) &&
                    (qc > 0 || mbar_test_wait(bar(M_Q), qj & 1))) {
                    const int g = qg;
                    tc_fence_after();
                    const uint32_t kvs = sbase + kOffKV + (g % kStages) * kStageBytes;
#pragma unroll
                    for (int i = 0; i < 3; ++i)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = smem_desc(qs + i * kSlab + kk * 32, 16, 1024, kSwizzle128B);
                            const uint64_t bd = smem_desc(kvs + i * kSlab + kk * 32, 16, 1024, kSwizzle128B);
                            mma_f16_ss(tmem + kColS + (g & 1) * kKeys, ad, bd, id_qk, (i > 0 || kk > 0) ? 1u : 0u);
                        }
                    mma_commit(bar(M_SFULL + (g & 1)));
                    ++qg;
                    if (++qc == qu.NT) {
                        qc = 0;
                        if (++qj < n_units) qu = unit(qj);
                    }
                    progressed = true;
                }
                if (pg < qg && mbar_test_wait(bar(M_PFULL + (pg & 1)), (pg >> 1) & 1)) {
                    const int g = pg;
                    tc_fence_after();
                    const uint32_t vs = sbase + kOffKV + (g % kStages) * kStageBytes + 3 * kSlab;
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk) {
                        // B = the V tile read MN-major: 64 values per 128-byte row,
                        // LBO = next 64 columns (slab), SBO = next 8 keys
                        const uint64_t bd = smem_desc(vs + kk * 2048, kSlab, 1024, kSwizzle128B);
                        mma_f16_ts(tmem + kColO, tmem + kColP + (g & 1) * 64 + kk * 8, bd, id_pv,
                                   (pc > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar(M_PVDONE + (g & 1)));
                    mma_commit(bar(M_KEMPTY + (g % kStages)));
                    ++pg;
                    if (++pc == pu.NT) {
                        pc = 0;
                        if (++pj < n_units) pu = unit(pj);
                    }
                    progressed = true;
                }
                if (progressed) {
                    t_idle = globaltimer_ns();
                } else if (*abort_flag) {
                    ok = false;
                } else if (globaltimer_ns() - t_idle > kWaitLimitNs) {
                    *abort_flag = 1;
                    report_timeout(M_PFULL, pg, 0);
                    ok = false;
                }
            }
            // every MMA issued completes before TMEM is released
            mma_commit(bar(M_DRAIN));
            const uint64_t t0n = globaltimer_ns();
            while (!mbar_try_wait(bar(M_DRAIN), 0) && globaltimer_ns() - t0n < kWaitLimitNs) {
            }
        }
    } else if (warp >= 4) {
        // --------------------------------------------- softmax + epilogue
        const int hs = (warp - 4) >> 2;
        const int i = (warp & 3) * 32 + lane;                  // query row of the tile = TMEM lane
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        float* red = reinterpret_cast<float*>(sgen + kOffRed);
        float* lsum_s = reinterpret_cast<float*>(sgen + kOffLsum);
        bool ok = true;
        int g0 = 0;
        for (int u = 0; ok && u < n_units; ++u) {
            const Unit w = unit(u);
            const int t = w.t0 + i, h = w.h, NT = w.NT;
            float m_use = -INFINITY, l = 0.f;
            // keys s <= t + shift (and s < S) of this row
            const int s_lim = t < T ? min(S - 1, t + shift) : -1;
            for (int j = 0; ok && j < NT; ++j) {
                const int g = g0 + j;
                const int b = g & 1;
                if (!wait_w(bar(M_SFULL + b), (g >> 1) & 1, abort_flag, 200, g)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[64];
                tmem_ld32(tmem + lane_addr + kColS + b * kKeys + 64 * hs, *reinterpret_cast<uint32_t(*)[32]>(sr));
                tmem_ld32(tmem + lane_addr + kColS + b * kKeys + 64 * hs + 32,
                          *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(M_SFREE + b));
                const int s0 = kKeys * j + 64 * hs;
                float x[64];
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    x[c] = s0 + c <= s_lim ? __uint_as_float(sr[c]) * scale_log2 : -INFINITY;
                float mx = x[0];
#pragma unroll
                for (int c = 1; c < 64; ++c) mx = fmaxf(mx, x[c]);
                // row maximum over both key halves (the other half lives in warp +-4)
                red[(b * 2 + hs) * kRows + i] = mx;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(M_RED + b));
                if (!wait_w(bar(M_RED + b), (g >> 1) & 1, abort_flag, 201, g)) { ok = false; break; }
                const float mc = fmaxf(mx, red[(b * 2 + (hs ^ 1)) * kRows + i]);
                const float m_new = fmaxf(m_use, mc);
                const bool raise = m_new > m_use + 8.f;
                const bool rescale = raise && m_use != -INFINITY;
                const float f = rescale ? ex2(m_use - m_new) : 1.f;
                if (__any_sync(0xffffffffu, rescale)) {
                    // O holds earlier tiles of this unit: rescale this half's 64
                    // columns once PV(g-1) has landed (warp-wide TMEM access; f = 1
                    // where the maximum did not move)
                    if (!wait_w(bar(M_PVDONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort_flag, 202, g)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int q2 = 0; q2 < 2; ++q2) {
                        uint32_t o[32];
                        const uint32_t ta = tmem + lane_addr + kColO + 64 * hs + 32 * q2;
                        tmem_ld32(ta, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                        tmem_st32(ta, o);
                    }
                    tmem_wait_st();
                }
                l *= f;
                if (raise) m_use = m_new;
                const float msub = m_use == -INFINITY ? 0.f : m_use;
                uint32_t pk[32];
                float ps = 0.f;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float p0 = ex2(x[2 * c] - msub), p1 = ex2(x[2 * c + 1] - msub);
                    ps += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
                l += ps;
                // P buffer b is free once PV(g-2) has read it
                if (g >= 2 && !wait_w(bar(M_PVDONE + b), ((g - 2) >> 1) & 1, abort_flag, 203, g)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_st32(tmem + lane_addr + kColP + b * 64 + 32 * hs, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(M_PFULL + b));
            }
            // row sum over both key halves (buffer u & 1)
            if (ok) {
                lsum_s[((u & 1) * 2 + hs) * kRows + i] = l;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(M_LSUM));
                ok = wait_w(bar(M_LSUM), u & 1, abort_flag, 204, u);
                if (ok) l += lsum_s[((u & 1) * 2 + (hs ^ 1)) * kRows + i];
            }
            if (ok) {
                const int gl = g0 + NT - 1;
                ok = wait_w(bar(M_PVDONE + (gl & 1)), (gl >> 1) & 1, abort_flag, 205, gl);
            }
            if (ok) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_addr + kColO + 64 * hs + 32 * q2, o);
                    tmem_wait_ld();
                    if (t < T) {
                        uint32_t wv[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)t * Hq + h) * kDv + 64 * hs + 32 * q2);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
                    }
                }
                // O is read: the next unit's first PV may overwrite it (its P
                // arrives only after this warp's next tile)
                tc_fence_before();
                if (hs == 0 && t < T)
                    lse[(size_t)t * Hq + h] = l > 0.f ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            }
            g0 += NT;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace mha_tc
}  // namespace dsa
