// Sparse MLA attention in MQA mode on the 5th-generation tensor cores.
//
//   u_t = Attn(h_t, {c_s : s selected}); all 128 query heads attend to the
//   same latent rows c_s of width 576 (512 latent + 64 rope); the value is the
//   latent part c_s[0:512] ("Paper Breakdown: DeepSeek-V3.2", section 2,
//   "Attention" and "DSA under MLA (MQA Mode)": the shared latent row is what
//   makes the heads one M = 128 tile of a single MMA).
//
// One thread-block cluster of two CTAs (two SMs) handles one query row. The
// output accumulator O [128 heads x 512] fp32 alone fills one SM's 256 KB of
// tensor memory, so the pair splits the latent columns: CTA r owns latent
// columns [256r, 256r+256) and rope columns [512+32r, 544+32r). Each CTA
// gathers only its 288 columns of every selected row and computes a partial
// logit tile S_r = Q[:, cols_r] . C[:, cols_r]^T (tcgen05, M=128 heads,
// N=64 keys, K=288). The partials are swapped through distributed shared
// memory as fp16 (already scaled by scale*log2(e)); both CTAs then hold the
// same S = S_0 + S_1 and run the same online softmax, and each accumulates its
// own half of O = P . C[:, 256r:256r+256] (tcgen05, A = P from TMEM, B = the
// gathered rows read MN-major, N = 256). No flop is done twice and every
// selected row crosses HBM/L2 once per query.
//
// Warp roles (256 threads per CTA): warp 0 allocates TMEM and issues MMAs
// (one thread); warp 1 loads Q with TMA tiles and gathers the selected rows
// with TMA tile::gather4 (four rows per instruction, 128B/64B swizzle applied
// by the TMA unit) into a 3-stage ring of 64-row chunks; warps 4-7 (one thread
// per head = TMEM lane) run the softmax, the exchange (st.async into the
// peer's shared memory, counted on the peer's mbarrier) and the epilogue;
// warps 2-3 only take part in set-up and tear-down.
// Shared memory per CTA: Q slice 72 KB + 3 x 36 KB ring + 2 x 16 KB exchange.
// TMEM: O cols [0,256), S double buffer [256,384), P (bf16 pairs) [384,448).
#pragma once
#include <cuda.h>

#include "sm100.cuh"

namespace dsa {
namespace attn_tc {

using namespace sm100;

constexpr int kHeads = 128;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kKeys = 64;
constexpr int kStages = 3;
constexpr int kThreads = 256;

constexpr int kQSlab = kHeads * 128;        // 64 columns x 128 rows, 128B swizzle
constexpr int kQBytes = 4 * kQSlab + kHeads * 64;
constexpr int kKSlab = kKeys * 128;
constexpr int kStageBytes = 4 * kKSlab + kKeys * 64;
constexpr int kXBytes = kHeads * 128;       // 64 fp16 partial logits per head
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffX = kOffKV + kStages * kStageBytes;
constexpr int kOffBar = kOffX + 2 * kXBytes;
constexpr int kOffMask = kOffBar + 256;                 // [kStages][2] validity bits
constexpr int kSmemBytes = kOffMask + kStages * 8 + 1024;  // + 1 KB alignment slack

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColP = 384;

enum : int {
    B_Q = 0, B_FULL = 1, B_EMPTY = 4, B_SFULL = 7, B_SFREE = 9, B_PFULL = 11, B_PVDONE = 13,
    B_XFULL = 15, B_XFREE = 17, B_DRAIN = 19, B_COUNT = 20
};

static_assert(kOffKV % 1024 == 0 && kStageBytes % 1024 == 0 && kOffX % 1024 == 0, "alignment");
static_assert(kSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_half2(uint32_t v)
{
    __half2 h = *reinterpret_cast<__half2*>(&v);
    return __half22float2(h);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_mla_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q128,
                          const __grid_constant__ CUtensorMap tm_q64,
                          const __grid_constant__ CUtensorMap tm_kv128,
                          const __grid_constant__ CUtensorMap tm_kv64,
                          const int* __restrict__ idx, const int* __restrict__ pos,
                          const int* __restrict__ k_base, int T, int S, int k, float scale_log2,
                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + kOffBar;
    uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sgen + kOffBar + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + kOffBar + 8 * B_COUNT + 8);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const int t = T - 1 - (int)(blockIdx.x >> 1);   // long rows first
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    const int p_last = n_cand - 1;
    const int n_row = min(k, n_cand);
    const int NC = ceil_div(n_row, kKeys);

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B_FULL + s), 1);
            mbar_init(bar(B_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_SFULL + b), 1);
            mbar_init(bar(B_SFREE + b), 4);
            mbar_init(bar(B_PFULL + b), 4);
            mbar_init(bar(B_PVDONE + b), 1);
            mbar_init(bar(B_XFULL + b), 1);   // receiver's expect_tx + the peer's bytes
            mbar_init(bar(B_XFREE + b), 4);   // one arrival per softmax warp of the peer
        }
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
    cluster_sync();   // the peer's barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *taddr_slot;
    const uint32_t qs = sbase + kOffQ;

    if (warp == 0) {
        // ------------------------------------------------------------- MMA
        if (lane == 0 && NC > 0) {
            const uint32_t id_qk = idesc_bf16(128, kKeys, false);
            const uint32_t id_pv = idesc_bf16(128, 256, true);
            bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
            auto pv = [&](int c) -> bool {
                if (!mbar_wait(bar(B_PFULL + (c & 1)), (c >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t kvs = sbase + kOffKV + (c % kStages) * kStageBytes;
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk) {
                    // B = gathered rows read MN-major: 64 values per 128-byte row,
                    // LBO = next 64 columns (slab), SBO = next 8 keys.
                    const uint64_t bd = smem_desc(kvs + kk * 16 * 128, kKSlab, 1024, kSwizzle128B);
                    mma_f16_ts(tmem + kColO, tmem + kColP + (c & 1) * 32 + kk * 8, bd, id_pv,
                               (c > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(B_PVDONE + (c & 1)));
                mma_commit(bar(B_EMPTY + (c % kStages)));
                return true;
            };
            for (int c = 0; ok && c < NC; ++c) {
                const int st = c % kStages;
                ok = mbar_wait(bar(B_FULL + st), (c / kStages) & 1, abort_flag);
                if (ok && c >= 2) ok = mbar_wait(bar(B_SFREE + (c & 1)), ((c - 2) >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kvs = sbase + kOffKV + st * kStageBytes;
                const uint32_t d = tmem + kColS + (c & 1) * kKeys;
                uint32_t acc = 0;
#pragma unroll
                for (int slab = 0; slab < 4; ++slab)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = smem_desc(qs + slab * kQSlab + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = smem_desc(kvs + slab * kKSlab + kk * 32, 16, 1024, kSwizzle128B);
                        mma_f16_ss(d, ad, bd, id_qk, acc);
                        acc = 1;
                    }
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint64_t ad = smem_desc(qs + 4 * kQSlab + kk * 32, 16, 512, kSwizzle64B);
                    const uint64_t bd = smem_desc(kvs + 4 * kKSlab + kk * 32, 16, 512, kSwizzle64B);
                    mma_f16_ss(d, ad, bd, id_qk, 1u);
                }
                mma_commit(bar(B_SFULL + (c & 1)));
                if (c >= 1) ok = pv(c - 1);
            }
            if (ok) pv(NC - 1);
            // drain: every MMA issued above completes before TMEM is released
            mma_commit(bar(B_DRAIN));
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bar(B_DRAIN), 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ TMA loads
        if (lane == 0) {
            prefetch_tmap(&tm_q128);
            prefetch_tmap(&tm_q64);
            prefetch_tmap(&tm_kv128);
            prefetch_tmap(&tm_kv64);
            mbar_arrive_expect_tx(bar(B_Q), kQBytes);
            for (int j = 0; j < 4; ++j)
                tma_load_2d(qs + j * kQSlab, &tm_q128, (int)rank * 256 + j * 64, t * kHeads, bar(B_Q));
            tma_load_2d(qs + 4 * kQSlab, &tm_q64, 512 + (int)rank * 32, t * kHeads, bar(B_Q));
        }
        const int* idx_row = idx + (size_t)t * k;
        uint32_t* smask = reinterpret_cast<uint32_t*>(sgen + kOffMask);
        // lane holds entries lane and lane + 32 of the next chunk (one chunk ahead)
        int sa = lane < n_row ? __ldg(idx_row + lane) : -1;
        int sb = lane + 32 < n_row ? __ldg(idx_row + lane + 32) : -1;
        int issued = 0;
        for (int c = 0; c < NC; ++c) {
            const int st = c % kStages;
            if (c >= kStages && !mbar_wait(bar(B_EMPTY + st), ((c - kStages) / kStages) & 1, abort_flag))
                break;
            const bool va = sa >= 0 && sa <= p_last, vb = sb >= 0 && sb <= p_last;
            // masked entries load row 0 of the sequence (finite data, weight 0)
            const int ra = va ? sa : 0, rb = vb ? sb : 0;
            const unsigned ma = __ballot_sync(0xffffffffu, va), mb = __ballot_sync(0xffffffffu, vb);
            if (lane == 0) {
                smask[st * 2] = ma;
                smask[st * 2 + 1] = mb;
            }
            const int i_next = (c + 1) * kKeys + lane;
            sa = i_next < n_row ? __ldg(idx_row + i_next) : -1;
            sb = i_next + 32 < n_row ? __ldg(idx_row + i_next + 32) : -1;
            int y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = 4 * (lane & 15) + e;
                const int from_a = __shfl_sync(0xffffffffu, ra, key & 31);
                const int from_b = __shfl_sync(0xffffffffu, rb, key & 31);
                y[e] = (int)(base + (key < 32 ? from_a : from_b));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(bar(B_FULL + st), kStageBytes);
            __syncwarp();
            if (lane < 16) {
                const uint32_t kvs = sbase + kOffKV + st * kStageBytes;
                const int r0 = 4 * lane;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tma_gather4(kvs + j * kKSlab + r0 * 128, &tm_kv128, (int)rank * 256 + j * 64,
                                y[0], y[1], y[2], y[3], bar(B_FULL + st));
                tma_gather4(kvs + 4 * kKSlab + r0 * 64, &tm_kv64, 512 + (int)rank * 32, y[0], y[1],
                            y[2], y[3], bar(B_FULL + st));
            }
            issued = c + 1;
        }
        if (issued < NC) {
            // aborted: let the loads already issued land before the CTA ends
            for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(bar(B_FULL + c % kStages), (c / kStages) & 1) &&
                       globaltimer_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else if (warp >= 4) {
        // --------------------------------------------- softmax + epilogue
        const int i = threadIdx.x - 128;                       // head = TMEM lane
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t xs = sbase + kOffX;
        const uint32_t x_peer = mapa(xs, peer);
        const uint32_t xfull_peer = mapa(bar(B_XFULL), peer);
        const uint32_t xfree_peer = mapa(bar(B_XFREE), peer);
        const uint32_t* smask = reinterpret_cast<const uint32_t*>(sgen + kOffMask);
        float m_use = -INFINITY, l = 0.f;
        bool ok = true;

        // this CTA's partial logits of chunk c, scaled, as fp16 pairs
        auto load_partial = [&](int c, uint32_t (&h)[32]) {
            uint32_t s0[32], s1[32];
            tmem_ld32(tmem + lane_addr + kColS + (c & 1) * kKeys, s0);
            tmem_ld32(tmem + lane_addr + kColS + (c & 1) * kKeys + 32, s1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                h[j] = pack_half2(__uint_as_float(s0[2 * j]) * scale_log2,
                                  __uint_as_float(s0[2 * j + 1]) * scale_log2);
                h[16 + j] = pack_half2(__uint_as_float(s1[2 * j]) * scale_log2,
                                       __uint_as_float(s1[2 * j + 1]) * scale_log2);
            }
        };
        // send chunk c's partial into the peer's exchange slot
        auto send = [&](int c) -> bool {
            const int b = c & 1;
            if (!mbar_wait(bar(B_SFULL + b), (c >> 1) & 1, abort_flag)) return false;
            tc_fence_after();
            uint32_t h[32];
            load_partial(c, h);
            if (c >= 2 && !mbar_wait<true>(bar(B_XFREE + b), ((c - 2) >> 1) & 1, abort_flag)) return false;
            const uint32_t xr_peer = x_peer + b * kXBytes + i * 128;
#pragma unroll
            for (int m = 0; m < 8; ++m)
                st_async_v4(xr_peer + (((m + i) & 7) << 4),
                            make_uint4(h[4 * m], h[4 * m + 1], h[4 * m + 2], h[4 * m + 3]),
                            xfull_peer + 8u * b);
            return true;
        };

        if (NC > 0) ok = send(0);
        for (int c = 0; ok && c < NC; ++c) {
            const int b = c & 1;
            // the next chunk's exchange overlaps this chunk's softmax
            if (c + 1 < NC && !send(c + 1)) { ok = false; break; }
            if (i == 0) mbar_arrive_expect_tx(bar(B_XFULL + b), kXBytes);
            if (!mbar_wait<true>(bar(B_XFULL + b), (c >> 1) & 1, abort_flag)) { ok = false; break; }
            uint32_t g[32], h[32];
            const uint32_t xr = xs + b * kXBytes + i * 128;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const uint4 v = ld_shared_v4(xr + (((m + i) & 7) << 4));
                g[4 * m] = v.x; g[4 * m + 1] = v.y; g[4 * m + 2] = v.z; g[4 * m + 3] = v.w;
            }
            load_partial(c, h);                     // same rounding as what was sent
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SFREE + b));
            // validity of the chunk's entries (published by the gather warps)
            if (!mbar_wait(bar(B_FULL + c % kStages), (c / kStages) & 1, abort_flag)) { ok = false; break; }
            const uint32_t mlo = smask[(c % kStages) * 2], mhi = smask[(c % kStages) * 2 + 1];

            // full logits (log2 domain), masked entries -> -inf
            float x[kKeys];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float2 a = unpack_half2(h[j]), o = unpack_half2(g[j]);
                const uint32_t mw = j < 16 ? mlo : mhi;
                x[2 * j] = (mw >> ((2 * j) & 31)) & 1u ? a.x + o.x : -INFINITY;
                x[2 * j + 1] = (mw >> ((2 * j + 1) & 31)) & 1u ? a.y + o.y : -INFINITY;
            }
            // the peer may refill this exchange slot once every warp has used it
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(xfree_peer + 8u * b);
            float mc = -INFINITY;
#pragma unroll
            for (int j = 0; j < kKeys; ++j) mc = fmaxf(mc, x[j]);
            const float m_new = fmaxf(m_use, mc);
            if (m_new > m_use + 8.f) {
                if (m_use != -INFINITY) {
                    // O holds earlier chunks: rescale once PV(c-1) has landed
                    const float f = ex2(m_use - m_new);
                    l *= f;
                    if (!mbar_wait(bar(B_PVDONE + ((c - 1) & 1)), ((c - 1) >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int q8 = 0; q8 < 8; ++q8) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_addr + kColO + q8 * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                        tmem_st32(tmem + lane_addr + kColO + q8 * 32, o);
                    }
                    tmem_wait_st();
                }
                m_use = m_new;
            }
            const float msub = m_use == -INFINITY ? 0.f : m_use;
            uint32_t pk[32];
            float lsum = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float p0 = ex2(x[2 * j] - msub), p1 = ex2(x[2 * j + 1] - msub);
                lsum += p0 + p1;
                pk[j] = pack_bf16x2(p0, p1);
            }
            l += lsum;
            if (c >= 2 && !mbar_wait(bar(B_PVDONE + b), ((c - 2) >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_st32(tmem + lane_addr + kColP + b * 32, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_PFULL + b));
        }
        // epilogue: O / l -> bf16, this CTA's 256 columns of head i
        __nv_bfloat16* orow = out + ((size_t)t * kHeads + i) * kDv + rank * 256;
        if (ok && NC > 0) {
            const int c = NC - 1;
            ok = mbar_wait(bar(B_PVDONE + (c & 1)), (c >> 1) & 1, abort_flag);
            if (ok) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
                for (int q8 = 0; q8 < 8; ++q8) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_addr + kColO + q8 * 32, o);
                    tmem_wait_ld();
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                           __uint_as_float(o[2 * e + 1]) * inv);
                    uint4* dst = reinterpret_cast<uint4*>(orow + q8 * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
        } else if (NC == 0) {
            uint4* dst = reinterpret_cast<uint4*>(orow);
            for (int v = 0; v < 32; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (rank == 0 && (ok || NC == 0))
            lse[(size_t)t * kHeads + i] = l > 0.f ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    cluster_sync();   // no CTA leaves while its peer may still touch its shared memory
}

}  // namespace attn_tc
}  // namespace dsa
