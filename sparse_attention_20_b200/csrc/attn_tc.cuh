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
// Decode variant (few rows): the selected set of a row can be split across
// `splits` clusters, each taking a contiguous range of the row's chunks; a
// cluster then writes its partial output normalised by its own softmax sum
// (fp32) and its log-sum-exp, and lse_merge_kernel combines the parts
// ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models",
// section "2.3 Inference Costs": decoding reads the cache, so the work of one
// query token is spread over more SMs).
//
// The kernel is persistent: one cluster per pair of SMs walks the work units
// (row, part) cid, cid + clusters, ... in order of decreasing row length. Every
// per-chunk barrier counts chunks across units, so the gather ring, the QK
// MMAs and the exchange run on into the next unit while the softmax warps
// finish the current one (its last chunk, the row-sum exchange, the
// epilogue): the per-row setup (barriers, TMEM, the first gathers and Q
// loads) is paid once per cluster, not once per row.
//
// Warp roles (512 threads per CTA): warp 0 allocates TMEM and issues the QK
// and PV MMAs and the Q TMA loads (one thread polling every kind of
// readiness, so a late chunk never holds back the PV of the previous one);
// warps 1-3 gather the selected rows with 16-byte cp.async into
// 128B/64B-swizzled shared memory (4-stage ring of 64-row chunks; completion
// is counted on the stage's mbarrier, so the gather runs up to four chunks
// ahead); warps 12-15
// (one per TMEM lane quarter) run the exchange: they stage the chunk's fp16
// partial logits locally and send them with one bulk copy per warp into the
// peer's shared memory, counted on the peer's mbarrier; warps 4-11 (two per
// lane quarter, each taking 32 of a chunk's 64 keys) run the softmax, write
// the next unit's latent Q columns into TMEM once the current unit's last
// QK has completed, and run the epilogue.
// Shared memory per CTA: Q 40 KB (latent columns 128..255 of the slice and the
// rope slice) + 4 x 36 KB ring + 16 KB receive slot + 16 KB staging.
// TMEM: O cols [0,256), S double buffer [256,384), latent Q [384,448), P
// (bf16 pairs) double buffer [448,512).
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
constexpr int kStages = 4;
constexpr int kThreads = 512;               // 16 warps: MMA, 3 gather, 8 softmax, 4 senders
constexpr int kGatherThreads = 96;

constexpr int kQSlab = kHeads * 128;        // 64 latent columns x 128 heads, 128B swizzle
// Q in shared memory: latent columns [128, 256) of this CTA's slice (two
// slabs) and the rope slice (32 columns, 64B swizzle). Latent columns [0, 128)
// live in TMEM.
constexpr int kQBytes = 2 * kQSlab + kHeads * 64;
constexpr int kKSlab = kKeys * 128;
constexpr int kStageBytes = 4 * kKSlab + kKeys * 64;
// Exchange slot: fp16 partial logits of one chunk, [head][64 keys], 128 B per
// head with the eight 16 B pieces rotated by the head index. One sender warp
// owns the contiguous 4 KB of its 32 heads and sends them as one bulk copy.
constexpr int kXBytes = kHeads * 128;
// One receive slot and one staging slot: chunk c+1 is staged and sent once
// the peer has taken chunk c out of its slot, which also proves that the
// bulk copy of c has finished reading the staging slot.
constexpr int kXSlots = 1;
constexpr int kXWarpBytes = 32 * 128;
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffX = kOffKV + kStages * kStageBytes;
constexpr int kOffXS = kOffX + kXSlots * kXBytes;         // staging of outgoing slots
constexpr int kOffBar = kOffXS + kXSlots * kXBytes;
constexpr int kOffMask = kOffBar + 256;                 // [kStages][2] validity bits
constexpr int kOffRed = kOffMask + 64;                  // [2 parity][2 halves][128] row maxima
constexpr int kOffLsum = kOffRed + 2 * 2 * kHeads * 4;  // [2 unit parities][2 halves][128] row sums
constexpr int kOffRows = kOffLsum + 2 * 2 * kHeads * 4;     // [3 gather warps][64] row byte offsets
constexpr int kSmemBytes = kOffRows + 3 * kKeys * 8 + 1024;  // + 1 KB alignment slack

constexpr uint32_t kTmemCols = 512;
// O [0,256); S double buffer [256,384); latent Q columns [0,128) of the
// slice [384,448); P double buffer (bf16 pairs) [448,512).
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 384, kColP = 448;

enum : int {
    B_Q = 0, B_QT = 1, B_FULL = 2, B_EMPTY = 6, B_SFULL = 10, B_PFULL = 12, B_PVDONE = 14,
    B_XFULL = 16, B_XFREE = 18, B_DRAIN = 20, B_RED = 21, B_LSUM = 23, B_SFREE = 24, B_COUNT = 26
};

static_assert(kOffKV % 1024 == 0 && kStageBytes % 1024 == 0 && kOffX % 1024 == 0, "alignment");
static_assert(8 * B_COUNT + 16 <= 256, "barrier area");
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

// Destination of 16-byte piece j (0..35) of gathered row r in a stage: pieces
// 0..31 go to four 128B-swizzled slabs of 64 columns, 32..35 to one
// 64B-swizzled slab of 32 columns (the layouts the MMA descriptors name).
__device__ __forceinline__ uint32_t piece_dst(uint32_t stage, int r, int j)
{
    if (j < 32) return stage + (j >> 3) * kKSlab + r * 128 + (((j & 7) ^ (r & 7)) << 4);
    return stage + 4 * kKSlab + r * 64 + (((j - 32) ^ ((r >> 1) & 3)) << 4);
}

// Source column of piece j for CTA `rank`.
__device__ __forceinline__ int piece_col(uint32_t rank, int j)
{
    return j < 32 ? (int)rank * 256 + j * 8 : 512 + (int)rank * 32 + (j - 32) * 8;
}

// Bounded wait whose outcome is the same for the whole warp.
__device__ __forceinline__ bool wait_warp(uint32_t b_addr, uint32_t par, volatile int* abort_flag,
                                          int tag, int c)
{
    return __all_sync(0xffffffffu, mbar_wait(b_addr, par, abort_flag, tag, c));
}

// A work unit of the persistent kernel: part `part` of query row t's
// selected set (unit u: t = T-1-u/splits, long rows first).
struct Unit {
    int t, part, e0, n_row, NC, p_last;
    long long base;
    const int* bt;   // block-table line of a paged cache, else NULL
};

__device__ __forceinline__ Unit unit_of(int u, const PagedRows& pg, const int* pos, const int* k_base, int T,
                                        int S, int k, int splits)
{
    Unit w;
    w.t = T - 1 - u / splits;
    w.part = u % splits;
    const int n_cand = row_keys(pg, pos, k_base, w.t, T, S, &w.base, &w.bt);
    w.p_last = n_cand - 1;
    // this unit's entries of the row: chunks [c0, c1) of its ceil(n/64)
    const int n_all = min(k, n_cand);
    const int nc_all = ceil_div(n_all, kKeys);
    const int c0 = (int)((long long)nc_all * w.part / splits);
    const int c1 = (int)((long long)nc_all * (w.part + 1) / splits);
    w.e0 = c0 * kKeys;
    w.n_row = max(0, min(c1 * kKeys, n_all) - w.e0);
    w.NC = ceil_div(w.n_row, kKeys);
    return w;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_mla_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q128,
                          const __grid_constant__ CUtensorMap tm_q64,
                          const __nv_bfloat16* __restrict__ q,
                          const __nv_bfloat16* __restrict__ kv,
                          const int* __restrict__ idx, const int* __restrict__ pos,
                          const int* __restrict__ k_base, int T, int S, int k, float scale_log2,
                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse, const PagedRows pg,
                          int splits, float* __restrict__ part_o, float* __restrict__ part_lse)
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
    griddep_wait();
    // units cid, cid + ncl, ... of the T * splits (every role walks the same
    // sequence; per-chunk barrier phases count chunks across units)
    const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
    const int n_units_all = T * splits;
    const int n_units = cid < n_units_all ? (n_units_all - cid + ncl - 1) / ncl : 0;
    auto unit = [&](int j) -> Unit { return unit_of(cid + j * ncl, pg, pos, k_base, T, S, k, splits); };

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q), 1);
        mbar_init(bar(B_QT), 8);        // latent Q written to TMEM by the softmax warps
        // S(c) read by every softmax and sender warp
        for (int b = 0; b < 2; ++b) mbar_init(bar(B_SFREE + b), 12);
        for (int s = 0; s < kStages; ++s) {
            // every gather thread's cp.async arrival + the mask publisher
            mbar_init(bar(B_FULL + s), kGatherThreads + 1);
            mbar_init(bar(B_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_SFULL + b), 1);
            mbar_init(bar(B_PFULL + b), 8);
            mbar_init(bar(B_PVDONE + b), 1);
            if (b < kXSlots) {
                mbar_init(bar(B_XFULL + b), 1);   // receiver's expect_tx + the peer senders' bytes
                mbar_init(bar(B_XFREE + b), 8);   // one arrival per softmax warp of the peer
            }
            mbar_init(bar(B_RED + b), 8);
        }
        mbar_init(bar(B_DRAIN), 1);     // the MMA issuer
        mbar_init(bar(B_LSUM), 8);
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
    bool issued_any = false;

    if (warp == 0) {
        // ------------------------------------------------- QK and PV MMAs
        // One thread issues both: QK(g) once chunk g is gathered and its S
        // buffer has been read (chunk g-2), PV(g) once the softmax has written
        // P(g); g counts chunks across this cluster's units. The Q tiles of a
        // unit are loaded once every QK of the previous unit has completed.
        // Readiness is polled without blocking so that neither kind of MMA
        // waits behind the other; the tensor pipe runs them in issue order.
        if (lane == 0) {
            prefetch_tmap(&tm_q128);
            prefetch_tmap(&tm_q64);
            const uint32_t id_qk = idesc_bf16(128, kKeys, false);
            const uint32_t id_pv = idesc_bf16(128, 256, true);
            bool ok = true;
            Unit qu{}, pu{};
            int qj = 0, qc = 0, qg = 0, qq = 0;   // QK cursor: unit, local chunk, global chunk, Q index
            int pj = 0, pc = 0, pgl = 0;          // PV cursor
            auto seek = [&](int& j, Unit& w) {
                for (; j < n_units; ++j) {
                    w = unit(j);
                    if (w.NC > 0) return;
                }
            };
            seek(qj, qu);
            pj = qj;
            pu = qu;
            int q_issued = 0;         // Q loads issued (units with entries)
            int g_prev_last = -1;     // last QK of the previous unit with entries
            uint64_t t_idle = globaltimer_ns();
            while (ok && pj < n_units) {
                bool progressed = false;
                if (qj < n_units && q_issued == qq &&
                    (g_prev_last < 0 ||
                     mbar_test_wait(bar(B_SFULL + (g_prev_last & 1)), (g_prev_last >> 1) & 1))) {
                    // Q of the unit at the QK cursor: latent columns [128,256) of
                    // the slice and the rope slice
                    mbar_arrive_expect_tx(bar(B_Q), kQBytes);
                    for (int j = 0; j < 2; ++j)
                        tma_load_2d(qs + j * kQSlab, &tm_q128, (int)rank * 256 + 128 + j * 64, qu.t * kHeads,
                                    bar(B_Q));
                    tma_load_2d(qs + 2 * kQSlab, &tm_q64, 512 + (int)rank * 32, qu.t * kHeads, bar(B_Q));
                    ++q_issued;
                    progressed = true;
                }
                if (qj < n_units && q_issued > qq &&
                    mbar_test_wait(bar(B_FULL + qg % kStages), (qg / kStages) & 1) &&
                    (qg < 2 || mbar_test_wait(bar(B_SFREE + (qg & 1)), ((qg - 2) >> 1) & 1)) &&
                    (qc > 0 || (mbar_test_wait(bar(B_Q), qq & 1) && mbar_test_wait(bar(B_QT), qq & 1)))) {
                    const int g = qg;
                    // the stage was written by cp.async (generic proxy); the MMA
                    // reads it through the async proxy
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t kvs = sbase + kOffKV + (g % kStages) * kStageBytes;
                    const uint32_t d = tmem + kColS + (g & 1) * kKeys;
                    // latent columns [0,128) of the slice: A = Q in TMEM (8 K-steps)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t bd = smem_desc(kvs + (kk >> 2) * kKSlab + (kk & 3) * 32, 16, 1024, kSwizzle128B);
                        mma_f16_ts(d, tmem + kColQ + kk * 8, bd, id_qk, kk > 0 ? 1u : 0u);
                    }
                    // latent columns [128,256): A = Q in shared memory (8 K-steps)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t ad = smem_desc(qs + (kk >> 2) * kQSlab + (kk & 3) * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = smem_desc(kvs + (2 + (kk >> 2)) * kKSlab + (kk & 3) * 32, 16, 1024, kSwizzle128B);
                        mma_f16_ss(d, ad, bd, id_qk, 1u);
                    }
                    // rope part: A = Q rope slice in shared memory
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const uint64_t ad = smem_desc(qs + 2 * kQSlab + kk * 32, 16, 512, kSwizzle64B);
                        const uint64_t bd = smem_desc(kvs + 4 * kKSlab + kk * 32, 16, 512, kSwizzle64B);
                        mma_f16_ss(d, ad, bd, id_qk, 1u);
                    }
                    mma_commit(bar(B_SFULL + (g & 1)));
                    issued_any = true;
                    ++qg;
                    if (++qc == qu.NC) {
                        g_prev_last = g;
                        ++qq;
                        qc = 0;
                        ++qj;
                        seek(qj, qu);
                    }
                    progressed = true;
                }
                if (pgl < qg && mbar_test_wait(bar(B_PFULL + (pgl & 1)), (pgl >> 1) & 1)) {
                    const int g = pgl;
                    tc_fence_after();
                    const uint32_t kvs = sbase + kOffKV + (g % kStages) * kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk) {
                        // B = gathered rows read MN-major: 64 values per 128-byte row,
                        // LBO = next 64 columns (slab), SBO = next 8 keys.
                        const uint64_t bd = smem_desc(kvs + kk * 16 * 128, kKSlab, 1024, kSwizzle128B);
                        mma_f16_ts(tmem + kColO, tmem + kColP + (g & 1) * 32 + kk * 8, bd, id_pv,
                                   (pc > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar(B_PVDONE + (g & 1)));
                    mma_commit(bar(B_EMPTY + (g % kStages)));
                    ++pgl;
                    if (++pc == pu.NC) {
                        pc = 0;
                        ++pj;
                        seek(pj, pu);
                    }
                    progressed = true;
                }
                if (progressed) {
                    t_idle = globaltimer_ns();
                } else if (*abort_flag) {
                    ok = false;
                } else if (globaltimer_ns() - t_idle > kWaitLimitNs) {
                    *abort_flag = 1;
                    report_timeout(B_PFULL, pgl, 0);
                    ok = false;
                }
            }
        }
    } else if (warp <= 3) {
        // ---------------------------------------------------------- gather
        // The 64 x 36 sixteen-byte pieces of a chunk are spread evenly over the
        // 96 gather threads: piece e = it*96 + g is row e/36, piece e%36. The
        // (row, piece) pattern of a thread repeats every three iterations with
        // the row advanced by 8, which keeps the swizzle phase, so a copy costs
        // one table load and one cp.async. Each warp keeps its own table of the
        // chunk's row byte offsets (-1 = masked entry, read as zeros). The ring
        // runs on across units: the next unit's first chunks are gathered
        // while the current one finishes.
        const int gw = warp - 1;
        const int g = threadIdx.x - 32;
        uint32_t* smask = reinterpret_cast<uint32_t*>(sgen + kOffMask);
        long long* rows_tab = reinterpret_cast<long long*>(sgen + kOffRows) + gw * kKeys;
        int r_q[3];
        uint32_t d_q[3], dstep_q[3];
        int col_q[3];
#pragma unroll
        for (int q3 = 0; q3 < 3; ++q3) {
            const int e = q3 * kGatherThreads + g;
            const int r = e / 36, j = e - r * 36;
            r_q[q3] = r;
            d_q[q3] = piece_dst(0, r, j);
            dstep_q[q3] = j < 32 ? 8 * 128 : 8 * 64;
            col_q[q3] = piece_col(rank, j) * 2;   // bytes
        }
        const char* kvb = reinterpret_cast<const char*>(kv);
        int gg = 0;
        bool ok = true;
        for (int j = 0; ok && j < n_units; ++j) {
            const Unit w = unit(j);
            if (w.NC == 0) continue;
            const int* idx_row = idx + (size_t)w.t * k + w.e0;
            int sa = lane < w.n_row ? __ldg(idx_row + lane) : -1;
            int sb = lane + 32 < w.n_row ? __ldg(idx_row + lane + 32) : -1;
            for (int c = 0; c < w.NC; ++c, ++gg) {
                const int st = gg % kStages;
                if (gg >= kStages) {
                    const bool got = mbar_wait(bar(B_EMPTY + st), ((gg - kStages) / kStages) & 1,
                                               abort_flag, 100 + B_EMPTY, gg);
                    if (!__all_sync(0xffffffffu, got)) {   // warp-uniform exit
                        ok = false;
                        break;
                    }
                }
                const bool va = sa >= 0 && sa <= w.p_last, vb = sb >= 0 && sb <= w.p_last;
                rows_tab[lane] = va ? key_row(pg, w.bt, w.base, sa) * (long long)(kDqk * 2) : -1ll;
                rows_tab[lane + 32] = vb ? key_row(pg, w.bt, w.base, sb) * (long long)(kDqk * 2) : -1ll;
                if (gw == 0) {
                    const unsigned ma = __ballot_sync(0xffffffffu, va), mb = __ballot_sync(0xffffffffu, vb);
                    if (lane == 0) {
                        smask[st * 2] = ma;
                        smask[st * 2 + 1] = mb;
                    }
                }
                const int i_next = (c + 1) * kKeys + lane;
                sa = i_next < w.n_row ? __ldg(idx_row + i_next) : -1;
                sb = i_next + 32 < w.n_row ? __ldg(idx_row + i_next + 32) : -1;
                __syncwarp();
                const uint32_t kvs = sbase + kOffKV + st * kStageBytes;
#pragma unroll
                for (int m = 0; m < 8; ++m)
#pragma unroll
                    for (int q3 = 0; q3 < 3; ++q3) {
                        const long long off = rows_tab[r_q[q3] + 8 * m];
                        const void* src = off >= 0 ? kvb + off + col_q[q3] : kvb;
                        cp_async16(kvs + d_q[q3] + m * dstep_q[q3], src, off >= 0 ? 16u : 0u);
                    }
                cp_async_arrive_noinc(bar(B_FULL + st));
                if (gw == 0 && lane == 0) mbar_arrive(bar(B_FULL + st));   // publishes the mask
                __syncwarp();   // the table is rewritten for the next chunk
            }
        }
        cp_async_wait_all();
    } else if (warp >= 12) {
        // ------------------------------------------------------- senders
        // Warps 12-15, one per TMEM lane quarter: ship this CTA's partial
        // logits of each chunk (scaled to log2 units, fp16) to the peer. A warp
        // stages its 32 heads x 64 keys locally and sends the 4 KB with one
        // bulk copy, counted in bytes on the peer's XFULL barrier.
        const int qd = warp & 3;
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        const uint32_t xwarp = (uint32_t)qd * kXWarpBytes;
        const uint32_t xrow = xwarp + (uint32_t)lane * 128;
        const uint32_t x_peer = mapa(sbase + kOffX, peer);
        const uint32_t xfull_peer = mapa(bar(B_XFULL), peer);
        const uint32_t xstage = sbase + kOffXS;
        int gs = 0;
        bool ok = true;
        for (int j = 0; ok && j < n_units; ++j) {
            const int NC = unit(j).NC;
            for (int c = 0; c < NC; ++c, ++gs) {
                const int b = gs & 1;
                if (!wait_warp(bar(B_SFULL + b), (gs >> 1) & 1, abort_flag, 500 + B_SFULL, gs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t s0[32], s1[32];
                tmem_ld32(tmem + lane_addr + kColS + b * kKeys, s0);
                tmem_ld32(tmem + lane_addr + kColS + b * kKeys + 32, s1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_SFREE + b));
                uint32_t h[32];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    h[jj] = pack_half2(__uint_as_float(s0[2 * jj]) * scale_log2,
                                       __uint_as_float(s0[2 * jj + 1]) * scale_log2);
                    h[16 + jj] = pack_half2(__uint_as_float(s1[2 * jj]) * scale_log2,
                                            __uint_as_float(s1[2 * jj + 1]) * scale_log2);
                }
                // The peer has consumed chunk gs-kXSlots from slot xb, so the bulk
                // copy of that chunk has landed: it has also finished reading
                // staging slot xb.
                const int xb = gs % kXSlots;
                if (gs >= kXSlots && !wait_warp(bar(B_XFREE + xb), ((gs - kXSlots) / kXSlots) & 1, abort_flag,
                                                500 + B_XFREE, gs)) {
                    ok = false;
                    break;
                }
                const uint32_t stg = xstage + xb * kXBytes;
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    st_shared_v4(stg + xrow + (((m + lane) & 7) << 4),
                                 make_uint4(h[4 * m], h[4 * m + 1], h[4 * m + 2], h[4 * m + 3]));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    bulk_s2cluster(x_peer + xb * kXBytes + xwarp, stg + xwarp, kXWarpBytes, xfull_peer + 8u * xb);
            }
        }
    } else if (warp >= 4) {
        // --------------------------------------------- softmax + epilogue
        // Warps 4-11: two warps per TMEM lane quarter; warp half hs takes keys
        // [32hs, 32hs+32) of every chunk and output columns [128hs, 128hs+128).
        const int hs = (warp - 4) >> 2;
        const int i = (warp & 3) * 32 + lane;                  // head = TMEM lane
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        // head i's 128 B row of an exchange slot
        const uint32_t xs = sbase + kOffX + (uint32_t)i * 128;
        const uint32_t xfree_peer = mapa(bar(B_XFREE), peer);
        const uint32_t* smask = reinterpret_cast<const uint32_t*>(sgen + kOffMask);
        float* red = reinterpret_cast<float*>(sgen + kOffRed);
        float* lsum_s = reinterpret_cast<float*>(sgen + kOffLsum);
        bool ok = true;
        auto wait_w = [&](uint32_t b_addr, uint32_t par, int tag, int c) -> bool {
            return wait_warp(b_addr, par, abort_flag, tag, c);
        };
        // latent Q columns [0,128) of a unit's row for head i into TMEM (A
        // operand of the QK MMAs): this half's 64 columns, two bf16 per 32-bit
        // TMEM column
        auto write_q = [&](int t) {
            const uint4* qsrc = reinterpret_cast<const uint4*>(
                q + ((size_t)t * kHeads + i) * kDqk + rank * 256 + 64 * hs);
            uint32_t w[32];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint4 x = __ldg(qsrc + v);
                w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
            }
            tmem_st32(tmem + lane_addr + kColQ + 32 * hs, w);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_QT));
        };
        // the next unit with entries after iteration j (n_units if none)
        auto next_with_entries = [&](int j, int* t_out) -> int {
            for (++j; j < n_units; ++j) {
                const Unit w = unit(j);
                if (w.NC > 0) {
                    *t_out = w.t;
                    return j;
                }
            }
            return n_units;
        };
        {
            int t_first;
            if (next_with_entries(-1, &t_first) < n_units) write_q(t_first);
        }
        int g0 = 0;
        for (int j = 0; j < n_units; ++j) {
            const Unit w = unit(j);
            const int NC = w.NC, t = w.t, part = w.part;
            float m_use = -INFINITY, l = 0.f;
            for (int c = 0; ok && c < NC; ++c) {
                const int gc = g0 + c;
                const int b = gc & 1;
                const int xb = gc % kXSlots;
                if (i == 0 && hs == 0) mbar_arrive_expect_tx(bar(B_XFULL + xb), kXBytes);
                // the chunk's validity bits (its gather completed long before S(c))
                if (!wait_w(bar(B_FULL + gc % kStages), (gc / kStages) & 1, 200 + B_FULL, gc)) { ok = false; break; }
                const uint32_t mw = smask[(gc % kStages) * 2 + hs];
                // this CTA's partial logits of chunk c (fp32, TMEM)
                if (!wait_w(bar(B_SFULL + b), (gc >> 1) & 1, 200 + B_SFULL, gc)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[32];
                tmem_ld32(tmem + lane_addr + kColS + b * kKeys + 32 * hs, sr);
                // the peer's (fp16, scaled) arrive by bulk copy, counted on this local barrier
                if (!wait_w(bar(B_XFULL + xb), (gc / kXSlots) & 1, 200 + B_XFULL, gc)) {
                    tmem_wait_ld();
                    ok = false;
                    break;
                }
                uint32_t gx[16];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint4 v = ld_shared_v4(xs + xb * kXBytes + (((4 * hs + m + lane) & 7) << 4));
                    gx[4 * m] = v.x; gx[4 * m + 1] = v.y; gx[4 * m + 2] = v.z; gx[4 * m + 3] = v.w;
                }
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_SFREE + b));   // S(c) fully read by this warp
                // logit (log2 domain) = own partial (fp32) + peer partial (fp16); masked -> -inf
                float x[32];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const float2 o = unpack_half2(gx[jj]);
                    x[2 * jj] = (mw >> (2 * jj)) & 1u ? fmaf(__uint_as_float(sr[2 * jj]), scale_log2, o.x)
                                                      : -INFINITY;
                    x[2 * jj + 1] = (mw >> (2 * jj + 1)) & 1u
                                        ? fmaf(__uint_as_float(sr[2 * jj + 1]), scale_log2, o.y)
                                        : -INFINITY;
                }
                // the peer may refill this exchange slot once every warp has used it
                // (the loaded values are consumed above, so a relaxed signal suffices)
                __syncwarp();
                if (lane == 0) mbar_arrive_remote_relaxed(xfree_peer + 8u * xb);
                float mx[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) mx[jj] = fmaxf(x[jj], x[jj + 16]);
#pragma unroll
                for (int ww = 8; ww >= 1; ww >>= 1)
#pragma unroll
                    for (int jj = 0; jj < ww; ++jj) mx[jj] = fmaxf(mx[jj], mx[jj + ww]);
                // row maximum over both key halves (the other half lives in warp +-4)
                red[(b * 2 + hs) * kHeads + i] = mx[0];
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_RED + b));
                if (!wait_w(bar(B_RED + b), (gc >> 1) & 1, 200 + B_RED, gc)) { ok = false; break; }
                const float mc = fmaxf(mx[0], red[(b * 2 + (hs ^ 1)) * kHeads + i]);
                const float m_new = fmaxf(m_use, mc);
                const bool raise = m_new > m_use + 8.f;
                const bool rescale = raise && m_use != -INFINITY;
                const float f = rescale ? ex2(m_use - m_new) : 1.f;
                if (__any_sync(0xffffffffu, rescale)) {
                    // O holds earlier chunks of this unit: rescale once PV(c-1)
                    // has landed. TMEM loads/stores are warp-wide, so every lane
                    // takes part (f = 1 for rows whose maximum did not move).
                    if (!wait_w(bar(B_PVDONE + ((gc - 1) & 1)), ((gc - 1) >> 1) & 1, 400 + B_PVDONE, gc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t o[32];
                        const uint32_t ta = tmem + lane_addr + kColO + 128 * hs + q4 * 32;
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
                uint32_t pk[16];
                float ps[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const float p0 = ex2(x[2 * jj] - msub), p1 = ex2(x[2 * jj + 1] - msub);
                    ps[jj] = p0 + p1;
                    pk[jj] = pack_bf16x2(p0, p1);
                }
#pragma unroll
                for (int ww = 8; ww >= 1; ww >>= 1)
#pragma unroll
                    for (int jj = 0; jj < ww; ++jj) ps[jj] += ps[jj + ww];
                l += ps[0];
                // P buffer b is free once PV(g-2) has read it
                if (gc >= 2 && !wait_w(bar(B_PVDONE + b), ((gc - 2) >> 1) & 1, 200 + B_PVDONE, gc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_st16(tmem + lane_addr + kColP + b * 32 + 16 * hs, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PFULL + b));
            }
            // every QK of this unit has completed (its last S was read): the
            // next unit's Q goes into TMEM now, so its first QKs overlap this
            // unit's epilogue
            if (ok && NC > 0) {
                int t_next;
                if (next_with_entries(j, &t_next) < n_units) write_q(t_next);
            }
            // row sum over both key halves (buffer j & 1)
            if (ok) {
                lsum_s[((j & 1) * 2 + hs) * kHeads + i] = l;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_LSUM));
                ok = wait_w(bar(B_LSUM), j & 1, 200 + B_LSUM, j);
                if (ok) l += lsum_s[((j & 1) * 2 + (hs ^ 1)) * kHeads + i];
            }
            // epilogue: O / l -> bf16 (or, for a part of a split row, fp32 into
            // the parts buffer), columns [128hs, 128hs+128) of this CTA's half
            const size_t prow = ((size_t)t * splits + part) * kHeads + i;   // parts layout [T, splits, 128]
            __nv_bfloat16* orow = out + ((size_t)t * kHeads + i) * kDv + rank * 256 + 128 * hs;
            float* porow = splits > 1 ? part_o + prow * kDv + rank * 256 + 128 * hs : nullptr;
            if (ok && NC > 0) {
                const int gl = g0 + NC - 1;
                ok = wait_w(bar(B_PVDONE + (gl & 1)), (gl >> 1) & 1, 300 + B_PVDONE, gl);
                if (ok) {
                    tc_fence_after();
                    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_addr + kColO + 128 * hs + q4 * 32, o);
                        tmem_wait_ld();
                        if (porow) {
                            float4* dst = reinterpret_cast<float4*>(porow + q4 * 32);
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                                     __uint_as_float(o[4 * v + 2]) * inv,
                                                     __uint_as_float(o[4 * v + 3]) * inv);
                            continue;
                        }
                        uint32_t wv[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                                __uint_as_float(o[2 * e + 1]) * inv);
                        uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 32);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
                    }
                    // O is read: the next unit's first PV may overwrite it (its
                    // P arrives only after this warp's next chunk)
                    tc_fence_before();
                }
            } else if (NC == 0) {
                if (porow) {
                    float4* dst = reinterpret_cast<float4*>(porow);
                    for (int v = 0; v < 32; ++v) dst[v] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(orow);
                    for (int v = 0; v < 16; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            if (rank == 0 && hs == 0 && (ok || NC == 0)) {
                const float lv = l > 0.f ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
                if (splits > 1)
                    part_lse[prow] = lv;
                else
                    lse[(size_t)t * kHeads + i] = lv;
            }
            g0 += NC;
            if (!ok) break;
        }
    }

    if (warp == 0 && lane == 0 && issued_any) {
        // every MMA issued completes before TMEM is released
        mma_commit(bar(B_DRAIN));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar(B_DRAIN), 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    cluster_sync();   // no CTA leaves while its peer may still touch its shared memory
}

// Log-sum-exp merge of a split row's parts (decode variant): for row t and
// head h, with parts z of (o_z normalised by its own softmax sum, lse_z),
//   lse = log sum_z exp(lse_z),  out = sum_z exp(lse_z - lse) o_z.
// One CTA of 128 threads per (row, 8 heads); each thread owns four
// consecutive columns of one head at a time (float4 loads of every part).
constexpr int kMergeHeads = 8;

__global__ void __launch_bounds__(128)
lse_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse, int T, int splits,
                 __nv_bfloat16* __restrict__ out, float* __restrict__ lse)
{
    __shared__ float wz[kMergeHeads][16];
    griddep_wait();
    const int t = blockIdx.x;
    const int h0 = blockIdx.y * kMergeHeads;
    if (threadIdx.x < kMergeHeads) {
        const int h = h0 + threadIdx.x;
        float m = -INFINITY;
        for (int z = 0; z < splits; ++z) m = fmaxf(m, part_lse[((size_t)t * splits + z) * kHeads + h]);
        float total = -INFINITY;
        if (m != -INFINITY) {
            float l = 0.f;
            for (int z = 0; z < splits; ++z) l += expf(part_lse[((size_t)t * splits + z) * kHeads + h] - m);
            total = m + logf(l);
        }
        for (int z = 0; z < splits; ++z) {
            const float lz = part_lse[((size_t)t * splits + z) * kHeads + h];
            wz[threadIdx.x][z] = (total == -INFINITY || lz == -INFINITY) ? 0.f : expf(lz - total);
        }
        lse[(size_t)t * kHeads + h] = total;
    }
    __syncthreads();
    // 8 heads x 512 columns = 1024 float4 groups, 8 per thread
    for (int e = threadIdx.x; e < kMergeHeads * kDv / 4; e += 128) {
        const int hh = e / (kDv / 4), c4 = e % (kDv / 4);
        const int h = h0 + hh;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int z = 0; z < splits; ++z) {
            const float wgt = wz[hh][z];
            const float4 v = reinterpret_cast<const float4*>(
                part_o + (((size_t)t * splits + z) * kHeads + h) * kDv)[c4];
            acc.x = fmaf(wgt, v.x, acc.x);
            acc.y = fmaf(wgt, v.y, acc.y);
            acc.z = fmaf(wgt, v.z, acc.z);
            acc.w = fmaf(wgt, v.w, acc.w);
        }
        uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
        reinterpret_cast<uint2*>(out + ((size_t)t * kHeads + h) * kDv)[c4] = pk;
    }
}

// Most parts a row is split into (the merge keeps one weight per part in
// shared memory).
constexpr int kMaxSplits = 16;

}  // namespace attn_tc
}  // namespace dsa
