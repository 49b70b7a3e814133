// Backward of the sparse MQA attention: the gradients that train the main
// model through the selected latent rows only (the sparse training stage of
// "Paper Breakdown: DeepSeek-V3.2", table "Continued Pre-Training (2.1.1)").
//
// Forward, per query row t and head h over the selected set (MQA: one latent
// row c_s serves every head): z_s = scale q_h.c_s, p = softmax(z),
// o_h = sum_s p_s c_s[0:d_v], lse_h = log sum_s exp(z_s). Given dout:
//   dp_s = dout_h . c_s[0:d_v]          D_h  = dout_h . o_h
//   dz_s = p_s (dp_s - D_h)             p_s  = exp(z_s - lse_h)
//   dq_h = scale sum_s dz_s c_s
//   dkv[row of s] += scale sum_h dz_{h,s} q_h + sum_h p_{h,s} dout_h[0:d_v]
//
// Two kernels, both on warp-level bf16 MMAs (m16n8k16, fp32 accumulate):
//  - attn_bwd_dkv_kernel, one CTA per (row, 64 selected slots): recomputes z
//    and dp for all heads against the 64 gathered rows, forms p and
//    g = scale dz (bf16), adds g^T q + p^T dout into dkv (float4 fp32
//    atomics, one per four columns of a slot) and stores g for the next kernel;
//  - attn_bwd_dq_kernel, one CTA per (row, 64 columns): dq = g . C over the
//    row's selected rows, no atomics.
// p and g are rounded to bf16 before they enter an MMA, as the forward rounds
// its probabilities; D comes from the forward's bf16 output.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace bwd {

using sm100::smem_u32;

constexpr int kSlots = 64;      // selected slots per CTA of the dkv kernel
constexpr int kCols = 64;       // column slice of the dC and dq tiles
constexpr int kThreads = 256;   // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kMaxHeads = 128;  // 8 warps x 16 heads
constexpr int kMaxDqk = 576;
constexpr int kPS = kCols + 8;  // row stride (bf16) of the [head][64] tiles: 144 B, conflict-free ldmatrix

__host__ __device__ inline int heads_pad(int Hq) { return (Hq + 15) / 16 * 16; }
__host__ __device__ inline int slots_pad(int k) { return (k + kSlots - 1) / kSlots * kSlots; }

// Shared memory of the dkv kernel (113 KB at Hq = 128, d_qk = 576: two CTAs per
// SM). Region A: the 64 gathered rows while z and dp are formed, then two
// double-buffered [hp][64] slices of q and dout for the dC products. Region B:
// a double-buffered [hp][64] tile of q or dout while z and dp are formed, then
// p and g. Plus the slots' cache rows and per-head D and lse.
__host__ __device__ inline size_t dkv_region_a(int hp, int d_qk)
{
    const size_t rows = (size_t)kSlots * (d_qk + 8), sl = (size_t)4 * hp * kPS;
    return rows > sl ? rows : sl;
}

__host__ __device__ inline size_t dkv_smem(int Hq, int d_qk)
{
    const int hp = heads_pad(Hq);
    return sizeof(__nv_bfloat16) * (dkv_region_a(hp, d_qk) + (size_t)2 * hp * kPS) +
           sizeof(long long) * kSlots + 2 * sizeof(float) * hp;
}

// Shared memory of the dq kernel: two buffers of {64 rows x 64 columns, g of hp heads x 64 slots}.
__host__ __device__ inline size_t dq_smem(int Hq)
{
    return sizeof(__nv_bfloat16) * 2 * ((size_t)kSlots * kPS + (size_t)heads_pad(Hq) * kPS);
}

// ------------------------------------------------------ warp-level helpers

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += a (16x16, row) * b (16x8, col); bf16 inputs, fp32 accumulators. A pure
// register operation (not volatile), so the compiler may schedule it freely; the
// ldmatrix loads stay volatile and in program order around the barriers.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Lane addresses of the four 8x8 matrices of one ldmatrix.x4 (lane l feeds row l % 8 of
// matrix l / 8), for the three operand forms used here. Shared tiles are row-major with
// a row stride of `ld` bf16.
// A fragment (16 x 16 at r0, c0) of a row-major [m][k] tile.
__device__ __forceinline__ uint32_t a_addr(uint32_t base, int ld, int r0, int c0, int lane)
{
    return base + 2u * (uint32_t)((r0 + (lane & 15)) * ld + c0 + (lane >> 4) * 8);
}
// A fragment of the transpose of a [k][m] tile (m0 = first m, k0 = first k); use with .trans.
__device__ __forceinline__ uint32_t at_addr(uint32_t base, int ld, int m0, int k0, int lane)
{
    return base + 2u * (uint32_t)((k0 + (lane & 7) + (lane >> 4) * 8) * ld + m0 + ((lane >> 3) & 1) * 8);
}
// B fragments of two n8 tiles (n0, n0 + 8) from a [n][k] tile (non-trans).
__device__ __forceinline__ uint32_t bn_addr(uint32_t base, int ld, int n0, int k0, int lane)
{
    return base + 2u * (uint32_t)((n0 + (lane & 7) + (lane >> 4) * 8) * ld + k0 + ((lane >> 3) & 1) * 8);
}
// B fragments of two n8 tiles (n0, n0 + 8) from a [k][n] tile; use with .trans.
__device__ __forceinline__ uint32_t bk_addr(uint32_t base, int ld, int n0, int k0, int lane)
{
    return base + 2u * (uint32_t)((k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + n0 + (lane >> 4) * 8);
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint32_t ld_pair(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint32_t*>(p)); }

// Cache row of slot i of row t (-1: not a candidate).
__device__ __forceinline__ long long slot_row(const int* idx, int k, int t, int i, long long base, int n_cand)
{
    if (i >= k) return -1;
    const int s = idx[(size_t)t * k + i];
    return (s >= 0 && s < n_cand) ? base + s : -1;
}

// ------------------------------------------------------------- dkv kernel

// grid: x = slot chunk (64 slots), y = query row within the batch [r0, r0 + gridDim.y).
// g_ws: bf16 [rows][heads_pad(Hq)][slots_pad(k)], g = scale * dz per slot; chunks past
// the row's min(k, candidates) entries are neither read nor written.
__global__ void __launch_bounds__(kThreads, 2)
attn_bwd_dkv_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv,
                    const int* __restrict__ idx, const int* __restrict__ pos, const int* __restrict__ k_base,
                    const __nv_bfloat16* __restrict__ out, const float* __restrict__ lse,
                    const __nv_bfloat16* __restrict__ dout, int r0, int T, int S, int Hq, int d_qk, int d_v,
                    int k, float scale, float* __restrict__ dkv, __nv_bfloat16* __restrict__ g_ws)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int hp = heads_pad(Hq), ldc = d_qk + 8, kp = slots_pad(k);
    __nv_bfloat16* cs = reinterpret_cast<__nv_bfloat16*>(smem_raw);   // A: [64][ldc] gathered rows
    __nv_bfloat16* bufB = cs + dkv_region_a(hp, d_qk);                // B: 2 x [hp][kPS] q or dout
    __nv_bfloat16* ps = bufB;                                         // B after z, dp: p [hp][kPS]
    __nv_bfloat16* gs = ps + (size_t)hp * kPS;                        //                g [hp][kPS]
    long long* rows = reinterpret_cast<long long*>(bufB + (size_t)2 * hp * kPS);  // [64]
    float* Dh = reinterpret_cast<float*>(rows + kSlots);              // [hp]
    float* lse2 = Dh + hp;                                            // [hp]

    const int tl = blockIdx.y, t = r0 + tl, i0 = blockIdx.x * kSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    constexpr float kLog2e = 1.4426950408889634f;
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    if (i0 >= min(k, n_cand)) return;   // whole chunk past the row's entries (uniform per CTA)
    const int n_slices = (d_qk + kCols - 1) / kCols;

    const int n_qs = n_slices, n_os = (d_v + kCols - 1) / kCols;

    // Columns c0 .. c0 + 63 of the rows of q (ld = d_qk, nvalid = d_qk) or dout
    // (ld = d_v, nvalid = d_v) into the [hp][kPS] tile at dst, zeros past nvalid
    // and Hq (cp.async; the caller commits).
    auto load_tile = [&](__nv_bfloat16* dst, const __nv_bfloat16* src, int ld, int nvalid, int c0) {
        for (int e = threadIdx.x; e < hp * (kCols / 8); e += kThreads) {
            const int h = e >> 3, c8 = (e & 7) * 8;
            const bool ok = h < Hq && c0 + c8 < nvalid;
            const __nv_bfloat16* g = ok ? src + ((size_t)t * Hq + h) * ld + c0 + c8 : src;
            sm100::cp_async16(smem_u32(dst + (size_t)h * kPS + c8), g, ok ? 16u : 0u);
        }
    };
    // z / dp stage st: q columns 64 st (st < n_qs), else dout columns 64 (st - n_qs); buffer st & 1
    auto load_stage = [&](int st) {
        __nv_bfloat16* dst = bufB + (size_t)(st & 1) * hp * kPS;
        if (st < n_qs) load_tile(dst, q, d_qk, d_qk, st * kCols);
        else load_tile(dst, dout, d_v, d_v, (st - n_qs) * kCols);
        cp_async_commit();
    };
    // dC slice sl: q and dout columns 64 sl, into pair sl & 1 of region A
    auto load_slice = [&](__nv_bfloat16* dst, int sl) {
        __nv_bfloat16* qsl = dst + (size_t)(sl & 1) * 2 * hp * kPS;
        load_tile(qsl, q, d_qk, d_qk, sl * kCols);
        load_tile(qsl + (size_t)hp * kPS, dout, d_v, d_v, sl * kCols);
        cp_async_commit();
    };
    if (threadIdx.x < kSlots) rows[threadIdx.x] = slot_row(idx, k, t, i0 + threadIdx.x, base, n_cand);
    __syncthreads();
    // gather the 64 selected rows (zeros for non-candidates) and the first q tile
    // with cp.async while D is formed
    {
        const int v8 = d_qk / 8;
        for (int e = threadIdx.x; e < kSlots * v8; e += kThreads) {
            const int j = e / v8, c8 = e - j * v8;
            const long long r = rows[j];
            const __nv_bfloat16* src = r >= 0 ? kv + (size_t)r * d_qk + c8 * 8 : kv;
            sm100::cp_async16(smem_u32(cs + (size_t)j * ldc + c8 * 8), src, r >= 0 ? 16u : 0u);
        }
        cp_async_commit();
    }
    load_stage(0);
    // D_h = dout_h . o_h and lse in base 2, one warp per head
    for (int h = warp; h < hp; h += kWarps) {
        float acc = 0.f;
        if (h < Hq) {
            const __nv_bfloat16* gr = dout + ((size_t)t * Hq + h) * d_v;
            const __nv_bfloat16* orow = out + ((size_t)t * Hq + h) * d_v;
            for (int c = 2 * lane; c < d_v; c += 64) {
                const uint32_t a = ld_pair(gr + c), b = ld_pair(orow + c);
                acc = fmaf(bf16_lo(a), bf16_lo(b), fmaf(bf16_hi(a), bf16_hi(b), acc));
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
            Dh[h] = acc;
            lse2[h] = h < Hq ? lse[(size_t)t * Hq + h] * kLog2e : 0.f;
        }
    }

    const uint32_t cs_u = smem_u32(cs), ps_u = smem_u32(ps), gs_u = smem_u32(gs);

    // z and dp: warp w takes heads 16 w .. + 16 against the 64 slots, one 64-column
    // tile of q (then of dout) at a time, the next tile loading meanwhile.
    const int h0 = warp * 16;
    const bool h_active = h0 < hp;
    float z[8][4], dp[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) z[n][e] = dp[n][e] = 0.f;
    const int n_stages = n_qs + n_os;
    for (int st = 0; st < n_stages; ++st) {
        if (st + 1 < n_stages) {
            load_stage(st + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_group<0>();
        }
        __syncthreads();
        const bool is_q = st < n_qs;
        const int c0 = (is_q ? st : st - n_qs) * kCols;
        const int nc = min(kCols, (is_q ? d_qk : d_v) - c0);   // a multiple of 16
        const uint32_t a_u = smem_u32(bufB + (size_t)(st & 1) * hp * kPS);
        auto tile_mma = [&](float (&acc)[8][4]) {
#pragma unroll 2
            for (int kk = 0; kk < nc; kk += 16) {
                uint32_t a[4], b[4][4];
                ldsm_x4(a_addr(a_u, kPS, h0, kk, lane), a);
#pragma unroll
                for (int np = 0; np < 4; ++np) ldsm_x4(bn_addr(cs_u, ldc, np * 16, c0 + kk, lane), b[np]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    mma_bf16(acc[2 * np], a, b[np][0], b[np][1]);
                    mma_bf16(acc[2 * np + 1], a, b[np][2], b[np][3]);
                }
            }
        };
        if (h_active) {
            if (is_q) tile_mma(z);
            else tile_mma(dp);
        }
        __syncthreads();
    }
    // p and g (region B is free: every warp is past its last slice)
    if (h_active) {
        const float zs = scale * kLog2e;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int hl = h0 + gq + 8 * half;
            const bool hok = hl < Hq;
            const float l2 = lse2[hl], D = Dh[hl];
            __nv_bfloat16* gw = g_ws + ((size_t)tl * hp + hl) * kp + i0;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int j = n * 8 + 2 * tq;
                float pv[2], gv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool ok = hok && rows[j + e] >= 0;
                    const float p = ok ? exp2f(fmaf(z[n][2 * half + e], zs, -l2)) : 0.f;
                    pv[e] = p;
                    gv[e] = ok ? scale * p * (dp[n][2 * half + e] - D) : 0.f;
                }
                const uint32_t pp = pack_bf16x2(pv[0], pv[1]), gg = pack_bf16x2(gv[0], gv[1]);
                *reinterpret_cast<uint32_t*>(ps + (size_t)hl * kPS + j) = pp;
                *reinterpret_cast<uint32_t*>(gs + (size_t)hl * kPS + j) = gg;
                *reinterpret_cast<uint32_t*>(gw + j) = gg;
            }
        }
    }
    __nv_bfloat16* slices = cs;   // region A: the gathered rows are dead
    load_slice(slices, 0);
    __syncthreads();

    // dC (64 slots x d_qk) = g^T q + p^T dout, 64 columns at a time, the next
    // slice of q / dout loading (cp.async) while this one is multiplied; warp w
    // owns slots 16 (w % 4) .. + 16 and columns 32 (w / 4) .. + 32 of a slice.
    const int mt = warp & 3, nh = warp >> 2;
    for (int sl = 0; sl < n_slices; ++sl) {
        if (sl + 1 < n_slices) {
            load_slice(slices, sl + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_group<0>();
        }
        __syncthreads();
        const int c0 = sl * kCols, nc = min(kCols, d_qk - c0);   // nc: a multiple of 16
        const uint32_t qsl_u = smem_u32(slices + (size_t)(sl & 1) * 2 * hp * kPS);
        const uint32_t osl_u = qsl_u + 2u * hp * kPS;
        if (nh * 32 < nc) {
            // g^T q and p^T dout in separate accumulators (no back-to-back MMA
            // dependence), all fragments of a k-step loaded before its MMAs
            float acc[4][4], accp[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[n][e] = accp[n][e] = 0.f;
            const int npairs = min(2, (nc - nh * 32) / 16);
            const bool with_v = c0 < d_v;
#pragma unroll 2
            for (int k0 = 0; k0 < hp; k0 += 16) {
                uint32_t ag[4], ap[4], bq[2][4], bo[2][4];
                ldsm_x4_t(at_addr(gs_u, kPS, mt * 16, k0, lane), ag);
#pragma unroll
                for (int np = 0; np < 2; ++np)
                    if (np < npairs) ldsm_x4_t(bk_addr(qsl_u, kPS, nh * 32 + np * 16, k0, lane), bq[np]);
                if (with_v) {
                    ldsm_x4_t(at_addr(ps_u, kPS, mt * 16, k0, lane), ap);
#pragma unroll
                    for (int np = 0; np < 2; ++np)
                        if (np < npairs) ldsm_x4_t(bk_addr(osl_u, kPS, nh * 32 + np * 16, k0, lane), bo[np]);
                }
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    if (np < npairs) {
                        mma_bf16(acc[2 * np], ag, bq[np][0], bq[np][1]);
                        mma_bf16(acc[2 * np + 1], ag, bq[np][2], bq[np][3]);
                        if (with_v) {
                            mma_bf16(accp[2 * np], ap, bo[np][0], bo[np][1]);
                            mma_bf16(accp[2 * np + 1], ap, bo[np][2], bo[np][3]);
                        }
                    }
                }
            }
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[n][e] += accp[n][e];
            // lane pairs (tq, tq ^ 1) swap halves so that each lane adds four
            // consecutive columns of one slot: even tq slot gq, odd tq slot gq + 8
            const bool odd = tq & 1;
            const long long r = rows[mt * 16 + gq + (odd ? 8 : 0)];
            float* dst = dkv + (r < 0 ? 0 : (size_t)r * d_qk) + c0 + nh * 32 + 4 * (tq >> 1);
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const float s0 = odd ? acc[n][0] : acc[n][2], s1 = odd ? acc[n][1] : acc[n][3];
                const float g0 = __shfl_xor_sync(0xffffffffu, s0, 1), g1 = __shfl_xor_sync(0xffffffffu, s1, 1);
                const float4 v = odd ? make_float4(g0, g1, acc[n][2], acc[n][3])
                                     : make_float4(acc[n][0], acc[n][1], g0, g1);
                if (n < 2 * npairs && r >= 0) atomicAdd(reinterpret_cast<float4*>(dst + n * 8), v);
            }
        }
        __syncthreads();
    }
}

// -------------------------------------------------------------- dq kernel

// grid: x = 64-column slice of d_qk, y = query row within the batch.
// dq fp32 [T][Hq][d_qk] = sum over the row's slots of g (from g_ws) times the row.
__global__ void __launch_bounds__(kThreads)
attn_bwd_dq_kernel(const __nv_bfloat16* __restrict__ kv, const int* __restrict__ idx,
                   const int* __restrict__ pos, const int* __restrict__ k_base,
                   const __nv_bfloat16* __restrict__ g_ws, int r0, int T, int S, int Hq, int d_qk, int k,
                   float* __restrict__ dq)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int hp = heads_pad(Hq), kp = slots_pad(k);
    __nv_bfloat16* csl = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // 2 x [64 slots][kPS] column slice
    __nv_bfloat16* gsm = csl + (size_t)2 * kSlots * kPS;               // 2 x [hp][kPS] g of 64 slots

    const int tl = blockIdx.y, t = r0 + tl, c0 = blockIdx.x * kCols;
    const int nc = min(kCols, d_qk - c0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    const int h0 = warp * 16;
    const bool active = h0 < hp;
    float acc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;

    // chunk c (slots 64 c .. + 64): the rows' column slice and g, into buffer c & 1 (cp.async)
    auto load_chunk = [&](int c) {
        const int i0 = c * kSlots;
        __nv_bfloat16* cb = csl + (size_t)(c & 1) * kSlots * kPS;
        __nv_bfloat16* gb = gsm + (size_t)(c & 1) * hp * kPS;
        for (int e = threadIdx.x; e < kSlots * (kCols / 8); e += kThreads) {
            const int j = e >> 3, c8 = (e & 7) * 8;
            const long long r = slot_row(idx, k, t, i0 + j, base, n_cand);
            const bool ok = r >= 0 && c8 < nc;
            sm100::cp_async16(smem_u32(cb + (size_t)j * kPS + c8), ok ? kv + (size_t)r * d_qk + c0 + c8 : kv,
                              ok ? 16u : 0u);
        }
        for (int e = threadIdx.x; e < hp * (kSlots / 8); e += kThreads) {
            const int h = e >> 3, j8 = (e & 7) * 8;
            sm100::cp_async16(smem_u32(gb + (size_t)h * kPS + j8), g_ws + ((size_t)tl * hp + h) * kp + i0 + j8,
                              16u);
        }
        cp_async_commit();
    };
    const int n_chunks = (min(k, n_cand) + kSlots - 1) / kSlots;
    if (n_chunks > 0) load_chunk(0);
    for (int c = 0; c < n_chunks; ++c) {
        if (c + 1 < n_chunks) {
            load_chunk(c + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_group<0>();
        }
        __syncthreads();
        if (active) {
            const uint32_t csl_u = smem_u32(csl + (size_t)(c & 1) * kSlots * kPS);
            const uint32_t gsm_u = smem_u32(gsm + (size_t)(c & 1) * hp * kPS);
#pragma unroll
            for (int k0 = 0; k0 < kSlots; k0 += 16) {
                uint32_t a[4], b[4][4];
                ldsm_x4(a_addr(gsm_u, kPS, h0, k0, lane), a);
#pragma unroll
                for (int np = 0; np < 4; ++np)
                    if (np * 16 < nc) ldsm_x4_t(bk_addr(csl_u, kPS, np * 16, k0, lane), b[np]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    if (np * 16 < nc) {
                        mma_bf16(acc[2 * np], a, b[np][0], b[np][1]);
                        mma_bf16(acc[2 * np + 1], a, b[np][2], b[np][3]);
                    }
                }
            }
        }
        __syncthreads();
    }
    if (!active) return;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int h = h0 + gq + 8 * half;
        if (h >= Hq) continue;
        float* dst = dq + ((size_t)t * Hq + h) * d_qk + c0 + 2 * tq;
#pragma unroll
        for (int n = 0; n < 8; ++n)
            if (n * 8 < nc)
                *reinterpret_cast<float2*>(dst + n * 8) = make_float2(acc[n][2 * half], acc[n][2 * half + 1]);
    }
}

}  // namespace bwd
}  // namespace dsa
