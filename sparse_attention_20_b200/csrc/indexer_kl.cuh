// Indexer KL loss and its gradient with respect to the indexer's inputs: the
// objective that trains the lightning indexer toward the main attention
// ("Paper Breakdown: DeepSeek-V3.2", table "Continued Pre-Training (2.1.1)":
// the dense warm-up uses L^I = sum_t D_KL(p_{t,:} || Softmax(I_{t,:})), the
// sparse stage the same KL over the selected set S_t, indexer input detached).
//
// p_{t,:} (left undefined by the pages) is read as the main attention of row t
// summed over the query heads and L1-normalised over S_t:
//   p_s  = sum_h P_{h,s} / sum_{s',h} P_{h,s'},  P_{h,s} = exp(scale q_h.c_s - lse_h)
//   I_s  = sum_j w_j ReLU(u_{j,s}),  u_{j,s} = q^I_j.k^I_s   (FP8 inputs, fp32 sums)
//   L_t  = sum_s p_s (log p_s - I_s + logsumexp_S(I)),   dI_s = softmax_S(I)_s - p_s
//   dw_j = sum_s dI_s ReLU(u_{j,s}); dq^I_j = sum_s dI_s w_j [u_{j,s} > 0] k^I_s;
//   dk^I_s += sum_j dI_s w_j [u_{j,s} > 0] q^I_j   (fp32 atomics; caller zeroes)
// The dense warm-up loss is the same call with every causal key selected.
//
// Two kernels:
//  - head_prob_sum_kernel, one CTA per (row, 64 selected slots): the gathered
//    latent rows against all query heads (warp-level bf16 MMAs, as the
//    attention backward forms z), P from the forward's lse, summed over heads:
//    psum [rows][slots_pad(k)] fp32;
//  - indexer_kl_row_kernel, one CTA per row: index scores of the selected keys
//    (CUDA cores, one slot per thread), the loss, and the three gradients.
#pragma once
#include "attn_bwd.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace kl {

using namespace dsa::bwd;

// ------------------------------------------------------ head-summed probabilities

// Region A: the 64 gathered rows [64][d_qk + 8]; region B: two [hp][kPS] q tiles
// (after the MMAs: the per-warp column sums [8][64] fp32). Then rows and lse.
__host__ __device__ inline size_t prob_smem(int Hq, int d_qk)
{
    const int hp = heads_pad(Hq);
    size_t b = (size_t)2 * hp * kPS * sizeof(__nv_bfloat16);
    if (b < (size_t)kWarps * kSlots * sizeof(float)) b = (size_t)kWarps * kSlots * sizeof(float);
    return (size_t)kSlots * (d_qk + 8) * sizeof(__nv_bfloat16) + b + sizeof(long long) * kSlots +
           sizeof(float) * hp;
}

// grid: x = slot chunk, y = query row within the pass [r0, r0 + gridDim.y).
// psum [rows][slots_pad(k)]: sum over heads of exp(scale q_h.c_s - lse_h), 0 for
// non-candidates; chunks past the row's min(k, candidates) entries are not written.
__global__ void __launch_bounds__(kThreads, 2)
head_prob_sum_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv,
                     const int* __restrict__ idx, const int* __restrict__ pos, const int* __restrict__ k_base,
                     const float* __restrict__ lse, int r0, int T, int S, int Hq, int d_qk, int k, float scale,
                     float* __restrict__ psum)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int hp = heads_pad(Hq), ldc = d_qk + 8, kp = slots_pad(k);
    __nv_bfloat16* cs = reinterpret_cast<__nv_bfloat16*>(smem_raw);
    unsigned char* regb = smem_raw + (size_t)kSlots * ldc * sizeof(__nv_bfloat16);
    size_t bbytes = (size_t)2 * hp * kPS * sizeof(__nv_bfloat16);
    if (bbytes < (size_t)kWarps * kSlots * sizeof(float)) bbytes = (size_t)kWarps * kSlots * sizeof(float);
    __nv_bfloat16* qbuf = reinterpret_cast<__nv_bfloat16*>(regb);   // 2 x [hp][kPS]
    float* red = reinterpret_cast<float*>(regb);                      // after the MMAs: [8][64]
    long long* rows = reinterpret_cast<long long*>(regb + bbytes);
    float* lse2 = reinterpret_cast<float*>(rows + kSlots);

    const int tl = blockIdx.y, t = r0 + tl, i0 = blockIdx.x * kSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    constexpr float kLog2e = 1.4426950408889634f;
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    if (i0 >= min(k, n_cand)) return;
    const int n_tiles = (d_qk + kCols - 1) / kCols;

    auto load_tile = [&](int st) {
        __nv_bfloat16* dst = qbuf + (size_t)(st & 1) * hp * kPS;
        const int c0 = st * kCols;
        for (int e = threadIdx.x; e < hp * (kCols / 8); e += kThreads) {
            const int h = e >> 3, c8 = (e & 7) * 8;
            const bool ok = h < Hq && c0 + c8 < d_qk;
            const __nv_bfloat16* g = ok ? q + ((size_t)t * Hq + h) * d_qk + c0 + c8 : q;
            sm100::cp_async16(smem_u32(dst + (size_t)h * kPS + c8), g, ok ? 16u : 0u);
        }
        cp_async_commit();
    };

    if (threadIdx.x < kSlots) rows[threadIdx.x] = slot_row(idx, k, t, i0 + threadIdx.x, base, n_cand);
    for (int h = threadIdx.x; h < hp; h += kThreads) lse2[h] = h < Hq ? lse[(size_t)t * Hq + h] * kLog2e : 0.f;
    __syncthreads();
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
    load_tile(0);

    const uint32_t cs_u = smem_u32(cs);
    const int h0 = warp * 16;
    const bool h_active = h0 < hp;
    float z[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) z[n][e] = 0.f;
    for (int st = 0; st < n_tiles; ++st) {
        if (st + 1 < n_tiles) {
            load_tile(st + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_group<0>();
        }
        __syncthreads();
        const int c0 = st * kCols, nc = min(kCols, d_qk - c0);
        const uint32_t a_u = smem_u32(qbuf + (size_t)(st & 1) * hp * kPS);
        if (h_active) {
#pragma unroll 2
            for (int kk = 0; kk < nc; kk += 16) {
                uint32_t a[4], b[4][4];
                ldsm_x4(a_addr(a_u, kPS, h0, kk, lane), a);
#pragma unroll
                for (int np = 0; np < 4; ++np) ldsm_x4(bn_addr(cs_u, ldc, np * 16, c0 + kk, lane), b[np]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    mma_bf16(z[2 * np], a, b[np][0], b[np][1]);
                    mma_bf16(z[2 * np + 1], a, b[np][2], b[np][3]);
                }
            }
        }
        __syncthreads();
    }
    // P summed over the warp's 16 heads per slot column, then over the warps
    float col[8][2];
    const float zs = scale * kLog2e;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float v = 0.f;
            if (h_active) {
                const int j = n * 8 + 2 * tq + e;
                const bool slot_ok = rows[j] >= 0;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int hl = h0 + gq + 8 * half;
                    if (slot_ok && hl < Hq) v += exp2f(fmaf(z[n][2 * half + e], zs, -lse2[hl]));
                }
            }
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            col[n][e] = v;
        }
    }
    if (gq == 0) {
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) red[warp * kSlots + n * 8 + 2 * tq + e] = col[n][e];
    }
    __syncthreads();
    if (threadIdx.x < kSlots) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w * kSlots + threadIdx.x];
        psum[(size_t)tl * kp + i0 + threadIdx.x] = s;
    }
}

// ------------------------------------------------------------- per-row loss

constexpr int kRowThreads = 256;
constexpr int kMaxHI = 16;
constexpr int kMaxDI = 256;
constexpr int kMaxQElems = 4096;   // H_I * d_I: 16 dq outputs per thread

__host__ __device__ inline size_t row_smem(int H_I, int d_I, int k)
{
    return sizeof(float) * (256 + (size_t)H_I * d_I + kMaxHI + slots_pad(k) + (size_t)kRowThreads * H_I + 64) +
           (size_t)kRowThreads * d_I;
}

__device__ __forceinline__ float block_sum(float v, float* red)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kRowThreads / 32; ++w) s += red[w];
    return s;
}

__device__ __forceinline__ float block_max(float v, float* red)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = -INFINITY;
#pragma unroll
    for (int w = 0; w < kRowThreads / 32; ++w) s = fmaxf(s, red[w]);
    return s;
}

// grid: one CTA per query row of the pass. loss [T], dw [T][H_I], dqi [T][H_I][d_I]
// written; dki [S][d_I] accumulated.
__global__ void __launch_bounds__(kRowThreads)
indexer_kl_row_kernel(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                      const uint8_t* __restrict__ k_idx, const int* __restrict__ idx, const int* __restrict__ pos,
                      const int* __restrict__ k_base, const float* __restrict__ psum, int r0, int T, int S,
                      int H_I, int d_I, int k, float* __restrict__ loss, float* __restrict__ dw,
                      float* __restrict__ dqi, float* __restrict__ dki)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int kp = slots_pad(k);
    float* lut = reinterpret_cast<float*>(smem_raw);        // [256] e4m3 byte -> value
    float* qf = lut + 256;                                  // [H_I][d_I]
    float* wv = qf + H_I * d_I;                             // [16]
    float* Ib = wv + kMaxHI;                                // [kp] index scores of the slots
    float* cch = Ib + kp;                                   // [256][H_I] dI w_j [u > 0] of a chunk
    float* red = cch + kRowThreads * H_I;                   // [64]
    uint8_t* kch = reinterpret_cast<uint8_t*>(red + 64);    // [256][d_I] key bytes of a chunk

    const int tl = blockIdx.x, t = r0 + tl, tid = threadIdx.x;
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    const int n_row = min(k, n_cand);
    const int nq = H_I * d_I, d16 = d_I / 16;

    {
        const float2 f = e4m3x2_to_float2((uint16_t)tid);   // byte tid in the low half
        lut[tid] = f.x;
    }
    __syncthreads();
    for (int e = tid; e < nq; e += kRowThreads) qf[e] = lut[q_idx[(size_t)t * nq + e]];
    if (tid < kMaxHI) wv[tid] = tid < H_I ? w[(size_t)t * H_I + tid] : 0.f;

    // stage the key rows of slots c0 .. c0 + 255 (zeros for non-candidates) and
    // return this thread's slot row (-1: none)
    auto stage = [&](int c0) -> long long {
        for (int e = tid; e < kRowThreads * d16; e += kRowThreads) {
            const int j = e / d16, part = e - j * d16;
            const long long r = c0 + j < n_row ? slot_row(idx, k, t, c0 + j, base, n_cand) : -1;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r >= 0) v = __ldg(reinterpret_cast<const uint4*>(k_idx + (size_t)r * d_I) + part);
            *reinterpret_cast<uint4*>(kch + (size_t)j * d_I + part * 16) = v;
        }
        return c0 + tid < n_row ? slot_row(idx, k, t, c0 + tid, base, n_cand) : -1;
    };
    // u_j of this thread's staged key
    auto scores = [&](float (&u)[kMaxHI]) {
#pragma unroll
        for (int j = 0; j < kMaxHI; ++j) u[j] = 0.f;
        const uint8_t* kr = kch + (size_t)tid * d_I;
        for (int part = 0; part < d16; ++part) {
            const uint4 v = *reinterpret_cast<const uint4*>(kr + part * 16);
            const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
            float kf[16];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float2 lo = e4m3x2_to_float2((uint16_t)(wd[m] & 0xFFFFu));
                const float2 hi = e4m3x2_to_float2((uint16_t)(wd[m] >> 16));
                kf[4 * m] = lo.x;
                kf[4 * m + 1] = lo.y;
                kf[4 * m + 2] = hi.x;
                kf[4 * m + 3] = hi.y;
            }
#pragma unroll
            for (int j = 0; j < kMaxHI; ++j) {
                if (j < H_I) {
                    const float4* qj = reinterpret_cast<const float4*>(qf + j * d_I + part * 16);
                    float s = u[j];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float4 qv = qj[m];
                        s = fmaf(qv.x, kf[4 * m], s);
                        s = fmaf(qv.y, kf[4 * m + 1], s);
                        s = fmaf(qv.z, kf[4 * m + 2], s);
                        s = fmaf(qv.w, kf[4 * m + 3], s);
                    }
                    u[j] = s;
                }
            }
        }
    };

    // pass A: index scores of the row's slots
    for (int c0 = 0; c0 < n_row; c0 += kRowThreads) {
        __syncthreads();
        const long long r = stage(c0);
        __syncthreads();
        if (c0 + tid < n_row) {
            float I = -INFINITY;
            if (r >= 0) {
                float u[kMaxHI];
                scores(u);
                I = 0.f;
#pragma unroll
                for (int j = 0; j < kMaxHI; ++j)
                    if (j < H_I) I = fmaf(wv[j], fmaxf(u[j], 0.f), I);
            }
            Ib[c0 + tid] = I;
        }
    }
    __syncthreads();
    // log-sum-exp of the scores, total of the head sums, the loss
    const float* ps = psum + (size_t)tl * kp;
    float m = -INFINITY, ptot = 0.f;
    for (int i = tid; i < n_row; i += kRowThreads) {
        m = fmaxf(m, Ib[i]);
        ptot += ps[i];
    }
    m = block_max(m, red);
    ptot = block_sum(ptot, red + 8);
    const bool any = m > -INFINITY && ptot > 0.f;
    float l = 0.f;
    if (any)
        for (int i = tid; i < n_row; i += kRowThreads) l += Ib[i] > -INFINITY ? __expf(Ib[i] - m) : 0.f;
    l = block_sum(l, red + 16);
    const float lseI = m + __logf(l), inv_ptot = any ? 1.f / ptot : 0.f;
    float L = 0.f;
    if (any)
        for (int i = tid; i < n_row; i += kRowThreads) {
            const float p = ps[i] * inv_ptot;
            if (p > 0.f && Ib[i] > -INFINITY) L += p * (__logf(p) - Ib[i] + lseI);
        }
    L = block_sum(L, red + 24);
    if (tid == 0) loss[t] = any ? L : 0.f;

    // pass B: gradients. dq: thread owns groups g = tid + 256 e of four
    // consecutive d of one head j (g < H_I d_I / 4)
    constexpr int kGroups = kMaxQElems / 4 / kRowThreads;
    float4 acc[kGroups];
#pragma unroll
    for (int e = 0; e < kGroups; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int d4 = d_I / 4, nq4 = nq / 4;
    float dwp[kMaxHI];
#pragma unroll
    for (int j = 0; j < kMaxHI; ++j) dwp[j] = 0.f;
    for (int c0 = 0; any && c0 < n_row; c0 += kRowThreads) {
        __syncthreads();
        const long long r = stage(c0);
        __syncthreads();
        float c[kMaxHI];
#pragma unroll
        for (int j = 0; j < kMaxHI; ++j) c[j] = 0.f;
        if (r >= 0) {
            float u[kMaxHI];
            scores(u);
            const int i = c0 + tid;
            const float dI = __expf(Ib[i] - lseI) - ps[i] * inv_ptot;
#pragma unroll
            for (int j = 0; j < kMaxHI; ++j) {
                if (j < H_I) {
                    dwp[j] = fmaf(dI, fmaxf(u[j], 0.f), dwp[j]);
                    c[j] = u[j] > 0.f ? dI * wv[j] : 0.f;
                }
            }
            float* dk = dki + (size_t)r * d_I;
            for (int d = 0; d < d_I; d += 4) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < kMaxHI; ++j) {
                    if (j < H_I) {
                        const float4 qv = *reinterpret_cast<const float4*>(qf + j * d_I + d);
                        v.x = fmaf(c[j], qv.x, v.x);
                        v.y = fmaf(c[j], qv.y, v.y);
                        v.z = fmaf(c[j], qv.z, v.z);
                        v.w = fmaf(c[j], qv.w, v.w);
                    }
                }
                atomicAdd(reinterpret_cast<float4*>(dk + d), v);
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxHI; ++j)
            if (j < H_I) cch[tid * H_I + j] = c[j];
        __syncthreads();
        const int ns = min(kRowThreads, n_row - c0);
#pragma unroll
        for (int e = 0; e < kGroups; ++e) {
            const int g = tid + e * kRowThreads;
            if (g < nq4) {
                const int j = g / d4, d0 = 4 * (g - j * d4);
                float4 a = acc[e];
                for (int sl = 0; sl < ns; ++sl) {
                    const float cj = cch[sl * H_I + j];
                    const uint32_t kb = *reinterpret_cast<const uint32_t*>(kch + (size_t)sl * d_I + d0);
                    const float2 lo = e4m3x2_to_float2((uint16_t)(kb & 0xFFFFu));
                    const float2 hi = e4m3x2_to_float2((uint16_t)(kb >> 16));
                    a.x = fmaf(cj, lo.x, a.x);
                    a.y = fmaf(cj, lo.y, a.y);
                    a.z = fmaf(cj, hi.x, a.z);
                    a.w = fmaf(cj, hi.y, a.w);
                }
                acc[e] = a;
            }
        }
    }
#pragma unroll
    for (int e = 0; e < kGroups; ++e) {
        const int g = tid + e * kRowThreads;
        if (g < nq4) *reinterpret_cast<float4*>(dqi + (size_t)t * nq + 4 * g) = acc[e];
    }
    // dw: per-thread partials summed over the block, one head at a time
    for (int j = 0; j < H_I; ++j) {
        float v = 0.f;
#pragma unroll
        for (int jj = 0; jj < kMaxHI; ++jj)
            if (jj == j) v = dwp[jj];
        v = block_sum(v, red + 32);
        if (tid == 0) dw[(size_t)t * H_I + j] = v;
    }
}

}  // namespace kl
}  // namespace dsa
